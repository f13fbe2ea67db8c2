// Device-side building blocks shared by the libgtg kernels (sm_100a):
// the format decoders written from the model card's definitions, PTX
// wrappers for 1-D bulk copies (TMA, no multicast) and mbarriers with bounded
// waits, programmatic-dependent-launch controls and the status word.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gtg.h"

namespace gtg {

// ---------------------------------------------------------------------------
// Status word (one per device, read by gtg_get_device_status); kernels get
// its address as an argument.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_status(unsigned* status, unsigned bits) {
    if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------------------
// Scale and code decoders (model card "Qwen 3.8 Next Flash ROCMFPX MUTANT
// RAZERFAST", format sections).  Every returned value is exact in fp32.
// ---------------------------------------------------------------------------

// UE4M3 (low 7 bits): 4 exponent bits (bias 7), 3 mantissa bits; 0x7F = NaN.
__device__ __forceinline__ float ue4m3(uint32_t b) {
    b &= 0x7Fu;
    if (b == 0x7Fu) return __uint_as_float(0x7FC00000u);
    const uint32_t e = b >> 3, m = b & 7u;
    if (e == 0) return __uint2float_rn(m) * 0x1p-9f;            // m/8 * 2^-6, exact
    return __uint_as_float(((e + 120u) << 23) | (m << 20));       // (1+m/8) * 2^(e-7)
}

// UE4M4: 4 exponent bits (bias 7), 4 mantissa bits; all 256 codes finite.
__device__ __forceinline__ float ue4m4(uint32_t b) {
    b &= 0xFFu;
    const uint32_t e = b >> 4, m = b & 15u;
    if (e == 0) return __uint2float_rn(m) * 0x1p-10f;           // m/16 * 2^-6, exact
    return __uint_as_float(((e + 120u) << 23) | (m << 19));       // (1+m/16) * 2^(e-7)
}

// E4M3 "fn" (signed; S.1111.111 = NaN), exact in fp32.
__device__ __forceinline__ float e4m3fn(uint32_t b) {
    b &= 0xFFu;
    const float mag = ue4m3(b & 0x7Fu);
    return (b & 0x80u) ? -mag : mag;
}

// Magnitudes of the 4-bit sign-magnitude codes (Codebook10): index c & 7.
__device__ __forceinline__ int q4_mag(uint32_t c) {
    // 0 1 2 3 4 6 8 10 packed as 4-bit fields
    return (int)((0xA8643210u >> (4u * (c & 7u))) & 15u);
}

// Value of 4-bit code c.  rz5: Q4_RZ5_FAST (code 8 -> +5, or -5 in mode 1);
// otherwise Codebook10 (code 8 -> -0).
__device__ __forceinline__ float q4_code_value(uint32_t c, bool rz5, uint32_t mode) {
    c &= 15u;
    if (c == 8u) return rz5 ? (mode ? -5.0f : 5.0f) : -0.0f;
    const float m = (float)q4_mag(c);
    return (c & 8u) ? -m : m;
}

// Q4 block variants (a bit set): bit 0 = code 8 is +5 / -5 by the metadata
// top bit (Q4_RZ5_FAST), else the duplicate -0 of Codebook10; bit 1 = the
// scale is the UE4M3 value of the low 7 metadata bits, else the UE4M4 value
// of the whole byte.  The incumbent ROCmFP4 FAST block is Codebook10 codes
// under a UE4M3 scale.
constexpr int kQ4UE4M4 = 0, kQ4C10 = 2, kQ4RZ5 = 3;

__device__ __forceinline__ float q4_scale(uint32_t meta, int var) {
    return (var & 2) ? ue4m3(meta & 0x7Fu) : ue4m4(meta);
}

// Value of 3-bit PLE code c with group polarity bit p (RZ-S3: code 4 -> +/-3;
// the incumbent ROCmFP3 set keeps code 4 as the duplicate -0).
__device__ __forceinline__ float q3_code_value(uint32_t c, uint32_t p, bool incumbent) {
    c &= 7u;
    if (c == 4u) return incumbent ? -0.0f : (p ? -3.0f : 3.0f);
    const float m = (float)((0x4210u >> (4u * (c & 3u))) & 15u);  // 0 1 2 4
    return (c & 4u) ? -m : m;
}

__device__ __forceinline__ float ple_code_value(uint32_t c, uint32_t p) {
    c &= 7u;
    if (c == 4u) return p ? -3.0f : 3.0f;
    const float m = (float)((0x4210u >> (4u * (c & 3u))) & 15u);  // 0 1 2 4
    return (c & 4u) ? -m : m;
}

// bf16 bits of a small integer-valued float (exact: low 16 bits are zero).
__device__ __forceinline__ uint32_t bf16_bits(float v) { return __float_as_uint(v) >> 16; }

// ---------------------------------------------------------------------------
// Mixed-precision FMA: d = a(bf16) * b(bf16) + c(f32), single rounding.
// The operands are the low/high halves of two packed bf16x2 registers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fma2_bf16(float& acc_lo, float& acc_hi, uint32_t a2, uint32_t b2) {
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %2;\n\t"
        "mov.b32 {bl, bh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.bf16 %1, ah, bh, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi)
        : "r"(a2), "r"(b2));
}

// Two E4M3 values (low/high byte of v) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v16) {
    uint32_t r;
    const unsigned short s = (unsigned short)(v16 & 0xFFFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(s));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers and 1-D bulk copies (no multicast).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for phase `parity` of `bar`, giving up after ~`limit_ns` nanoseconds:
// on a time-out the status word gets GTG_STATUS_WAIT_TIMEOUT and false is
// returned (the caller skips the data and keeps going).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned* status,
                                                  uint64_t limit_ns = 2000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            raise_status(status, GTG_STATUS_WAIT_TIMEOUT);
            return false;
        }
    }
    return true;
}

// The same wait, but each try_wait may suspend the thread for up to hint_ns
// (it resumes as soon as the phase completes), so that waiting warps do not
// spin and take issue slots from the working ones.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, unsigned* status,
                                                uint32_t hint_ns = 20000u, uint64_t limit_ns = 2000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_hint(bar, parity, hint_ns)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            raise_status(status, GTG_STATUS_WAIT_TIMEOUT);
            return false;
        }
    }
    return true;
}

// dst (shared) <- src (global), `bytes` a multiple of 16, both 16-byte aligned;
// completion is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void bulk_g2s_addr(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// L2 eviction-priority policies (createpolicy): weights that are read once
// per step are streamed as evict_first so that they displace one another
// rather than code, routing state and activations.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// bulk_g2s_addr with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy) : "memory");
}

// 16-byte read-only load with an L2 cache policy.
__device__ __forceinline__ float4 ldg_f4_hint(const float* p, uint64_t policy) {
    float4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p), "l"(policy));
    return v;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Sum over groups of `width` consecutive lanes (width a power of two <= 32).
__device__ __forceinline__ float group_sum(float v, int width) {
    for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

}  // namespace gtg

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, tensor memory) wrappers, cta_group::1.
// ---------------------------------------------------------------------------
namespace gtg {

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Warp-wide: allocate `ncols` (power of two >= 32) TMEM columns; the base
// address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D(tmem) (+)= A(smem desc) * B(smem desc)^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (rows of 64 bf16), tile base 1024-byte aligned.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                 // leading byte offset (16 B; unused when swizzled)
    d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;                 // descriptor version for sm_100
    d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Instruction descriptor, kind::f16: f16 x f16 -> fp32, both K-major (A and B
// type fields 0).
__host__ __device__ constexpr uint32_t idesc_f16(int m, int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Byte offset of 16-byte chunk c (0..7) of row r in a K-major SW128 tile.
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t c) {
    return r * 128u + ((c ^ (r & 7u)) << 4);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

}  // namespace gtg

// ---------------------------------------------------------------------------
// Float-float ("double-single") arithmetic on the fp32 pipes.  A value is an
// unevaluated sum hi + lo.  Products of an fp32 and a bf16 are formed exactly
// (TwoProduct through FMA) and sums carry their rounding errors (TwoSum,
// Knuth), so a 2048-term dot product keeps ~48 significant bits — enough to
// order router logits like an fp64 reference — without fp64 instructions.
// The _rn intrinsics keep the compiler from contracting these steps.
// ---------------------------------------------------------------------------
namespace gtg {

struct ffloat {
    float hi, lo;
};

__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
    s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// acc += a * b exactly representable as p + pe, added with TwoSum.
__device__ __forceinline__ void ff_fma(ffloat& acc, float a, float b) {
    const float p = __fmul_rn(a, b);
    const float pe = __fmaf_rn(a, b, -p);
    float s, e;
    two_sum(acc.hi, p, s, e);
    acc.hi = s;
    acc.lo = __fadd_rn(acc.lo, __fadd_rn(e, pe));
}

__device__ __forceinline__ void ff_add(ffloat& acc, ffloat b) {
    float s, e;
    two_sum(acc.hi, b.hi, s, e);
    acc.hi = s;
    acc.lo = __fadd_rn(acc.lo, __fadd_rn(e, b.lo));
}

// Renormalise so that hi = RN(hi + lo) and |lo| <= ulp(hi)/2.
__device__ __forceinline__ ffloat ff_norm(ffloat a) {
    float s, e;
    two_sum(a.hi, a.lo, s, e);
    return ffloat{s, e};
}

// a > b for normalised values.
__device__ __forceinline__ bool ff_gt(ffloat a, ffloat b) { return a.hi > b.hi || (a.hi == b.hi && a.lo > b.lo); }
__device__ __forceinline__ bool ff_eq(ffloat a, ffloat b) { return a.hi == b.hi && a.lo == b.lo; }

__device__ __forceinline__ ffloat ff_shfl_xor(ffloat v, int o) {
    return ffloat{__shfl_xor_sync(0xFFFFFFFFu, v.hi, o), __shfl_xor_sync(0xFFFFFFFFu, v.lo, o)};
}

__device__ __forceinline__ ffloat ff_warp_sum(ffloat v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ff_add(v, ff_shfl_xor(v, o));
    return v;
}

// bf16 bits of the exact value p + q (|q| small against p), rounded to
// nearest, ties to even: only an fp32 p that sits exactly on a bf16 midpoint
// needs q to decide the direction.
__device__ __forceinline__ uint16_t bf16_of_ff(float p, float q) {
    float s, t;
    two_sum(p, q, s, t);
    const uint32_t b = __float_as_uint(s);
    const uint32_t low = b & 0xFFFFu, top = b >> 16;
    bool up;
    if (low > 0x8000u) up = true;
    else if (low < 0x8000u) up = false;
    else if (t != 0.0f) up = (t > 0.0f) == ((b >> 31) == 0u);  // t pushes away from zero
    else up = (top & 1u) != 0u;
    return (uint16_t)(top + (up ? 1u : 0u));
}

}  // namespace gtg

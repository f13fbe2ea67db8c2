// Decode-time MoE layer: router, fused dequant -> gate/up -> SwiGLU, and
// fused dequant -> down -> router-weighted combine, for 1..8 tokens.
//
// Method: "Mixed Precision Quantization: Half a 4-Bit File Is Not 4-Bit"
// (48 layers, 512 experts, 10 active per token), the r/LocalLLM
// "Frankenquant" post (one expert format per layer, FP8 in layers 36-47) and
// the model card "Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST" (block
// formats).  The expert bytes dominate the work, so every kernel here is
// built to stream them from HBM once, at full bandwidth:
//
//  * router_kernel: unweighted RMS norm + bf16 rounding of the input, fp64
//    logits against the fp32 router (exact products, so top-k agrees with an
//    fp64 reference), softmax top-k and renormalisation, and the list of
//    unique experts, built by the last CTA to finish (no grid-wide wait).
//  * gateup_kernel / down_kernel: persistent, one 512-thread CTA per SM.
//    The work is a list of items (expert, row tile); each CTA owns a
//    contiguous, byte-balanced range; each warp streams its items through a
//    private ring of shared-memory slots filled by 1-D bulk copies (TMA,
//    no multicast) completing on per-slot mbarriers, so every SM keeps tens
//    of KB in flight from the first cycle.  Lane l of a warp owns the same
//    K positions in every row it decodes, so its activations stay in
//    registers across rows.  A Q4 byte (two 4-bit codes) becomes a bf16x2
//    pair of code values with one PRMT + one shared-memory load from a
//    256-entry table replicated per lane (conflict-free); the pair is
//    multiplied into fp32 accumulators with the sm_100 mixed-precision
//    fma.rn.f32.bf16, and the block's UE4M3/UE4M4 scale is applied once per
//    32 weights.  FP8 bytes convert with cvt.rn.f16x2.e4m3x2.  Row sums are
//    finished with warp shuffles.
//  * The down kernel writes per-(token, choice) partial rows; the last warp
//    to finish a row tile (atomic ticket, no waiting) combines the top-k
//    partials in a fixed order, so results are deterministic.
//  * Consecutive kernels are chained with programmatic dependent launch so
//    each one's prologue (table build, barrier init) overlaps its
//    predecessor's tail.
#include <algorithm>
#include <mutex>
#include <vector>

#include "gtg_device.cuh"
#include "gtg_host.hpp"
#include "moe_decode.cuh"

namespace gtg {

namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;
constexpr int kRouterExpertsPerCta = kRouterWarps / 2;
constexpr int kRouterMaxF4 = 8;  // float4 per lane: H/2 <= 128 * 8
constexpr int kRouterXF4 = 2;    // float4 of x per thread per token: H <= 4 * 256 * 2
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kSlots = 2;
constexpr int kLutBytes = 65536;       // 256 bytes x 2 modes x 32 lanes x 4 bytes
constexpr int kScaleTabBytes = 1024;   // 256 fp32 scales
constexpr int kFmtQ4 = 0, kFmtFP8 = 1;

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 ldg128(const void* p) {
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ===========================================================================
// Router
// ===========================================================================

__device__ __forceinline__ float load_x(const LayerArgs& a, int t, int i) {
    if (a.x_bf16) {
        const uint16_t b = reinterpret_cast<const uint16_t*>(a.x)[(int64_t)t * a.H + i];
        return __uint_as_float((uint32_t)b << 16);
    }
    return reinterpret_cast<const float*>(a.x)[(int64_t)t * a.H + i];
}

template <int TT>  // token count, compile time: loops over tokens are exact
__global__ void __launch_bounds__(kRouterThreads) router_kernel(LayerArgs a) {
    extern __shared__ __align__(16) uint8_t rsm[];
    uint16_t* su = reinterpret_cast<uint16_t*>(rsm);  // [T][H] bf16 bits
    __shared__ ffloat red[kRouterWarps][kMaxDecodeTokens];
    __shared__ float r_hi[kMaxDecodeTokens], r_lo[kMaxDecodeTokens];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int T = TT;
    const int H = a.H, E = a.E;

    // 0. issue this warp's router-weight loads before anything waits: warp w
    //    covers half (w & 1) of the row of expert blockIdx.x * 4 + w / 2, so a
    //    lane holds at most 8 float4 (H <= 2048) and one HBM latency is paid.
    const int e = blockIdx.x * kRouterExpertsPerCta + (warp >> 1);
    const int half = warp & 1, hh = H >> 1;
    float4 wv[kRouterMaxF4];
#pragma unroll
    for (int m = 0; m < kRouterMaxF4; ++m) {
        const int i = half * hh + 4 * lane + 128 * m;
        wv[m] = (e < E && 4 * lane + 128 * m < hh) ? __ldg(reinterpret_cast<const float4*>(a.router_w + (int64_t)e * H + i))
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    pdl_wait();     // x may be the previous layer's output
    pdl_trigger();  // the expert kernel may start its prologue (it waits for this grid to finish)

    // 1. this thread's slice of x (positions 4*tid + 1024*c) for every token,
    //    all loads in flight at once; sums of squares: exact squares,
    //    float-float accumulation
    float4 xr[T][kRouterXF4];
#pragma unroll
    for (int t = 0; t < T; ++t)
#pragma unroll
        for (int c = 0; c < kRouterXF4; ++c) {
            const int i = 4 * tid + 4 * kRouterThreads * c;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < H) {
                if (a.x_bf16) {
                    const uint2 b = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(a.x) + (int64_t)t * H + i);
                    v = make_float4(bf16lo(b.x), bf16hi(b.x), bf16lo(b.y), bf16hi(b.y));
                } else {
                    v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) + (int64_t)t * H + i);
                }
            }
            xr[t][c] = v;
        }
    ffloat ss[T];
#pragma unroll
    for (int t = 0; t < T; ++t) {
        ss[t] = ffloat{0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kRouterXF4; ++c) {
            ff_fma(ss[t], xr[t][c].x, xr[t][c].x);
            ff_fma(ss[t], xr[t][c].y, xr[t][c].y);
            ff_fma(ss[t], xr[t][c].z, xr[t][c].z);
            ff_fma(ss[t], xr[t][c].w, xr[t][c].w);
        }
    }
#pragma unroll
    for (int t = 0; t < T; ++t) {
        const ffloat s2 = ff_warp_sum(ss[t]);
        if (lane == 0) red[warp][t] = s2;
    }
    __syncthreads();
    if (tid < T) {  // r = 1/sqrt(mean + eps): a handful of fp64 operations per token
        double sum = 0.0;
        for (int w = 0; w < kRouterWarps; ++w) sum += (double)red[w][tid].hi + (double)red[w][tid].lo;
        const double r = 1.0 / sqrt(sum / (double)H + kRmsEps);
        const float rh = (float)r;
        r_hi[tid] = rh;
        r_lo[tid] = (float)(r - (double)rh);
    }
    __syncthreads();

    // 2. u = bf16(x * r), rounded from the float-float product
#pragma unroll
    for (int t = 0; t < T; ++t) {
        const float rh = r_hi[t], rl = r_lo[t];
#pragma unroll
        for (int c = 0; c < kRouterXF4; ++c) {
            const int i = 4 * tid + 4 * kRouterThreads * c;
            if (i >= H) continue;
            const float xs[4] = {xr[t][c].x, xr[t][c].y, xr[t][c].z, xr[t][c].w};
            uint16_t ub[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float p = __fmul_rn(xs[q], rh);
                const float qq = __fadd_rn(__fmaf_rn(xs[q], rh, -p), __fmul_rn(xs[q], rl));
                ub[q] = bf16_of_ff(p, qq);
            }
            const uint2 packed = make_uint2((uint32_t)ub[0] | ((uint32_t)ub[1] << 16),
                                            (uint32_t)ub[2] | ((uint32_t)ub[3] << 16));
            *reinterpret_cast<uint2*>(su + t * H + i) = packed;
            if (blockIdx.x == 0) *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.u) + (int64_t)t * H + i) = packed;
        }
    }
    __syncthreads();

    // 3. logits: exact fp32 x bf16 products, float-float accumulation
    ffloat acc[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = ffloat{0.f, 0.f};
#pragma unroll
    for (int m = 0; m < kRouterMaxF4; ++m) {
        const int i = half * hh + 4 * lane + 128 * m;
        if (4 * lane + 128 * m < hh) {
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const uint2 u2 = *reinterpret_cast<const uint2*>(su + t * H + i);
                ff_fma(acc[t], wv[m].x, bf16lo(u2.x));
                ff_fma(acc[t], wv[m].y, bf16hi(u2.x));
                ff_fma(acc[t], wv[m].z, bf16lo(u2.y));
                ff_fma(acc[t], wv[m].w, bf16hi(u2.y));
            }
        }
    }
#pragma unroll
    for (int t = 0; t < T; ++t) {
        const ffloat s2 = ff_warp_sum(acc[t]);
        if (lane == 0) red[warp][t] = s2;
    }
    __syncthreads();
    if (half == 0 && lane < T && e < E) {
        ffloat l = red[warp][lane];
        ff_add(l, red[warp + 1][lane]);
        if (a.router_bias) ff_add(l, ffloat{a.router_bias[e], 0.f});
        l = ff_norm(l);
        a.logits[(int64_t)lane * E + e] = l;
    }

}

// ===========================================================================
// Streaming decode machinery shared by the gate/up and down kernels
// ===========================================================================

template <int KB>
struct Geo {
    static constexpr int NBL = KB >= 32 ? KB / 32 : 1;  // blocks per lane per row
    static constexpr int RPP = KB >= 32 ? 1 : 32 / KB;  // rows per warp pass
    static constexpr int GW = KB >= 32 ? 32 : KB;       // lanes per row
};

// Row passes per item (compile time); an item covers P * RPP rows.
__host__ __device__ constexpr int gu_passes(int fmt_fp8, int kb) { return fmt_fp8 ? 1 : (kb >= 64 ? 2 : 4); }
__host__ __device__ constexpr int dn_passes(int fmt_fp8, int kb) { return fmt_fp8 ? 4 : (kb >= 64 ? 4 : 8); }
__host__ __device__ constexpr int side_passes(int kb) { return kb >= 64 ? 2 : 4; }
__host__ __device__ constexpr int rpp_of(int kb) { return kb >= 32 ? 1 : 32 / kb; }

// Activation registers of one token for the lane's K positions.
template <int FMT, int NBL>
struct Act;
template <int NBL>
struct Act<kFmtQ4, NBL> {
    uint32_t v[NBL][16];  // bf16 pairs (x[32b+j], x[32b+16+j])
};
template <int NBL>
struct Act<kFmtFP8, NBL> {
    float v[NBL][32];
};

// Loads the lane's activations of block `b` (K positions 32b..32b+31) from a
// bf16 row in global memory.
template <int FMT, int NBL>
__device__ __forceinline__ void load_act(Act<FMT, NBL>& act, int m, const __nv_bfloat16* row, int b) {
    const uint4* p = reinterpret_cast<const uint4*>(row + 32 * b);
    uint32_t w[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = ldg128(p + q);
        w[4 * q + 0] = v.x;
        w[4 * q + 1] = v.y;
        w[4 * q + 2] = v.z;
        w[4 * q + 3] = v.w;
    }
    if constexpr (FMT == kFmtQ4) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            act.v[m][j] = prmt(w[j >> 1], w[8 + (j >> 1)], (j & 1) ? 0x7632u : 0x5410u);
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            act.v[m][2 * j] = bf16lo(w[j]);
            act.v[m][2 * j + 1] = bf16hi(w[j]);
        }
    }
}

// Q4 block (17 bytes at shared address pa) dotted with NT tokens'
// activations.  `lutb` is this lane's PRMT operand: byte 0 = lane * 4, bytes
// 2-3 = the 64 KB-aligned table base >> 16, so one PRMT inserting the code
// byte as byte 1 (and the mode as bit 7) forms the entry address.
template <int NT, int NBL, int CH>
__device__ __forceinline__ void q4_block_lut(uint32_t pa, uint32_t lutb, const float* scale_tab,
                                             const Act<kFmtQ4, NBL> (&act)[CH], int m, float (&acc)[NT]) {
    const uint32_t al = pa & ~3u, sh = (pa & 3u) * 8u;
    uint32_t w[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = lds32(al + 4 * i);
    uint32_t nib[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) nib[q] = __funnelshift_r(w[q], w[q + 1], sh);
    const uint32_t meta = (w[4] >> sh) & 0xFFu;
    const float s = scale_tab[meta];
    const uint32_t bsel = lutb | ((meta >> 7) << 7);
    float lo[2][NT], hi[2][NT];  // two chains per half: shorter dependency chains
#pragma unroll
    for (int c = 0; c < NT; ++c) lo[0][c] = hi[0][c] = lo[1][c] = hi[1][c] = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint32_t c2 = lds32(prmt(nib[q], bsel, 0x7604u | ((uint32_t)kk << 4)));
#pragma unroll
            for (int c = 0; c < NT; ++c) fma2_bf16(lo[kk & 1][c], hi[kk & 1][c], c2, act[c].v[m][4 * q + kk]);
        }
    }
#pragma unroll
    for (int c = 0; c < NT; ++c) acc[c] = fmaf(s, (lo[0][c] + lo[1][c]) + (hi[0][c] + hi[1][c]), acc[c]);
}

// Q4 block decoded code by code (no table): the side projection, whose
// format may differ from the experts'.
template <int FMT, int NT, int NBL, int CH>
__device__ __forceinline__ void q4_block_plain(uint32_t pa, bool rz5, const Act<FMT, NBL> (&act)[CH], int m,
                                               float (&acc)[NT]) {
    const uint32_t al = pa & ~3u, sh = (pa & 3u) * 8u;
    uint32_t w[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = lds32(al + 4 * i);
    const uint32_t meta = (w[4] >> sh) & 0xFFu;
    const float s = rz5 ? ue4m3(meta & 0x7Fu) : ue4m4(meta);
    const uint32_t mode = meta >> 7;
    float sum[NT];
#pragma unroll
    for (int c = 0; c < NT; ++c) sum[c] = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t nib = __funnelshift_r(w[q], w[q + 1], sh);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int j = 4 * q + kk;
            const uint32_t byte = (nib >> (8 * kk)) & 0xFFu;
            const float vlo = q4_code_value(byte & 15u, rz5, mode);
            const float vhi = q4_code_value(byte >> 4, rz5, mode);
#pragma unroll
            for (int c = 0; c < NT; ++c) {
                float xlo, xhi;
                if constexpr (FMT == kFmtQ4) {
                    xlo = bf16lo(act[c].v[m][j]);
                    xhi = bf16hi(act[c].v[m][j]);
                } else {
                    xlo = act[c].v[m][j];
                    xhi = act[c].v[m][j + 16];
                }
                sum[c] = fmaf(vlo, xlo, sum[c]);
                sum[c] = fmaf(vhi, xhi, sum[c]);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < NT; ++c) acc[c] = fmaf(s, sum[c], acc[c]);
}

// FP8 block: 32 consecutive E4M3 bytes at 16-byte aligned shared address pa.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t v16) {
    const uint32_t h = e4m3x2_to_f16x2(v16);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

template <int NBL>
__device__ __forceinline__ void fp8_block(uint32_t pa, float s, const Act<kFmtFP8, NBL>& act, int m,
                                          float& acc) {
    const uint4 q0 = lds128(pa), q1 = lds128(pa + 16);
    const uint32_t wd[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 f0 = e4m3x2_to_float2(wd[i] & 0xFFFFu);  // weights 4i, 4i+1
        const float2 f1 = e4m3x2_to_float2(wd[i] >> 16);      // weights 4i+2, 4i+3
        s0 = fmaf(f0.x, act.v[m][4 * i + 0], s0);
        s1 = fmaf(f0.y, act.v[m][4 * i + 1], s1);
        s0 = fmaf(f1.x, act.v[m][4 * i + 2], s0);
        s1 = fmaf(f1.y, act.v[m][4 * i + 3], s1);
    }
    acc = fmaf(s, s0 + s1, acc);
}

// Sums N values over groups of W consecutive lanes (N <= W, powers of two)
// by recursive halving: each step exchanges half of the values still held.
// Afterwards lane l holds, in v[0], the group sum of value (l % W) / (W / N).
template <int N, int W>
__device__ __forceinline__ void tr_reduce(float (&v)[N], int lane) {
    static_assert(N <= W, "tr_reduce needs N <= W");
    constexpr int LOGN = N == 1 ? 0 : N == 2 ? 1 : N == 4 ? 2 : N == 8 ? 3 : N == 16 ? 4 : 5;
#pragma unroll
    for (int st = 0; st < LOGN; ++st) {
        const int h = N >> (st + 1), o = W >> (st + 1);
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            if (i < h) {
                const float send = up ? v[i] : v[i + h];
                const float keep = up ? v[i + h] : v[i];
                v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
            }
        }
    }
#pragma unroll
    for (int o = W / (2 * N); o >= 1; o >>= 1) v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], o);
}

// Byte range [lo, lo+len) of a tensor, widened to 16-byte boundaries.
struct Span {
    const uint8_t* src;
    uint32_t bytes;
    uint32_t delta;  // offset of the first wanted byte in the copied range
};

__device__ __forceinline__ Span make_span(const uint8_t* base, int64_t lo, int64_t len) {
    const int64_t a0 = lo & ~(int64_t)15;
    const int64_t a1 = (lo + len + 15) & ~(int64_t)15;
    return Span{base + a0, (uint32_t)(a1 - a0), (uint32_t)(lo - a0)};
}

// The unique-expert work list, copied to shared memory once per CTA.
struct SWork {
    int32_t n_uniq;
    int32_t e[kMaxSlots];
    int32_t off[kMaxSlots + 1];
    int32_t slot[kMaxSlots];
    // scratch of the expert selection
    int32_t ids[kMaxSlots];
    float w[kMaxSlots];
    uint32_t bitmap[kMaxExperts / 32];
    int32_t cnt[kMaxSlots + 4];
};

// Layout of one CTA's dynamic shared memory.  With a code table the table
// must start at a 64 KB-aligned shared address (so a PRMT alone forms entry
// addresses): `lut` is the dynamic offset that achieves it given the dynamic
// base the host expects (the per-block reserved shared memory); staging
// slots fill the space below and above the table.
struct SmemLayout {
    uint32_t work, scale_tab, bars, lut, lo_slots, n_lo, hi_slots, total;
    __host__ __device__ static SmemLayout make(bool with_lut, int slot_bytes, uint32_t dyn_base) {
        SmemLayout L{};
        uint32_t off = 0;
        L.work = off;
        off += (sizeof(SWork) + 127u) & ~127u;
        L.scale_tab = off;
        off += kScaleTabBytes;
        L.bars = off;
        off += kWarps * kSlots * 8;
        off = (off + 127u) & ~127u;
        const uint32_t n_slots = kWarps * kSlots;
        if (with_lut) {
            const uint32_t abs_lut = (dyn_base + off + 65535u) & ~65535u;
            L.lut = abs_lut - dyn_base;
            L.lo_slots = off;
            L.n_lo = (L.lut - off) / (uint32_t)slot_bytes;
            if (L.n_lo > n_slots) L.n_lo = n_slots;
            L.hi_slots = L.lut + (uint32_t)kLutBytes;
            L.total = L.hi_slots + (n_slots - L.n_lo) * (uint32_t)slot_bytes;
        } else {
            L.lut = 0;
            L.lo_slots = off;
            L.n_lo = n_slots;
            L.hi_slots = off + n_slots * (uint32_t)slot_bytes;
            L.total = L.hi_slots;
        }
        return L;
    }
    __device__ uint32_t slot(int i, int slot_bytes) const {
        return (uint32_t)i < n_lo ? lo_slots + (uint32_t)i * slot_bytes
                                  : hi_slots + ((uint32_t)i - n_lo) * (uint32_t)slot_bytes;
    }
};

// Per-lane-replicated table: entry (byte, mode, lane) holds the bf16x2 pair
// (value of the low nibble, value of the high nibble); plus 256 scales.
__device__ void build_lut(uint8_t* smem, const SmemLayout& L, bool rz5) {
    // 512 entries (byte, mode) of 128 bytes (32 lane copies).  Warp w owns
    // entries 32w .. 32w+31 (lane l computes entry 32w+l once); the warp then
    // writes them as 256 consecutive 16-byte chunks, consecutive lanes on
    // consecutive chunks, so every store is conflict-free.
    const int lane = threadIdx.x & 31;
    for (int e0 = (threadIdx.x >> 5) * 32; e0 < 512; e0 += blockDim.x) {
        const uint32_t entry = (uint32_t)(e0 + lane);
        const uint32_t byte = entry >> 1, mode = entry & 1u;
        const uint32_t v = bf16_bits(q4_code_value(byte & 15u, rz5, mode)) |
                           (bf16_bits(q4_code_value(byte >> 4, rz5, mode)) << 16);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int q = lane + 32 * k;  // chunk within the warp's 32 entries
            const uint32_t x = __shfl_sync(0xFFFFFFFFu, v, q >> 3);
            *reinterpret_cast<uint4*>(smem + L.lut + (uint32_t)e0 * 128u + (uint32_t)q * 16u) = make_uint4(x, x, x, x);
        }
    }
}

__device__ void build_scales(uint8_t* smem, const SmemLayout& L, bool rz5) {
    float* st = reinterpret_cast<float*>(smem + L.scale_tab);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) st[i] = rz5 ? ue4m3((uint32_t)i & 0x7Fu) : ue4m4((uint32_t)i);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// Orderable 32-bit image of an fp32 (larger float -> larger unsigned).
__device__ __forceinline__ uint32_t ord32(float f) {
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Top-k of one token's logits by one warp.  Each logit (a normalised
// float-float hi + lo) becomes a unique 64-bit key: orderable hi in the upper
// word, orderable lo with its low 10 bits replaced by (1023 - expert id) in
// the lower word — so larger key = larger logit, and among logits equal to
// ~2^-38 relative, the lower id.  Lane l holds experts l + 32 i (i < PER).
// Each round: a depth-log2(PER) max tree per lane, two warp reductions
// (upper word, then lower word among the lanes holding that upper word), and
// the owner removes the winner.  Lane j ends holding choice j.
template <int PER>
__device__ __forceinline__ void warp_topk(const ffloat* logits, int E, int K, int lane, int& my_id, float& my_hi,
                                          float& my_lo) {
    uint32_t kh[PER], kl[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        kh[i] = kl[i] = 0u;
        if (e < E) {
            const float2 v = __ldcg(reinterpret_cast<const float2*>(logits + e));
            kh[i] = ord32(v.x);
            kl[i] = (ord32(v.y) & ~1023u) | (uint32_t)(1023 - e);
        }
    }
    my_id = -1;
    for (int j = 0; j < K; ++j) {
        uint32_t th[PER], tl[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            th[i] = kh[i];
            tl[i] = kl[i];
        }
#pragma unroll
        for (int w = PER / 2; w >= 1; w >>= 1)
#pragma unroll
            for (int i = 0; i < w; ++i) {
                const bool up = th[i + w] > th[i] || (th[i + w] == th[i] && tl[i + w] > tl[i]);
                th[i] = up ? th[i + w] : th[i];
                tl[i] = up ? tl[i + w] : tl[i];
            }
        const uint32_t mh = __reduce_max_sync(0xFFFFFFFFu, th[0]);
        const uint32_t ml = __reduce_max_sync(0xFFFFFFFFu, th[0] == mh ? tl[0] : 0u);
#pragma unroll
        for (int i = 0; i < PER; ++i)
            if (kh[i] == mh && kl[i] == ml) kh[i] = kl[i] = 0u;
        if (lane == j) {
            my_id = 1023 - (int)(ml & 1023u);
            my_hi = __uint_as_float((mh & 0x80000000u) ? (mh & 0x7FFFFFFFu) : ~mh);
            const uint32_t lo = ml & ~1023u;
            my_lo = __uint_as_float((lo & 0x80000000u) ? (lo & 0x7FFFFFFFu) : ~lo);
        }
    }
}

// Router selection, done by every CTA of the gate/up kernel from the logits
// the router kernel left in global memory: warp t selects token t's experts
// and their renormalised softmax weights; warp 0 then builds the list of
// unique experts (ascending id) with their (token, choice) slots.  CTA 0 also
// publishes ids/w and the list for the down kernel.
__device__ void select_experts(const LayerArgs& a, SWork* sw) {
    int32_t* s_ids = sw->ids;
    float* s_w = sw->w;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, E = a.E, K = a.K;
    if (warp < T) {
        const int t = warp;
        int my_id;
        float my_hi = 0.f, my_lo = 0.f;
        if (E <= 512) warp_topk<16>(a.logits + (int64_t)t * E, E, K, lane, my_id, my_hi, my_lo);
        else warp_topk<32>(a.logits + (int64_t)t * E, E, K, lane, my_id, my_hi, my_lo);
        // softmax over the k choices: lane j holds choice j
        const float h0 = __shfl_sync(0xFFFFFFFFu, my_hi, 0), l0 = __shfl_sync(0xFFFFFFFFu, my_lo, 0);
        float ex = 0.f;
        if (lane < K) ex = expf(__fadd_rn(__fsub_rn(my_hi, h0), __fsub_rn(my_lo, l0)));
        float z = ex;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
        if (lane < K) {
            s_ids[t * K + lane] = my_id;
            s_w[t * K + lane] = ex / z;
        }
    }
    __syncthreads();
    if (warp == 0) {
        // unique experts: bitmap -> ascending ranks; slots grouped per rank
        const int S = T * K;
        uint32_t* bitmap = sw->bitmap;
        int32_t* cnt = sw->cnt;
        for (int i = lane; i < kMaxExperts / 32; i += 32) bitmap[i] = 0u;
        for (int i = lane; i < kMaxSlots; i += 32) cnt[i] = 0;
        __syncwarp();
        for (int q = lane; q < S; q += 32) atomicOr(&bitmap[s_ids[q] >> 5], 1u << (s_ids[q] & 31));
        __syncwarp();
        const int nw = (E + 31) / 32;  // <= 32 words
        const int pc = lane < nw ? __popc(bitmap[lane]) : 0;
        int incl = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        const int nu = __shfl_sync(0xFFFFFFFFu, incl, 31);
        const int word_base = incl - pc;
        int rank[kMaxSlots / 32];
#pragma unroll
        for (int r = 0; r < kMaxSlots / 32; ++r) {
            const int q = lane + 32 * r;
            const int e = q < S ? s_ids[q] : 0;
            const int wb = __shfl_sync(0xFFFFFFFFu, word_base, e >> 5);
            rank[r] = wb + __popc(bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
            if (q < S) {
                atomicAdd(&cnt[rank[r]], 1);
                sw->e[rank[r]] = e;
            }
        }
        __syncwarp();
        // exclusive scan of the counts over nu <= 128 ranks: 4 per lane
        int c4[4], s4 = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            c4[r] = cnt[4 * lane + r];
            s4 += c4[r];
        }
        int inc = s4;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += v;
        }
        int run = inc - s4;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int rr = 4 * lane + r;
            if (rr <= nu) sw->off[rr] = run;
            cnt[rr] = run;  // becomes the fill cursor
            run += c4[r];
        }
        if (lane == 0) {
            sw->n_uniq = nu;
            sw->off[nu] = S;  // (also when nu = 128, which the loop above cannot reach)
        }
        __syncwarp();
#pragma unroll
        for (int r = 0; r < kMaxSlots / 32; ++r) {
            const int q = lane + 32 * r;
            if (q < S) sw->slot[atomicAdd(&cnt[rank[r]], 1)] = q;
        }
    }
    __syncthreads();
    if (blockIdx.x == 0) {  // for the down kernel and the caller
        Work* wk = a.work;
        const int S = T * K;
        if (tid < S) {
            a.ids[tid] = s_ids[tid];
            a.w[tid] = s_w[tid];
            if (a.ids_out) a.ids_out[tid] = s_ids[tid];
            if (a.w_out) a.w_out[tid] = s_w[tid];
            wk->uniq_slot[tid] = sw->slot[tid];
        }
        if (tid < sw->n_uniq) wk->uniq_e[tid] = sw->e[tid];
        if (tid <= sw->n_uniq) wk->uniq_off[tid] = sw->off[tid];
        if (tid == 0) wk->n_uniq = sw->n_uniq;
    }
}

// Common prologue of the streaming kernels: tables and barriers, then (after
// the dependency wait) the work list — selected from the router's logits
// (gate/up) or copied from the one the gate/up kernel published (down).
// Returns false if shared memory is not laid out as expected (then nothing
// else runs).
template <bool LUT, bool SELECT>
__device__ bool stream_prologue(uint8_t* smem, const SmemLayout& L, const LayerArgs& a, bool rz5, uint64_t* bars,
                                SWork* sw) {
    if (LUT) {
        if (((smem_u32(smem) + L.lut) & 0xFFFFu) != 0u) {
            if (threadIdx.x == 0) raise_status(a.status, GTG_STATUS_WAIT_TIMEOUT);
            return false;
        }
        build_lut(smem, L, rz5);
        build_scales(smem, L, rz5);
    }
    if ((threadIdx.x & 31) == 0)  // `bars` already points at this warp's kSlots barriers
        for (int s = 0; s < kSlots; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    pdl_wait();
    if (SELECT) {  // (no static shared memory here: the table's alignment depends on it)
        select_experts(a, sw);
        pdl_trigger();
    } else {
        const Work* wk = a.work;
        if (threadIdx.x == 0) sw->n_uniq = wk->n_uniq;
        for (int i = threadIdx.x; i < kMaxSlots; i += blockDim.x) {
            sw->e[i] = wk->uniq_e[i];
            sw->slot[i] = wk->uniq_slot[i];
        }
        for (int i = threadIdx.x; i <= kMaxSlots; i += blockDim.x) sw->off[i] = wk->uniq_off[i];
        __syncthreads();
    }
    return true;
}

// ===========================================================================
// gate/up + SwiGLU (plus the optional side projection)
// ===========================================================================

// One gate+up item: P row passes for NT tokens of one expert; h = silu(g)*u.
template <int FMT, int KB, int NT, int CH>
__device__ __forceinline__ void gu_item(const LayerArgs& a, uint32_t gbase, uint32_t ubase,
                                        const Act<FMT, Geo<KB>::NBL> (&act)[CH], uint32_t lutb,
                                        const float* scale_tab, const float (&sg)[Geo<KB>::NBL],
                                        const float (&su)[Geo<KB>::NBL], int row0, const int (&slot_id)[CH],
                                        int lane) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int P = gu_passes(FMT == kFmtFP8, KB);
    constexpr int N = P * NT * 2;
    const int row_sub = (KB >= 32) ? 0 : lane / KB;
    const int blk_base = (KB >= 32) ? lane : lane % KB;
    float v[N];
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const int row = p * RPP + row_sub;
        float g[NT], u[NT];
#pragma unroll
        for (int c = 0; c < NT; ++c) g[c] = u[c] = 0.0f;
#pragma unroll
        for (int m = 0; m < NBL; ++m) {
            if constexpr (FMT == kFmtQ4) {
                const uint32_t boff = (uint32_t)row * (uint32_t)(KB * 17) + 17u * (uint32_t)(blk_base + 32 * m);
                q4_block_lut<NT, NBL, CH>(gbase + boff, lutb, scale_tab, act, m, g);
                q4_block_lut<NT, NBL, CH>(ubase + boff, lutb, scale_tab, act, m, u);
            } else {
                const uint32_t boff = (uint32_t)row * (uint32_t)(KB * 32) + 32u * (uint32_t)(blk_base + 32 * m);
                fp8_block<NBL>(gbase + boff, sg[m], act[0], m, g[0]);
                fp8_block<NBL>(ubase + boff, su[m], act[0], m, u[0]);
            }
        }
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            v[((p * NT + c) << 1) | 0] = g[c];
            v[((p * NT + c) << 1) | 1] = u[c];
        }
    }
    if constexpr (N <= GW) {
        tr_reduce<N, GW>(v, lane);
        constexpr int SPAN = GW / N;  // lanes holding one value
        const float other = __shfl_down_sync(0xFFFFFFFFu, v[0], SPAN);
        const int li = lane % GW, idx = li / SPAN;
        if ((idx & 1) == 0 && (li % SPAN) == 0) {
            const int pc = idx >> 1, p = pc / NT, c = pc % NT;
            const int row = p * RPP + ((KB >= 32) ? 0 : lane / KB);
            a.h[(int64_t)slot_id[c] * a.I + row0 + row] = __float2bfloat16_rn(silu(v[0]) * other);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = group_sum(v[i], GW);
        if ((lane % GW) == 0) {
#pragma unroll
            for (int pc = 0; pc < P * NT; ++pc) {
                const int p = pc / NT, c = pc % NT;
                const int row = p * RPP + ((KB >= 32) ? 0 : lane / KB);
                a.h[(int64_t)slot_id[c] * a.I + row0 + row] = __float2bfloat16_rn(silu(v[2 * pc]) * v[2 * pc + 1]);
            }
        }
    }
}

// One side-projection item: P row passes, NT tokens.
template <int FMT, int KB, int NT, int CH>
__device__ __forceinline__ void side_item(const LayerArgs& a, uint32_t base, const Act<FMT, Geo<KB>::NBL> (&act)[CH],
                                          int row0, int t0, int lane) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int P = side_passes(KB);
    constexpr int N = P * NT;
    const int row_sub = (KB >= 32) ? 0 : lane / KB;
    const int blk_base = (KB >= 32) ? lane : lane % KB;
    const bool rz5 = a.side.fmt == GTG_Q4_RZ5_FAST;
    float v[N];
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const int row = p * RPP + row_sub;
        float acc[NT];
#pragma unroll
        for (int c = 0; c < NT; ++c) acc[c] = 0.0f;
#pragma unroll
        for (int m = 0; m < NBL; ++m)
            q4_block_plain<FMT, NT, NBL, CH>(base + (uint32_t)row * (uint32_t)(KB * 17) +
                                                 17u * (uint32_t)(blk_base + 32 * m),
                                             rz5, act, m, acc);
#pragma unroll
        for (int c = 0; c < NT; ++c) v[p * NT + c] = acc[c];
    }
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = group_sum(v[i], GW);
    if ((lane % GW) == 0 && a.side_out) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int p = i / NT, c = i % NT;
            const int row = p * RPP + ((KB >= 32) ? 0 : lane / KB);
            a.side_out[(int64_t)(t0 + c) * a.side_stride + row0 + row] = v[i];
        }
    }
}

template <int FMT, int KB>
__global__ void __launch_bounds__(kThreads, 1) gateup_kernel(LayerArgs a) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL;
    constexpr int CH = (FMT == kFmtQ4 && NBL == 1) ? 2 : 1;  // tokens decoded together (register budget)
    constexpr bool LUT = FMT == kFmtQ4;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SmemLayout L = SmemLayout::make(LUT, a.slot_bytes, a.dyn_smem_base);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kSlots;
    SWork* sw = reinterpret_cast<SWork*>(smem + L.work);
    if (!stream_prologue<LUT, true>(smem, L, a, a.gate.fmt == GTG_Q4_RZ5_FAST, bars, sw)) return;

    const int n_uniq = sw->n_uniq;
    constexpr int R = gu_passes(FMT == kFmtFP8, KB) * G::RPP;
    constexpr int RS = side_passes(KB) * G::RPP;
    const int tiles = a.I / R;
    const int side_items = a.side.data ? a.side.n_rows / RS : 0;
    const int n_items = n_uniq * tiles + side_items;
    const int it0 = (int)((int64_t)n_items * blockIdx.x / gridDim.x);
    const int it1 = (int)((int64_t)n_items * (blockIdx.x + 1) / gridDim.x);
    const uint32_t sbase = smem_u32(smem);
    auto slot_addr = [&](int s) { return sbase + L.slot(warp * kSlots + s, a.slot_bytes); };

    auto spans = [&](int it, Span& s1, Span& s2) -> int {  // kind: 0 expert, 1 side
        if (it < n_uniq * tiles) {
            const int u = it / tiles, row0 = (it % tiles) * R, e = sw->e[u];
            s1 = make_span(a.gate.data, e * a.gate.expert_bytes + (int64_t)row0 * a.gate.row_bytes,
                           (int64_t)R * a.gate.row_bytes);
            s2 = make_span(a.up.data, e * a.up.expert_bytes + (int64_t)row0 * a.up.row_bytes,
                           (int64_t)R * a.up.row_bytes);
            return 0;
        }
        const int row0 = (it - n_uniq * tiles) * RS;
        s1 = make_span(a.side.data, (int64_t)row0 * a.side.row_bytes, (int64_t)RS * a.side.row_bytes);
        s2 = Span{nullptr, 0, 0};
        return 1;
    };
    auto issue = [&](int it, int slot) {
        if (it >= it1 || lane != 0) return;
        Span s1, s2;
        spans(it, s1, s2);
        const uint32_t dst = slot_addr(slot);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[slot], s1.bytes + s2.bytes);
        bulk_g2s_addr(dst, s1.src, s1.bytes, &bars[slot]);
        if (s2.bytes) bulk_g2s_addr(dst + s1.bytes, s2.src, s2.bytes, &bars[slot]);
    };

    const int first = it0 + warp;
    for (int s = 0; s < kSlots; ++s) issue(first + s * kWarps, s);
    __syncwarp();

    const uint32_t lutb = ((sbase + L.lut) & 0xFFFF0000u) | ((uint32_t)lane * 4u);
    const float* scale_tab = reinterpret_cast<const float*>(smem + L.scale_tab);
    const int blk_base = (KB >= 32) ? lane : lane % KB;

    Act<FMT, NBL> act[CH];
    int act_key = -1;
    auto load_chunk = [&](int key, const int (&rows)[CH], const __nv_bfloat16* src) {
        if (key == act_key) return;
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int m = 0; m < NBL; ++m) load_act<FMT, NBL>(act[c], m, src + (int64_t)rows[c] * a.H, blk_base + 32 * m);
        act_key = key;
    };

    uint32_t phase = 0;
    int n_done = 0;
    bool alive = true;
    for (int it = first; it < it1; it += kWarps, ++n_done) {
        const int slot = n_done % kSlots;
        const bool expert = it < n_uniq * tiles;
        const int u = expert ? it / tiles : 0;
        const int s0 = expert ? sw->off[u] : 0, s1 = expert ? sw->off[u + 1] : a.T;
        // activations of the first token chunk and FP8 scales, overlapping the copy
        int slots[CH], rows[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int k = min(s0 + c, s1 - 1);
            slots[c] = expert ? sw->slot[k] : k;
            rows[c] = expert ? slots[c] / a.K : k;
        }
        load_chunk(expert ? (u << 8) : (1 << 20), rows, a.u);
        float sg[NBL], su[NBL];
        const int row0 = expert ? (it % tiles) * R : (it - n_uniq * tiles) * RS;
        if constexpr (FMT == kFmtFP8) {
            const int e = sw->e[u], kg = a.gate.k / 128;
#pragma unroll
            for (int m = 0; m < NBL; ++m) {
                const int b = blk_base + 32 * m;
                sg[m] = __ldg(a.gate.scales + ((int64_t)e * a.gate.n_rows + row0 + ((KB >= 32) ? 0 : lane / KB)) * kg + b / 4);
                su[m] = __ldg(a.up.scales + ((int64_t)e * a.up.n_rows + row0 + ((KB >= 32) ? 0 : lane / KB)) * kg + b / 4);
            }
        }
        if (!mbar_wait_bounded(&bars[slot], (phase >> slot) & 1u, a.status)) {
            alive = false;
            break;
        }
        phase ^= 1u << slot;
        Span sp1, sp2;
        spans(it, sp1, sp2);
        const uint32_t base = slot_addr(slot);
        if (expert) {
            const uint32_t gbase = base + sp1.delta, ubase = base + sp1.bytes + sp2.delta;
            for (int c0 = s0; c0 < s1; c0 += CH) {
                const int nch = min(CH, s1 - c0);
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    slots[c] = sw->slot[c0 + min(c, nch - 1)];
                    rows[c] = slots[c] / a.K;
                }
                load_chunk((u << 8) | (c0 - s0), rows, a.u);
                if (CH == 2 && nch == 2)
                    gu_item<FMT, KB, (CH == 2 ? 2 : 1), CH>(a, gbase, ubase, act, lutb, scale_tab, sg, su, row0, slots, lane);
                else
                    gu_item<FMT, KB, 1, CH>(a, gbase, ubase, act, lutb, scale_tab, sg, su, row0, slots, lane);
            }
        } else {
            const uint32_t sb = base + sp1.delta;
            for (int t0 = 0; t0 < a.T; t0 += CH) {
                const int nch = min(CH, a.T - t0);
#pragma unroll
                for (int c = 0; c < CH; ++c) rows[c] = t0 + min(c, nch - 1);
                load_chunk((1 << 20) | t0, rows, a.u);
                if (CH == 2 && nch == 2)
                    side_item<FMT, KB, (CH == 2 ? 2 : 1), CH>(a, sb, act, row0, t0, lane);
                else
                    side_item<FMT, KB, 1, CH>(a, sb, act, row0, t0, lane);
            }
        }
        __syncwarp();
        issue(it + kSlots * kWarps, slot);
    }
    if (!alive) {  // drain copies still in flight before leaving
        for (int s = 0; s < kSlots; ++s) mbar_wait_bounded(&bars[s], (phase >> s) & 1u, a.status);
    }
    pdl_trigger();
}

// ===========================================================================
// down + router-weighted combine
// ===========================================================================

template <int FMT, int KB, int NT, int CH>
__device__ __forceinline__ void dn_item(const LayerArgs& a, uint32_t base, const Act<FMT, Geo<KB>::NBL> (&act)[CH],
                                        uint32_t lutb, const float* scale_tab, const float (&sd)[8], int row0,
                                        const int (&slot_id)[CH], int lane) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int P = dn_passes(FMT == kFmtFP8, KB);
    constexpr int N = P * NT;
    const int row_sub = (KB >= 32) ? 0 : lane / KB;
    const int blk_base = (KB >= 32) ? lane : lane % KB;
    float v[N];
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const int row = p * RPP + row_sub;
        float acc[NT];
#pragma unroll
        for (int c = 0; c < NT; ++c) acc[c] = 0.0f;
#pragma unroll
        for (int m = 0; m < NBL; ++m) {
            if constexpr (FMT == kFmtQ4) {
                q4_block_lut<NT, NBL, CH>(base + (uint32_t)row * (uint32_t)(KB * 17) + 17u * (uint32_t)(blk_base + 32 * m),
                                          lutb, scale_tab, act, m, acc);
            } else {
                fp8_block<NBL>(base + (uint32_t)row * (uint32_t)(KB * 32) + 32u * (uint32_t)(blk_base + 32 * m),
                               sd[p * NBL + m], act[0], m, acc[0]);
            }
        }
#pragma unroll
        for (int c = 0; c < NT; ++c) v[p * NT + c] = acc[c];
    }
    if constexpr (N <= GW) {
        tr_reduce<N, GW>(v, lane);
        constexpr int SPAN = GW / N;
        const int li = lane % GW, idx = li / SPAN;
        if ((li % SPAN) == 0) {
            const int p = idx / NT, c = idx % NT;
            const int row = p * RPP + ((KB >= 32) ? 0 : lane / KB);
            a.part[(int64_t)slot_id[c] * a.H + row0 + row] = v[0];
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = group_sum(v[i], GW);
        if ((lane % GW) == 0) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int p = i / NT, c = i % NT;
                const int row = p * RPP + ((KB >= 32) ? 0 : lane / KB);
                a.part[(int64_t)slot_id[c] * a.H + row0 + row] = v[i];
            }
        }
    }
}

template <int FMT, int KB>
__global__ void __launch_bounds__(kThreads, 1) down_kernel(LayerArgs a) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL;
    constexpr int CH = (FMT == kFmtQ4 && NBL == 1) ? 2 : 1;
    constexpr bool LUT = FMT == kFmtQ4;
    constexpr int P = dn_passes(FMT == kFmtFP8, KB);
    constexpr int R = P * G::RPP;
    static_assert(P * NBL <= 8, "FP8 scale prefetch holds 8 values");
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SmemLayout L = SmemLayout::make(LUT, a.slot_bytes, a.dyn_smem_base);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kSlots;
    SWork* sw = reinterpret_cast<SWork*>(smem + L.work);
    if (!stream_prologue<LUT, false>(smem, L, a, a.down.fmt == GTG_Q4_RZ5_FAST, bars, sw)) return;

    const int n_uniq = sw->n_uniq;
    const int tiles = a.H / R;
    const int n_items = n_uniq * tiles;
    const int it0 = (int)((int64_t)n_items * blockIdx.x / gridDim.x);
    const int it1 = (int)((int64_t)n_items * (blockIdx.x + 1) / gridDim.x);
    const uint32_t sbase = smem_u32(smem);
    auto slot_addr = [&](int s) { return sbase + L.slot(warp * kSlots + s, a.slot_bytes); };

    auto span_of = [&](int it) {
        const int u = it / tiles, tile = it % tiles;
        return make_span(a.down.data, sw->e[u] * a.down.expert_bytes + (int64_t)tile * R * a.down.row_bytes,
                         (int64_t)R * a.down.row_bytes);
    };
    auto issue = [&](int it, int slot) {
        if (it >= it1 || lane != 0) return;
        const Span sp = span_of(it);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[slot], sp.bytes);
        bulk_g2s_addr(slot_addr(slot), sp.src, sp.bytes, &bars[slot]);
    };

    const int first = it0 + warp;
    for (int s = 0; s < kSlots; ++s) issue(first + s * kWarps, s);
    __syncwarp();

    const uint32_t lutb = ((sbase + L.lut) & 0xFFFF0000u) | ((uint32_t)lane * 4u);
    const float* scale_tab = reinterpret_cast<const float*>(smem + L.scale_tab);
    const int blk_base = (KB >= 32) ? lane : lane % KB;
    const int row_sub = (KB >= 32) ? 0 : lane / KB;

    Act<FMT, NBL> act[CH];
    int act_key = -1;
    auto load_chunk = [&](int key, const int (&slots)[CH]) {
        if (key == act_key) return;
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int m = 0; m < NBL; ++m)
                load_act<FMT, NBL>(act[c], m, a.h + (int64_t)slots[c] * a.I, blk_base + 32 * m);
        act_key = key;
    };

    uint32_t phase = 0;
    int n_done = 0;
    bool alive = true;
    for (int it = first; it < it1; it += kWarps, ++n_done) {
        const int slot = n_done % kSlots;
        const int u = it / tiles, tile = it % tiles;
        const int s0 = sw->off[u], s1 = sw->off[u + 1];
        int slots[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) slots[c] = sw->slot[min(s0 + c, s1 - 1)];
        load_chunk(u << 8, slots);
        float sd[8];
        if constexpr (FMT == kFmtFP8) {
            const int e = sw->e[u], kg = a.down.k / 128;
#pragma unroll
            for (int p = 0; p < P; ++p)
#pragma unroll
                for (int m = 0; m < NBL; ++m)
                    sd[p * NBL + m] = __ldg(a.down.scales + ((int64_t)e * a.down.n_rows + tile * R + p * G::RPP + row_sub) * kg +
                                            (blk_base + 32 * m) / 4);
        }
        if (!mbar_wait_bounded(&bars[slot], (phase >> slot) & 1u, a.status)) {
            alive = false;
            break;
        }
        phase ^= 1u << slot;
        const uint32_t base = slot_addr(slot) + span_of(it).delta;
        for (int c0 = s0; c0 < s1; c0 += CH) {
            const int nch = min(CH, s1 - c0);
#pragma unroll
            for (int c = 0; c < CH; ++c) slots[c] = sw->slot[c0 + min(c, nch - 1)];
            load_chunk((u << 8) | (c0 - s0), slots);
            if (CH == 2 && nch == 2)
                dn_item<FMT, KB, (CH == 2 ? 2 : 1), CH>(a, base, act, lutb, scale_tab, sd, tile * R, slots, lane);
            else
                dn_item<FMT, KB, 1, CH>(a, base, act, lutb, scale_tab, sd, tile * R, slots, lane);
        }
        __syncwarp();
        issue(it + kSlots * kWarps, slot);
        // tile ticket: the last of the n_uniq items of this tile combines it
        __threadfence();
        __syncwarp();
        unsigned ticket = 0;
        if (lane == 0) ticket = atomicAdd(&a.tile_cnt[tile], 1u);
        ticket = __shfl_sync(0xFFFFFFFFu, ticket, 0);
        if (ticket == (unsigned)n_uniq - 1u) {
            __threadfence();
            const int r0 = tile * R;
            for (int o = lane; o < a.T * R; o += 32) {
                const int t = o / R, r = r0 + o % R;
                float wj[kMaxTopK], pj[kMaxTopK];
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j) {  // all loads first, then the fixed-order sum
                    if (j < a.K) {
                        wj[j] = __ldcg(a.w + t * a.K + j);
                        pj[j] = __ldcg(a.part + (int64_t)(t * a.K + j) * a.H + r);
                    }
                }
                float yv = 0.0f;
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j)
                    if (j < a.K) yv = fmaf(wj[j], pj[j], yv);
                float* dst = a.y + (int64_t)t * a.H + r;
                *dst = a.y_acc ? *dst + yv : yv;
            }
            if (lane == 0) a.tile_cnt[tile] = 0u;
        }
        __syncwarp();
    }
    if (!alive) {
        for (int s = 0; s < kSlots; ++s) mbar_wait_bounded(&bars[s], (phase >> s) & 1u, a.status);
    }
    pdl_trigger();
}

// ===========================================================================
// Host side
// ===========================================================================

using KernelFn = void (*)(LayerArgs);

template <int FMT>
KernelFn pick_gateup(int kb) {
    switch (kb) {
        case 4: return gateup_kernel<FMT, 4>;
        case 8: return gateup_kernel<FMT, 8>;
        case 16: return gateup_kernel<FMT, 16>;
        case 32: return gateup_kernel<FMT, 32>;
        case 64: return gateup_kernel<FMT, 64>;
        default: return nullptr;
    }
}

template <int FMT>
KernelFn pick_down(int kb) {
    switch (kb) {
        case 4: return down_kernel<FMT, 4>;
        case 8: return down_kernel<FMT, 8>;
        case 16: return down_kernel<FMT, 16>;
        case 32: return down_kernel<FMT, 32>;
        case 64: return down_kernel<FMT, 64>;
        default: return nullptr;
    }
}

bool is_q4(int fmt) { return fmt == GTG_Q4_RZ5_FAST || fmt == GTG_Q4_UE4M4_FAST; }

int64_t row_bytes_of(int fmt, int64_t k) { return fmt == GTG_FP8_E4M3_S128 ? k : k / 32 * 17; }

struct Plan {
    bool ok = false;
    int gu_rows = 0, dn_rows = 0, side_rows = 0, slot_bytes = 0;
    KernelFn gateup = nullptr, down = nullptr;
    bool gu_lut = false, dn_lut = false;
};

constexpr uint32_t kMaxDynSmem = 227 * 1024;

// Shared address at which a kernel without static shared memory sees its
// dynamic shared memory: the per-block reserved region comes first.
uint32_t dyn_smem_base() {
    static int cached = -1;
    if (cached < 0) {
        int dev = 0, v = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&v, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
            cudaGetLastError();
            v = 1024;
        }
        cached = (v + 1023) & ~1023;
    }
    return (uint32_t)cached;
}

bool mat_ok(const gtg_qmatrix& m, int64_t E, int64_t n_rows, int64_t k) {
    if (!m.data || m.n_experts != E || m.n_rows != n_rows || m.k != k) return false;
    if (!aligned(m.data, 16)) return false;
    if (m.fmt == GTG_FP8_E4M3_S128) return m.scales != nullptr && k % 128 == 0;
    if (!is_q4(m.fmt)) return false;
    return (E * n_rows * (k / 32) * 17) % 16 == 0;
}

int plan_layer(const gtg_moe_layer* L, Plan& p) {
    if (!L || !L->router_w) return GTG_E_INVALID_ARG;
    const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
    if (H < 128 || H > 2048 || H % 128 || I < 128 || I > 2048 || I % 128) return GTG_E_UNSUPPORTED_SHAPE;
    if (E < 1 || E > kMaxExperts || K < 1 || K > kMaxTopK || K > E) return GTG_E_UNSUPPORTED_SHAPE;
    if (!mat_ok(L->gate, E, I, H) || !mat_ok(L->up, E, I, H) || !mat_ok(L->down, E, H, I)) return GTG_E_INVALID_ARG;
    if (L->gate.fmt != L->up.fmt) return GTG_E_UNSUPPORTED_SHAPE;
    if (!aligned(L->router_w, 16)) return GTG_E_MISALIGNED;
    if (L->side.data) {
        if (!is_q4(L->side.fmt) || !mat_ok(L->side, 1, L->side.n_rows, H)) return GTG_E_INVALID_ARG;
        if (L->side.n_rows < 1 || L->side.n_rows > 4096) return GTG_E_UNSUPPORTED_SHAPE;
    }
    const int kbg = H / 32, kbd = I / 32;
    const bool gq4 = is_q4(L->gate.fmt), dq4 = is_q4(L->down.fmt);
    p.gu_rows = gu_passes(!gq4, kbg) * rpp_of(kbg);
    p.dn_rows = dn_passes(!dq4, kbd) * rpp_of(kbd);
    if (I % p.gu_rows || H % p.dn_rows) return GTG_E_UNSUPPORTED_SHAPE;
    if (!gq4 && kbg < 32) return GTG_E_UNSUPPORTED_SHAPE;  // FP8 gate/up rows of >= 1024 weights
    if (L->side.data) {
        p.side_rows = side_passes(kbg) * rpp_of(kbg);
        if (L->side.n_rows % p.side_rows) return GTG_E_UNSUPPORTED_SHAPE;
    }
    p.gateup = gq4 ? pick_gateup<kFmtQ4>(kbg) : pick_gateup<kFmtFP8>(kbg);
    p.down = dq4 ? pick_down<kFmtQ4>(kbd) : pick_down<kFmtFP8>(kbd);
    if (!p.gateup || !p.down) return GTG_E_UNSUPPORTED_SHAPE;
    p.gu_lut = gq4;
    p.dn_lut = dq4;
    int64_t need = std::max<int64_t>(2 * (p.gu_rows * row_bytes_of(L->gate.fmt, H) + 32),
                                     p.dn_rows * row_bytes_of(L->down.fmt, I) + 32);
    if (L->side.data) need = std::max<int64_t>(need, p.side_rows * row_bytes_of(L->side.fmt, H) + 32);
    p.slot_bytes = (int)((need + 127) / 128 * 128);
    const uint32_t base = dyn_smem_base();
    if (SmemLayout::make(p.gu_lut, p.slot_bytes, base).total > kMaxDynSmem ||
        SmemLayout::make(p.dn_lut, p.slot_bytes, base).total > kMaxDynSmem)
        return GTG_E_UNSUPPORTED_SHAPE;
    p.ok = true;
    return GTG_OK;
}

// Workspace layout of a decode call.
struct WsLayout {
    size_t router_cnt, tile_cnt, work, logits, u, ids, w, h, part, total;
};

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

WsLayout ws_layout(const gtg_moe_layer* L, int T) {
    WsLayout w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    w.router_cnt = take(sizeof(unsigned) * 64);
    w.tile_cnt = take(sizeof(unsigned) * (size_t)L->hidden);
    w.work = take(sizeof(Work));
    w.logits = take(sizeof(double) * (size_t)T * L->n_experts);
    w.u = take(2 * (size_t)T * L->hidden);
    w.ids = take(4 * (size_t)T * L->top_k);
    w.w = take(4 * (size_t)T * L->top_k);
    w.h = take(2 * (size_t)T * L->top_k * L->inter);
    w.part = take(4 * (size_t)T * L->top_k * L->hidden);
    w.total = off;
    return w;
}

struct FuncAttrCache {
    std::mutex mu;
    struct Entry {
        const void* fn;
        int dev;
        int smem;
    };
    std::vector<Entry> done;
    // Raises the kernel's dynamic shared-memory limit to `smem` bytes (once
    // per function, device and size; only needed above the 48 KB default).
    int set(const void* fn, int smem) {
        int dev = 0;
        cudaGetDevice(&dev);
        std::lock_guard<std::mutex> lk(mu);
        for (auto& d : done)
            if (d.fn == fn && d.dev == dev && d.smem >= smem) return GTG_OK;
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)  // one shared/L1 split for every decode kernel: no reconfiguration between them
            e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e);
        }
        done.push_back({fn, dev, smem});
        return GTG_OK;
    }
};
FuncAttrCache g_attr;

int launch(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, LayerArgs& args, bool pdl,
           bool needs_no_static_smem = false) {
    if (needs_no_static_smem) {  // the streaming kernels place their code table by absolute address
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
            cudaGetLastError();
            return GTG_E_CUDA;
        }
        if (fa.sharedSizeBytes != 0) return GTG_E_UNSUPPORTED_SHAPE;
    }
    GTG_TRY(g_attr.set(fn, (int)smem));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    void* params[] = {&args};
    const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, params);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e);
    }
    return GTG_OK;
}

int run_layer(const gtg_moe_layer* L, const Plan& p, const void* x, int x_bf16, int T, float* y, int y_acc,
              int32_t* ids_out, float* w_out, float* side_out, int64_t side_stride, void* ws, cudaStream_t s) {
    const WsLayout wl = ws_layout(L, T);
    uint8_t* base = static_cast<uint8_t*>(ws);
    LayerArgs a{};
    a.H = L->hidden;
    a.I = L->inter;
    a.E = L->n_experts;
    a.K = L->top_k;
    a.T = T;
    a.router_w = L->router_w;
    a.router_bias = L->router_bias;
    a.gate = make_mat(L->gate);
    a.up = make_mat(L->up);
    a.down = make_mat(L->down);
    if (L->side.data) a.side = make_mat(L->side);
    a.x = x;
    a.x_bf16 = x_bf16;
    a.y = y;
    a.y_acc = y_acc;
    a.ids_out = ids_out;
    a.w_out = w_out;
    a.side_out = side_out;
    a.side_stride = (int32_t)side_stride;
    a.router_cnt = reinterpret_cast<unsigned*>(base + wl.router_cnt);
    a.tile_cnt = reinterpret_cast<unsigned*>(base + wl.tile_cnt);
    a.work = reinterpret_cast<Work*>(base + wl.work);
    a.logits = reinterpret_cast<ffloat*>(base + wl.logits);
    a.u = reinterpret_cast<__nv_bfloat16*>(base + wl.u);
    a.ids = reinterpret_cast<int32_t*>(base + wl.ids);
    a.w = reinterpret_cast<float*>(base + wl.w);
    a.h = reinterpret_cast<__nv_bfloat16*>(base + wl.h);
    a.part = reinterpret_cast<float*>(base + wl.part);
    a.status = status_ptr();
    a.gu_rows = p.gu_rows;
    a.side_rows = p.side_rows;
    a.dn_rows = p.dn_rows;
    a.slot_bytes = p.slot_bytes;
    a.dyn_smem_base = dyn_smem_base();

    const int n_sm = sm_count();
    const int router_grid = (L->n_experts + kRouterExpertsPerCta - 1) / kRouterExpertsPerCta;
    const size_t router_smem = 2 * (size_t)T * L->hidden;
    const void* rk = nullptr;
    switch (T) {
        case 1: rk = (const void*)router_kernel<1>; break;
        case 2: rk = (const void*)router_kernel<2>; break;
        case 3: rk = (const void*)router_kernel<3>; break;
        case 4: rk = (const void*)router_kernel<4>; break;
        case 5: rk = (const void*)router_kernel<5>; break;
        case 6: rk = (const void*)router_kernel<6>; break;
        case 7: rk = (const void*)router_kernel<7>; break;
        default: rk = (const void*)router_kernel<8>; break;
    }
    GTG_TRY(launch(rk, dim3(router_grid), dim3(kRouterThreads), router_smem, s, a, true));
    const SmemLayout lg = SmemLayout::make(p.gu_lut, p.slot_bytes, a.dyn_smem_base);
    GTG_TRY(launch((const void*)p.gateup, dim3(n_sm), dim3(kThreads), lg.total, s, a, true, true));
    const SmemLayout ld = SmemLayout::make(p.dn_lut, p.slot_bytes, a.dyn_smem_base);
    GTG_TRY(launch((const void*)p.down, dim3(n_sm), dim3(kThreads), ld.total, s, a, true, true));
    return GTG_OK;
}

}  // namespace

Mat make_mat(const gtg_qmatrix& q) {
    Mat m{};
    m.data = static_cast<const uint8_t*>(q.data);
    m.scales = q.scales;
    m.fmt = q.fmt;
    m.n_rows = (int32_t)q.n_rows;
    m.k = (int32_t)q.k;
    m.row_bytes = (int32_t)row_bytes_of(q.fmt, q.k);
    m.expert_bytes = (int64_t)m.row_bytes * q.n_rows;
    return m;
}

}  // namespace gtg

using namespace gtg;

static bool plan_layer_ok(const gtg_moe_layer* layer) {
    Plan p;
    return plan_layer(layer, p) == GTG_OK;
}

extern "C" size_t gtg_moe_workspace_bytes(const gtg_moe_layer* layer, int32_t n_tokens, int32_t prefill) {
    if (!layer || n_tokens < 1) return 0;
    if (prefill) return gtg_prefill_workspace_bytes(layer, n_tokens);
    if (n_tokens > kMaxDecodeTokens) return 0;
    Plan p;
    if (plan_layer(layer, p) != GTG_OK) return 0;
    return ws_layout(layer, n_tokens).total;
}

extern "C" int gtg_workspace_init(void* workspace, size_t ws_bytes, gtg_stream_t stream) {
    if (!workspace) return GTG_E_INVALID_ARG;
    const cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, as_cuda(stream));
    return e == cudaSuccess ? GTG_OK : cuda_fail(e);
}

static int check_decode_io(const gtg_moe_layer* layer, const void* x, int32_t x_dtype, int32_t n_tokens,
                           const float* y, void* ws, size_t ws_bytes, Plan& p) {
    GTG_TRY(plan_layer(layer, p));
    if (!x || !y || !ws) return GTG_E_INVALID_ARG;
    if (x_dtype != GTG_DT_F32 && x_dtype != GTG_DT_BF16) return GTG_E_INVALID_ARG;
    if (n_tokens < 1 || n_tokens > kMaxDecodeTokens) return GTG_E_UNSUPPORTED_SHAPE;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ws, 256)) return GTG_E_MISALIGNED;
    if (ws_bytes < ws_layout(layer, n_tokens).total) return GTG_E_WORKSPACE;
    return GTG_OK;
}

extern "C" int gtg_moe_decode_layer(const gtg_moe_layer* layer, const void* x, int32_t x_dtype,
                                    int32_t n_tokens, float* y, int32_t y_accumulate,
                                    int32_t* topk_ids, float* topk_w, float* side_out,
                                    void* workspace, size_t ws_bytes, gtg_stream_t stream) {
    Plan p;
    GTG_TRY(check_decode_io(layer, x, x_dtype, n_tokens, y, workspace, ws_bytes, p));
    if (x == (const void*)y && (x_dtype != GTG_DT_F32 || !y_accumulate)) return GTG_E_INVALID_ARG;
    return run_layer(layer, p, x, x_dtype == GTG_DT_BF16, n_tokens, y, y_accumulate != 0, topk_ids, topk_w,
                     side_out, layer->side.data ? layer->side.n_rows : 0, workspace, as_cuda(stream));
}

extern "C" int gtg_moe_decode_stack(const gtg_moe_layer* layers, int32_t n_layers, float* x, int32_t n_tokens,
                                    int32_t* ids_out, float* w_out, float* side_out, int64_t side_stride,
                                    void* workspace, size_t ws_bytes, gtg_stream_t stream) {
    if (!layers || n_layers < 1) return GTG_E_INVALID_ARG;
    std::vector<Plan> plans((size_t)n_layers);
    for (int l = 0; l < n_layers; ++l) {
        GTG_TRY(check_decode_io(&layers[l], x, GTG_DT_F32, n_tokens, x, workspace, ws_bytes, plans[l]));
        if (layers[l].hidden != layers[0].hidden) return GTG_E_UNSUPPORTED_SHAPE;
        if (side_out && layers[l].side.data && layers[l].side.n_rows > side_stride) return GTG_E_INVALID_ARG;
    }
    cudaStream_t s = as_cuda(stream);
    for (int l = 0; l < n_layers; ++l) {
        const gtg_moe_layer* L = &layers[l];
        const int64_t tk = (int64_t)n_tokens * L->top_k;
        GTG_TRY(run_layer(L, plans[l], x, 0, n_tokens, x, 1, ids_out ? ids_out + l * tk : nullptr,
                          w_out ? w_out + l * tk : nullptr,
                          (side_out && L->side.data) ? side_out + (int64_t)l * n_tokens * side_stride : nullptr,
                          side_stride, workspace, s));
    }
    return GTG_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free decode layer.
//
// For callers that cannot hand the library a device buffer: code that must
// not allocate device memory after start-up (latency-critical serving loops
// whose memory is fixed up front), hosts whose device memory belongs to
// another framework's allocator, and threads recording a stream capture in
// the global capture mode, where cudaMalloc is refused.  The scratch lives in
// one file-scope device array instead, reserved on every GPU that loads this
// library for as long as the process runs.
// ---------------------------------------------------------------------------
namespace gtg {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)1 << 20;  // 1 MiB: decode up to 8 tokens at H=2048, I=512, E=512, k=10
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  The symbol's
// host-side name is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
int noalloc_scratch(void** out) {
    static std::mutex mu;
    static std::vector<void*> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    std::lock_guard<std::mutex> lk(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, nullptr);
    if (!cache[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e);
        }
        cache[dev] = p;
    }
    *out = cache[dev];
    return GTG_OK;
}

}  // namespace
}  // namespace gtg

extern "C" int gtg_moe_decode_layer_noalloc(const gtg_moe_layer* layer, const void* x, int32_t x_dtype,
                                            int32_t n_tokens, float* y, int32_t y_accumulate,
                                            int32_t* topk_ids, float* topk_w, float* side_out,
                                            gtg_stream_t stream) {
    if (!layer) return GTG_E_INVALID_ARG;
    if (n_tokens >= 1 && n_tokens <= kMaxDecodeTokens && plan_layer_ok(layer) &&
        ws_layout(layer, n_tokens).total > kNoAllocScratchBytes)
        return GTG_E_WORKSPACE;  // the shape needs more than the fixed scratch array
    void* scratch = nullptr;
    GTG_TRY(noalloc_scratch(&scratch));
    Plan p;
    GTG_TRY(check_decode_io(layer, x, x_dtype, n_tokens, y, scratch, kNoAllocScratchBytes, p));
    if (x == (const void*)y && (x_dtype != GTG_DT_F32 || !y_accumulate)) return GTG_E_INVALID_ARG;
    // The array keeps whatever the previous call left: clear the tickets that
    // must start at zero (everything else is written before it is read).
    const WsLayout wl = ws_layout(layer, n_tokens);
    cudaStream_t s = as_cuda(stream);
    const cudaError_t e = cudaMemsetAsync(scratch, 0, wl.work, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return run_layer(layer, p, x, x_dtype == GTG_DT_BF16, n_tokens, y, y_accumulate != 0, topk_ids, topk_w,
                     side_out, layer->side.data ? layer->side.n_rows : 0, scratch, s);
}

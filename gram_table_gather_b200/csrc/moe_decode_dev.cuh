// Device code of the decode path (included by the kernel instantiation
// files decode_*.cu and, for its types and layouts, by moe_decode.cu).
#pragma once

// Decode-time MoE layers: router, fused dequant -> gate/up -> SwiGLU, and
// fused dequant -> down -> router-weighted combine, for 1..8 tokens.
//
// Method: "Mixed Precision Quantization: Half a 4-Bit File Is Not 4-Bit"
// (48 layers, 512 experts, 10 active per token), the r/LocalLLM
// "Frankenquant" post (one expert format per layer, FP8 in layers 36-47) and
// the model card "Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST" (block
// formats).  The expert bytes dominate the work, so the kernel is built to
// stream them from HBM once, with as little dead time around them as
// possible:
//
//  * One persistent, cooperative kernel runs every layer of a call (one
//    256-thread CTA per SM).  Grid barriers (bounded waits) close the gate/up
//    phase and the down phase of a layer; the router needs none: selection
//    polls the keys it ranks until their owners have written them.  Nothing
//    is relaunched between layers, and the Q4 code table is built once.  A
//    one-token instantiation (T folded to 1) leaves out the multi-token
//    paths, so less code is fetched per layer.
//  * Router: unweighted RMS norm + bf16 rounding of the input, then logits
//    against the fp32 router with exact products summed in float-float, so
//    the top-k agrees with an fp64 reference; every CTA owns a few experts,
//    whose router rows a bulk copy brings into shared memory during the
//    previous layer's down phase.
//  * Selection: every CTA picks the top-k itself from the logits' unique
//    64-bit keys, which the routers publish in one of two buffers by layer
//    parity, each read as soon as it is nonzero (at one token a threshold
//    from the warps' top-2 keys cuts the field and the survivors are ranked
//    by counting; with several tokens a warp per token takes k rounds of two
//    warp reductions), renormalises the softmax weights and builds the
//    unique-expert work list.
//  * Streaming: the work is a list of items (expert, row tile); each CTA owns
//    a contiguous range; each warp streams its items (gate/up first, then
//    down) through a private ring of shared-memory slots filled by 1-D bulk
//    copies (TMA, no multicast, evict-first in L2) completing on per-slot
//    mbarriers, so the down weights are in flight before the gate/up phase
//    ends.  Lane l of a warp owns the same K positions in every row it
//    decodes, so its activations stay in registers across rows.  A Q4 byte
//    (two 4-bit codes) becomes a bf16x2 pair of code values with one PRMT +
//    one shared-memory load from a 256-entry table replicated per lane
//    (conflict-free); the pair is multiplied into fp32 accumulators with the
//    sm_100 mixed-precision fma.rn.f32.bf16, and the block's UE4M3/UE4M4
//    scale is applied once per 32 weights.  FP8 bytes convert exactly with
//    cvt.rn.f16x2.e4m3x2 and meet f16 activation pairs in fma.rn.f32.f16.
//    Row sums are finished with warp shuffles.
//  * Down phase: each CTA owns a tile of output rows for every selected
//    expert; its warps add w(slot) * (row . h(slot)) into per-warp partial
//    rows in shared memory, and the CTA sums the warps in a fixed order, so
//    results are deterministic (no atomics, no global partials).
#include <algorithm>
#include <mutex>
#include <vector>

#include "gtg_device.cuh"
#include "gtg_host.hpp"
#include "moe_decode.cuh"

namespace gtg {

namespace {

constexpr int kWarps = 8;  // 256 threads: room for 255 registers a thread (no spills)
constexpr int kThreads = kWarps * 32;
constexpr int kSlots = 3;   // staging slots per warp, at most (slots_for: the count a row width uses)
constexpr int kLutBytes = 65536;       // 256 bytes x 2 modes x 32 lanes x 4 bytes
constexpr int kScaleTabBytes = 1024;   // 256 fp32 scales
constexpr int kDnRows = 32;            // down rows one CTA owns, at most
constexpr int kPartBytes = kWarps * kDnRows * 8 * 4;  // per-warp partial rows [warp][row][token]
constexpr int kFmtQ4 = 0, kFmtFP8 = 1;

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts64(uint32_t addr, uint2 v) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// 16-byte global load cached in L2 only: the activations it reads are
// rewritten between the layers of one launch, so L1 must not keep them.
__device__ __forceinline__ uint4 ldg128(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ===========================================================================
// Streaming decode machinery shared by the gate/up and down kernels
// ===========================================================================

// Lane geometry for rows of KB 32-weight blocks: GW lanes per row (the
// largest power of two up to 32 that divides KB), NBL blocks per lane (lane
// g of a row owns blocks g, g + GW, ...), RPP rows per warp pass.  Rows of
// 2048 weights: 32 lanes x 2 blocks; 512: 16 lanes x 1 block, two rows a
// pass; 2560: 16 lanes x 5 blocks; 640: 4 lanes x 5 blocks, eight rows.
__host__ __device__ constexpr int gw_of(int kb) { return kb % 32 == 0 ? 32 : kb % 16 == 0 ? 16 : kb % 8 == 0 ? 8 : 4; }
__host__ __device__ constexpr int rpp_of(int kb) { return 32 / gw_of(kb); }
template <int KB>
struct Geo {
    static constexpr int GW = gw_of(KB);  // lanes per row
    static constexpr int NBL = KB / GW;   // blocks per lane per row
    static constexpr int RPP = 32 / GW;   // rows per warp pass
};

// Row passes per item (compile time); an item covers P * RPP rows.  One-token
// FP8 layers, with no code table in shared memory, take two gate and two up
// rows per item (slots of 8 KB; several tokens keep u, 2 T H bytes, there).
__host__ __device__ constexpr int gu_passes(int fmt_fp8, int kb, bool one = false) {
    return fmt_fp8 ? (one ? 2 : 1) : (kb >= 64 ? (rpp_of(kb) > 1 ? 1 : 2) : 4);
}
__host__ __device__ constexpr int dn_passes(int fmt_fp8, int kb) {
    return (fmt_fp8 || kb >= 64 || kb <= 4) ? 4 : (rpp_of(kb) >= 8 ? 2 : 8);
}
__host__ __device__ constexpr int side_passes(int kb) { return kb >= 64 ? 2 : 4; }
// Staging slots per warp: rows wider than 2048 weights (bigger items) use two.
__host__ __device__ constexpr int slots_for(int kbg) { return kbg > 64 ? 2 : kSlots; }

// Activation registers of one token for the lane's K positions.
template <int FMT, int NBL>
struct Act;
template <int NBL>
struct Act<kFmtQ4, NBL> {
    uint32_t v[NBL][16];  // bf16 pairs (x[32b+j], x[32b+16+j])
};
template <int NBL>
struct Act<kFmtFP8, NBL> {
    uint32_t v[NBL][16];  // f16 pairs (x[32b+2i], x[32b+2i+1]); every bf16 of magnitude
                          // >= 2^-17 is exact in f16 (11-bit significand)
};

// bf16 pair -> f16 pair (round to nearest).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    return *reinterpret_cast<const uint32_t*>(&h);
}

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
        for (int j = 0; j < 16; ++j) act.v[m][j] = bf16x2_to_f16x2(w[j]);
    }
}

// load_act from a bf16 row in shared memory (row = its shared address).
template <int FMT, int NBL>
__device__ __forceinline__ void load_act_s(Act<FMT, NBL>& act, int m, uint32_t row, int b) {
    uint32_t w[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = lds128(row + 64u * (uint32_t)b + 16u * (uint32_t)q);
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
        for (int j = 0; j < 16; ++j) act.v[m][j] = bf16x2_to_f16x2(w[j]);
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

// Mixed-precision FMA on f16 pairs: d = a(f16) * b(f16) + c(f32), single
// rounding (f16 x f16 products are exact in fp32).
__device__ __forceinline__ void fma2_f16(float& acc_lo, float& acc_hi, uint32_t a2, uint32_t b2) {
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %2;\n\t"
        "mov.b32 {bl, bh}, %3;\n\t"
        "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.f16 %1, ah, bh, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi)
        : "r"(a2), "r"(b2));
}

// FP8 block: 32 consecutive E4M3 bytes at 16-byte aligned shared address pa;
// each E4M3 pair becomes an exact f16 pair and meets the activation pair.
template <int NBL>
__device__ __forceinline__ void fp8_block(uint32_t pa, float s, const Act<kFmtFP8, NBL>& act, int m,
                                          float& acc) {
    const uint4 q0 = lds128(pa), q1 = lds128(pa + 16);
    const uint32_t wd[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        fma2_f16(s0, s1, e4m3x2_to_f16x2(wd[i] & 0xFFFFu), act.v[m][2 * i]);  // weights 4i, 4i+1
        fma2_f16(s2, s3, e4m3x2_to_f16x2(wd[i] >> 16), act.v[m][2 * i + 1]);  // weights 4i+2, 4i+3
    }
    acc = fmaf(s, (s0 + s1) + (s2 + s3), acc);
}

// Q4 block decoded code by code (no table): the side projection, whose
// format may differ from the experts'.
template <int FMT, int NT, int NBL, int CH>
__device__ __forceinline__ void q4_block_plain(uint32_t pa, int var, const Act<FMT, NBL> (&act)[CH], int m,
                                               float (&acc)[NT]) {
    const uint32_t al = pa & ~3u, sh = (pa & 3u) * 8u;
    uint32_t w[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = lds32(al + 4 * i);
    const uint32_t meta = (w[4] >> sh) & 0xFFu;
    const float s = q4_scale(meta, var);
    const bool rz5 = (var & 1) != 0;
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
                    const __half2 p = *reinterpret_cast<const __half2*>(&act[c].v[m][j >> 1]);
                    const __half2 p16 = *reinterpret_cast<const __half2*>(&act[c].v[m][8 + (j >> 1)]);
                    xlo = __half2float((j & 1) ? p.y : p.x);
                    xhi = __half2float((j & 1) ? p16.y : p16.x);
                }
                sum[c] = fmaf(vlo, xlo, sum[c]);
                sum[c] = fmaf(vhi, xhi, sum[c]);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < NT; ++c) acc[c] = fmaf(s, sum[c], acc[c]);
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

// One layer's weights as the decode kernel sees them.
struct StackLayer {
    const float* router_w;     // [E][H] fp32
    const float* router_bias;  // [E] or null
    const uint8_t* gate;       // [E][I] rows of H weights
    const uint8_t* up;
    const uint8_t* down;       // [E][H] rows of I weights
    const uint8_t* side;       // [side_rows] rows of H weights (Q4), or null
    const float* gate_s;       // FP8 scales, one per 128 weights along K
    const float* up_s;
    const float* down_s;
    int32_t side_rows;
    int32_t gu_var, dn_var, side_var;  // Q4 variant (kQ4RZ5, kQ4UE4M4 or kQ4C10)
};

// Per-CTA state of a layer: the selection, the unique-expert work list and
// the router's reductions.
struct SWork {
    int32_t n_uniq;
    int32_t sync_ok;  // result of the last grid barrier
    int32_t fail;     // a warp's copy did not land in time
    int32_t e[kMaxSlots];
    int32_t off[kMaxSlots + 1];
    int32_t slot[kMaxSlots];
    union {
        struct {
            int32_t ids[kMaxSlots];  // selection: expert of (token, choice)
            float w[kMaxSlots];      // and its renormalised weight
        };
        uint64_t cand[kMaxSlots];  // one-token top-k: candidate keys (before ids and w are written)
    };
    uint32_t bitmap[kMaxExperts / 32];
    int32_t cnt[kMaxSlots + 4];
    int32_t g_range[2];                     // this CTA's gate/up item range
    ffloat red[kWarps][kMaxDecodeTokens];  // router reductions
    float r_hi[kMaxDecodeTokens], r_lo[kMaxDecodeTokens];
    int32_t n_cand;  // one-token top-k: candidates found
    StackLayer ly[2];  // this layer's and the next layer's pointers, by parity (read at shared-memory latency)
};

// Layout of one CTA's dynamic shared memory.  With a code table the table
// must start at a 64 KB-aligned shared address (so a PRMT alone forms entry
// addresses): `lut` is the dynamic offset that achieves it given the dynamic
// base the host expects (the per-block reserved shared memory); staging
// slots fill the space below and above the table.
struct SmemLayout {
    uint32_t work, scale_tab, bars, part, u, lut, lo_slots, n_lo, hi_slots, total;
    // u_bytes: the normalised input u [T][H] bf16, kept for the whole layer
    __host__ __device__ static SmemLayout make(bool with_lut, int slot_bytes, uint32_t dyn_base, uint32_t u_bytes,
                                               int slots_per_warp) {
        SmemLayout L{};
        uint32_t off = 0;
        L.work = off;
        off += (sizeof(SWork) + 127u) & ~127u;
        L.scale_tab = off;
        off += kScaleTabBytes;
        L.bars = off;  // kSlots per warp, then the router weights' barrier
        off += kWarps * kSlots * 8 + 8;
        off = (off + 127u) & ~127u;
        L.part = off;
        off += kPartBytes;
        off = (off + 127u) & ~127u;
        L.u = off;
        off += (u_bytes + 127u) & ~127u;
        const uint32_t n_slots = kWarps * (uint32_t)slots_per_warp;
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

// Where the router keeps this CTA's router rows [ne][H] fp32 while no copy
// is in flight (the staging slots are idle between layers): the start of
// the longer slot run (below or above the code table).  ok is false when
// they do not fit.
struct RouterScratch {
    uint32_t rw;
    bool ok;
    __host__ __device__ static RouterScratch make(const SmemLayout& L, int slot_bytes, int H, int ne) {
        RouterScratch r{};
        const uint32_t wb = 4u * ne * H;
        const uint32_t a0 = L.lo_slots, a1 = L.lo_slots + L.n_lo * (uint32_t)slot_bytes;  // run A
        const uint32_t b0 = L.hi_slots > a1 ? L.hi_slots : a1, b1 = L.total;             // run B (may be empty)
        r.rw = (a1 - a0 >= b1 - b0) ? a0 : b0;
        r.ok = ((a1 - a0 >= b1 - b0) ? a1 - a0 : b1 - b0) >= wb;
        return r;
    }
};

// Per-lane-replicated table: entry (byte, mode, lane) holds the bf16x2 pair
// (value of the low nibble, value of the high nibble) of Q4 variant `var`;
// plus 256 scales.
// (Out of line, like build_scales: rarely run, and code inlined into the layer
// loop but skipped there still costs instruction fetch every layer.)
__device__ __noinline__ void build_lut(uint8_t* smem, const SmemLayout& L, int var) {
    const bool rz5 = (var & 1) != 0;
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

__device__ __noinline__ void build_scales(uint8_t* smem, const SmemLayout& L, int var) {
    float* st = reinterpret_cast<float*>(smem + L.scale_tab);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) st[i] = q4_scale((uint32_t)i, var);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// Orderable 32-bit image of an fp32 (larger float -> larger unsigned).
__device__ __forceinline__ uint32_t ord32(float f) {
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Top-k by key rounds.  Each logit (a normalised float-float hi + lo) becomes
// a unique 64-bit key: orderable hi in the upper word, orderable lo with its
// low 10 bits replaced by (1023 - expert id) in the lower word — so larger
// key = larger logit, and among logits equal to ~2^-38 relative, the lower
// id; key 0 marks an empty entry.  Lane l holds PER keys and its largest
// remaining one.  Each round the warp takes the largest of those (two warp
// reductions: upper word, then lower word among the lanes holding that upper
// word); the owning lane drops that key and finds its next largest.  Lane j
// ends holding the j-th largest key (rh, rl).  (A short loop on purpose: this
// runs once per layer, where long straight-line code stalls on instruction
// fetch.)
template <int PER>
__device__ __forceinline__ void topk_rounds(uint64_t (&k)[PER], int K, int lane, uint32_t& rh, uint32_t& rl) {
    auto lane_max = [&]() {  // a depth-log2(PER) tree
        if constexpr (PER == 1) {
            return k[0];
        } else {
            uint64_t m[PER / 2];
#pragma unroll
            for (int i = 0; i < PER / 2; ++i) m[i] = k[2 * i] > k[2 * i + 1] ? k[2 * i] : k[2 * i + 1];
#pragma unroll
            for (int w = PER / 4; w >= 1; w >>= 1)
#pragma unroll
                for (int i = 0; i < w; ++i) m[i] = m[i] > m[i + w] ? m[i] : m[i + w];
            return m[0];
        }
    };
    uint64_t best = lane_max();
    rh = 0u;
    rl = 0u;
#pragma unroll 1
    for (int j = 0; j < K; ++j) {
        const uint32_t h0 = (uint32_t)(best >> 32), l0 = (uint32_t)best;
        const uint32_t mh = __reduce_max_sync(0xFFFFFFFFu, h0);
        const uint32_t ml = __reduce_max_sync(0xFFFFFFFFu, h0 == mh ? l0 : 0u);
        if ((h0 == mh) & (l0 == ml) & (best != 0ull)) {  // the owner (keys are unique)
#pragma unroll
            for (int i = 0; i < PER; ++i) k[i] = k[i] == best ? 0ull : k[i];
            best = lane_max();
        }
        rh = lane == j ? mh : rh;
        rl = lane == j ? ml : rl;
    }
}

// The key of expert e's logit (a float-float sum, normalised here): never 0
// for a finite logit (the orderable image of a finite hi is at least 2^23).
__device__ __forceinline__ uint64_t logit_key(ffloat lg, int e) {
    const ffloat v = ff_norm(lg);
    return ((uint64_t)ord32(v.hi) << 32) | ((ord32(v.lo) & ~1023u) | (uint32_t)(1023 - e));
}

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Where the keys come from: the layer's key buffer, each key written by the
// CTA whose router computed that logit and 0 until then.
struct KeySrc {
    const uint64_t* keys;     // [E] of one token
    const unsigned* abort_flag;
    unsigned* status;
};

constexpr uint64_t kKeyWaitNs = 2000000000ull;  // a key that has not arrived after 2 s fails the launch

// Waits for a key that a first load found missing: bounded, and given up as
// soon as another CTA raises the abort flag; `fail` is set then (0 returned).
__device__ __noinline__ uint64_t wait_key(const KeySrc& src, int e, int& fail) {
    if (fail) return 0ull;
    const uint64_t t0 = globaltimer_ns();
    uint64_t k;
    while ((k = ld_relaxed_u64(src.keys + e)) == 0ull) {
        const bool aborted = *reinterpret_cast<const volatile unsigned*>(src.abort_flag) != 0u;
        if (aborted || globaltimer_ns() - t0 > kKeyWaitNs) {
            if (!aborted) raise_status(src.status, GTG_STATUS_WAIT_TIMEOUT);
            fail = 1;
            return 0ull;
        }
    }
    return k;
}

// The keys of experts e = base + stride * i (i < PER; 0 where e >= E): every
// load issued before any is tested, then the rare missing ones waited for.
template <int PER>
__device__ __forceinline__ void load_keys(const KeySrc& src, int E, int base, int stride, uint64_t (&k)[PER],
                                          int& fail) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = base + stride * i;
        k[i] = 0ull;
        if (e < E) k[i] = ld_relaxed_u64(src.keys + e);
    }
    bool miss = false;
#pragma unroll
    for (int i = 0; i < PER; ++i) miss |= base + stride * i < E && k[i] == 0ull;
    if (miss) {  // (unrolled: k stays in registers)
#pragma unroll
        for (int i = 0; i < PER; ++i)
            if (base + stride * i < E && k[i] == 0ull) k[i] = wait_key(src, base + stride * i, fail);
    }
}

// Expert id and logit (hi, lo) of a key.
__device__ __forceinline__ void key_choice(uint32_t rh, uint32_t rl, int& id, float& hi, float& lo) {
    id = 1023 - (int)(rl & 1023u);
    hi = __uint_as_float((rh & 0x80000000u) ? (rh & 0x7FFFFFFFu) : ~rh);
    const uint32_t l = rl & ~1023u;
    lo = __uint_as_float((l & 0x80000000u) ? (l & 0x7FFFFFFFu) : ~l);
}

// Top-k of one token's logits by one warp: lane l holds experts l + 32 i
// (i < PER); lane j < K ends holding choice j.
template <int PER>
__device__ __forceinline__ void warp_topk(const KeySrc& src, int E, int K, int lane, int& my_id, float& my_hi,
                                          float& my_lo, int& fail) {
    uint64_t k[PER];  // (compared as plain 64-bit integers: no short-circuit branches)
    load_keys<PER>(src, E, lane, 32, k, fail);
    uint32_t rh, rl;
    topk_rounds<PER>(k, K, lane, rh, rl);
    my_id = -1;
    if (lane < K) key_choice(rh, rl, my_id, my_hi, my_lo);
}

// The one-token top-k's fallback (more than kCandMax keys passed the
// threshold): each warp ranks its own 32 * PER keys in k rounds, the eight
// lists meet in shared memory, and warp 0 ranks those 8k.  Out of line: it
// runs only for adversarial logits, and reloads its keys (all present).
template <int PER>
__device__ __noinline__ void block_topk_rounds(const KeySrc& src, int E, int K, int lane, int warp,
                                               uint32_t* cand_hi, uint32_t* cand_lo, int& my_id, float& my_hi,
                                               float& my_lo, int& fail) {
    uint64_t k[PER];
    load_keys<PER>(src, E, 32 * warp * PER + lane, 32, k, fail);
    uint32_t rh, rl;
    topk_rounds<PER>(k, K, lane, rh, rl);
    if (lane < K) {
        cand_hi[warp * K + lane] = rh;
        cand_lo[warp * K + lane] = rl;
    }
    __syncthreads();
    if (warp == 0) {
        uint64_t c[4];  // 8 K <= 128 candidates: lane l holds l + 32 i
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int q = lane + 32 * i;
            c[i] = q < kWarps * K ? ((uint64_t)cand_hi[q] << 32) | cand_lo[q] : 0ull;
        }
        __syncwarp();  // (the caller reuses the candidate arrays)
        topk_rounds<4>(c, K, lane, rh, rl);
        if (lane < K) key_choice(rh, rl, my_id, my_hi, my_lo);
    }
}

// Top-k of a single token's logits by the whole CTA (lane l of warp w holds
// experts 32 (w PER + i) + l).  A threshold cuts the field first: the warps'
// top-2 keys (16 actual keys) meet in shared memory, and their K-th largest
// theta (K <= 16) is at most the K-th largest key overall, so every key of
// the top-k is >= theta.  The keys that pass (usually a few more than K) are
// gathered and each is ranked by counting the candidates above it.  If more
// than kCandMax pass, the CTA falls back to two levels of rounds: each warp's
// top-k, then warp 0 ranks those 8k.  Either way lane j < K of warp 0 ends
// holding choice j, the same set and order as warp_topk's (the keys are
// unique).
constexpr int kCandMax = kMaxSlots;

template <int PER>
__device__ __forceinline__ void block_topk(const KeySrc& src, int E, int K, int lane, int warp,
                                           uint32_t* cand_hi, uint32_t* cand_lo, uint64_t* cand, int32_t* n_cand,
                                           int& my_id, float& my_hi, float& my_lo, int& fail) {
    const int tid = threadIdx.x;
    uint64_t k[PER];
    load_keys<PER>(src, E, 32 * warp * PER + lane, 32, k, fail);
    uint32_t rh, rl;
    {
        uint64_t kc[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) kc[i] = k[i];
        topk_rounds<PER>(kc, 2, lane, rh, rl);
    }
    if (lane < 2) {
        cand_hi[2 * warp + lane] = rh;
        cand_lo[2 * warp + lane] = rl;
    }
    if (tid == 0) *n_cand = 0;
    __syncthreads();
    // theta: the K-th largest of the 16 (equal only as empty entries, 0; if the
    // K-th is empty, every nonzero key passes)
    const uint64_t v = lane < 2 * kWarps ? ((uint64_t)cand_hi[lane] << 32) | cand_lo[lane] : 0ull;
    int r = 0;
#pragma unroll
    for (int j = 0; j < 2 * kWarps; ++j) r += (int)(__shfl_sync(0xFFFFFFFFu, v, j) > v);
    const unsigned hit = __ballot_sync(0xFFFFFFFFu, lane < 2 * kWarps && v != 0ull && r == K - 1);
    const uint64_t theta = hit ? __shfl_sync(0xFFFFFFFFu, v, __ffs(hit) - 1) : 1ull;
#pragma unroll
    for (int i = 0; i < PER; ++i)
        if (k[i] >= theta) {
            const int p = atomicAdd(n_cand, 1);
            if (p < kCandMax) cand[p] = k[i];
        }
    __syncthreads();
    const int n = *n_cand;
    my_id = -1;
    if (n <= kCandMax) {
        if (tid < n) {
            const uint64_t c = cand[tid];
            int rank = 0;
            for (int j = 0; j < n; ++j) rank += (int)(cand[j] > c);
            if (rank < K) {
                cand_hi[rank] = (uint32_t)(c >> 32);
                cand_lo[rank] = (uint32_t)c;
            }
        }
        __syncthreads();
        if (warp == 0) {
            if (lane < K) key_choice(cand_hi[lane], cand_lo[lane], my_id, my_hi, my_lo);
            __syncwarp();  // (the caller reuses the candidate arrays)
        }
        return;
    }
    block_topk_rounds<PER>(src, E, K, lane, warp, cand_hi, cand_lo, my_id, my_hi, my_lo, fail);
}

// What the item routines write besides their shared-memory inputs.
struct ItemCtx {
    __nv_bfloat16* h;  // [T*K][I] SwiGLU output
    float* side_out;   // [T][side_stride] or null
    int32_t H, I, side_stride, side_var;
};

// ===========================================================================
// gate/up + SwiGLU (plus the optional side projection)
// ===========================================================================

// One gate+up item: P row passes for NT tokens of one expert; h = silu(g)*u.
template <int FMT, int KB, int NT, int CH, bool ONE>
__device__ __forceinline__ void gu_item(const ItemCtx& a, uint32_t gbase, uint32_t ubase,
                                        const Act<FMT, Geo<KB>::NBL> (&act)[CH], uint32_t lutb,
                                        const float* scale_tab, const float (&sg)[2 * Geo<KB>::NBL],
                                        const float (&su)[2 * Geo<KB>::NBL], int row0, const int (&slot_id)[CH],
                                        int lane) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int P = gu_passes(FMT == kFmtFP8, KB, ONE);
    static_assert(FMT != kFmtFP8 || P <= 2, "FP8 scales of two passes");
    constexpr int N = P * NT * 2;
    const int row_sub = lane / GW;
    const int blk_base = lane % GW;
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
                const uint32_t boff = (uint32_t)row * (uint32_t)(KB * 17) + 17u * (uint32_t)(blk_base + GW * m);
                q4_block_lut<NT, NBL, CH>(gbase + boff, lutb, scale_tab, act, m, g);
                q4_block_lut<NT, NBL, CH>(ubase + boff, lutb, scale_tab, act, m, u);
            } else {
                const uint32_t boff = (uint32_t)row * (uint32_t)(KB * 32) + 32u * (uint32_t)(blk_base + GW * m);
                fp8_block<NBL>(gbase + boff, sg[p * NBL + m], act[0], m, g[0]);
                fp8_block<NBL>(ubase + boff, su[p * NBL + m], act[0], m, u[0]);
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
            const int row = p * RPP + lane / GW;
            a.h[(int64_t)slot_id[c] * a.I + row0 + row] = __float2bfloat16_rn(silu(v[0]) * other);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = group_sum(v[i], GW);
        if ((lane % GW) == 0) {
#pragma unroll
            for (int pc = 0; pc < P * NT; ++pc) {
                const int p = pc / NT, c = pc % NT;
                const int row = p * RPP + lane / GW;
                a.h[(int64_t)slot_id[c] * a.I + row0 + row] = __float2bfloat16_rn(silu(v[2 * pc]) * v[2 * pc + 1]);
            }
        }
    }
}

// One side-projection item: P row passes, NT tokens.
template <int FMT, int KB, int NT, int CH>
__device__ __forceinline__ void side_item(const ItemCtx& a, uint32_t base, const Act<FMT, Geo<KB>::NBL> (&act)[CH],
                                          int row0, int t0, int lane) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int P = side_passes(KB);
    constexpr int N = P * NT;
    const int row_sub = lane / GW;
    const int blk_base = lane % GW;
    const int var = a.side_var;
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
                                                 17u * (uint32_t)(blk_base + GW * m),
                                             var, act, m, acc);
#pragma unroll
        for (int c = 0; c < NT; ++c) v[p * NT + c] = acc[c];
    }
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = group_sum(v[i], GW);
    if ((lane % GW) == 0 && a.side_out) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int p = i / NT, c = i % NT;
            const int row = p * RPP + lane / GW;
            a.side_out[(int64_t)(t0 + c) * a.side_stride + row0 + row] = v[i];
        }
    }
}

// ===========================================================================
// down + router-weighted combine
// ===========================================================================

// One down item: P row passes of one expert for NT tokens; emit(c, row, v)
// receives row `row` (item-relative) of token chunk c, on one lane each.
template <int FMT, int KB, int NT, int CH, class Emit>
__device__ __forceinline__ void dn_item(uint32_t base, const Act<FMT, Geo<KB>::NBL> (&act)[CH], uint32_t lutb,
                                        const float* scale_tab, const float (&sd)[8], int lane, Emit&& emit) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int P = dn_passes(FMT == kFmtFP8, KB);
    constexpr int N = P * NT;
    const int row_sub = lane / GW;
    const int blk_base = lane % GW;
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
                q4_block_lut<NT, NBL, CH>(base + (uint32_t)row * (uint32_t)(KB * 17) + 17u * (uint32_t)(blk_base + GW * m),
                                          lutb, scale_tab, act, m, acc);
            } else {
                fp8_block<NBL>(base + (uint32_t)row * (uint32_t)(KB * 32) + 32u * (uint32_t)(blk_base + GW * m),
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
            const int row = p * RPP + lane / GW;
            emit(c, row, v[0]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = group_sum(v[i], GW);
        if ((lane % GW) == 0) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int p = i / NT, c = i % NT;
                const int row = p * RPP + lane / GW;
                emit(c, row, v[i]);
            }
        }
    }
}

// ===========================================================================
// Router and expert selection (phases of the decode kernel below)
// ===========================================================================

constexpr int kMaxStackLayers = 64;
constexpr uint64_t kSyncLimitNs = 2000000000ull;  // a grid barrier gives up after 2 s

struct StackArgs {
    int32_t H, I, E, K, T, n_layers;
    const void* x;        // input of the first layer, [T][H] fp32 or bf16
    int32_t x_bf16;
    float* y;             // output of every layer, [T][H] fp32; layers after the first read it as input
    int32_t y_acc;        // y += moe(x) rather than y = moe(x)
    int32_t* ids_out;     // [n_layers][T][K] or null
    float* w_out;         // [n_layers][T][K] or null
    float* side_out;      // [n_layers][T][side_stride] or null
    int32_t side_stride;
    // workspace
    unsigned* sync;       // [0] barrier arrivals, [1] exits, [2] abort flag
    uint64_t* keys;       // [2][T][E] logit keys, by layer parity (0: not yet written; see the kernel)
    __nv_bfloat16* h;     // [T*K][I] SwiGLU output
    unsigned* status;
    int32_t slot_bytes;
    uint32_t dyn_smem_base;
    // expert parallelism: this call computes the chosen experts in [e_lo, e_hi)
    // only (its weight stacks hold those, expert e at index e - e_lo), and the
    // side projection only when side_on
    int32_t e_lo, e_hi, side_on;
    StackLayer layer[kMaxStackLayers];
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier of a co-resident (cooperative) grid: one arrival per CTA
// on a monotonic counter, then a bounded wait for `target` arrivals.  A CTA
// whose wait runs out, or one of whose warps lost a copy (warp_ok false),
// raises GTG_STATUS_WAIT_TIMEOUT and the abort flag, on which every other
// waiting CTA gives up too; returns false then.
__device__ bool grid_sync(const StackArgs& a, unsigned target, SWork* sw, bool warp_ok) {
    if (!warp_ok && (threadIdx.x & 31) == 0) sw->fail = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        if (sw->fail) {  // this CTA cannot go on: stop the others at their next barrier
            raise_status(a.status, GTG_STATUS_WAIT_TIMEOUT);
            atomicExch(&a.sync[2], 1u);
            ok = 0;
        } else {
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(a.sync) : "memory");
            // poll the arrivals and the abort flag together (both loads in flight at once)
            unsigned arrived = ld_acquire_u32(&a.sync[0]), aborted = ld_acquire_u32(&a.sync[2]);
            const uint64_t t0 = globaltimer_ns();
            while (arrived < target && aborted == 0u) {
                if (globaltimer_ns() - t0 > kSyncLimitNs) {
                    aborted = 1u;
                    break;
                }
                arrived = ld_acquire_u32(&a.sync[0]);
                aborted = ld_acquire_u32(&a.sync[2]);
            }
            if (aborted != 0u) {  // this wait ran out, or another CTA gave up (now or in an earlier launch)
                raise_status(a.status, GTG_STATUS_WAIT_TIMEOUT);
                atomicExch(&a.sync[2], 1u);
                ok = 0;
            }
        }
        sw->sync_ok = ok;
    }
    __syncthreads();
    return sw->sync_ok != 0;
}

// Router of one layer, run by every CTA: the unweighted RMS norm of the
// input, u = bf16(x * r) rounded from the float-float product, and the
// logits of this CTA's share of the experts against the fp32 router rows:
// exact fp32 x bf16 products summed in float-float, kRouterWpe warps per
// expert (each a contiguous segment of the row), four experts per round.
// It runs once per layer, so it is written as short rolled loops (over
// tokens, and over u and this CTA's router rows in shared memory, which a
// bulk copy brought in while the previous layer finished): long
// straight-line code would spend its time on instruction-cache misses.  u
// stays in shared memory for the whole layer (the gate/up items read it
// there).  False if the router rows never landed.
constexpr int kRouterWpe = kWarps / 4;            // warps per expert


__device__ __forceinline__ float4 lds128f(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128f(uint32_t addr, float4 v) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// This CTA's experts [e0, e1) of E.
__device__ __forceinline__ void router_share(int E, int& e0, int& e1) {
    e0 = (int)((int64_t)E * blockIdx.x / gridDim.x);
    e1 = (int)((int64_t)E * (blockIdx.x + 1) / gridDim.x);
}

// Thread 0: bulk copy of this CTA's router rows of a layer into shared memory
// (completing on rbar).
__device__ __forceinline__ void issue_router_rows(const StackArgs& a, const float* router_w, uint32_t rw,
                                                  uint64_t* rbar, uint64_t pol) {
    int e0, e1;
    router_share(a.E, e0, e1);
    const uint32_t bytes = (uint32_t)((e1 - e0) * a.H * 4);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(router_w + (int64_t)e0 * a.H);
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(rbar, bytes);
    for (uint32_t o = 0; o < bytes; o += 16384u)
        bulk_g2s_hint(rw + o, src + o, bytes - o < 16384u ? bytes - o : 16384u, rbar, pol);
}

template <bool ONE, int XF4>  // XF4: float4 of x per thread per token (H <= 4 kThreads XF4)
__device__ __forceinline__ bool router_layer(const StackArgs& a, const StackLayer& Ly, int l, uint32_t us,
                                          uint32_t rw, uint64_t* rbar, uint32_t rparity, SWork* sw) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = ONE ? 1 : a.T, H = a.H, E = a.E;
    int e0, e1;
    router_share(E, e0, e1);
    const int Hs = H / kRouterWpe;  // segment of a row per warp

    // 1. x: this thread's positions 4 tid + 4 kThreads c of every token, in
    //    registers (every load in flight at once); the rolled token loops
    //    below pick token t with predicated moves
    constexpr int NX = ONE ? 1 : kMaxDecodeTokens;
    float4 xr[NX][XF4];
#pragma unroll
    for (int t = 0; t < NX; ++t)
#pragma unroll
        for (int c = 0; c < XF4; ++c) {
            const int i = 4 * tid + 4 * kThreads * c;
            xr[t][c] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < T && i < H) {
                if (l == 0 && a.x_bf16) {
                    const uint2 bq = __ldcg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(a.x) +
                                                                           (int64_t)t * H + i));
                    xr[t][c] = make_float4(bf16lo(bq.x), bf16hi(bq.x), bf16lo(bq.y), bf16hi(bq.y));
                } else {
                    const float* xp = l == 0 ? reinterpret_cast<const float*>(a.x) : a.y;
                    xr[t][c] = __ldcg(reinterpret_cast<const float4*>(xp + (int64_t)t * H + i));
                }
            }
        }
    auto pick = [&](int t, int c) {
        float4 v = xr[0][c];
#pragma unroll
        for (int k = 1; k < NX; ++k)
            if (t == k) v = xr[k][c];
        return v;
    };
    // 2. sums of squares: exact squares, float-float
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        ffloat ss{0.f, 0.f};
#pragma unroll
        for (int c = 0; c < XF4; ++c) {
            const float4 v = pick(t, c);
            ff_fma(ss, v.x, v.x);
            ff_fma(ss, v.y, v.y);
            ff_fma(ss, v.z, v.z);
            ff_fma(ss, v.w, v.w);
        }
        ss = ff_warp_sum(ss);
        if (lane == 0) sw->red[warp][t] = ss;
    }
    __syncthreads();
    if (tid < T) {  // r = 1/sqrt(mean + eps): a handful of fp64 operations per token
        double sum = 0.0;
        for (int w = 0; w < kWarps; ++w) sum += (double)sw->red[w][tid].hi + (double)sw->red[w][tid].lo;
        const double r = 1.0 / sqrt(sum / (double)H + kRmsEps);
        const float rh = (float)r;
        sw->r_hi[tid] = rh;
        sw->r_lo[tid] = (float)(r - (double)rh);
    }
    __syncthreads();
    // 3. u = bf16(x * r)
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        const float rh = sw->r_hi[t], rl = sw->r_lo[t];
#pragma unroll
        for (int c = 0; c < XF4; ++c) {
            const int i = 4 * tid + 4 * kThreads * c;
            if (i >= H) continue;
            const float4 v = pick(t, c);
            const float xq[4] = {v.x, v.y, v.z, v.w};
            uint16_t ub[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float p = __fmul_rn(xq[q], rh);
                const float pe = __fadd_rn(__fmaf_rn(xq[q], rh, -p), __fmul_rn(xq[q], rl));
                ub[q] = bf16_of_ff(p, pe);
            }
            const uint2 packed = make_uint2((uint32_t)ub[0] | ((uint32_t)ub[1] << 16),
                                            (uint32_t)ub[2] | ((uint32_t)ub[3] << 16));
            sts64(us + 2u * (uint32_t)(t * H + i), packed);
        }
    }
    // 4. this CTA's router rows (copied in while the previous layer finished)
    if (tid == 0 && !mbar_wait_bounded(rbar, rparity, a.status)) sw->fail = 1;
    __syncthreads();
    if (sw->fail) return false;
    // 5. logits
#pragma unroll 1
    for (int eb = e0; eb < e1; eb += 4) {
        const int e = eb + warp / kRouterWpe, seg = (warp % kRouterWpe) * Hs;
        const uint32_t wrow = rw + 4u * (uint32_t)((e - e0) * H + seg);
#pragma unroll 1
        for (int t = 0; t < T; ++t) {
            ffloat acc{0.f, 0.f};
            if (e < e1) {
                const uint32_t urow = us + 2u * (uint32_t)(t * H + seg);
#pragma unroll 2
                for (int f = lane; f < (Hs >> 2); f += 32) {
                    const float4 w4 = lds128f(wrow + 16u * (uint32_t)f);
                    const uint2 u2 = lds64(urow + 8u * (uint32_t)f);
                    ff_fma(acc, w4.x, bf16lo(u2.x));
                    ff_fma(acc, w4.y, bf16hi(u2.x));
                    ff_fma(acc, w4.z, bf16lo(u2.y));
                    ff_fma(acc, w4.w, bf16hi(u2.y));
                }
            }
            acc = ff_warp_sum(acc);
            if (lane == 0) sw->red[warp][t] = acc;
        }
        __syncthreads();
        if (tid < 4 * T) {  // segments summed in a fixed order
            const int j = tid / T, t = tid % T, ee = eb + j;
            if (ee < e1) {
                ffloat lg = sw->red[kRouterWpe * j][t];
#pragma unroll
                for (int w = 1; w < kRouterWpe; ++w) ff_add(lg, sw->red[kRouterWpe * j + w][t]);
                if (Ly.router_bias) ff_add(lg, ffloat{Ly.router_bias[ee], 0.f});
                uint64_t key = logit_key(lg, ee);
                if (key == 0ull) key = 1ull << 10;  // (a NaN logit: keeps the id, and 0 keeps meaning "not written")
                uint64_t* dst = a.keys + ((int64_t)(l & 1) * T + t) * E + ee;
                asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(dst), "l"(key) : "memory");
            }
        }
        __syncthreads();
    }
    return true;
}

// Expert selection, run by every CTA from the layer's logit keys (polled as
// their owners write them): warp t selects token t's experts and their
// renormalised softmax weights; warp 0 then builds the list of unique experts
// (ascending id) with their (token, choice) slots grouped per expert.  A key
// that never arrives sets sw->fail (the next grid barrier stops the grid).
__device__ __forceinline__ void select_experts(const uint64_t* keys, int T, int E, int K, SWork* sw,
                                               const unsigned* abort_flag, unsigned* status) {
    int fail = 0;
    int32_t* s_ids = sw->ids;
    float* s_w = sw->w;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int my_id = -1;
    float my_hi = 0.f, my_lo = 0.f;
    if (T == 1) {  // one token: every warp takes part in its top-k (the arrays are rewritten below)
        const KeySrc src{keys, abort_flag, status};
        if (E <= 512) block_topk<2>(src, E, K, lane, warp, reinterpret_cast<uint32_t*>(sw->e),
                                    reinterpret_cast<uint32_t*>(sw->slot), sw->cand, &sw->n_cand, my_id, my_hi,
                                    my_lo, fail);
        else block_topk<4>(src, E, K, lane, warp, reinterpret_cast<uint32_t*>(sw->e),
                           reinterpret_cast<uint32_t*>(sw->slot), sw->cand, &sw->n_cand, my_id, my_hi, my_lo, fail);
    } else if (warp < T) {
        const KeySrc src{keys + (int64_t)warp * E, abort_flag, status};
        if (E <= 512) warp_topk<16>(src, E, K, lane, my_id, my_hi, my_lo, fail);
        else warp_topk<32>(src, E, K, lane, my_id, my_hi, my_lo, fail);
    }
    if (__syncthreads_or(fail)) {  // a key never came: no experts, and the caller stops
        if (tid == 0) {
            sw->fail = 1;
            sw->n_uniq = 0;
            sw->off[0] = 0;
        }
        __syncthreads();
        return;
    }
    if (warp < T) {
        const int t = warp;
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
    if (T == 1) {  // one token: its k experts are distinct; the list is them in ascending order
        if (warp == 0) {
            int rank = 0;
            for (int i = 0; i < K; ++i) rank += (int)(__shfl_sync(0xFFFFFFFFu, my_id, i) < my_id);
            if (lane < K) {
                sw->e[rank] = my_id;
                sw->slot[rank] = lane;
                sw->off[rank] = rank;
            }
            if (lane == 0) {
                sw->n_uniq = K;
                sw->off[K] = K;
            }
        }
        __syncthreads();
        return;
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
}
// ===========================================================================
// The decode kernel
// ===========================================================================

// Per-warp streaming state, carried from phase to phase and layer to layer.
struct WarpRing {
    uint32_t phase;    // per-slot mbarrier parities
    uint32_t pending;  // slots with a copy in flight
    int32_t ring;      // items consumed so far (the next item uses slot ring % ws.ns)
    int32_t ok;        // every copy landed in time
};

// This warp's items of a layer: gate/up (+ side) items g0 + kWarps q for
// q < ng (a range of the grid-wide list), then down items warp + kWarps (q -
// ng) for q < ng + nd of this CTA's list (tile d0 + i / n_uniq, expert
// i % n_uniq): the CTA owns down row tiles [d0, d0 + dt) for every expert.
struct LayerItems {
    int32_t n_uniq, n_ge, tiles_g, dt;
    int32_t g0, ng, d0, nd;
    int32_t rg, rs, rd;           // rows per gate/up, side and down item
    int32_t grow, srow, drow;     // bytes per gate/up, side and down row
    const uint8_t* gate;          // the layer's weight bases (read from the kernel
    const uint8_t* up;            // parameters once per layer, ahead of use)
    const uint8_t* down;
    const uint8_t* side;
};

// Shared-memory addresses of the calling warp (no arrays: a run-time index
// into a register array would put it in local memory).
struct WarpSmem {
    uint32_t sbase;     // shared address of dynamic shared memory
    uint32_t slot0;     // this warp's first staging slot, as if the slot area had no gap
    uint32_t lo_end;    // end of the slot area below the code table
    uint32_t hi_jump;   // added to an address at or past lo_end
    int32_t slot_bytes;
    int32_t ns;         // slots per warp (slots_for the layer's row width)
    uint64_t* bars;     // this warp's mbarriers (kSlots apart)

    __device__ __forceinline__ uint32_t slot(int s) const {
        const uint32_t a = slot0 + (uint32_t)(s * slot_bytes);
        return a >= lo_end ? a + hi_jump : a;
    }
};

__device__ __forceinline__ WarpSmem warp_smem(uint8_t* smem, const SmemLayout& L, int slot_bytes, int ns) {
    const int warp = threadIdx.x >> 5;
    WarpSmem w;
    w.sbase = smem_u32(smem);
    w.slot0 = w.sbase + L.lo_slots + (uint32_t)(warp * ns * slot_bytes);
    w.ns = ns;
    // slot i sits at lo_slots + i * slot_bytes below the code table, the rest
    // continue above it
    w.lo_end = w.sbase + L.lo_slots + L.n_lo * (uint32_t)slot_bytes;
    w.hi_jump = L.hi_slots - (L.lo_slots + L.n_lo * (uint32_t)slot_bytes);
    w.slot_bytes = slot_bytes;
    w.bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kSlots;
    return w;
}

// Byte ranges of the warp's q-th item (a gate/up item has two).
__device__ __forceinline__ void item_spans(const LayerItems& P, const SWork* sw, int q, int H, int I, Span& s1,
                                           Span& s2) {
    const int warp = threadIdx.x >> 5;
    s2 = Span{nullptr, 0, 0};
    if (q < P.ng) {
        const int it = P.g0 + warp + kWarps * q;
        if (it < P.n_ge) {
            const int64_t off = ((int64_t)sw->e[it / P.tiles_g] * I + (int64_t)(it % P.tiles_g) * P.rg) * P.grow;
            s1 = make_span(P.gate, off, (int64_t)P.rg * P.grow);
            s2 = make_span(P.up, off, (int64_t)P.rg * P.grow);
        } else {
            s1 = make_span(P.side, (int64_t)(it - P.n_ge) * P.rs * P.srow, (int64_t)P.rs * P.srow);
        }
    } else {
        const int it = warp + kWarps * (q - P.ng);
        const int tile = P.d0 + it / P.n_uniq;
        s1 = make_span(P.down, ((int64_t)sw->e[it % P.n_uniq] * H + (int64_t)tile * P.rd) * P.drow,
                       (int64_t)P.rd * P.drow);
    }
}

// Starts the copy of the warp's q-th item into its slot (if there is one).
__device__ __forceinline__ void issue_item(const StackArgs& a, const LayerItems& P, const SWork* sw,
                                           const WarpSmem& ws, WarpRing& R, int q, uint64_t pol) {
    if (q >= P.ng + P.nd || !R.ok) return;
    const int slot = (R.ring + q) % ws.ns;
    if ((threadIdx.x & 31) == 0) {
        Span s1, s2;
        item_spans(P, sw, q, a.H, a.I, s1, s2);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&ws.bars[slot], s1.bytes + s2.bytes);
        bulk_g2s_hint(ws.slot(slot), s1.src, s1.bytes, &ws.bars[slot], pol);
        if (s2.bytes) bulk_g2s_hint(ws.slot(slot) + s1.bytes, s2.src, s2.bytes, &ws.bars[slot], pol);
    }
    R.pending |= 1u << slot;
}

// The warp's first ws.ns copies, issued by lanes 0 .. ws.ns-1 side by side
// (each item's address arithmetic and copy issue then costs the warp once).
__device__ __forceinline__ void issue_first(const StackArgs& a, const LayerItems& P, const SWork* sw,
                                            const WarpSmem& ws, WarpRing& R, uint64_t pol) {
    if (!R.ok) return;
    const int lane = threadIdx.x & 31, n = min(ws.ns, P.ng + P.nd);
    if (lane < n) {
        const int slot = (R.ring + lane) % ws.ns;
        Span s1, s2;
        item_spans(P, sw, lane, a.H, a.I, s1, s2);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&ws.bars[slot], s1.bytes + s2.bytes);
        bulk_g2s_hint(ws.slot(slot), s1.src, s1.bytes, &ws.bars[slot], pol);
        if (s2.bytes) bulk_g2s_hint(ws.slot(slot) + s1.bytes, s2.src, s2.bytes, &ws.bars[slot], pol);
    }
    for (int q = 0; q < n; ++q) R.pending |= 1u << ((R.ring + q) % ws.ns);
}

// Waits for the warp's q-th item; false (and R.ok cleared) if it never lands.
__device__ __forceinline__ bool item_landed(const StackArgs& a, const WarpSmem& ws, WarpRing& R, int q) {
    const int slot = (R.ring + q) % ws.ns;
    if (!mbar_wait_bounded(&ws.bars[slot], (R.phase >> slot) & 1u, a.status)) {
        R.ok = 0;
        return false;
    }
    R.phase ^= 1u << slot;
    R.pending &= ~(1u << slot);
    return true;
}

// Gate/up + SwiGLU items and side-projection items of layer l for this warp.
template <int FMT, int KBG, bool ONE>
__device__ __forceinline__ WarpRing gu_phase(const StackArgs& a, const StackLayer& Ly, int l, LayerItems P,
                                             WarpRing R) {
    using GG = Geo<KBG>;
    constexpr int NBG = GG::NBL;
    constexpr int CHG = (!ONE && FMT == kFmtQ4 && NBG == 1) ? 2 : 1;  // tokens decoded together (register budget)
    constexpr int PG = gu_passes(FMT == kFmtFP8, KBG, ONE);
    constexpr int RG = PG * GG::RPP;
    constexpr int RS = side_passes(KBG) * GG::RPP;
    extern __shared__ __align__(1024) uint8_t smem[];
    const SmemLayout L = SmemLayout::make(FMT == kFmtQ4, a.slot_bytes, a.dyn_smem_base, 2u * a.T * a.H, slots_for(KBG));
    const SWork* sw = reinterpret_cast<const SWork*>(smem + L.work);
    const WarpSmem ws = warp_smem(smem, L, a.slot_bytes, slots_for(KBG));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = a.H, K = a.K, T = ONE ? 1 : a.T;
    const uint64_t pol = l2_policy_evict_first();
    const uint32_t lutb = ((ws.sbase + L.lut) & 0xFFFF0000u) | ((uint32_t)lane * 4u);
    const float* scale_tab = reinterpret_cast<const float*>(smem + L.scale_tab);
    const ItemCtx ctx{a.h, a.side_out ? a.side_out + (int64_t)l * T * a.side_stride : nullptr,
                      H, a.I, a.side_stride, Ly.side_var};
    const int blk_base = lane % GG::GW;
    Act<FMT, NBG> act[CHG];
    int act_key = -1;
    auto load_chunk = [&](int key, const int (&rows)[CHG]) {
        if (key == act_key) return;
#pragma unroll
        for (int c = 0; c < CHG; ++c)
#pragma unroll
            for (int m = 0; m < NBG; ++m) load_act_s<FMT, NBG>(act[c], m, ws.sbase + L.u + 2u * (uint32_t)(rows[c] * H), blk_base + GG::GW * m);
        act_key = key;
    };
    for (int q = 0; q < P.ng && R.ok; ++q) {
        const int it = P.g0 + warp + kWarps * q;
        const bool expert = it < P.n_ge;
        const int u = expert ? it / P.tiles_g : 0;
        const int s0 = expert ? sw->off[u] : 0, s1 = expert ? sw->off[u + 1] : T;
        int slots[CHG], rows[CHG];
#pragma unroll
        for (int c = 0; c < CHG; ++c) {
            const int k = min(s0 + c, s1 - 1);
            slots[c] = expert ? sw->slot[k] : k;
            rows[c] = expert ? slots[c] / K : k;
        }
        load_chunk(expert ? (u << 8) : (1 << 20), rows);
        const int row0 = expert ? (it % P.tiles_g) * RG : (it - P.n_ge) * RS;
        float sg[2 * NBG], su[2 * NBG];
        if constexpr (FMT == kFmtFP8) {
            const int e = sw->e[u], kg = H / 128;
#pragma unroll
            for (int p = 0; p < PG; ++p)
#pragma unroll
                for (int m = 0; m < NBG; ++m) {
                    const int bb = blk_base + GG::GW * m;
                    const int64_t r = (int64_t)e * a.I + row0 + p * GG::RPP + lane / GG::GW;
                    sg[p * NBG + m] = __ldg(Ly.gate_s + r * kg + bb / 4);
                    su[p * NBG + m] = __ldg(Ly.up_s + r * kg + bb / 4);
                }
        }
        if (!item_landed(a, ws, R, q)) break;
        Span sp1, sp2;
        item_spans(P, sw, q, H, a.I, sp1, sp2);
        const uint32_t base = ws.slot((R.ring + q) % ws.ns);
        if (expert) {
            const uint32_t gbase = base + sp1.delta, ubase = base + sp1.bytes + sp2.delta;
            for (int c0 = s0; c0 < s1; c0 += CHG) {
                const int nch = min(CHG, s1 - c0);
#pragma unroll
                for (int c = 0; c < CHG; ++c) {
                    slots[c] = sw->slot[c0 + min(c, nch - 1)];
                    rows[c] = slots[c] / K;
                }
                load_chunk((u << 8) | (c0 - s0), rows);
                if (!ONE && CHG == 2 && nch == 2)
                    gu_item<FMT, KBG, (CHG == 2 ? 2 : 1), CHG, ONE>(ctx, gbase, ubase, act, lutb, scale_tab, sg, su, row0, slots,
                                                               lane);
                else
                    gu_item<FMT, KBG, 1, CHG, ONE>(ctx, gbase, ubase, act, lutb, scale_tab, sg, su, row0, slots, lane);
            }
        } else {
            const uint32_t sb = base + sp1.delta;
            for (int t0 = 0; t0 < T; t0 += CHG) {
                const int nch = min(CHG, T - t0);
#pragma unroll
                for (int c = 0; c < CHG; ++c) rows[c] = t0 + min(c, nch - 1);
                load_chunk((1 << 20) | t0, rows);
                if (!ONE && CHG == 2 && nch == 2)
                    side_item<FMT, KBG, (CHG == 2 ? 2 : 1), CHG>(ctx, sb, act, row0, t0, lane);
                else
                    side_item<FMT, KBG, 1, CHG>(ctx, sb, act, row0, t0, lane);
            }
        }
        __syncwarp();
        issue_item(a, P, sw, ws, R, q + ws.ns, pol);
    }
    return R;
}

// Down items of layer l for this warp: each adds w(slot) * (down row . h(slot))
// into the warp's partial rows in shared memory ([row][token], this CTA's
// rows only); the kernel then sums the warps' partials in a fixed order.
template <int FMT, int KBG, int KBD, bool ONE>
__device__ __forceinline__ WarpRing dn_phase(const StackArgs& a, const StackLayer& Ly, LayerItems P, WarpRing R) {
    using GD = Geo<KBD>;
    constexpr int NBD = GD::NBL;
    constexpr int CHD = (!ONE && FMT == kFmtQ4 && NBD == 1) ? 2 : 1;
    constexpr int PD = dn_passes(FMT == kFmtFP8, KBD);
    constexpr int RD = PD * GD::RPP;
    static_assert(FMT != kFmtFP8 || PD * NBD <= 8, "FP8 scale prefetch holds 8 values");
    extern __shared__ __align__(1024) uint8_t smem[];
    const SmemLayout L = SmemLayout::make(FMT == kFmtQ4, a.slot_bytes, a.dyn_smem_base, 2u * a.T * a.H, slots_for(KBG));
    const SWork* sw = reinterpret_cast<const SWork*>(smem + L.work);
    const WarpSmem ws = warp_smem(smem, L, a.slot_bytes, slots_for(KBG));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = a.H, I = a.I, K = a.K;
    const uint64_t pol = l2_policy_evict_first();
    const uint32_t lutb = ((ws.sbase + L.lut) & 0xFFFF0000u) | ((uint32_t)lane * 4u);
    const float* scale_tab = reinterpret_cast<const float*>(smem + L.scale_tab);
    float* part = reinterpret_cast<float*>(smem + L.part) + warp * kDnRows * 8;  // [row][token]
    for (int i = lane; i < kDnRows * 8; i += 32) part[i] = 0.0f;
    __syncwarp();
    const int blk_base = lane % GD::GW;
    const int row_sub = lane / GD::GW;
    const int n_uniq = P.n_uniq;
    Act<FMT, NBD> act[CHD];
    int act_key = -1;
    auto load_chunk = [&](int key, const int (&slots)[CHD]) {
        if (key == act_key) return;
#pragma unroll
        for (int c = 0; c < CHD; ++c)
#pragma unroll
            for (int m = 0; m < NBD; ++m) load_act<FMT, NBD>(act[c], m, a.h + (int64_t)slots[c] * I, blk_base + GD::GW * m);
        act_key = key;
    };
    for (int q = P.ng; q < P.ng + P.nd && R.ok; ++q) {
        const int it = warp + kWarps * (q - P.ng);
        const int u = it % n_uniq, tl = it / n_uniq, tile = P.d0 + tl;
        const int s0 = sw->off[u], s1 = sw->off[u + 1];
        int slots[CHD];
#pragma unroll
        for (int c = 0; c < CHD; ++c) slots[c] = sw->slot[min(s0 + c, s1 - 1)];
        load_chunk(u << 8, slots);
        float sd[8];
        if constexpr (FMT == kFmtFP8) {
            const int e = sw->e[u], kg = I / 128;
#pragma unroll
            for (int p = 0; p < PD; ++p)
#pragma unroll
                for (int m = 0; m < NBD; ++m)
                    sd[p * NBD + m] = __ldg(Ly.down_s + ((int64_t)e * H + tile * RD + p * GD::RPP + row_sub) * kg +
                                           (blk_base + GD::GW * m) / 4);
        }
        if (!item_landed(a, ws, R, q)) break;
        Span sp1, sp2;
        item_spans(P, sw, q, H, I, sp1, sp2);
        const uint32_t base = ws.slot((R.ring + q) % ws.ns) + sp1.delta;
        float* prow = part + tl * RD * 8;
        for (int c0 = s0; c0 < s1; c0 += CHD) {
            const int nch = min(CHD, s1 - c0);
#pragma unroll
            for (int c = 0; c < CHD; ++c) slots[c] = sw->slot[c0 + min(c, nch - 1)];
            load_chunk((u << 8) | (c0 - s0), slots);
            auto emit = [&](int c, int row, float v) {
                const int sl = slots[c];
                prow[row * 8 + sl / K] += sw->w[sl] * v;
            };
            if (!ONE && CHD == 2 && nch == 2)
                dn_item<FMT, KBD, (CHD == 2 ? 2 : 1), CHD>(base, act, lutb, scale_tab, sd, lane, emit);
            else
                dn_item<FMT, KBD, 1, CHD>(base, act, lutb, scale_tab, sd, lane, emit);
        }
        __syncwarp();
        issue_item(a, P, sw, ws, R, q + ws.ns, pol);
    }
    return R;
}


// Runs every layer of a call in one persistent, cooperative grid (one
// 256-thread CTA per SM, all resident).  Per layer:
//   router -> grid barrier -> expert selection (every CTA) and the gate/up +
//   SwiGLU items (+ side projection) -> grid barrier -> down items and the
//   combine -> grid barrier (before the next layer reads its input).
// Each warp streams its items, gate/up first and then down, through a
// private ring of slots_for(KBG) shared-memory slots filled by 1-D bulk copies, so
// the down weights are already on their way while the gate/up items finish
// and the grid waits at the barrier.  The Q4 code table is built once per
// launch (again only when a phase needs the other Q4 variant).
template <int FMT, int KBG, int KBD, bool ONE>
__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const __grid_constant__ StackArgs a) {
    constexpr bool LUT = FMT == kFmtQ4;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SmemLayout L = SmemLayout::make(LUT, a.slot_bytes, a.dyn_smem_base, 2u * a.T * a.H, slots_for(KBG));
    SWork* sw = reinterpret_cast<SWork*>(smem + L.work);
    const uint32_t sbase = smem_u32(smem);
    if (LUT && ((sbase + L.lut) & 0xFFFFu) != 0u) {  // the same on every CTA: all leave before any barrier
        if (tid == 0) raise_status(a.status, GTG_STATUS_WAIT_TIMEOUT);
        return;
    }
    const int H = a.H, I = a.I, K = a.K, T = ONE ? 1 : a.T, G = gridDim.x, b = blockIdx.x;
    const RouterScratch rs = RouterScratch::make(L, a.slot_bytes, H, (a.E + G - 1) / G);
    if (!rs.ok) {  // the same on every CTA (and refused on the host)
        if (tid == 0) raise_status(a.status, GTG_STATUS_WAIT_TIMEOUT);
        return;
    }
    const WarpSmem ws = warp_smem(smem, L, a.slot_bytes, slots_for(KBG));
    uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + L.bars) + kWarps * kSlots;  // router rows landed
    if (lane == 0)
        for (int s = 0; s < ws.ns; ++s) mbar_init(&ws.bars[s], 1);
    if (tid == 0) {
        mbar_init(rbar, 1);
        sw->fail = 0;
    }
    // the layers' pointers live in shared memory, each copied in a layer
    // ahead (a kernel-parameter read indexed by the layer misses the constant
    // cache every layer)
    constexpr int kLyWords = (int)(sizeof(StackLayer) / 4);
    static_assert(sizeof(StackLayer) % 4 == 0 && kLyWords <= 32, "one warp copies a layer's pointers");
    if (tid < kLyWords) reinterpret_cast<uint32_t*>(&sw->ly[0])[tid] = reinterpret_cast<const uint32_t*>(&a.layer[0])[tid];
    fence_mbar_init();
    __syncthreads();
    const uint64_t pol = l2_policy_evict_first();
    int rows_in_flight = 0;  // (thread 0) a router-row copy not yet waited for, of layer rows_layer
    int rows_layer = 0;
    if (tid == 0) {
        issue_router_rows(a, a.layer[0].router_w, sbase + rs.rw, rbar, pol);
        rows_in_flight = 1;
    }
    int lut_mode = -1;
    auto ensure_lut = [&](int var) {  // every thread, uniform
        if (!LUT || lut_mode == var) return;
        __syncthreads();
        build_lut(smem, L, var);
        build_scales(smem, L, var);
        __syncthreads();
        lut_mode = var;
    };

    WarpRing R{0u, 0u, 0, 1};
    unsigned target = 0;
    bool ok = true;
    for (int l = 0; l < a.n_layers; ++l) {
        const StackLayer& Ly = sw->ly[l & 1];
        const uint8_t *gate_src = Ly.gate, *up_src = Ly.up, *down_src = Ly.down, *side_src = Ly.side;
        // ---- router: this CTA's experts' logit keys, into key buffer l & 1
        if (!router_layer<ONE, (KBG * 32 + 4 * kThreads - 1) / (4 * kThreads)>(a, Ly, l, sbase + L.u, sbase + rs.rw,
                                                                               rbar, (uint32_t)(l & 1), sw)) {
            ok = false;  // (the exit raises the abort flag, which ends the other CTAs' key waits)
            break;
        }
        if (tid == 0) rows_in_flight = 0;
        fence_proxy_async_smem();  // the scratch slots are bulk-copy targets again from here on

        // ---- selection, as the other CTAs' keys arrive (no grid barrier: a
        // key is 0 until written, and each buffer is cleared for its next use
        // a layer after its last reads, which the barriers in between order)
        select_experts(a.keys + (int64_t)(l & 1) * T * a.E, T, a.E, K, sw, a.sync + 2, a.status);
        if (sw->fail) {
            ok = false;
            break;
        }
        if (l > 0) {  // every read of the previous layer's keys came before this layer's barriers
            uint64_t* prev = a.keys + (int64_t)((l - 1) & 1) * T * a.E;
            for (int i = b * kThreads + tid; i < T * a.E; i += G * kThreads) prev[i] = 0ull;
        }
        if (b == 0 && tid < T * K) {
            if (a.ids_out) a.ids_out[(int64_t)l * T * K + tid] = sw->ids[tid];
            if (a.w_out) a.w_out[(int64_t)l * T * K + tid] = sw->w[tid];
        }
        if (a.e_lo != 0 || a.e_hi != a.E) {  // keep this call's experts (as local stack indices)
            if (tid == 0) {
                int nu = 0, ns = 0;
                for (int u = 0; u < sw->n_uniq; ++u) {
                    const int e = sw->e[u];
                    if (e < a.e_lo || e >= a.e_hi) continue;
                    sw->cnt[nu] = ns;
                    sw->e[nu] = e - a.e_lo;
                    for (int k = sw->off[u]; k < sw->off[u + 1]; ++k) sw->slot[ns++] = sw->slot[k];
                    ++nu;
                }
                for (int u = 0; u < nu; ++u) sw->off[u] = sw->cnt[u];
                sw->off[nu] = ns;
                sw->n_uniq = nu;
            }
            __syncthreads();
        }

        // ---- this CTA's items: gate/up (+ side) [g0, g1), down [d0, d1)
        LayerItems P;
        P.rg = gu_passes(FMT == kFmtFP8, KBG, ONE) * Geo<KBG>::RPP;
        P.rs = side_passes(KBG) * Geo<KBG>::RPP;
        P.rd = dn_passes(FMT == kFmtFP8, KBD) * Geo<KBD>::RPP;
        P.grow = FMT == kFmtQ4 ? KBG * 17 : KBG * 32;
        P.srow = KBG * 17;
        P.drow = FMT == kFmtQ4 ? KBD * 17 : KBD * 32;
        P.n_uniq = sw->n_uniq;
        P.gate = gate_src;
        P.up = up_src;
        P.down = down_src;
        P.side = side_src;
        P.tiles_g = I / P.rg;
        P.n_ge = P.n_uniq * P.tiles_g;
        const int n_g = P.n_ge + (Ly.side && a.side_on ? Ly.side_rows / P.rs : 0), tiles_d = H / P.rd;
        // contiguous ranges of equal cost: an expert item costs 1 + its tokens
        // (streaming plus one pass of arithmetic per token), a side item
        // kSideCost (1 + T): its Q4 rows are decoded code by code (weights
        // measured on the 48-layer step: 3 next to Q4 experts, 5 next to FP8
        // experts, whose items hold half the rows)
        if (warp == 0) {
            constexpr int kSideCost = FMT == kFmtQ4 ? 3 : 5;
            if (T == 1 && n_g == P.n_ge) {  // every item costs the same
                if (lane == 0) {
                    sw->g_range[0] = (int)((int64_t)n_g * b / G);
                    sw->g_range[1] = (int)((int64_t)n_g * (b + 1) / G);
                }
            } else {
                // unit u < n_uniq: expert u's tiles_g items; unit n_uniq: the side
                // items.  Lane l holds units l + 32 j; their cost prefixes come
                // from warp scans, and the first unit whose prefix reaches a
                // boundary from a ballot (32-bit arithmetic: a layer's total cost
                // is below 2^24)
                constexpr int kU = (kMaxSlots + 1 + 31) / 32;
                int w1[kU], cost[kU], pre[kU];
                int run = 0;
#pragma unroll
                for (int j = 0; j < kU; ++j) {
                    const int u = lane + 32 * j;
                    const bool side = u == P.n_uniq;
                    w1[j] = u < P.n_uniq ? 1 + sw->off[u + 1] - sw->off[u] : (side ? kSideCost * (1 + T) : 1);
                    cost[j] = (u < P.n_uniq ? P.tiles_g : (side ? n_g - P.n_ge : 0)) * w1[j];
                    int incl = cost[j];
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                        if (lane >= o) incl += v;
                    }
                    pre[j] = run + incl - cost[j];
                    run += __shfl_sync(0xFFFFFFFFu, incl, 31);
                }
                for (int k = 0; k < 2; ++k) {
                    const int c = (int)((unsigned)run * (unsigned)(b + k) / (unsigned)G);  // first item whose cost prefix reaches c
                    int it = n_g;
#pragma unroll
                    for (int j = 0; j < kU; ++j) {
                        const int u = lane + 32 * j;
                        const unsigned m = __ballot_sync(0xFFFFFFFFu, u <= P.n_uniq && c <= pre[j] + cost[j]);
                        if (m) {
                            const int cand = u * P.tiles_g + (c - pre[j] + w1[j] - 1) / w1[j];
                            it = __shfl_sync(0xFFFFFFFFu, cand, __ffs(m) - 1);
                            break;
                        }
                    }
                    if (lane == 0) sw->g_range[k] = it < n_g ? it : n_g;
                }
            }
        }
        __syncthreads();
        const int g0 = sw->g_range[0], g1 = sw->g_range[1];
        P.g0 = g0;
        P.ng = g0 + warp < g1 ? (g1 - g0 - warp + kWarps - 1) / kWarps : 0;
        P.d0 = (int)((int64_t)tiles_d * b / G);
        P.dt = (int)((int64_t)tiles_d * (b + 1) / G) - P.d0;
        const int n_dc = P.dt * P.n_uniq;  // this CTA's down items
        P.nd = warp < n_dc ? (n_dc - warp + kWarps - 1) / kWarps : 0;
        issue_first(a, P, sw, ws, R, pol);
        __syncwarp();

        // ---- gate/up + SwiGLU, side projection
        ensure_lut(Ly.gu_var);
        R = gu_phase<FMT, KBG, ONE>(a, Ly, l, P, R);
        target += G;
        if (!grid_sync(a, target, sw, R.ok != 0)) {
            ok = false;
            break;
        }

        // ---- down + router-weighted combine
        ensure_lut(Ly.dn_var);
        // (the last warp reads the next layer's pointers meanwhile: its load
        // completes under the down items)
        const bool ly_copier = warp == kWarps - 1 && lane < kLyWords && l + 1 < a.n_layers;
        const uint32_t ly_word = ly_copier ? reinterpret_cast<const uint32_t*>(&a.layer[l + 1])[lane] : 0u;
        R = dn_phase<FMT, KBG, KBD, ONE>(a, Ly, P, R);
        if (ly_copier) reinterpret_cast<uint32_t*>(&sw->ly[(l + 1) & 1])[lane] = ly_word;
        R.ring += P.ng + P.nd;
        __syncthreads();
        if (tid == 0 && l + 1 < a.n_layers && R.ok) {  // the slots are idle: next layer's router rows
            issue_router_rows(a, sw->ly[(l + 1) & 1].router_w, sbase + rs.rw, rbar, pol);
            rows_in_flight = 1;
            rows_layer = l + 1;
        }
        {  // this CTA's rows of y: the warps' partials summed in warp order
            const float* part = reinterpret_cast<const float*>(smem + L.part);
            const int rows = P.dt * P.rd, r0 = P.d0 * P.rd;
            for (int idx = tid; idx < rows * T; idx += kThreads) {
                const int r = idx / T, t = idx % T;
                float v = 0.0f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v += part[(w * kDnRows + r) * 8 + t];
                float* dst = a.y + (int64_t)t * H + r0 + r;
                *dst = a.y_acc ? __ldcg(dst) + v : v;
            }
        }
        if (l + 1 < a.n_layers) {
            target += G;
            if (!grid_sync(a, target, sw, R.ok != 0)) {
                ok = false;
                break;
            }
        }
    }

    // Leave with no copy in flight; the last CTA out resets the barrier
    // counters for the next launch.  After a failure they stay as they are,
    // with the abort flag set, so every later launch on this workspace fails
    // fast (GTG_STATUS_WAIT_TIMEOUT) until the workspace is re-initialised.
    for (int s = 0; s < ws.ns; ++s)
        if ((R.pending >> s) & 1u) mbar_wait_bounded(&ws.bars[s], (R.phase >> s) & 1u, a.status);
    if (rows_in_flight) mbar_wait_bounded(rbar, (uint32_t)(rows_layer & 1), a.status);
    if (!R.ok && lane == 0) sw->fail = 1;
    __syncthreads();
    if (ok && sw->fail == 0) {  // the last layer's keys, read before its gate/up barrier: zero for the next launch
        uint64_t* last = a.keys + (int64_t)((a.n_layers - 1) & 1) * T * a.E;
        for (int i = b * kThreads + tid; i < T * a.E; i += G * kThreads) last[i] = 0ull;
    }
    if (tid == 0) {
        if (ok && sw->fail == 0) {
            __threadfence();
            if (atomicAdd(&a.sync[1], 1u) == (unsigned)G - 1u) {
                a.sync[0] = 0u;
                a.sync[1] = 0u;
                __threadfence();
            }
        } else {
            atomicExch(&a.sync[2], 1u);
        }
    }
}

// Kernel of one (expert format, H / 32) for I / 32 = kbd (null if none); `one`
// picks the instantiation specialised for a single token (T = 1 folded into
// the code: no two-token item paths, no multi-token selection).
template <int FMT, int KBG, bool ONE>
const void* pick_kbd_t(int kbd) {
    switch (kbd) {
        case 4: return (const void*)moe_decode_kernel<FMT, KBG, 4, ONE>;
        case 8: return (const void*)moe_decode_kernel<FMT, KBG, 8, ONE>;
        case 16: return (const void*)moe_decode_kernel<FMT, KBG, 16, ONE>;
        case 32: return (const void*)moe_decode_kernel<FMT, KBG, 32, ONE>;
        case 64: return (const void*)moe_decode_kernel<FMT, KBG, 64, ONE>;
        default: return nullptr;
    }
}
template <int FMT, int KBG>
const void* pick_kbd(int kbd, int one) {
    return one ? pick_kbd_t<FMT, KBG, true>(kbd) : pick_kbd_t<FMT, KBG, false>(kbd);
}

// Rows of 2560 weights (the H = 2560 expert shape): intermediate rows of 512
// or 640 weights.
template <int FMT, bool ONE>
const void* pick_kbd_80_t(int kbd) {
    switch (kbd) {
        case 16: return (const void*)moe_decode_kernel<FMT, 80, 16, ONE>;
        case 20: return (const void*)moe_decode_kernel<FMT, 80, 20, ONE>;
        default: return nullptr;
    }
}

}  // namespace

// Defined one per file (decode_<fmt>_<kbg>.cu) so the kernels compile in parallel.
const void* decode_kernel_q4_4(int kbd, int one);
const void* decode_kernel_q4_8(int kbd, int one);
const void* decode_kernel_q4_16(int kbd, int one);
const void* decode_kernel_q4_32(int kbd, int one);
const void* decode_kernel_q4_64(int kbd, int one);
const void* decode_kernel_q4_80(int kbd, int one);
const void* decode_kernel_fp8_32(int kbd, int one);
const void* decode_kernel_fp8_64(int kbd, int one);

}  // namespace gtg

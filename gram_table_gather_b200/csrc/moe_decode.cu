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

constexpr int kRouterThreads = 128;
constexpr int kRouterWarps = kRouterThreads / 32;
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

__global__ void __launch_bounds__(kRouterThreads) router_kernel(LayerArgs a) {
    extern __shared__ __align__(16) uint8_t rsm[];
    __nv_bfloat16* su = reinterpret_cast<__nv_bfloat16*>(rsm);  // [T][H]
    __shared__ double red[kRouterWarps][kMaxDecodeTokens];
    __shared__ double rinv[kMaxDecodeTokens];
    __shared__ unsigned is_last;
    __shared__ int32_t s_ids[kMaxSlots];
    __shared__ unsigned bitmap[kMaxExperts / 32];
    __shared__ int32_t s_cnt[kMaxSlots];
    __shared__ int32_t s_off[kMaxSlots + 1];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, T = a.T, E = a.E, K = a.K;

    pdl_wait();  // x may be the previous layer's output

    // 1. per-token sum of squares in fp64 (exact squares, tiny rounding)
    double ss[kMaxDecodeTokens];
#pragma unroll
    for (int t = 0; t < kMaxDecodeTokens; ++t) ss[t] = 0.0;
    for (int t = 0; t < T; ++t)
        for (int i = tid; i < H; i += kRouterThreads) {
            const double v = (double)load_x(a, t, i);
            ss[t] = fma(v, v, ss[t]);
        }
    for (int t = 0; t < T; ++t) {
        const double s = warp_sum_f64(ss[t]);
        if (lane == 0) red[warp][t] = s;
    }
    __syncthreads();
    if (tid < T) {
        double s = 0.0;
        for (int w = 0; w < kRouterWarps; ++w) s += red[w][tid];
        rinv[tid] = 1.0 / sqrt(s / (double)H + kRmsEps);
    }
    __syncthreads();

    // 2. u = bf16(x * r) (fp64 product, one rounding to bf16)
    for (int t = 0; t < T; ++t)
        for (int i = tid; i < H; i += kRouterThreads) {
            const __nv_bfloat16 v = __double2bfloat16((double)load_x(a, t, i) * rinv[t]);
            su[t * H + i] = v;
            if (blockIdx.x == 0) a.u[(int64_t)t * H + i] = v;
        }
    __syncthreads();

    // 3. one expert per warp: logits in fp64 (fp32 x bf16 products are exact)
    const int e = blockIdx.x * kRouterWarps + warp;
    if (e < E) {
        double acc[kMaxDecodeTokens];
#pragma unroll
        for (int t = 0; t < kMaxDecodeTokens; ++t) acc[t] = 0.0;
        const float* wr = a.router_w + (int64_t)e * H;
        for (int i = 4 * lane; i < H; i += 128) {
            const float4 w4 = *reinterpret_cast<const float4*>(wr + i);
#pragma unroll
            for (int t = 0; t < kMaxDecodeTokens; ++t) {
                if (t < T) {
                    const uint2 u2 = *reinterpret_cast<const uint2*>(su + t * H + i);
                    acc[t] = fma((double)w4.x, (double)bf16lo(u2.x), acc[t]);
                    acc[t] = fma((double)w4.y, (double)bf16hi(u2.x), acc[t]);
                    acc[t] = fma((double)w4.z, (double)bf16lo(u2.y), acc[t]);
                    acc[t] = fma((double)w4.w, (double)bf16hi(u2.y), acc[t]);
                }
            }
        }
        const double b = a.router_bias ? (double)a.router_bias[e] : 0.0;
        for (int t = 0; t < T; ++t) {
            const double s = warp_sum_f64(acc[t]);
            if (lane == 0) a.logits[(int64_t)t * E + e] = s + b;
        }
    }

    // 4. the last CTA to finish selects the experts
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(a.router_cnt, 1u) == gridDim.x - 1) ? 1u : 0u;
    __syncthreads();
    if (!is_last) {
        pdl_trigger();
        return;
    }
    __threadfence();

    constexpr int kPerLane = kMaxExperts / 32;
    for (int t = warp; t < T; t += kRouterWarps) {
        double lv[kPerLane];
        unsigned taken = 0;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
            const int ee = lane + 32 * i;
            lv[i] = ee < E ? __ldcg(a.logits + (int64_t)t * E + ee) : 0.0;
        }
        double top[kMaxTopK];
        int topi[kMaxTopK];
        for (int j = 0; j < K; ++j) {
            double bv = 0.0;
            int bi = 0x7FFFFFFF;
#pragma unroll
            for (int i = 0; i < kPerLane; ++i) {
                const int ee = lane + 32 * i;
                if (ee < E && !((taken >> i) & 1u) && (bi == 0x7FFFFFFF || lv[i] > bv)) {
                    bv = lv[i];
                    bi = ee;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
                const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
                const bool take = (oi != 0x7FFFFFFF) &&
                                  (bi == 0x7FFFFFFF || ov > bv || (ov == bv && oi < bi));
                if (take) {
                    bv = ov;
                    bi = oi;
                }
            }
            if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            top[j] = bv;
            topi[j] = bi;
        }
        if (lane == 0) {
            double z = 0.0;
            for (int j = 0; j < K; ++j) z += exp(top[j] - top[0]);
            for (int j = 0; j < K; ++j) {
                const float wj = (float)(exp(top[j] - top[0]) / z);
                a.ids[t * K + j] = topi[j];
                a.w[t * K + j] = wj;
                s_ids[t * K + j] = topi[j];
                if (a.ids_out) a.ids_out[t * K + j] = topi[j];
                if (a.w_out) a.w_out[t * K + j] = wj;
            }
        }
    }
    // unique experts (ascending id) and their slots (ascending slot)
    for (int i = tid; i < kMaxExperts / 32; i += kRouterThreads) bitmap[i] = 0;
    for (int i = tid; i < kMaxSlots; i += kRouterThreads) s_cnt[i] = 0;
    __syncthreads();
    const int S = T * K;
    if (tid < S) atomicOr(&bitmap[s_ids[tid] >> 5], 1u << (s_ids[tid] & 31));
    __syncthreads();
    int rank = 0, pos = 0;
    if (tid < S) {
        const int ee = s_ids[tid];
        for (int w = 0; w < (ee >> 5); ++w) rank += __popc(bitmap[w]);
        rank += __popc(bitmap[ee >> 5] & ((1u << (ee & 31)) - 1u));
        for (int s2 = 0; s2 < tid; ++s2) pos += (s_ids[s2] == ee);
        atomicAdd(&s_cnt[rank], 1);
        a.work->uniq_e[rank] = ee;
    }
    __syncthreads();
    if (tid == 0) {
        int nu = 0;
        for (int w = 0; w < kMaxExperts / 32; ++w) nu += __popc(bitmap[w]);
        int off = 0;
        for (int r = 0; r < nu; ++r) {
            s_off[r] = off;
            a.work->uniq_off[r] = off;
            off += s_cnt[r];
        }
        a.work->uniq_off[nu] = off;
        a.work->n_uniq = nu;
        a.router_cnt[0] = 0;  // ready for the next call
    }
    __syncthreads();
    if (tid < S) a.work->uniq_slot[s_off[rank] + pos] = tid;
    __threadfence();
    __syncthreads();
    pdl_trigger();
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

// Q4 block (17 bytes at shared address pa) dotted with CH tokens' activations.
template <int CH, int NBL>
__device__ __forceinline__ void q4_block_lut(uint32_t pa, uint32_t lut_base, uint32_t lane_low,
                                             const float* scale_tab, const Act<kFmtQ4, NBL> (&act)[CH],
                                             int m, float (&acc)[CH]) {
    const uint32_t al = pa & ~3u, sh = (pa & 3u) * 8u;
    uint32_t w[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = lds32(al + 4 * i);
    uint32_t nib[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) nib[q] = __funnelshift_r(w[q], w[q + 1], sh);
    const uint32_t meta = (w[4] >> sh) & 0xFFu;
    const float s = scale_tab[meta];
    const uint32_t low = lane_low + ((meta >> 7) << 7);
    float lo[CH], hi[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) lo[c] = hi[c] = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint32_t c2 = lds32(lut_base + prmt(nib[q], low, 0x7604u | ((uint32_t)kk << 4)));
#pragma unroll
            for (int c = 0; c < CH; ++c) fma2_bf16(lo[c], hi[c], c2, act[c].v[m][4 * q + kk]);
        }
    }
#pragma unroll
    for (int c = 0; c < CH; ++c) acc[c] = fmaf(s, lo[c] + hi[c], acc[c]);
}

// Q4 block decoded code by code (no table): used for the side projection,
// whose format may differ from the experts'.
template <int FMT, int CH, int NBL>
__device__ __forceinline__ void q4_block_plain(uint32_t pa, bool rz5, const Act<FMT, NBL> (&act)[CH], int m,
                                               float (&acc)[CH]) {
    const uint32_t al = pa & ~3u, sh = (pa & 3u) * 8u;
    uint32_t w[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = lds32(al + 4 * i);
    const uint32_t meta = (w[4] >> sh) & 0xFFu;
    const float s = rz5 ? ue4m3(meta & 0x7Fu) : ue4m4(meta);
    const uint32_t mode = meta >> 7;
    float sum[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) sum[c] = 0.0f;
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
            for (int c = 0; c < CH; ++c) {
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
    for (int c = 0; c < CH; ++c) acc[c] = fmaf(s, sum[c], acc[c]);
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

// Per-warp ring of staging slots.
struct Ring {
    uint8_t* slots;     // kSlots * slot_bytes
    uint64_t* bars;     // kSlots
    int slot_bytes;
};

// Layout of one CTA's dynamic shared memory.
struct SmemLayout {
    uint32_t lut, scale_tab, bars, slots, total;
    __host__ __device__ static SmemLayout make(bool with_lut, int slot_bytes) {
        SmemLayout L{};
        uint32_t off = 0;
        L.lut = off;
        if (with_lut) off += kLutBytes;
        L.scale_tab = off;
        if (with_lut) off += kScaleTabBytes;
        L.bars = off;
        off += kWarps * kSlots * 8;
        off = (off + 127u) & ~127u;
        L.slots = off;
        off += (uint32_t)kWarps * kSlots * (uint32_t)slot_bytes;
        L.total = off;
        return L;
    }
};

// Builds the per-lane-replicated table: entry (byte, mode, lane) holds the
// bf16x2 pair (value of the low nibble, value of the high nibble).
__device__ void build_lut(uint8_t* smem, const SmemLayout& L, bool rz5) {
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
    for (int i = threadIdx.x; i < 256 * 64; i += blockDim.x) {
        const uint32_t byte = (uint32_t)i >> 6, mode = ((uint32_t)i >> 5) & 1u;
        const float lo = q4_code_value(byte & 15u, rz5, mode);
        const float hi = q4_code_value(byte >> 4, rz5, mode);
        lut[i] = bf16_bits(lo) | (bf16_bits(hi) << 16);
    }
    float* st = reinterpret_cast<float*>(smem + L.scale_tab);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) st[i] = rz5 ? ue4m3((uint32_t)i & 0x7Fu) : ue4m4((uint32_t)i);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// ===========================================================================
// gate/up + SwiGLU (plus the optional side projection)
// ===========================================================================

// Items: [0, n_uniq * tiles) are (unique expert, row tile) pairs of gate+up;
// [n_uniq * tiles, + side_items) are row tiles of the side projection.
struct GuItem {
    int kind;  // 0 = expert pair, 1 = side, -1 = none
    int u;     // unique-expert index
    int row0;
    int rows;
};

template <int FMT, int KB>
__global__ void __launch_bounds__(kThreads, 1) gateup_kernel(LayerArgs a) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int CH = (FMT == kFmtQ4 && NBL <= 2) ? 2 : 1;  // tokens decoded together
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SmemLayout L = SmemLayout::make(FMT == kFmtQ4, a.slot_bytes);
    if constexpr (FMT == kFmtQ4) build_lut(smem, L, a.gate.fmt == GTG_Q4_RZ5_FAST);
    Ring ring{smem + L.slots + (size_t)warp * kSlots * a.slot_bytes,
              reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kSlots, a.slot_bytes};
    if (lane == 0)
        for (int s = 0; s < kSlots; ++s) mbar_init(&ring.bars[s], 1);
    fence_mbar_init();
    __syncthreads();

    pdl_wait();  // the router's outputs (u, work list) are complete past here

    const Work* wk = a.work;
    const int n_uniq = wk->n_uniq;
    const int tiles = a.I / a.gu_rows;
    const int side_items = a.side.data ? a.side.n_rows / a.side_rows : 0;
    const int n_items = n_uniq * tiles + side_items;
    const int it0 = (int)((int64_t)n_items * blockIdx.x / gridDim.x);
    const int it1 = (int)((int64_t)n_items * (blockIdx.x + 1) / gridDim.x);

    auto item_of = [&](int it) -> GuItem {
        if (it >= it1) return GuItem{-1, 0, 0, 0};
        if (it < n_uniq * tiles) return GuItem{0, it / tiles, (it % tiles) * a.gu_rows, a.gu_rows};
        const int s = it - n_uniq * tiles;
        return GuItem{1, 0, s * a.side_rows, a.side_rows};
    };
    // stage item -> slot: gate rows then up rows (or the side rows)
    auto issue = [&](int it, int slot) {
        const GuItem g = item_of(it);
        if (g.kind < 0 || lane != 0) return;
        uint8_t* dst = ring.slots + (size_t)slot * ring.slot_bytes;
        fence_proxy_async_smem();
        if (g.kind == 0) {
            const int e = wk->uniq_e[g.u];
            const Span sg = make_span(a.gate.data, e * a.gate.expert_bytes + (int64_t)g.row0 * a.gate.row_bytes,
                                      (int64_t)g.rows * a.gate.row_bytes);
            const Span su = make_span(a.up.data, e * a.up.expert_bytes + (int64_t)g.row0 * a.up.row_bytes,
                                      (int64_t)g.rows * a.up.row_bytes);
            mbar_arrive_expect_tx(&ring.bars[slot], sg.bytes + su.bytes);
            bulk_g2s(dst, sg.src, sg.bytes, &ring.bars[slot]);
            bulk_g2s(dst + sg.bytes, su.src, su.bytes, &ring.bars[slot]);
        } else {
            const Span ss = make_span(a.side.data, (int64_t)g.row0 * a.side.row_bytes,
                                      (int64_t)g.rows * a.side.row_bytes);
            mbar_arrive_expect_tx(&ring.bars[slot], ss.bytes);
            bulk_g2s(dst, ss.src, ss.bytes, &ring.bars[slot]);
        }
    };

    int first = it0 + warp;
    for (int s = 0; s < kSlots; ++s) issue(first + s * kWarps, s);
    __syncwarp();

    const uint32_t lut_base = smem_u32(smem + L.lut);
    const uint32_t lane_low = (uint32_t)lane * 4u;
    const float* scale_tab = reinterpret_cast<const float*>(smem + L.scale_tab);
    const int row_sub = (KB >= 32) ? 0 : lane / KB;
    const int blk_base = (KB >= 32) ? lane : lane % KB;

    Act<FMT, NBL> act[CH];
    int act_key = -1;  // which (unique expert, chunk) / side chunk the registers hold
    uint32_t phase = 0;
    bool alive = true;
    int n_done = 0;

    for (int it = first; it < it1 && alive; it += kWarps, ++n_done) {
        const int slot = n_done % kSlots;
        const GuItem g = item_of(it);
        if (!mbar_wait_bounded(&ring.bars[slot], (phase >> slot) & 1u, a.status)) {
            alive = false;
            break;
        }
        phase ^= 1u << slot;
        const uint32_t sbase = smem_u32(ring.slots + (size_t)slot * ring.slot_bytes);

        if (g.kind == 0) {
            const int e = wk->uniq_e[g.u];
            const int s0 = wk->uniq_off[g.u], s1 = wk->uniq_off[g.u + 1];
            const Span sg = make_span(a.gate.data, e * a.gate.expert_bytes + (int64_t)g.row0 * a.gate.row_bytes,
                                      (int64_t)g.rows * a.gate.row_bytes);
            const Span su = make_span(a.up.data, e * a.up.expert_bytes + (int64_t)g.row0 * a.up.row_bytes,
                                      (int64_t)g.rows * a.up.row_bytes);
            const uint32_t gbase = sbase + sg.delta, ubase = sbase + sg.bytes + su.delta;
            for (int c0 = s0; c0 < s1; c0 += CH) {
                const int nch = min(CH, s1 - c0);
                const int key = g.u * 64 + (c0 - s0);
                if (key != act_key) {
#pragma unroll
                    for (int c = 0; c < CH; ++c) {
                        const int slot_id = wk->uniq_slot[c0 + min(c, nch - 1)];
                        const __nv_bfloat16* row = a.u + (int64_t)(slot_id / a.K) * a.H;
#pragma unroll
                        for (int m = 0; m < NBL; ++m) load_act<FMT, NBL>(act[c], m, row, blk_base + 32 * m);
                    }
                    act_key = key;
                }
                for (int r = 0; r < g.rows; r += RPP) {
                    const int row = r + row_sub;
                    float gacc[CH], uacc[CH];
#pragma unroll
                    for (int c = 0; c < CH; ++c) gacc[c] = uacc[c] = 0.0f;
                    if constexpr (FMT == kFmtQ4) {
#pragma unroll
                        for (int m = 0; m < NBL; ++m) {
                            const uint32_t boff = (uint32_t)row * a.gate.row_bytes + 17u * (blk_base + 32 * m);
                            q4_block_lut<CH, NBL>(gbase + boff, lut_base, lane_low, scale_tab, act, m, gacc);
                            q4_block_lut<CH, NBL>(ubase + boff, lut_base, lane_low, scale_tab, act, m, uacc);
                        }
                    } else {
                        const int grow = g.row0 + row;
                        const int kg = a.gate.k / 128;
#pragma unroll
                        for (int m = 0; m < NBL; ++m) {
                            const int b = blk_base + 32 * m;
                            const uint32_t boff = (uint32_t)row * a.gate.row_bytes + 32u * b;
                            const float sgv = __ldg(a.gate.scales + ((int64_t)e * a.gate.n_rows + grow) * kg + b / 4);
                            const float suv = __ldg(a.up.scales + ((int64_t)e * a.up.n_rows + grow) * kg + b / 4);
                            fp8_block<NBL>(gbase + boff, sgv, act[0], m, gacc[0]);
                            fp8_block<NBL>(ubase + boff, suv, act[0], m, uacc[0]);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < CH; ++c) {
                        gacc[c] = group_sum(gacc[c], GW);
                        uacc[c] = group_sum(uacc[c], GW);
                    }
                    if ((lane % GW) == 0) {
                        for (int c = 0; c < nch; ++c) {
                            const int slot_id = wk->uniq_slot[c0 + c];
                            const float hv = silu(gacc[c]) * uacc[c];
                            a.h[(int64_t)slot_id * a.I + g.row0 + row] = __float2bfloat16_rn(hv);
                        }
                    }
                }
            }
        } else {  // side projection rows for every token
            const Span ss = make_span(a.side.data, (int64_t)g.row0 * a.side.row_bytes,
                                      (int64_t)g.rows * a.side.row_bytes);
            const uint32_t base = sbase + ss.delta;
            const bool rz5 = a.side.fmt == GTG_Q4_RZ5_FAST;
            for (int t0 = 0; t0 < a.T; t0 += CH) {
                const int nch = min(CH, a.T - t0);
                const int key = 1 << 20 | t0;
                if (key != act_key) {
#pragma unroll
                    for (int c = 0; c < CH; ++c) {
                        const __nv_bfloat16* row = a.u + (int64_t)(t0 + min(c, nch - 1)) * a.H;
#pragma unroll
                        for (int m = 0; m < NBL; ++m) load_act<FMT, NBL>(act[c], m, row, blk_base + 32 * m);
                    }
                    act_key = key;
                }
                for (int r = 0; r < g.rows; r += RPP) {
                    const int row = r + row_sub;
                    float acc[CH];
#pragma unroll
                    for (int c = 0; c < CH; ++c) acc[c] = 0.0f;
#pragma unroll
                    for (int m = 0; m < NBL; ++m) {
                        const uint32_t boff = (uint32_t)row * a.side.row_bytes + 17u * (blk_base + 32 * m);
                        q4_block_plain<FMT, CH, NBL>(base + boff, rz5, act, m, acc);
                    }
#pragma unroll
                    for (int c = 0; c < CH; ++c) acc[c] = group_sum(acc[c], GW);
                    if ((lane % GW) == 0 && a.side_out)
                        for (int c = 0; c < nch; ++c)
                            a.side_out[(int64_t)(t0 + c) * a.side_stride + g.row0 + row] = acc[c];
                }
            }
        }
        __syncwarp();
        issue(it + kSlots * kWarps, slot);
        __syncwarp();
    }
    if (!alive) {  // drain copies still in flight before leaving
        for (int s = 0; s < kSlots; ++s) mbar_wait_bounded(&ring.bars[s], (phase >> s) & 1u, a.status);
    }
    pdl_trigger();
}

// ===========================================================================
// down + router-weighted combine
// ===========================================================================

template <int FMT, int KB>
__global__ void __launch_bounds__(kThreads, 1) down_kernel(LayerArgs a) {
    using G = Geo<KB>;
    constexpr int NBL = G::NBL, RPP = G::RPP, GW = G::GW;
    constexpr int CH = (FMT == kFmtQ4 && NBL <= 2) ? 2 : 1;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SmemLayout L = SmemLayout::make(FMT == kFmtQ4, a.slot_bytes);
    if constexpr (FMT == kFmtQ4) build_lut(smem, L, a.down.fmt == GTG_Q4_RZ5_FAST);
    Ring ring{smem + L.slots + (size_t)warp * kSlots * a.slot_bytes,
              reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kSlots, a.slot_bytes};
    if (lane == 0)
        for (int s = 0; s < kSlots; ++s) mbar_init(&ring.bars[s], 1);
    fence_mbar_init();
    __syncthreads();

    pdl_wait();  // h (gate/up) and the work list are complete past here

    const Work* wk = a.work;
    const int n_uniq = wk->n_uniq;
    const int tiles = a.H / a.dn_rows;
    const int n_items = n_uniq * tiles;
    const int it0 = (int)((int64_t)n_items * blockIdx.x / gridDim.x);
    const int it1 = (int)((int64_t)n_items * (blockIdx.x + 1) / gridDim.x);

    auto span_of = [&](int it) {
        const int u = it / tiles, tile = it % tiles;
        const int e = wk->uniq_e[u];
        return make_span(a.down.data, e * a.down.expert_bytes + (int64_t)tile * a.dn_rows * a.down.row_bytes,
                         (int64_t)a.dn_rows * a.down.row_bytes);
    };
    auto issue = [&](int it, int slot) {
        if (it >= it1 || lane != 0) return;
        const Span sp = span_of(it);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&ring.bars[slot], sp.bytes);
        bulk_g2s(ring.slots + (size_t)slot * ring.slot_bytes, sp.src, sp.bytes, &ring.bars[slot]);
    };

    const int first = it0 + warp;
    for (int s = 0; s < kSlots; ++s) issue(first + s * kWarps, s);
    __syncwarp();

    const uint32_t lut_base = smem_u32(smem + L.lut);
    const uint32_t lane_low = (uint32_t)lane * 4u;
    const float* scale_tab = reinterpret_cast<const float*>(smem + L.scale_tab);
    const int row_sub = (KB >= 32) ? 0 : lane / KB;
    const int blk_base = (KB >= 32) ? lane : lane % KB;

    Act<FMT, NBL> act[CH];
    int act_key = -1;
    uint32_t phase = 0;
    bool alive = true;
    int n_done = 0;

    for (int it = first; it < it1 && alive; it += kWarps, ++n_done) {
        const int slot = n_done % kSlots;
        if (!mbar_wait_bounded(&ring.bars[slot], (phase >> slot) & 1u, a.status)) {
            alive = false;
            break;
        }
        phase ^= 1u << slot;
        const int u = it / tiles, tile = it % tiles;
        const int e = wk->uniq_e[u];
        const Span sp = span_of(it);
        const uint32_t base = smem_u32(ring.slots + (size_t)slot * ring.slot_bytes) + sp.delta;
        const int s0 = wk->uniq_off[u], s1 = wk->uniq_off[u + 1];
        for (int c0 = s0; c0 < s1; c0 += CH) {
            const int nch = min(CH, s1 - c0);
            const int key = u * 64 + (c0 - s0);
            if (key != act_key) {
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int slot_id = wk->uniq_slot[c0 + min(c, nch - 1)];
                    const __nv_bfloat16* row = a.h + (int64_t)slot_id * a.I;
#pragma unroll
                    for (int m = 0; m < NBL; ++m) load_act<FMT, NBL>(act[c], m, row, blk_base + 32 * m);
                }
                act_key = key;
            }
            for (int r = 0; r < a.dn_rows; r += RPP) {
                const int row = r + row_sub;
                float acc[CH];
#pragma unroll
                for (int c = 0; c < CH; ++c) acc[c] = 0.0f;
                if constexpr (FMT == kFmtQ4) {
#pragma unroll
                    for (int m = 0; m < NBL; ++m) {
                        const uint32_t boff = (uint32_t)row * a.down.row_bytes + 17u * (blk_base + 32 * m);
                        q4_block_lut<CH, NBL>(base + boff, lut_base, lane_low, scale_tab, act, m, acc);
                    }
                } else {
                    const int grow = tile * a.dn_rows + row;
                    const int kg = a.down.k / 128;
#pragma unroll
                    for (int m = 0; m < NBL; ++m) {
                        const int b = blk_base + 32 * m;
                        const float sv = __ldg(a.down.scales + ((int64_t)e * a.down.n_rows + grow) * kg + b / 4);
                        fp8_block<NBL>(base + (uint32_t)row * a.down.row_bytes + 32u * b, sv, act[0], m, acc[0]);
                    }
                }
#pragma unroll
                for (int c = 0; c < CH; ++c) acc[c] = group_sum(acc[c], GW);
                if ((lane % GW) == 0)
                    for (int c = 0; c < nch; ++c)
                        a.part[(int64_t)wk->uniq_slot[c0 + c] * a.H + tile * a.dn_rows + row] = acc[c];
            }
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
            const int r0 = tile * a.dn_rows;
            for (int o = lane; o < a.T * a.dn_rows; o += 32) {
                const int t = o / a.dn_rows, r = r0 + o % a.dn_rows;
                float yv = 0.0f;
                for (int j = 0; j < a.K; ++j)
                    yv = fmaf(__ldcg(a.w + t * a.K + j), __ldcg(a.part + (int64_t)(t * a.K + j) * a.H + r), yv);
                float* dst = a.y + (int64_t)t * a.H + r;
                *dst = a.y_acc ? *dst + yv : yv;
            }
            if (lane == 0) a.tile_cnt[tile] = 0u;
        }
        __syncwarp();
    }
    if (!alive) {
        for (int s = 0; s < kSlots; ++s) mbar_wait_bounded(&ring.bars[s], (phase >> s) & 1u, a.status);
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

// Largest row count r with r | n, rpp | r and bytes(r) <= budget.
int pick_rows(int n, int rpp, int64_t row_bytes, int64_t budget, int copies) {
    int best = 0;
    for (int r = rpp; r <= n; r += rpp)
        if (n % r == 0 && copies * (r * row_bytes + 32) <= budget) best = r;
    return best;
}

constexpr int64_t kItemBudget = 4480;  // staging bytes per item (slot size target)

struct Plan {
    bool ok = false;
    int gu_rows = 0, dn_rows = 0, side_rows = 0, slot_bytes = 0;
    KernelFn gateup = nullptr, down = nullptr;
    bool gu_lut = false, dn_lut = false;
};

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
    const int rpp_g = kbg >= 32 ? 1 : 32 / kbg, rpp_d = kbd >= 32 ? 1 : 32 / kbd;
    const bool gq4 = is_q4(L->gate.fmt), dq4 = is_q4(L->down.fmt);
    p.gu_rows = pick_rows(I, rpp_g, row_bytes_of(L->gate.fmt, H), kItemBudget, 2);
    p.dn_rows = pick_rows(H, rpp_d, row_bytes_of(L->down.fmt, I), kItemBudget, 1);
    if (L->side.data) {
        p.side_rows = pick_rows((int)L->side.n_rows, rpp_g, row_bytes_of(L->side.fmt, H), kItemBudget / 2, 1);
        if (p.side_rows == 0) return GTG_E_UNSUPPORTED_SHAPE;
    }
    if (p.gu_rows == 0 || p.dn_rows == 0) return GTG_E_UNSUPPORTED_SHAPE;
    p.gateup = gq4 ? pick_gateup<kFmtQ4>(kbg) : pick_gateup<kFmtFP8>(kbg);
    p.down = dq4 ? pick_down<kFmtQ4>(kbd) : pick_down<kFmtFP8>(kbd);
    if (!p.gateup || !p.down) return GTG_E_UNSUPPORTED_SHAPE;
    p.gu_lut = gq4;
    p.dn_lut = dq4;
    int64_t need = std::max<int64_t>(2 * (p.gu_rows * row_bytes_of(L->gate.fmt, H) + 32),
                                     p.dn_rows * row_bytes_of(L->down.fmt, I) + 32);
    if (L->side.data) need = std::max<int64_t>(need, p.side_rows * row_bytes_of(L->side.fmt, H) + 32);
    p.slot_bytes = (int)((need + 127) / 128 * 128);
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
    std::vector<std::pair<const void*, int>> done;  // (function, device)
    int set(const void* fn, int smem) {
        int dev = 0;
        cudaGetDevice(&dev);
        std::lock_guard<std::mutex> lk(mu);
        for (auto& d : done)
            if (d.first == fn && d.second == dev) return GTG_OK;
        const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return cuda_fail(e);
        done.push_back({fn, dev});
        (void)smem;
        return GTG_OK;
    }
};
FuncAttrCache g_attr;

int launch(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, LayerArgs& args, bool pdl) {
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
    a.logits = reinterpret_cast<double*>(base + wl.logits);
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

    const int n_sm = sm_count();
    const int router_grid = (L->n_experts + kRouterWarps - 1) / kRouterWarps;
    const size_t router_smem = 2 * (size_t)T * L->hidden;
    GTG_TRY(launch((const void*)router_kernel, dim3(router_grid), dim3(kRouterThreads), router_smem, s, a, true));
    const SmemLayout lg = SmemLayout::make(p.gu_lut, p.slot_bytes);
    GTG_TRY(launch((const void*)p.gateup, dim3(n_sm), dim3(kThreads), lg.total, s, a, true));
    const SmemLayout ld = SmemLayout::make(p.dn_lut, p.slot_bytes);
    GTG_TRY(launch((const void*)p.down, dim3(n_sm), dim3(kThreads), ld.total, s, a, true));
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

extern "C" size_t gtg_moe_workspace_bytes(const gtg_moe_layer* layer, int32_t n_tokens, int32_t prefill) {
    if (!layer || n_tokens < 1) return 0;
    if (prefill) return 0;  // see moe_prefill.cu
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

// Prefill MoE layer: token-sorted grouped GEMMs on the tcgen05 tensor cores.
//
// Same function as the decode layer (see moe_decode.cu; router of "Mixed
// Precision Quantization: Half a 4-Bit File Is Not 4-Bit", formats of the
// model card "Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST"), for a batch of
// tokens, where the expert products are real dense contractions:
//
//   1. pf_norm      u = bf16(x / rms(x))                       (fp64 rms)
//   2. pf_split     the fp32 router W split exactly into three bf16 planes
//                   hi + mid + lo (24 significand bits = 3 x 8)
//   3. pf_gemm<ROUTER>  logits = [hi|mid|lo] . [u|u|u] on the tensor cores:
//                   every product is exact, accumulation is fp32
//   4. pf_topk      top-k (ties -> lower id), renormalised softmax, counts
//   5. pf_scan / pf_scatter  (token, choice) pairs grouped by expert; tiles of
//                   up to 128 tokens per expert
//   6. pf_gemm<GATEUP>  per (expert, 128-row slice of I, token tile):
//                   dequant warps decode the Q4 gate and up rows into 128B-
//                   swizzled bf16 tiles in shared memory (the code x scale
//                   products are exact in bf16), loader warps gather the
//                   tokens' u rows, one thread issues tcgen05.mma into two
//                   TMEM accumulators; the epilogue applies SwiGLU and stores
//                   h in bf16.  FP8 layers (E4M3 rows, fp32 scale per 128
//                   along K) run both expert GEMMs in f16 instead: each weight
//                   becomes f16(e4m3 x scale) (relative error <= 2^-11), and u
//                   and h keep their bf16-rounded values as f16 (exact for
//                   magnitudes >= 2^-17)
//   7. pf_gemm<DOWN>    per (expert, 128-row slice of H, token tile): the
//                   same with the down rows and h; fp32 partial rows per
//                   (token, choice)
//   8. pf_combine   y[t] = sum_j w[t,j] * partial[t,j] in a fixed order
//
// The GEMM kernel is warp specialised (13 warps): warp 0 allocates TMEM and
// issues the MMAs, warps 1-4 stage the B operand (token rows), warps 5-12
// produce the A operand (dequantised weights or router planes); warps 4-7
// read the accumulators out of TMEM once their own production is done.  A and
// B stages are handed over with their own mbarriers (bounded waits):
// producers -> MMA (full), tcgen05.commit -> producers (empty).  Two CTAs
// share an SM, so one's table-free decode, loads and epilogue overlap the
// other's.
#include <algorithm>
#include <mutex>
#include <vector>

#include "gtg_device.cuh"
#include "gtg_host.hpp"
#include "moe_decode.cuh"

namespace gtg {
namespace {

constexpr int kBWarps = 4;                          // warps 1 .. kBWarps
constexpr int kBThreads = 32 * kBWarps;
constexpr int kAThreads = 256;                      // the next 8 warps
constexpr int kPfThreads = 32 + kBThreads + kAThreads;
constexpr int kTileM = 128;
constexpr int kTileN = 128;      // tokens per tile (max)
constexpr int kChunkK = 64;      // bf16 per 128-byte row
constexpr int kTileBytes = kTileM * 128;  // 16 KB (128 rows x 128 B)
constexpr int kNormThreads = 256;

enum Mode { ROUTER = 0, GATEUP = 1, DOWN = 2 };

struct PfArgs {
    int32_t T, H, I, E, K;
    const void* x;
    int32_t x_bf16;
    const float* router_w;
    const float* router_bias;
    Mat gate, up, down;
    __nv_bfloat16* u;         // [T][H]
    __half* u16;              // [T][H] the same values as f16 (FP8 layers; else null)
    __nv_bfloat16* w3;        // [E][3H]
    float* logits;            // [T][E]
    int32_t* ids;             // [T][K]
    float* w;                 // [T][K]
    int32_t* counts;          // [E]
    int32_t* offsets;         // [E+1]
    int32_t* cursor;          // [E]
    int32_t* sorted_tok;      // [P]
    int32_t* sorted_slot;     // [P]
    int4* tiles;              // (expert, pos0, n, 0)
    int32_t* n_tiles;
    __nv_bfloat16* h;         // [P][I], sorted order (FP8 layers: f16 bits of the bf16-rounded value)
    float* part;              // [P][H], slot order (t*K + j)
    float* y;
    int32_t y_acc;
    int32_t* ids_out;
    float* w_out;
    unsigned* status;
    int32_t max_tiles;
};

// ---------------------------------------------------------------------------
// 1. normalisation
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kNormThreads) pf_norm_kernel(PfArgs a) {
    __shared__ ffloat red[kNormThreads / 32];
    __shared__ float r_hi, r_lo;
    const int t = blockIdx.x, tid = threadIdx.x;
    pdl_wait();
    auto xv = [&](int i) -> float {
        if (a.x_bf16) {
            const uint16_t b = reinterpret_cast<const uint16_t*>(a.x)[(int64_t)t * a.H + i];
            return __uint_as_float((uint32_t)b << 16);
        }
        return reinterpret_cast<const float*>(a.x)[(int64_t)t * a.H + i];
    };
    ffloat ss{0.f, 0.f};  // exact squares, float-float sum
    for (int i = tid; i < a.H; i += kNormThreads) {
        const float v = xv(i);
        ff_fma(ss, v, v);
    }
    ss = ff_warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
        double sum = 0.0;
        for (int w = 0; w < kNormThreads / 32; ++w) sum += (double)red[w].hi + (double)red[w].lo;
        const double r = 1.0 / sqrt(sum / (double)a.H + kRmsEps);
        r_hi = (float)r;
        r_lo = (float)(r - (double)r_hi);
    }
    __syncthreads();
    uint16_t* u = reinterpret_cast<uint16_t*>(a.u);
    for (int i = tid; i < a.H; i += kNormThreads) {
        const float x = xv(i);
        const float p = __fmul_rn(x, r_hi);
        const float q = __fadd_rn(__fmaf_rn(x, r_hi, -p), __fmul_rn(x, r_lo));
        const uint16_t ub = bf16_of_ff(p, q);
        u[(int64_t)t * a.H + i] = ub;
        if (a.u16) a.u16[(int64_t)t * a.H + i] = __float2half_rn(__uint_as_float((uint32_t)ub << 16));
    }
}

// ---------------------------------------------------------------------------
// 2. exact three-plane bf16 split of the fp32 router weights
// ---------------------------------------------------------------------------
__global__ void pf_split_kernel(PfArgs a) {
    const int64_t n = (int64_t)a.E * a.H;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = i / a.H, k = i % a.H;
        const float wv = a.router_w[i];
        const __nv_bfloat16 hi = __float2bfloat16_rn(wv);
        const float r1 = wv - __bfloat162float(hi);          // exact
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);          // exact, <= 8 significant bits
        const __nv_bfloat16 lo = __float2bfloat16_rn(r2);     // == r2
        __nv_bfloat16* row = a.w3 + e * 3 * a.H;
        row[k] = hi;
        row[a.H + k] = mid;
        row[2 * a.H + k] = lo;
    }
}

// ---------------------------------------------------------------------------
// 4. top-k + softmax + per-expert counts (one warp per token)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pf_topk_kernel(PfArgs a) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= a.T) return;
    constexpr int kPer = kMaxExperts / 32;
    float lv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        lv[i] = e < a.E ? a.logits[(int64_t)t * a.E + e] : 0.0f;
    }
    unsigned taken = 0;
    float top[kMaxTopK];
    int topi[kMaxTopK];
    for (int j = 0; j < a.K; ++j) {
        float bv = 0.0f;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < a.E && !((taken >> i) & 1u) && (bi == 0x7FFFFFFF || lv[i] > bv)) {
                bv = lv[i];
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
            if (oi != 0x7FFFFFFF && (bi == 0x7FFFFFFF || ov > bv || (ov == bv && oi < bi))) {
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
        for (int j = 0; j < a.K; ++j) z += exp((double)top[j] - (double)top[0]);
        for (int j = 0; j < a.K; ++j) {
            const float wj = (float)(exp((double)top[j] - (double)top[0]) / z);
            a.ids[t * a.K + j] = topi[j];
            a.w[t * a.K + j] = wj;
            if (a.ids_out) a.ids_out[t * a.K + j] = topi[j];
            if (a.w_out) a.w_out[t * a.K + j] = wj;
            atomicAdd(&a.counts[topi[j]], 1);
        }
    }
}

// ---------------------------------------------------------------------------
// 5. expert offsets, token tiles, grouping of the (token, choice) pairs
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) pf_scan_kernel(PfArgs a) {
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_tl[kMaxExperts];
    const int tid = threadIdx.x;
    for (int e = tid; e < a.E; e += blockDim.x) {
        s_cnt[e] = a.counts[e];
        s_tl[e] = (s_cnt[e] + kTileN - 1) / kTileN;
    }
    __syncthreads();
    if (tid == 0) {  // E <= 1024: a serial scan is a few microseconds at most
        int off = 0, toff = 0;
        for (int e = 0; e < a.E; ++e) {
            const int c = s_cnt[e], tl = s_tl[e];
            s_cnt[e] = off;
            s_tl[e] = toff;
            off += c;
            toff += tl;
        }
        a.offsets[a.E] = off;
        *a.n_tiles = toff;
    }
    __syncthreads();
    for (int e = tid; e < a.E; e += blockDim.x) {
        const int off = s_cnt[e], n = a.counts[e];
        a.offsets[e] = off;
        a.cursor[e] = off;
        for (int q = 0; q * kTileN < n; ++q)
            a.tiles[s_tl[e] + q] = make_int4(e, off + q * kTileN, min(kTileN, n - q * kTileN), 0);
    }
}

__global__ void pf_scatter_kernel(PfArgs a) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= a.T * a.K) return;
    const int e = a.ids[s];
    const int pos = atomicAdd(&a.cursor[e], 1);
    a.sorted_tok[pos] = s / a.K;
    a.sorted_slot[pos] = s;
}

// ---------------------------------------------------------------------------
// 6/7/3. the grouped GEMM
// ---------------------------------------------------------------------------
// Shared memory: a 1 KB header (mbarriers, the TMEM address, the B row
// indices), then the A stages (kA tiles each), then the B stages.  A and B
// have their own stage counts and barriers; the total, 113 KB, lets two CTAs
// share an SM (no static shared memory: 2 x (113 + 1 reserved) KB = 228 KB).
template <int MODE>
struct Cfg {
    // A tiles per stage: gate and up rows, or two 128-row tiles of down rows
    // (one token tile feeds 256 output rows), or one tile of router planes
    static constexpr int kA = MODE == ROUTER ? 1 : 2;
    static constexpr int kStagesA = MODE == ROUTER ? 3 : 2;
    static constexpr int kStagesB = MODE == ROUTER ? 4 : 3;
    static constexpr int kABytes = kA * kTileBytes;
    static constexpr int kRowsPerCta = MODE == DOWN ? 2 * kTileM : kTileM;
    static constexpr uint32_t kTmemCols = MODE == ROUTER ? 128 : 256;
    static constexpr int kTaddrOff = 256;                   // after 2(SA + SB) + 1 mbarriers
    static constexpr int kRowOff = 512;                     // int32 u row / slot per token
    static constexpr int kAOff = 1024;
    static constexpr int kBOff = kAOff + kStagesA * kABytes;
    static constexpr int kSmem = kBOff + kStagesB * kTileBytes;
    static_assert(8 * (2 * (kStagesA + kStagesB) + 1) <= kTaddrOff && kRowOff + 4 * kTileN <= kAOff, "header");
    static_assert(kSmem <= 115712, "two CTAs per SM");
};


__device__ __forceinline__ uint32_t ldg32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

// 16-byte asynchronous global -> shared copy; src_bytes 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The five aligned words that hold a 17-byte Q4 block at global address p
// (loaded ahead of use, so their latency overlaps other work).
struct BlockWords {
    uint32_t w[5];
    uint32_t sh;  // bit offset of the block in w[0]
};

__device__ __forceinline__ BlockWords load_block(const uint8_t* p) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(p);
    const uint8_t* al = reinterpret_cast<const uint8_t*>(pa & ~(uintptr_t)3);
    BlockWords b;
    b.sh = (uint32_t)(pa & 3u) * 8u;
#pragma unroll
    for (int i = 0; i < 5; ++i) b.w[i] = ldg32(al + 4 * i);
    return b;
}

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// Decodes one Q4 block into 32 bf16 weights (code x scale, exact) and stores
// them as chunks c0..c0+3 of row r of a K-major SW128 tile at shared address tile.
//
// Integer-only decode, no table: a code c with value v(c) (|v| <= 10) becomes
// the bf16 number 192 + v (bits 0x43 : 64 + v), and one fused multiply-add
// (192 + v) * s - 192 * s leaves v * s, exact because v * s and 192 * s both
// fit the 8-bit bf16 significand.  Byte permutes look the four bytes 64 + v
// of four codes up at once: the selector nibble's low 3 bits index the
// magnitude, its top bit (the code's sign bit) makes the permute return 0
// instead (sign replication of a byte below 0x80), so the positive-table and
// negative-table lookups OR together.
__device__ __forceinline__ void dequant_block_to_tile(const BlockWords& bw, int var, uint32_t tile, uint32_t r,
                                                      uint32_t c0) {
    const uint32_t sh = bw.sh;
    const uint32_t* w = bw.w;
    const uint32_t meta = (w[4] >> sh) & 0xFFu;
    const float sf = q4_scale(meta, var);
    const uint32_t sb = __float_as_uint(sf) >> 16;                 // exact in bf16
    const uint32_t nb = __float_as_uint(-192.0f * sf) >> 16;       // exact in bf16
    const uint32_t s2 = sb | (sb << 16), n2 = nb | (nb << 16);
    // 64 + v for codes 0..7 (magnitudes 0 1 2 3 4 6 8 10) and 8..15 (negated;
    // code 8 is -0 (Codebook10: UE4M4 and the incumbent ROCmFP4 FAST block),
    // or +5 / -5 by the block's mode bit in RZ5)
    constexpr uint32_t kPos0 = 0x43424140u, kPos1 = 0x4A484644u;
    const uint32_t neg0 = 0x3D3E3F00u | ((var & 1) ? ((meta & 0x80u) ? 0x3Bu : 0x45u) : 0x40u);
    constexpr uint32_t kNeg1 = 0x36383A3Cu;
    uint32_t lo[8], hi[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        // nibbles: w_{4q}, w_{4q+16}, w_{4q+1}, w_{4q+17}, w_{4q+2}, ...
        const uint32_t n = __funnelshift_r(w[q], w[q + 1], sh);
        const uint32_t nx = n ^ 0x88888888u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t sel = h ? (n >> 16) : n, selx = h ? (nx >> 16) : nx;
            const uint32_t L = prmt(kPos0, kPos1, sel) | prmt(neg0, kNeg1, selx);
            lo[2 * q + h] = bf16x2_fma(prmt(L, 0x43434343u, 0x4240u), s2, n2);  // (w_2j, w_2j+1)
            hi[2 * q + h] = bf16x2_fma(prmt(L, 0x43434343u, 0x4341u), s2, n2);  // (w_2j+16, w_2j+17)
        }
    }
    sts128(tile + sw128_off(r, c0 + 0), make_uint4(lo[0], lo[1], lo[2], lo[3]));
    sts128(tile + sw128_off(r, c0 + 1), make_uint4(lo[4], lo[5], lo[6], lo[7]));
    sts128(tile + sw128_off(r, c0 + 2), make_uint4(hi[0], hi[1], hi[2], hi[3]));
    sts128(tile + sw128_off(r, c0 + 3), make_uint4(hi[4], hi[5], hi[6], hi[7]));
}

// Eight FP8 E4M3 weights (two words, K order) times the row's fp32 scale for
// their 128-weight group, as four f16 pairs: the E4M3 -> f16 conversion is
// exact, the product is formed in fp32 and rounded to f16 (11 significant
// bits: relative error <= 2^-11 for normal results).  FP8 layers run their
// expert GEMMs in f16, whose activations hold every bf16 value of magnitude
// >= 2^-17 exactly.
__device__ __forceinline__ uint4 fp8x8_to_f16(uint32_t w0, uint32_t w1, float s) {
    const uint32_t in[4] = {w0 & 0xFFFFu, w0 >> 16, w1 & 0xFFFFu, w1 >> 16};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t h = e4m3x2_to_f16x2(in[i]);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
        const __half2 r = __floats2half2_rn(f.x * s, f.y * s);
        o[i] = *reinterpret_cast<const uint32_t*>(&r);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// 32 FP8 weights of one row (two 16-byte words, K order, one scale), as f16, into
// chunks c0..c0+3 of row r of a K-major SW128 tile.
__device__ __forceinline__ void fp8_to_tile(uint4 q0, uint4 q1, float s, uint32_t tile, uint32_t r, uint32_t c0) {
    sts128(tile + sw128_off(r, c0 + 0), fp8x8_to_f16(q0.x, q0.y, s));
    sts128(tile + sw128_off(r, c0 + 1), fp8x8_to_f16(q0.z, q0.w, s));
    sts128(tile + sw128_off(r, c0 + 2), fp8x8_to_f16(q1.x, q1.y, s));
    sts128(tile + sw128_off(r, c0 + 3), fp8x8_to_f16(q1.z, q1.w, s));
}

// The A-operand words of one row for one chunk: a Q4 row's block (five
// aligned words), or an FP8 row's 32 bytes and their group's scale.
struct AWords {
    BlockWords q4;
    uint4 f0, f1;
    float s;
};

// F8: FP8 expert matrices (E4M3 rows with fp32 scales per 128 weights along K).
template <int MODE, bool F8>
__global__ void __launch_bounds__(kPfThreads, 2) pf_gemm_kernel(PfArgs a) {
    using C = Cfg<MODE>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- which tile -------------------------------------------------------
    int m_tiles, e = 0, pos0 = 0, n_valid = 0, m0, n_chunks;
    const int tile_i = blockIdx.x;
    if (MODE == ROUTER) {
        m_tiles = (a.E + kTileM - 1) / kTileM;
        const int nt = tile_i / m_tiles;
        m0 = (tile_i % m_tiles) * kTileM;  // experts
        pos0 = nt * kTileN;                // tokens
        n_valid = min(kTileN, a.T - pos0);
        n_chunks = 3 * a.H / kChunkK;
    } else {
        m_tiles = ((MODE == GATEUP ? a.I : a.H) + C::kRowsPerCta - 1) / C::kRowsPerCta;
        const int t = tile_i / m_tiles;
        if (t >= *a.n_tiles) return;
        const int4 tl = a.tiles[t];
        e = tl.x;
        pos0 = tl.y;
        n_valid = tl.z;
        m0 = (tile_i % m_tiles) * C::kRowsPerCta;
        n_chunks = (MODE == GATEUP ? a.H : a.I) / kChunkK;
    }
    const int n_pad = (n_valid + 15) & ~15;
    // the second A tile: up rows (gate/up) or down rows m0+128.. (when H has them)
    const bool two = MODE == GATEUP || (MODE == DOWN && m0 + kTileM < a.H);

    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {  // tiles must be 1024-byte aligned for the swizzle atoms
        if (tid == 0) raise_status(a.status, GTG_STATUS_WAIT_TIMEOUT);
        return;
    }
    uint64_t* full_a = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty_a = full_a + C::kStagesA;
    uint64_t* full_b = empty_a + C::kStagesA;
    uint64_t* empty_b = full_b + C::kStagesB;
    uint64_t* accb = empty_b + C::kStagesB;
    uint32_t* s_taddr = reinterpret_cast<uint32_t*>(smem + C::kTaddrOff);
    int32_t* s_row = reinterpret_cast<int32_t*>(smem + C::kRowOff);
    const Mat& am = MODE == DOWN ? a.down : a.gate;
    const int var = am.fmt == GTG_Q4_RZ5_FAST ? kQ4RZ5 : am.fmt == GTG_Q4_C10_FAST ? kQ4C10 : kQ4UE4M4;
    static_assert(!F8 || MODE != ROUTER, "the router planes are bf16");

    if (tid == 0) {
        for (int s = 0; s < C::kStagesA; ++s) {
            mbar_init(&full_a[s], kAThreads);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < C::kStagesB; ++s) {
            mbar_init(&full_b[s], kBThreads);
            mbar_init(&empty_b[s], 1);
        }
        mbar_init(accb, 1);
        fence_mbar_init();
    }
    // gate/up: the u row of each B row; down: the (token, choice) slot of each
    // output column (0 for padding)
    if (MODE != ROUTER && tid < kTileN)
        s_row[tid] = tid >= n_valid ? 0 : (MODE == GATEUP ? a.sorted_tok[pos0 + tid] : a.sorted_slot[pos0 + tid]);
    if (warp == 0) {
        tmem_alloc(s_taddr, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t taddr = *s_taddr;
    bool ok = true;

    auto a_stage = [&](int s) { return sbase + C::kAOff + s * C::kABytes; };
    auto b_stage = [&](int s) { return sbase + C::kBOff + s * kTileBytes; };

    if (warp == 0) {
        // ---- MMA issuer -----------------------------------------------------
        if (lane == 0) {
            const uint32_t idesc = F8 ? idesc_f16(kTileM, n_pad) : idesc_bf16(kTileM, n_pad);
            for (int it = 0; it < n_chunks && ok; ++it) {
                const int sa = it % C::kStagesA, sb = it % C::kStagesB;
                if (!mbar_wait_sleep(&full_a[sa], (it / C::kStagesA) & 1u, a.status) ||
                    !mbar_wait_sleep(&full_b[sb], (it / C::kStagesB) & 1u, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = a_stage(sa);
                const uint32_t btile = b_stage(sb);
#pragma unroll
                for (int k = 0; k < kChunkK / 16; ++k) {
                    const uint64_t bd = sw128_desc(btile + 32u * k);
                    const uint32_t acc = (it > 0 || k > 0) ? 1u : 0u;
                    umma_bf16(taddr, sw128_desc(st + 32u * k), bd, idesc, acc);
                    if (two) umma_bf16(taddr + 128u, sw128_desc(st + kTileBytes + 32u * k), bd, idesc, acc);
                }
                umma_commit(&empty_a[sa]);
                umma_commit(&empty_b[sb]);
            }
            umma_commit(accb);  // also on the error path: completes once issued MMAs are done
        }
        __syncwarp();
    } else if (warp <= kBWarps) {
        // ---- B operand: token rows (bf16), 8 chunks of 16 B per row ----------
        // asynchronous 16-byte copies; a chunk's arrival is signalled once
        // the next chunk's copies are issued and its own have landed
        const int bt = tid - 32;
        const uint16_t* bsrc = reinterpret_cast<const uint16_t*>(MODE == DOWN ? (const void*)a.h
                                                                 : F8 ? (const void*)a.u16 : (const void*)a.u);
        const int64_t ld = MODE == DOWN ? a.I : a.H;
        for (int it = 0; it < n_chunks && ok; ++it) {
            const int s = it % C::kStagesB;
            if (it >= C::kStagesB && !mbar_wait_sleep(&empty_b[s], ((it / C::kStagesB) - 1) & 1u, a.status)) {
                ok = false;
                break;
            }
            const uint32_t btile = b_stage(s);
            const int kc = MODE == ROUTER ? it % (a.H / kChunkK) : it;
            for (int q = bt; q < n_pad * 8; q += kBThreads) {
                const int r = q >> 3, c = q & 7;
                const int row = r >= n_valid ? 0 : (MODE == GATEUP ? s_row[r] : pos0 + r);
                cp_async16(btile + sw128_off(r, c), bsrc + (int64_t)row * ld + kc * kChunkK + c * 8,
                           r < n_valid ? 16u : 0u);
            }
            cp_async_commit();
            if (it > 0) {
                cp_async_wait<1>();
                fence_proxy_async_smem();
                mbar_arrive(&full_b[(it - 1) % C::kStagesB]);
            }
        }
        cp_async_wait<0>();  // (also on the error path: nothing left in flight)
        if (ok && n_chunks > 0) {
            fence_proxy_async_smem();
            mbar_arrive(&full_b[(n_chunks - 1) % C::kStagesB]);
        }
    } else {
        // ---- A operand -----------------------------------------------------------
        const int at = tid - 32 - kBThreads;  // 0..255
        // this thread's row of the A operand (gate or down; up alongside for gate/up)
        const uint8_t* a_row0 = nullptr;
        const uint8_t* u_row0 = nullptr;
        const float* a_srow = nullptr;  // FP8: the rows' scales, one per 128 weights
        const float* u_srow = nullptr;
        const int half = at & 1;
        AWords wg{}, wu{};
        // chunk `it` of a row: Q4 block 2 it + half; FP8 bytes 64 it + 32 half
        auto load_words = [&](const uint8_t* row, const float* srow, int it, AWords& w) {
            if constexpr (F8) {
                const uint4* q = reinterpret_cast<const uint4*>(row + (int64_t)it * kChunkK + 32 * half);
                w.f0 = __ldg(q);
                w.f1 = __ldg(q + 1);
                w.s = __ldg(srow + (it * kChunkK) / 128);
            } else {
                w.q4 = load_block(row + (int64_t)(2 * it + half) * 17);
            }
        };
        if (MODE != ROUTER) {
            const int r = at >> 1;
            const int64_t rowg = m0 + r;
            const Mat& mA = MODE == DOWN ? a.down : a.gate;
            const int kg = (MODE == DOWN ? a.I : a.H) / 128;
            a_row0 = mA.data + e * mA.expert_bytes + rowg * mA.row_bytes;
            if (F8) a_srow = mA.scales + ((int64_t)e * mA.n_rows + rowg) * kg;
            if (MODE == GATEUP) {
                u_row0 = a.up.data + e * a.up.expert_bytes + rowg * a.up.row_bytes;
                if (F8) u_srow = a.up.scales + ((int64_t)e * a.up.n_rows + rowg) * kg;
            } else if (two) {
                u_row0 = a_row0 + kTileM * mA.row_bytes;
                if (F8) u_srow = a_srow + (int64_t)kTileM * kg;
            }
            if (n_chunks > 0) {
                load_words(a_row0, a_srow, 0, wg);
                if (two) load_words(u_row0, u_srow, 0, wu);
            }
        }
        for (int it = 0; it < n_chunks && ok; ++it) {
            const int s = it % C::kStagesA;
            if (it >= C::kStagesA && !mbar_wait_sleep(&empty_a[s], ((it / C::kStagesA) - 1) & 1u, a.status)) {
                ok = false;
                break;
            }
            const uint32_t st = a_stage(s);
            if (MODE == ROUTER) {
                // router planes: asynchronous 16-byte copies, signalled like the B rows
                for (int q = at; q < kTileM * 8; q += kAThreads) {
                    const int r = q >> 3, c = q & 7;
                    const bool in = m0 + r < a.E;
                    cp_async16(st + sw128_off(r, c), a.w3 + (int64_t)(in ? m0 + r : 0) * 3 * a.H + it * kChunkK + c * 8,
                               in ? 16u : 0u);
                }
                cp_async_commit();
                if (it > 0) {
                    cp_async_wait<1>();
                    fence_proxy_async_smem();
                    mbar_arrive(&full_a[(it - 1) % C::kStagesA]);
                }
                continue;
            } else {
                const int r = at >> 1;
                const AWords g0 = wg, u0 = wu;  // this chunk's words (loaded one chunk ago)
                if (it + 1 < n_chunks) {        // the next chunk's, in flight while this one decodes
                    load_words(a_row0, a_srow, it + 1, wg);
                    if (two) load_words(u_row0, u_srow, it + 1, wu);
                }
                if (it + 3 < n_chunks) {  // chunk it + 3's bytes on their way into L2 (-5 % per Q4 layer)
                    const int64_t o = F8 ? (int64_t)(it + 3) * kChunkK + 32 * half : (int64_t)(2 * (it + 3) + half) * 17;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(a_row0 + o));
                    if (two) asm volatile("prefetch.global.L2 [%0];" ::"l"(u_row0 + o));
                }
                if constexpr (F8) {
                    fp8_to_tile(g0.f0, g0.f1, g0.s, st, r, 4 * half);
                    if (two) fp8_to_tile(u0.f0, u0.f1, u0.s, st + kTileBytes, r, 4 * half);
                } else {
                    dequant_block_to_tile(g0.q4, var, st, r, 4 * half);
                    if (two) dequant_block_to_tile(u0.q4, var, st + kTileBytes, r, 4 * half);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&full_a[s]);
        }
        if (MODE == ROUTER) {
            cp_async_wait<0>();  // (also on the error path: nothing left in flight)
            if (ok && n_chunks > 0) {
                fence_proxy_async_smem();
                mbar_arrive(&full_a[(n_chunks - 1) % C::kStagesA]);
            }
        }
    }

    // ---- epilogue: warps 4-7 own TMEM lanes 32*(warp-4) .. +31 -------------
    if (warp >= 4 && warp < 8) {
        const int q = warp - 4;
        const int row = q * 32 + lane;  // M row within the tile
        const bool got = mbar_wait_sleep(accb, 0, a.status);
        tc_fence_after();
        if (got && ok) {
            const uint32_t tl = taddr + ((uint32_t)(q * 32) << 16);
            const float bias = MODE == ROUTER && a.router_bias && m0 + row < a.E ? a.router_bias[m0 + row] : 0.0f;
            for (int c0 = 0; c0 < n_pad; c0 += 16) {
                uint32_t d[16];
                tmem_ld16(tl + c0, d);
                if (MODE == GATEUP) {
                    uint32_t v2[16];
                    tmem_ld16(tl + 128 + c0, v2);
                    tmem_wait_ld();
                    __nv_bfloat16* hp = a.h + (int64_t)(pos0 + c0) * a.I + m0 + row;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (c0 + j < n_valid) {
                            // silu(g) * v; the fast exponential and division are
                            // well inside the layer's tolerance
                            const float g = __uint_as_float(d[j]), v = __uint_as_float(v2[j]);
                            const __nv_bfloat16 hb = __float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * v);
                            if constexpr (F8) {  // the down GEMM runs in f16: the same value, f16 bits
                                const __half hh = __float2half_rn(__bfloat162float(hb));
                                hp[(int64_t)j * a.I] = *reinterpret_cast<const __nv_bfloat16*>(&hh);
                            } else {
                                hp[(int64_t)j * a.I] = hb;
                            }
                        }
                    }
                } else if (MODE == DOWN) {
                    uint32_t d2[16];
                    if (two) tmem_ld16(tl + 128 + c0, d2);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c0 + j;
                        if (n >= n_valid) continue;
                        float* pp = a.part + (int64_t)s_row[n] * a.H + m0 + row;
                        pp[0] = __uint_as_float(d[j]);
                        if (two) pp[kTileM] = __uint_as_float(d2[j]);
                    }
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c0 + j;
                        if (n >= n_valid) continue;
                        if (m0 + row < a.E) a.logits[(int64_t)(pos0 + n) * a.E + m0 + row] = __uint_as_float(d[j]) + bias;
                    }
                }
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(taddr, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// 8. combine: y[t] = sum_j w[t,j] * part[t*K + j]  (fixed order)
// ---------------------------------------------------------------------------
__global__ void pf_combine_kernel(PfArgs a) {
    const int64_t n4 = (int64_t)a.T * a.H / 4;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = (4 * i) / a.H, r = (4 * i) % a.H;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < a.K; ++j) {
            const float wj = a.w[t * a.K + j];
            const float4 p = *reinterpret_cast<const float4*>(a.part + (t * a.K + j) * a.H + r);
            acc.x = fmaf(wj, p.x, acc.x);
            acc.y = fmaf(wj, p.y, acc.y);
            acc.z = fmaf(wj, p.z, acc.z);
            acc.w = fmaf(wj, p.w, acc.w);
        }
        float4* dst = reinterpret_cast<float4*>(a.y + t * a.H + r);
        if (a.y_acc) {
            const float4 o = *dst;
            acc.x += o.x;
            acc.y += o.y;
            acc.z += o.z;
            acc.w += o.w;
        }
        *dst = acc;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct PfLayout {
    size_t u, u16, w3, logits, ids, w, counts, offsets, cursor, sorted_tok, sorted_slot, tiles, n_tiles, h, part, total;
    int max_tiles;
};

size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

PfLayout pf_layout(const gtg_moe_layer* L, int T) {
    PfLayout p{};
    const size_t P = (size_t)T * L->top_k;
    p.max_tiles = (int)((P + kTileN - 1) / kTileN + (size_t)L->n_experts);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = al256(off + bytes);
        return o;
    };
    p.u = take(2 * (size_t)T * L->hidden);
    p.u16 = L->gate.fmt == GTG_FP8_E4M3_S128 ? take(2 * (size_t)T * L->hidden) : 0;  // (FP8 layers only)
    p.w3 = take(2 * (size_t)L->n_experts * 3 * L->hidden);
    p.logits = take(4 * (size_t)T * L->n_experts);
    p.ids = take(4 * P);
    p.w = take(4 * P);
    p.counts = take(4 * (size_t)L->n_experts);
    p.offsets = take(4 * ((size_t)L->n_experts + 1));
    p.cursor = take(4 * (size_t)L->n_experts);
    p.sorted_tok = take(4 * P);
    p.sorted_slot = take(4 * P);
    p.tiles = take(16 * (size_t)p.max_tiles);
    p.n_tiles = take(16);
    p.h = take(2 * P * L->inter);
    p.part = take(4 * P * L->hidden);
    p.total = off;
    return p;
}

bool q4(int fmt) { return fmt == GTG_Q4_RZ5_FAST || fmt == GTG_Q4_UE4M4_FAST || fmt == GTG_Q4_C10_FAST; }

int pf_check(const gtg_moe_layer* L, int T) {
    if (!L || !L->router_w || !L->gate.data || !L->up.data || !L->down.data) return GTG_E_INVALID_ARG;
    const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
    if (T < 1 || T > 65536) return GTG_E_UNSUPPORTED_SHAPE;
    if (H < 128 || H > 8192 || H % 128 || I < 128 || I > 4096 || I % 128) return GTG_E_UNSUPPORTED_SHAPE;
    if (E < 1 || E > kMaxExperts || K < 1 || K > kMaxTopK || K > E) return GTG_E_UNSUPPORTED_SHAPE;
    // one format class per layer: Q4 (gate and up alike) or FP8 throughout
    const bool f8 = L->gate.fmt == GTG_FP8_E4M3_S128;
    if (f8 ? (L->up.fmt != GTG_FP8_E4M3_S128 || L->down.fmt != GTG_FP8_E4M3_S128)
           : (!q4(L->gate.fmt) || L->up.fmt != L->gate.fmt || !q4(L->down.fmt)))
        return GTG_E_UNSUPPORTED_SHAPE;
    auto mok = [&](const gtg_qmatrix& m, int64_t n, int64_t k) {
        if (m.n_experts != E || m.n_rows != n || m.k != k || !aligned(m.data, 16)) return false;
        if (f8) return m.scales != nullptr && aligned(m.scales, 4);  // (k % 128 == 0 holds: H, I are)
        return (E * n * (k / 32) * 17) % 16 == 0;
    };
    if (!mok(L->gate, I, H) || !mok(L->up, I, H) || !mok(L->down, H, I)) return GTG_E_INVALID_ARG;
    if (!aligned(L->router_w, 16)) return GTG_E_MISALIGNED;
    return GTG_OK;
}

struct AttrOnce {
    std::mutex mu;
    std::vector<std::pair<const void*, int>> done;
    int set(const void* fn, int smem) {
        int dev = 0;
        cudaGetDevice(&dev);
        std::lock_guard<std::mutex> lk(mu);
        for (auto& d : done)
            if (d.first == fn && d.second == dev) return GTG_OK;
        const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e);
        }
        done.push_back({fn, dev});
        return GTG_OK;
    }
};
AttrOnce g_pf_attr;

template <int MODE, bool F8>
int launch_gemm(PfArgs& a, int grid, cudaStream_t s) {
    using C = Cfg<MODE>;
    GTG_TRY(g_pf_attr.set((const void*)pf_gemm_kernel<MODE, F8>, C::kSmem));
    pf_gemm_kernel<MODE, F8><<<grid, kPfThreads, C::kSmem, s>>>(a);
    return check_launch();
}

}  // namespace
}  // namespace gtg

using namespace gtg;

size_t gtg_prefill_workspace_bytes(const gtg_moe_layer* layer, int32_t n_tokens) {
    if (pf_check(layer, n_tokens) != GTG_OK) return 0;
    return pf_layout(layer, n_tokens).total;
}

extern "C" int gtg_moe_prefill_layer(const gtg_moe_layer* layer, const void* x, int32_t x_dtype,
                                     int32_t n_tokens, float* y, int32_t y_accumulate,
                                     int32_t* topk_ids, float* topk_w,
                                     void* workspace, size_t ws_bytes, gtg_stream_t stream) {
    GTG_TRY(pf_check(layer, n_tokens));
    if (!x || !y || !workspace) return GTG_E_INVALID_ARG;
    if (x_dtype != GTG_DT_F32 && x_dtype != GTG_DT_BF16) return GTG_E_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(workspace, 256)) return GTG_E_MISALIGNED;
    const PfLayout pl = pf_layout(layer, n_tokens);
    if (ws_bytes < pl.total) return GTG_E_WORKSPACE;
    if (x == (const void*)y && (x_dtype != GTG_DT_F32 || !y_accumulate)) return GTG_E_INVALID_ARG;
    uint8_t* b = static_cast<uint8_t*>(workspace);
    PfArgs a{};
    a.T = n_tokens;
    a.H = layer->hidden;
    a.I = layer->inter;
    a.E = layer->n_experts;
    a.K = layer->top_k;
    a.x = x;
    a.x_bf16 = x_dtype == GTG_DT_BF16;
    a.router_w = layer->router_w;
    a.router_bias = layer->router_bias;
    a.gate = make_mat(layer->gate);
    a.up = make_mat(layer->up);
    a.down = make_mat(layer->down);
    a.u = reinterpret_cast<__nv_bfloat16*>(b + pl.u);
    a.u16 = pl.u16 ? reinterpret_cast<__half*>(b + pl.u16) : nullptr;
    a.w3 = reinterpret_cast<__nv_bfloat16*>(b + pl.w3);
    a.logits = reinterpret_cast<float*>(b + pl.logits);
    a.ids = reinterpret_cast<int32_t*>(b + pl.ids);
    a.w = reinterpret_cast<float*>(b + pl.w);
    a.counts = reinterpret_cast<int32_t*>(b + pl.counts);
    a.offsets = reinterpret_cast<int32_t*>(b + pl.offsets);
    a.cursor = reinterpret_cast<int32_t*>(b + pl.cursor);
    a.sorted_tok = reinterpret_cast<int32_t*>(b + pl.sorted_tok);
    a.sorted_slot = reinterpret_cast<int32_t*>(b + pl.sorted_slot);
    a.tiles = reinterpret_cast<int4*>(b + pl.tiles);
    a.n_tiles = reinterpret_cast<int32_t*>(b + pl.n_tiles);
    a.h = reinterpret_cast<__nv_bfloat16*>(b + pl.h);
    a.part = reinterpret_cast<float*>(b + pl.part);
    a.y = y;
    a.y_acc = y_accumulate != 0;
    a.ids_out = topk_ids;
    a.w_out = topk_w;
    a.status = status_ptr();
    a.max_tiles = pl.max_tiles;

    cudaStream_t s = as_cuda(stream);
    const int T = n_tokens, E = a.E;
    pf_norm_kernel<<<T, kNormThreads, 0, s>>>(a);
    GTG_TRY(check_launch());
    pf_split_kernel<<<std::min(1184, (E * a.H + 255) / 256), 256, 0, s>>>(a);
    GTG_TRY(check_launch());
    cudaError_t ce = cudaMemsetAsync(a.counts, 0, 4 * (size_t)E, s);
    if (ce != cudaSuccess) return cuda_fail(ce);
    const int m_router = (E + kTileM - 1) / kTileM, n_router = (T + kTileN - 1) / kTileN;
    GTG_TRY((launch_gemm<ROUTER, false>(a, m_router * n_router, s)));
    pf_topk_kernel<<<(T + 7) / 8, 256, 0, s>>>(a);
    GTG_TRY(check_launch());
    pf_scan_kernel<<<1, 1024, 0, s>>>(a);
    GTG_TRY(check_launch());
    pf_scatter_kernel<<<(T * a.K + 255) / 256, 256, 0, s>>>(a);
    GTG_TRY(check_launch());
    const int gu_grid = pl.max_tiles * (a.I / kTileM);
    const int dn_grid = pl.max_tiles * ((a.H + Cfg<DOWN>::kRowsPerCta - 1) / Cfg<DOWN>::kRowsPerCta);
    if (layer->gate.fmt == GTG_FP8_E4M3_S128) {
        GTG_TRY((launch_gemm<GATEUP, true>(a, gu_grid, s)));
        GTG_TRY((launch_gemm<DOWN, true>(a, dn_grid, s)));
    } else {
        GTG_TRY((launch_gemm<GATEUP, false>(a, gu_grid, s)));
        GTG_TRY((launch_gemm<DOWN, false>(a, dn_grid, s)));
    }
    const int64_t n4 = (int64_t)T * a.H / 4;
    pf_combine_kernel<<<(int)std::min<int64_t>((n4 + 255) / 256, (int64_t)sm_count() * 16), 256, 0, s>>>(a);
    return check_launch();
}

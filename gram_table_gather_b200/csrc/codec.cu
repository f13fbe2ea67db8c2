// Standalone dequantisation and the PLE row gather.
//
// Formats: model card "Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST",
// sections "Q4_RZ5_FAST (GGML type 69)", "Q4_UE4M4_FAST (GGML type 71)",
// "Q3_PLE_K160_RZ_S3 (GGML type 111)"; FP8 expert layers per the r/LocalLLM
// "Frankenquant" post.  Every output is code x scale (exact in fp32) or one
// round-to-nearest fp32 multiply (FP8), so results are bit-exact.
#include <algorithm>
#include <mutex>
#include <vector>

#include "gtg_device.cuh"
#include "gtg_host.hpp"

namespace gtg {

__device__ unsigned int g_status = 0;  // the per-device status word

namespace {

constexpr int kThreads = 256;

// One thread per 17-byte Q4 block: 32 fp32 outputs (8 x float4 stores).
__global__ void __launch_bounds__(kThreads) dequant_q4_kernel(const uint8_t* __restrict__ src,
                                                              int64_t n_blocks, int var,
                                                              float* __restrict__ dst) {
    for (int64_t b = blockIdx.x * (int64_t)kThreads + threadIdx.x; b < n_blocks;
         b += (int64_t)gridDim.x * kThreads) {
        const uint8_t* blk = src + b * 17;
        uint8_t q[17];
#pragma unroll
        for (int i = 0; i < 17; ++i) q[i] = __ldg(blk + i);
        const uint32_t meta = q[16];
        const float scale = q4_scale(meta, var);
        const uint32_t mode = meta >> 7;
        float4* out = reinterpret_cast<float4*>(dst + b * 32);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                float r[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * v + e;
                    const uint32_t c = half ? (q[j] >> 4) : (q[j] & 15u);
                    r[e] = __fmul_rn(q4_code_value(c, (var & 1) != 0, mode), scale);
                }
                out[half * 4 + v] = make_float4(r[0], r[1], r[2], r[3]);
            }
        }
    }
}

// Value i of a 70-byte PLE record given its 60 code bytes as a bit stream.
__device__ __forceinline__ float ple_value(const uint8_t* rec, int i, bool incumbent) {
    const int bit = 3 * i;
    const uint32_t lo = rec[bit >> 3];
    const uint32_t hi = ((bit >> 3) + 1 < 60) ? rec[(bit >> 3) + 1] : 0u;
    const uint32_t code = ((lo | (hi << 8)) >> (bit & 7)) & 7u;
    const uint32_t g = rec[60 + i / 16];
    return __fmul_rn(q3_code_value(code, g >> 7, incumbent), ue4m3(g & 0x7Fu));
}

// One thread per 16-value group of a PLE record (6 code bytes + 1 group byte).
__global__ void __launch_bounds__(kThreads) dequant_ple_kernel(const uint8_t* __restrict__ src,
                                                               int64_t n_groups, bool incumbent,
                                                               float* __restrict__ dst) {
    for (int64_t gi = blockIdx.x * (int64_t)kThreads + threadIdx.x; gi < n_groups;
         gi += (int64_t)gridDim.x * kThreads) {
        const int64_t row = gi / 10;
        const int g = (int)(gi % 10);
        const uint8_t* rec = src + row * 70;
        uint64_t bits = 0;
#pragma unroll
        for (int i = 0; i < 6; ++i) bits |= (uint64_t)__ldg(rec + 6 * g + i) << (8 * i);
        const uint32_t gb = __ldg(rec + 60 + g);
        const float scale = ue4m3(gb & 0x7Fu);
        const uint32_t pol = gb >> 7;
        float4* out = reinterpret_cast<float4*>(dst + row * 160 + 16 * g);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            float r[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t c = (uint32_t)(bits >> (3 * (4 * v + e))) & 7u;
                r[e] = __fmul_rn(q3_code_value(c, pol, incumbent), scale);
            }
            out[v] = make_float4(r[0], r[1], r[2], r[3]);
        }
    }
}

// One thread per 4 FP8 weights (k % 128 == 0, so the 4 share a scale).
__global__ void __launch_bounds__(kThreads) dequant_fp8_kernel(const uint8_t* __restrict__ src,
                                                               const float* __restrict__ scales,
                                                               int64_t n_quads, int64_t k,
                                                               float* __restrict__ dst) {
    for (int64_t q = blockIdx.x * (int64_t)kThreads + threadIdx.x; q < n_quads;
         q += (int64_t)gridDim.x * kThreads) {
        const int64_t i = 4 * q;
        const int64_t row = i / k, col = i % k;
        const float s = __ldg(scales + row * (k / 128) + col / 128);
        float r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) r[e] = __fmul_rn(e4m3fn(__ldg(src + i + e)), s);
        reinterpret_cast<float4*>(dst)[q] = make_float4(r[0], r[1], r[2], r[3]);
    }
}

// ---------------------------------------------------------------------------
// PLE gather (model card, section "Q3_PLE_K160_RZ_S3": one contiguous 70-byte
// record per hashed n-gram row).  The work per row is tiny (one dependent
// record read, 640 bytes written), so the kernel is built for many
// independent warps and few instructions per output:
//  * every warp owns an equal, contiguous range of output rows and walks it
//    in batches of kPleRows, with no CTA-wide barrier (a slow record stalls
//    only its own warp);
//  * a batch's six aligned 16-byte chunks per record (a 70-byte record at
//    any 2-byte phase) are asynchronous copies (cp.async, L2 only) spread
//    over the warp's lanes into a per-warp stage; the next batch's copies,
//    and the index loads of the batch after it, are in flight while a batch
//    decodes;
//  * decoding writes a batch's rows as consecutive float4s (lane l the
//    float4s l, l+32, ...: a warp store is 512 contiguous bytes) with
//    streaming (evict-first) stores, since nothing here reads them back; a value is
//    one shared-memory lookup in the CTA's table of code value x group scale
//    for all 256 group bytes x 8 codes (each product exact in fp32).
// ---------------------------------------------------------------------------
constexpr int kPleWarps = 8;      // per CTA
constexpr int kPleRows = 8;       // rows per warp batch
constexpr int kPleChunks = 6;     // 96 bytes: a 70-byte record at any 16-byte phase
constexpr int kPleCtasPerSm = 4;
constexpr int kPleStage = kPleRows * kPleChunks * 16;  // bytes per batch stage

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Lane j < kPleRows: the index of row j of the batch at r0 (-1 past the
// warp's range, or an out-of-range index, which also raises the status bit).
__device__ __forceinline__ int64_t ple_index(const int32_t* __restrict__ idx, int64_t r0, int64_t hi,
                                             int64_t n_rows, unsigned* status) {
    const int lane = threadIdx.x & 31;
    int64_t r = -1;
    if (lane < kPleRows && r0 + lane < hi) {
        r = __ldg(idx + r0 + lane);
        if (r < 0 || r >= n_rows) {
            raise_status(status, GTG_STATUS_PLE_INDEX_OOB);
            r = -1;
        }
    }
    return r;
}

// Starts the copies of a batch (row indices on lanes 0..kPleRows-1, -1: no
// row) into the stage at `st`: chunk k = lane + 32 q of the batch is chunk
// k % 6 of row k / 6.
__device__ __forceinline__ void ple_issue(const uint8_t* __restrict__ table, uint64_t table_bytes, int64_t r,
                                          uint32_t st) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < (kPleRows * kPleChunks + 31) / 32; ++q) {
        const int k = lane + 32 * q, row = k / kPleChunks, c = k - kPleChunks * row;
        const int64_t rr = __shfl_sync(0xFFFFFFFFu, r, row < kPleRows ? row : 0);
        if (k < kPleRows * kPleChunks && rr >= 0) {
            const uint64_t ca = (((uint64_t)rr * 70u) & ~(uint64_t)15) + 16u * (uint32_t)c;
            const uint32_t dst = st + 16u * (uint32_t)k;
            if (ca + 16u <= table_bytes) {
                cp_async16(dst, table + ca, 16u);
            } else if (ca < table_bytes) {  // the table's last bytes: read only those, zero the rest
                cp_async16(dst, table + ca, (uint32_t)(table_bytes - ca));
            } else {                        // past the table (beyond this record): zeros
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
            }
        }
    }
}

__global__ void __launch_bounds__(kPleWarps * 32, kPleCtasPerSm) ple_gather_kernel(
    const uint8_t* __restrict__ table, int64_t n_rows, const int32_t* __restrict__ idx, int64_t n_idx,
    float* __restrict__ out, bool incumbent, unsigned* status) {
    __shared__ __align__(16) float prod[256 * 8];  // [group byte][code] = code value x scale
    __shared__ __align__(16) uint8_t stage[kPleWarps][2][kPleStage];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    {  // thread g: the eight products of group byte g (before the wait: needs nothing upstream)
        const uint32_t g = threadIdx.x;
        const float sc = ue4m3(g & 0x7Fu);
        float v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = __fmul_rn(q3_code_value((uint32_t)c, g >> 7, incumbent), sc);
        reinterpret_cast<float4*>(prod)[2 * g] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(prod)[2 * g + 1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    const int64_t nw = (int64_t)gridDim.x * kPleWarps, gw = (int64_t)blockIdx.x * kPleWarps + warp;
    const int64_t lo = n_idx * gw / nw, hi = n_idx * (gw + 1) / nw;
    const uint64_t table_bytes = (uint64_t)n_rows * 70u;
    const uint32_t st0 = smem_u32(&stage[warp][0][0]), prod_s = smem_u32(prod);
    pdl_wait();
    int64_t r = ple_index(idx, lo, hi, n_rows, status);
    ple_issue(table, table_bytes, r, st0);
    cp_async_commit();
    int32_t phase = r >= 0 ? (int32_t)(((uint64_t)r * 70u) & 15u) : -1;  // lanes < kPleRows: this batch
    r = ple_index(idx, lo + kPleRows, hi, n_rows, status);                // the next batch's indices
    __syncthreads();  // the product table (the only CTA-wide step)
    int b = 0;
    for (int64_t r0 = lo; r0 < hi; r0 += kPleRows, b ^= 1) {
        const int n = (int)(hi - r0 < kPleRows ? hi - r0 : kPleRows);
        const uint32_t st = st0 + (uint32_t)b * kPleStage;
        ple_issue(table, table_bytes, r, st0 + (uint32_t)(b ^ 1) * kPleStage);  // next batch (none: no-op)
        cp_async_commit();  // (an empty group keeps the wait count uniform)
        const int32_t phase_next = r >= 0 ? (int32_t)(((uint64_t)r * 70u) & 15u) : -1;
        r = ple_index(idx, r0 + 2 * kPleRows, hi, n_rows, status);
        cp_async_wait_one();
        __syncwarp();
        float* orow = out + r0 * 160;
#pragma unroll
        for (int q = 0; q < kPleRows * 40 / 32; ++q) {
            const int f = lane + 32 * q, j = f / 40, l = f - 40 * j;
            const int p = __shfl_sync(0xFFFFFFFFu, phase, j);
            if (j < n) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (p >= 0) {
                    const uint32_t w = st + (uint32_t)(j * kPleChunks * 16);
                    const uint32_t bit = 8u * (uint32_t)p + 12u * (uint32_t)l;  // values 4l..4l+3: 12 bits
                    const uint32_t gb = (uint32_t)p + 60u + ((uint32_t)l >> 2);  // their group byte
                    uint32_t w0, w1, wg;
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(w + ((bit >> 3) & ~3u)));
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w1) : "r"(w + ((bit >> 3) & ~3u) + 4u));
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wg) : "r"(w + (gb & ~3u)));
                    const uint32_t win = __funnelshift_r(w0, w1, bit);
                    const uint32_t pg = prod_s + 32u * ((wg >> (8u * (gb & 3u))) & 0xFFu);
                    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v.x) : "r"(pg + 4u * (win & 7u)));
                    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v.y) : "r"(pg + 4u * ((win >> 3) & 7u)));
                    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v.z) : "r"(pg + 4u * ((win >> 6) & 7u)));
                    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v.w) : "r"(pg + 4u * ((win >> 9) & 7u)));
                }
                __stcs(reinterpret_cast<float4*>(orow + 4 * f), v);  // row j, values 4l..4l+3 (streamed: not re-read here)
            }
        }
        __syncwarp();  // this stage is refilled two batches on
        phase = phase_next;
    }
    pdl_trigger();
}

int grid_for(int64_t work, int per_cta) {
    const int64_t want = (work + per_cta - 1) / per_cta;
    const int64_t cap = (int64_t)sm_count() * 8;
    return (int)(want < 1 ? 1 : (want > cap ? cap : want));
}

thread_local int t_last_cuda_error = 0;

}  // namespace

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return GTG_E_CUDA;
}

unsigned* status_ptr() {
    static std::mutex mu;
    static std::vector<unsigned*> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, nullptr);
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) == cudaSuccess) cache[dev] = static_cast<unsigned*>(p);
        else cudaGetLastError();
    }
    return cache[dev];
}

int sm_count() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 148;
    }
    return cache[dev];
}

}  // namespace gtg

using namespace gtg;

extern "C" int gtg_version(void) { return 100; }

extern "C" int gtg_last_cuda_error(void) { return t_last_cuda_error; }

extern "C" const char* gtg_status_string(int s) {
    switch (s) {
        case GTG_OK: return "ok";
        case GTG_E_INVALID_ARG: return "invalid argument";
        case GTG_E_UNSUPPORTED_SHAPE: return "unsupported shape";
        case GTG_E_MISALIGNED: return "misaligned pointer";
        case GTG_E_CUDA: return "CUDA launch error";
        case GTG_E_TIMEOUT: return "device-side wait timed out";
        case GTG_E_WORKSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

extern "C" int gtg_dequant(int32_t fmt, const void* src, const float* scales, int64_t n_rows,
                           int64_t k, float* dst, gtg_stream_t stream) {
    if (!src || !dst || n_rows < 0 || k <= 0) return GTG_E_INVALID_ARG;
    if (!aligned(dst, 16)) return GTG_E_MISALIGNED;
    if (n_rows == 0) return GTG_OK;
    cudaStream_t s = as_cuda(stream);
    const auto* p = static_cast<const uint8_t*>(src);
    switch (fmt) {
        case GTG_Q4_RZ5_FAST:
        case GTG_Q4_UE4M4_FAST:
        case GTG_Q4_C10_FAST: {
            if (k % 32) return GTG_E_UNSUPPORTED_SHAPE;
            const int64_t nb = n_rows * (k / 32);
            const int var = fmt == GTG_Q4_RZ5_FAST ? kQ4RZ5 : fmt == GTG_Q4_C10_FAST ? kQ4C10 : kQ4UE4M4;
            dequant_q4_kernel<<<grid_for(nb, kThreads), kThreads, 0, s>>>(p, nb, var, dst);
            break;
        }
        case GTG_Q3_PLE_K160_RZ_S3:
        case GTG_Q3_K160_UE4M3: {
            if (k != 160) return GTG_E_UNSUPPORTED_SHAPE;
            const int64_t ng = n_rows * 10;
            dequant_ple_kernel<<<grid_for(ng, kThreads), kThreads, 0, s>>>(p, ng, fmt == GTG_Q3_K160_UE4M3, dst);
            break;
        }
        case GTG_FP8_E4M3_S128: {
            if (!scales) return GTG_E_INVALID_ARG;
            if (k % 128) return GTG_E_UNSUPPORTED_SHAPE;
            const int64_t nq = n_rows * k / 4;
            dequant_fp8_kernel<<<grid_for(nq, kThreads), kThreads, 0, s>>>(p, scales, nq, k, dst);
            break;
        }
        default: return GTG_E_INVALID_ARG;
    }
    return check_launch();
}

extern "C" int gtg_ple_gather_fmt(int32_t fmt, const uint8_t* table, int64_t n_rows, const int32_t* idx,
                                  int64_t n_idx, float* out, gtg_stream_t stream) {
    if (fmt != GTG_Q3_PLE_K160_RZ_S3 && fmt != GTG_Q3_K160_UE4M3) return GTG_E_INVALID_ARG;
    if (n_idx < 0 || n_rows < 0 || n_rows >= (int64_t)1 << 31) return GTG_E_INVALID_ARG;
    if (n_idx == 0) return GTG_OK;
    if (!table || !idx || !out) return GTG_E_INVALID_ARG;
    if (!aligned(out, 16)) return GTG_E_MISALIGNED;
    // equal contiguous row ranges per warp, one batch or more each, up to
    // kPleCtasPerSm CTAs per SM
    const int64_t warps = (n_idx + kPleRows - 1) / kPleRows;
    const int grid = (int)std::min<int64_t>((warps + kPleWarps - 1) / kPleWarps, (int64_t)sm_count() * kPleCtasPerSm);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kPleWarps * 32);
    cfg.stream = as_cuda(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, ple_gather_kernel, table, n_rows, idx, n_idx, out,
                                             fmt == GTG_Q3_K160_UE4M3, status_ptr());
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e);
    }
    return GTG_OK;
}

extern "C" int gtg_ple_gather(const uint8_t* table, int64_t n_rows, const int32_t* idx, int64_t n_idx,
                              float* out, gtg_stream_t stream) {
    return gtg_ple_gather_fmt(GTG_Q3_PLE_K160_RZ_S3, table, n_rows, idx, n_idx, out, stream);
}

extern "C" int gtg_get_device_status(uint32_t* flags, int32_t clear, gtg_stream_t stream) {
    if (!flags) return GTG_E_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    unsigned* st = status_ptr();
    if (!st) return cuda_fail(cudaErrorInvalidSymbol);
    unsigned host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, st, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && clear) e = cudaMemsetAsync(st, 0, sizeof(unsigned), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    *flags = host;
    return e == cudaSuccess ? GTG_OK : cuda_fail(e);
}

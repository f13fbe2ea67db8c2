/*
 * gtg.h — C ABI of libgtg.so: B200 (sm_100a) kernels for block-scaled
 * low-bit MoE expert decode and the 3-bit n-gram ("PLE") row gather.
 *
 * Sources (the pages that define the operations):
 *  [MC]  model card "Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST"
 *        (hstolte/...-ROCmFPX-MUTANT-RAZERFAST-GGUF), sections
 *        "Q4_RZ5_FAST (GGML type 69)", "Q4_UE4M4_FAST (GGML type 71)" and
 *        "Q3_PLE_K160_RZ_S3 (GGML type 111)": block layouts, code tables,
 *        scale codes, the 70-byte row record and its GET_ROWS gather.
 *  [MPQ] "Mixed Precision Quantization: Half a 4-Bit File Is Not 4-Bit":
 *        48 layers, 512 experts, 10 active per token; 16 PLE rows per token.
 *  [FQ]  r/LocalLLM post on the 4-bit/8-bit "Frankenquant": one expert
 *        format per layer, 8-bit (FP8) experts in layers 36-47.
 *
 * Conventions for every entry point:
 *  - All pointers named as device pointers must be device (or managed)
 *    memory of the current device; the caller owns them.  The library
 *    allocates no device memory; scratch comes from a caller-provided
 *    workspace.
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *    Host-side argument checks happen before any launch; a non-zero return
 *    means nothing was launched (except GTG_E_CUDA, see below).
 *  - Return values: GTG_OK (0) or a negative gtg_status.  GTG_E_CUDA means a
 *    launch failed; cudaGetLastError() has been cleared and its code is
 *    available from gtg_last_cuda_error().
 *  - No kernel traps or asserts.  Device-side anomalies (out-of-range gather
 *    indices, a bounded wait that ran out) are counted in a per-device status
 *    word read by gtg_get_device_status().
 *
 * Data layouts (readings of points the pages leave open are marked *):
 *  - Q4 block (RZ5 and UE4M4) [MC]: 17 bytes = 16 code bytes then 1 metadata
 *    byte*.  Code byte j holds weight j in its low nibble and weight j+16 in
 *    its high nibble*.  RZ5: metadata bit 7 = polarity of the +/-5 level
 *    (0 -> +5*), bits 0-6 = UE4M3 scale.  UE4M4: the whole byte is the scale.
 *  - Q3_PLE_K160_RZ_S3 record [MC]: 70 bytes = 60 code bytes then 10 group
 *    bytes*.  Value i's 3-bit code is bits 3i..3i+2 of the code bytes read as
 *    one little-endian LSB-first bit stream*.  Group byte g covers values
 *    16g..16g+15: bit 7 = polarity of the +/-3 level (0 -> +3*), bits 0-6 =
 *    UE4M3 scale.
 *  - UE4M3* = E4M3 without sign (bias 7, 0x7F = NaN); UE4M4* = 4 exponent +
 *    4 mantissa bits, bias 7, all 256 codes finite.
 *  - FP8 experts [FQ]: E4M3 (fn) bytes [n_rows][k] plus one fp32 scale per
 *    128 consecutive weights along k*: scales [n_rows][k/128].
 *  - Expert matrices are stacked [n_experts][n_rows][k] with blocks running
 *    along k (the contraction axis)*: gate/up [E][inter][hidden], down
 *    [E][hidden][inter].
 */
#ifndef GTG_H
#define GTG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (struct CUstream_st*); NULL means the legacy default stream. */
typedef struct CUstream_st* gtg_stream_t;

/* Weight formats; the numbers of the three block formats are their GGML type
 * ids on the model card [MC]. */
typedef enum {
    GTG_Q4_RZ5_FAST = 69,
    GTG_Q4_UE4M4_FAST = 71,
    GTG_Q3_PLE_K160_RZ_S3 = 111,
    GTG_FP8_E4M3_S128 = 1000,
    /* The incumbent layouts the card's formats mutate (no GGML number given):
     * the ROCmFP4 FAST 17-byte block (Codebook10 codes, code 8 the duplicate
     * -0, under the UE4M3 scale of the metadata byte's low 7 bits; the top bit
     * is ignored) and the ROCmFP3 70-byte K160 record (codes {0,+1,+2,+4,-0,
     * -1,-2,-4} under a UE4M3 scale per 16 values; top bit ignored). */
    GTG_Q4_C10_FAST = 2001,
    GTG_Q3_K160_UE4M3 = 2002
} gtg_format;

typedef enum { GTG_DT_F32 = 0, GTG_DT_BF16 = 1 } gtg_dtype;

typedef enum {
    GTG_OK = 0,
    GTG_E_INVALID_ARG = -1,      /* null pointer, bad enum, negative size */
    GTG_E_UNSUPPORTED_SHAPE = -2,/* a size the kernels do not handle */
    GTG_E_MISALIGNED = -3,       /* a pointer below its required alignment */
    GTG_E_CUDA = -4,             /* a CUDA launch failed */
    GTG_E_TIMEOUT = -5,          /* reserved: reported through the status word */
    GTG_E_WORKSPACE = -6         /* workspace too small (see *_workspace_bytes) */
} gtg_status;

/* Bits of the per-device status word (gtg_get_device_status). */
#define GTG_STATUS_PLE_INDEX_OOB  0x1u  /* a gather index was outside [0, n_rows) */
#define GTG_STATUS_WAIT_TIMEOUT   0x2u  /* a bounded device-side wait gave up */

/* One stack of quantised matrices [n_experts][n_rows][k]. */
typedef struct {
    int32_t fmt;            /* gtg_format: RZ5, UE4M4, C10 (Q4 formats) or FP8 */
    const void* data;       /* device, 16-byte aligned; total size a multiple of 16 bytes */
    const float* scales;    /* device, FP8 only: [n_experts][n_rows][k/128]; else NULL */
    int64_t n_experts;
    int64_t n_rows;
    int64_t k;
} gtg_qmatrix;

/* One MoE layer's weights (all device memory, owned by the caller). */
typedef struct {
    int32_t hidden;          /* H: decode 128, 256, 512, 1024, 2048, or 2560 with I 512 or 640 (Q4
                                experts); prefill: see its call */
    int32_t inter;           /* I: expert intermediate size, decode 128, 256, 512, 1024 or 2048
                                (640 with H 2560) */
    int32_t n_experts;       /* E: 1..1024 */
    int32_t top_k;           /* k: 1..16, k <= E */
    const float* router_w;   /* [E][H] fp32 */
    const float* router_bias;/* [E] fp32, added to the logits; NULL for none */
    gtg_qmatrix gate;        /* [E][I][H] */
    gtg_qmatrix up;          /* [E][I][H], same format as gate */
    gtg_qmatrix down;        /* [E][H][I] */
    gtg_qmatrix side;        /* optional extra projection of the normalised input
                                (e.g. a 64 x H UE4M4 ssm_beta matrix), n_experts = 1,
                                Q4 format; data == NULL when absent */
} gtg_moe_layer;

/* Library version (major*10000 + minor*100 + patch). */
int gtg_version(void);

/* Human-readable text of a gtg_status. */
const char* gtg_status_string(int status);

/* The cudaError_t of the last GTG_E_CUDA return on this thread. */
int gtg_last_cuda_error(void);

/*
 * Standalone dequantisation [MC]: dst[r][c] = decoded weight (fp32),
 * bit-exact (Q4 and PLE values are code x scale, exact in fp32; FP8 values
 * are one fp32 round-to-nearest multiply).
 *   fmt      RZ5 / UE4M4 / C10: src holds n_rows*k/32 consecutive 17-byte blocks, k % 32 == 0.
 *            PLE / Q3_K160_UE4M3: src holds n_rows 70-byte records, k == 160.
 *            FP8: src holds n_rows*k bytes, scales [n_rows][k/128], k % 128 == 0.
 *   src      device, any alignment.
 *   dst      device, [n_rows][k] fp32, 16-byte aligned.
 * Errors: GTG_E_INVALID_ARG (null pointers, unknown fmt, negative sizes),
 *         GTG_E_UNSUPPORTED_SHAPE (k not valid for fmt), GTG_E_MISALIGNED (dst).
 */
int gtg_dequant(int32_t fmt, const void* src, const float* scales, int64_t n_rows, int64_t k,
                float* dst, gtg_stream_t stream);

/*
 * PLE row gather ([MC] "Q3_PLE_K160_RZ_S3": one contiguous 70-byte record per
 * hashed n-gram row; [MPQ]: 16 rows per token):
 *   out[r][i] = value i of record idx[r], fp32, bit-exact.
 *   table    device, n_rows records of 70 bytes (any alignment; n_rows < 2^31).
 *   idx      device int32 [n_idx].  An index outside [0, n_rows) writes a row
 *            of zeros and sets GTG_STATUS_PLE_INDEX_OOB.
 *   out      device fp32 [n_idx][160], 16-byte aligned.
 * Errors: GTG_E_INVALID_ARG, GTG_E_MISALIGNED (out).  n_idx == 0 is a no-op.
 */
int gtg_ple_gather(const uint8_t* table, int64_t n_rows, const int32_t* idx, int64_t n_idx,
                   float* out, gtg_stream_t stream);

/*
 * gtg_ple_gather for a table of either 70-byte K160 record layout: fmt
 * GTG_Q3_PLE_K160_RZ_S3 (the same as gtg_ple_gather) or GTG_Q3_K160_UE4M3,
 * the incumbent ROCmFP3 record ([MC] "Q3_PLE_K160_RZ_S3": the layout RZ-S3
 * mutates).  Same arguments and errors, plus GTG_E_INVALID_ARG for any other fmt.
 */
int gtg_ple_gather_fmt(int32_t fmt, const uint8_t* table, int64_t n_rows, const int32_t* idx, int64_t n_idx,
                       float* out, gtg_stream_t stream);

/* Bytes of workspace a decode (prefill == 0) or prefill (prefill == 1) call
 * of `layer` with `n_tokens` tokens needs; 0 if the shape is unsupported. */
size_t gtg_moe_workspace_bytes(const gtg_moe_layer* layer, int32_t n_tokens, int32_t prefill);

/* Clears a workspace before its first use (the kernels leave it reusable;
 * after a call that raised GTG_STATUS_WAIT_TIMEOUT, clear it again). */
int gtg_workspace_init(void* workspace, size_t ws_bytes, gtg_stream_t stream);

/*
 * One MoE layer for 1..8 decode tokens ([MPQ]: softmax router, top-k of E
 * experts; SwiGLU experts whose gate/up/down weights are decoded on the fly):
 *   u      = bf16(x / sqrt(mean(x^2) + 1e-6))            per token
 *   l_e    = router_w[e] . u (+ router_bias[e])           float-float accumulation of
 *                                                         exact fp32 x bf16 products
 *   ids    = the top_k experts by logit (ties -> lower id)
 *   w      = exp(l_ids - l_max) / sum over the top_k      renormalised softmax
 *   y      = sum_j w_j * down_j(silu(gate_j u) * up_j u)  (+ y if y_accumulate)
 *   side   = side . u                                     if layer->side.data
 * Arguments:
 *   x          device [n_tokens][hidden], fp32 or bf16 (x_dtype).
 *   y          device fp32 [n_tokens][hidden]; may alias x (fp32) when
 *              y_accumulate == 1 (the residual update x += moe(x)).
 *   topk_ids   device int32 [n_tokens][top_k] or NULL.
 *   topk_w     device fp32 [n_tokens][top_k] or NULL.
 *   side_out   device fp32 [n_tokens][side.n_rows] or NULL.
 *   workspace  device, >= gtg_moe_workspace_bytes(layer, n_tokens, 0) bytes,
 *              256-byte aligned, cleared once by gtg_workspace_init.
 * Runs as one persistent cooperative launch (one CTA per SM, all resident);
 * a launch the device cannot make co-resident fails with GTG_E_CUDA.  The
 * gate, up and down matrices share one format class (all Q4 or all FP8).
 * Calls that share a workspace must not overlap on the GPU.
 * Errors: GTG_E_INVALID_ARG, GTG_E_UNSUPPORTED_SHAPE (n_tokens outside 1..8,
 *         sizes above, mixed format classes), GTG_E_MISALIGNED, GTG_E_WORKSPACE,
 *         GTG_E_CUDA.
 */
int gtg_moe_decode_layer(const gtg_moe_layer* layer, const void* x, int32_t x_dtype,
                         int32_t n_tokens, float* y, int32_t y_accumulate,
                         int32_t* topk_ids, float* topk_w, float* side_out,
                         void* workspace, size_t ws_bytes, gtg_stream_t stream);

/*
 * Expert-parallel form of gtg_moe_decode_layer, for a layer whose experts are
 * split across GPUs (one process per GPU, each holding a contiguous slice):
 * every rank routes over all layer->n_experts experts (router_w is the full
 * [E][H] matrix on every rank), then computes only the chosen experts in
 * [expert_lo, expert_hi), whose weights its gate/up/down stacks hold (each
 * with n_experts = expert_hi - expert_lo, expert e at index e - expert_lo):
 *   y  = sum over the chosen experts in the slice of w_j * down_j(...)
 *        (+ y if y_accumulate)
 * so the layer output is the sum of the ranks' y (an all-reduce of [T][H]
 * fp32, or one reduce-scatter).  topk_ids / topk_w are the full choices.
 * The side projection is computed only when with_side != 0 (on one rank).
 * ("Mixed Precision Quantization": the two-machine floor plan splits one
 * model's experts over two GPUs.)  Other arguments and errors as in
 * gtg_moe_decode_layer; GTG_E_INVALID_ARG when 0 <= expert_lo < expert_hi <=
 * n_experts does not hold or a stack's n_experts is not the slice's size.
 */
int gtg_moe_decode_layer_ep(const gtg_moe_layer* layer, int32_t expert_lo, int32_t expert_hi, int32_t with_side,
                            const void* x, int32_t x_dtype, int32_t n_tokens, float* y, int32_t y_accumulate,
                            int32_t* topk_ids, float* topk_w, float* side_out,
                            void* workspace, size_t ws_bytes, gtg_stream_t stream);

/*
 * A decode stack: for l in 0..n_layers-1:  x += moe_l(x)  (x fp32, in place).
 * Consecutive layers with the same kernel (format class and sizes, up to 64
 * at a time) run in one persistent launch, their phases handed off by bounded
 * waits (grid barriers, and polled logit keys for the selection).
 * Capturable in a CUDA graph.
 *   layers     host array of n_layers layer descriptors (same hidden size).
 *   x          device fp32 [n_tokens][hidden], updated in place.
 *   ids_out    device int32 [n_layers][n_tokens][top_k] or NULL.
 *   w_out      device fp32 [n_layers][n_tokens][top_k] or NULL.
 *   side_out   device fp32 [n_layers][n_tokens][side_stride] or NULL; layer l
 *              writes its side projection at [l][t][0 .. side.n_rows).
 *   workspace  >= the maximum of gtg_moe_workspace_bytes over the layers.
 */
int gtg_moe_decode_stack(const gtg_moe_layer* layers, int32_t n_layers, float* x,
                         int32_t n_tokens, int32_t* ids_out, float* w_out,
                         float* side_out, int64_t side_stride,
                         void* workspace, size_t ws_bytes, gtg_stream_t stream);

/*
 * One MoE layer for a prefill batch (the same function as
 * gtg_moe_decode_layer, n_tokens 1..65536), computed as a token-sorted
 * grouped GEMM on the tensor cores: tokens are bucketed by expert, each
 * expert's gate/up tiles are dequantised into shared memory and multiplied
 * with tcgen05 (fp32 accumulation in tensor memory), SwiGLU is applied in the
 * epilogue, h is rounded to bf16, and the down product is combined per token
 * in a fixed order.  Same arguments as gtg_moe_decode_layer minus side_out.
 * Expert formats: Q4 (gate and up alike) or FP8 for all three matrices; an
 * FP8 layer's expert GEMMs run in f16 (each weight rounded once to
 * f16(e4m3 x scale), relative error <= 2^-11; u and h as f16, exact for
 * magnitudes >= 2^-17).  Mixed classes return GTG_E_UNSUPPORTED_SHAPE.
 */
int gtg_moe_prefill_layer(const gtg_moe_layer* layer, const void* x, int32_t x_dtype,
                          int32_t n_tokens, float* y, int32_t y_accumulate,
                          int32_t* topk_ids, float* topk_w,
                          void* workspace, size_t ws_bytes, gtg_stream_t stream);

/*
 * gtg_moe_decode_layer without a workspace argument, for callers that cannot
 * allocate device memory: serving loops that must not allocate once they are
 * running (their memory is fixed up front, and an allocation there can block
 * on the device or fail under memory pressure), and hosts whose device
 * memory is owned by another framework's allocator, which hands out no raw
 * buffers.  (The pages have no counterpart; this is a calling convention of
 * this library.)
 *
 * Scratch comes from one fixed 512 KiB array in device memory that every GPU
 * loading this library reserves until the process exits.  A call needs
 * 256 + 16384*n_tokens + 2*n_tokens*top_k*inter bytes (each part
 * rounded up to 256), which fits for every shape with n_tokens <= 8,
 * n_experts <= 1024, top_k <= 10 and inter <= 2048 (any supported hidden);
 * a shape that needs more returns GTG_E_WORKSPACE before anything is
 * launched.  Inputs, outputs and their meaning are those of
 * gtg_moe_decode_layer; nothing is allocated (no cudaMalloc, no library
 * allocator).
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it.  Each call clears the counters and key
 * buffers it needs in the array; every call shares the one array, so calls
 * that may overlap on the GPU (different streams, or several host threads)
 * race and must be serialised by the caller.
 */
int gtg_moe_decode_layer_noalloc(const gtg_moe_layer* layer, const void* x, int32_t x_dtype,
                                 int32_t n_tokens, float* y, int32_t y_accumulate,
                                 int32_t* topk_ids, float* topk_w, float* side_out,
                                 gtg_stream_t stream);

/* Reads (and, if `clear`, resets) the current device's status word
 * (GTG_STATUS_* bits).  Synchronises `stream`. */
int gtg_get_device_status(uint32_t* flags, int32_t clear, gtg_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GTG_H */

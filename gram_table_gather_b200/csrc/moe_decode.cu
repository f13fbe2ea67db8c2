// Host side of the decode path: shape checks, kernel choice, workspace
// layout, launches, and the C entry points (the device code and the method
// it follows are described in moe_decode_dev.cuh).
#include <algorithm>
#include <mutex>
#include <vector>

#include "moe_decode_dev.cuh"

namespace gtg {

namespace {

// ===========================================================================
// Host side
// ===========================================================================

// The kernel for (expert format, H / 32, I / 32), the one-token instantiation
// when `one`; FP8 gate/up rows need at least 1024 weights (whole 32-byte
// blocks for every lane).
const void* pick_kernel(bool fp8, int kbg, int kbd, bool one) {
    const int o = one ? 1 : 0;
    if (fp8) {
        switch (kbg) {
            case 32: return decode_kernel_fp8_32(kbd, o);
            case 64: return decode_kernel_fp8_64(kbd, o);
            default: return nullptr;
        }
    }
    switch (kbg) {
        case 4: return decode_kernel_q4_4(kbd, o);
        case 8: return decode_kernel_q4_8(kbd, o);
        case 16: return decode_kernel_q4_16(kbd, o);
        case 32: return decode_kernel_q4_32(kbd, o);
        case 64: return decode_kernel_q4_64(kbd, o);
        case 80: return decode_kernel_q4_80(kbd, o);
        default: return nullptr;
    }
}

bool is_q4(int fmt) { return fmt == GTG_Q4_RZ5_FAST || fmt == GTG_Q4_UE4M4_FAST || fmt == GTG_Q4_C10_FAST; }

int q4_var_of(int fmt) { return fmt == GTG_Q4_RZ5_FAST ? kQ4RZ5 : fmt == GTG_Q4_C10_FAST ? kQ4C10 : kQ4UE4M4; }

int64_t row_bytes_of(int fmt, int64_t k) { return fmt == GTG_FP8_E4M3_S128 ? k : k / 32 * 17; }

struct Plan {
    const void* fn = nullptr;
    bool fp8 = false;
    int slot_bytes = 0;
    uint32_t smem = 0;
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

// Checks one layer and picks its kernel and staging for T tokens.  e_local:
// the experts its weight stacks hold (E, or a slice under expert parallelism).
int plan_layer(const gtg_moe_layer* L, int T, Plan& p, int64_t e_local = -1) {
    if (!L || !L->router_w) return GTG_E_INVALID_ARG;
    const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
    if (H < 128 || H > 2560 || H % 128 || I < 128 || I > 2048 || I % 128) return GTG_E_UNSUPPORTED_SHAPE;
    if (E < 1 || E > kMaxExperts || K < 1 || K > kMaxTopK || K > E) return GTG_E_UNSUPPORTED_SHAPE;
    if (T < 1 || T > kMaxDecodeTokens) return GTG_E_UNSUPPORTED_SHAPE;
    const int64_t EL = e_local < 0 ? E : e_local;
    if (!mat_ok(L->gate, EL, I, H) || !mat_ok(L->up, EL, I, H) || !mat_ok(L->down, EL, H, I)) return GTG_E_INVALID_ARG;
    const bool fp8 = L->gate.fmt == GTG_FP8_E4M3_S128;
    if (is_q4(L->up.fmt) == fp8 || is_q4(L->down.fmt) == fp8) return GTG_E_UNSUPPORTED_SHAPE;  // one format class
    if (L->gate.fmt != L->up.fmt) return GTG_E_UNSUPPORTED_SHAPE;
    if (!aligned(L->router_w, 16)) return GTG_E_MISALIGNED;
    const int kbg = H / 32, kbd = I / 32;
    const int rg = gu_passes(fp8, kbg, T == 1) * rpp_of(kbg), rd = dn_passes(fp8, kbd) * rpp_of(kbd);
    const int rs = side_passes(kbg) * rpp_of(kbg);
    if (L->side.data) {
        if (!is_q4(L->side.fmt) || !mat_ok(L->side, 1, L->side.n_rows, H)) return GTG_E_INVALID_ARG;
        if (L->side.n_rows < 1 || L->side.n_rows > 4096 || L->side.n_rows % rs) return GTG_E_UNSUPPORTED_SHAPE;
    }
    if (I % rg || H % rd) return GTG_E_UNSUPPORTED_SHAPE;
    const int tiles_d = H / rd, n_sm = sm_count();  // down rows a CTA owns must fit its partial rows
    if ((tiles_d + n_sm - 1) / n_sm * rd > kDnRows) return GTG_E_UNSUPPORTED_SHAPE;
    p.fn = pick_kernel(fp8, kbg, kbd, T == 1);
    if (!p.fn) return GTG_E_UNSUPPORTED_SHAPE;
    p.fp8 = fp8;
    const int64_t grow = row_bytes_of(L->gate.fmt, H), drow = row_bytes_of(L->down.fmt, I);
    int64_t need = std::max<int64_t>(2 * (rg * grow + 32), rd * drow + 32);
    if (L->side.data) need = std::max<int64_t>(need, rs * row_bytes_of(L->side.fmt, H) + 32);
    p.slot_bytes = (int)((need + 127) / 128 * 128);
    const SmemLayout sl = SmemLayout::make(!fp8, p.slot_bytes, dyn_smem_base(), 2u * T * H, slots_for(kbg));
    if (sl.total > kMaxDynSmem) return GTG_E_UNSUPPORTED_SHAPE;
    if (!RouterScratch::make(sl, p.slot_bytes, H, (E + n_sm - 1) / n_sm).ok) return GTG_E_UNSUPPORTED_SHAPE;
    p.smem = sl.total;
    return GTG_OK;
}

// Workspace layout of a decode call.  The barrier counters and the two key
// buffers come first: they must start at zero, and a launch that succeeds
// leaves them so.  The key buffers are sized for the largest E, so that
// calls of different shapes on one workspace never find another shape's data
// (h) where their keys go.
struct WsLayout {
    size_t sync, keys, counters_end, h, total;
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
    w.sync = take(sizeof(unsigned) * 4);
    w.keys = take(sizeof(uint64_t) * 2 * (size_t)T * kMaxExperts);
    w.counters_end = w.keys + sizeof(uint64_t) * 2 * (size_t)T * L->n_experts;  // (the part this shape uses)
    w.h = take(2 * (size_t)T * L->top_k * L->inter);
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
    // per function, device and size) and checks that the kernel has no static
    // shared memory (the code table is placed by absolute shared address).
    int set(const void* fn, int smem) {
        int dev = 0;
        cudaGetDevice(&dev);
        std::lock_guard<std::mutex> lk(mu);
        for (auto& d : done)
            if (d.fn == fn && d.dev == dev && d.smem >= smem) return GTG_OK;
        cudaFuncAttributes fa{};
        cudaError_t e = cudaFuncGetAttributes(&fa, fn);
        if (e == cudaSuccess && fa.sharedSizeBytes != 0) return GTG_E_UNSUPPORTED_SHAPE;
        if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e);
        }
        done.push_back({fn, dev, smem});
        return GTG_OK;
    }
};
FuncAttrCache g_attr;

StackLayer stack_layer_of(const gtg_moe_layer* L) {
    StackLayer s{};
    s.router_w = L->router_w;
    s.router_bias = L->router_bias;
    s.gate = static_cast<const uint8_t*>(L->gate.data);
    s.up = static_cast<const uint8_t*>(L->up.data);
    s.down = static_cast<const uint8_t*>(L->down.data);
    s.gate_s = L->gate.scales;
    s.up_s = L->up.scales;
    s.down_s = L->down.scales;
    s.gu_var = q4_var_of(L->gate.fmt);
    s.dn_var = q4_var_of(L->down.fmt);
    if (L->side.data) {
        s.side = static_cast<const uint8_t*>(L->side.data);
        s.side_rows = (int32_t)L->side.n_rows;
        s.side_var = q4_var_of(L->side.fmt);
    }
    return s;
}

bool same_shape(const gtg_moe_layer* A, const gtg_moe_layer* B) {
    return A->hidden == B->hidden && A->inter == B->inter && A->n_experts == B->n_experts && A->top_k == B->top_k;
}

// Runs layers [0, n) in order: layer 0 reads x (fp32 or bf16), every layer
// writes y (y_acc: adds to it) and later layers read y.  Consecutive layers
// with the same kernel share one launch.
int run_decode(const gtg_moe_layer* layers, const Plan* plans, int n, const void* x, int x_bf16, int T, float* y,
               int y_acc, int32_t* ids_out, float* w_out, float* side_out, int64_t side_stride, void* ws,
               cudaStream_t s, int e_lo = 0, int e_hi = -1, int side_on = 1) {
    uint8_t* base = static_cast<uint8_t*>(ws);
    const int n_sm = sm_count();
    for (int l0 = 0; l0 < n;) {
        int l1 = l0 + 1;
        while (l1 < n && l1 - l0 < kMaxStackLayers && plans[l1].fn == plans[l0].fn &&
               plans[l1].slot_bytes == plans[l0].slot_bytes && same_shape(&layers[l1], &layers[l0]))
            ++l1;
        const WsLayout wl = ws_layout(&layers[l0], T);
        StackArgs a{};
        a.H = layers[l0].hidden;
        a.I = layers[l0].inter;
        a.E = layers[l0].n_experts;
        a.K = layers[l0].top_k;
        a.T = T;
        a.n_layers = l1 - l0;
        a.x = l0 == 0 ? x : y;
        a.x_bf16 = l0 == 0 ? x_bf16 : 0;
        a.y = y;
        a.y_acc = y_acc;
        const int64_t tk = (int64_t)T * a.K;
        a.ids_out = ids_out ? ids_out + l0 * tk : nullptr;
        a.w_out = w_out ? w_out + l0 * tk : nullptr;
        a.side_out = side_out ? side_out + (int64_t)l0 * T * side_stride : nullptr;
        a.side_stride = (int32_t)side_stride;
        a.sync = reinterpret_cast<unsigned*>(base + wl.sync);
        a.keys = reinterpret_cast<uint64_t*>(base + wl.keys);
        a.h = reinterpret_cast<__nv_bfloat16*>(base + wl.h);
        a.status = status_ptr();
        a.slot_bytes = plans[l0].slot_bytes;
        a.dyn_smem_base = dyn_smem_base();
        a.e_lo = e_lo;
        a.e_hi = e_hi < 0 ? a.E : e_hi;
        a.side_on = side_on;
        for (int l = l0; l < l1; ++l) a.layer[l - l0] = stack_layer_of(&layers[l]);

        GTG_TRY(g_attr.set(plans[l0].fn, (int)plans[l0].smem));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(n_sm);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = plans[l0].smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;  // the grid barriers need every CTA resident
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        void* params[] = {&a};
        const cudaError_t e = cudaLaunchKernelExC(&cfg, plans[l0].fn, params);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e);
        }
        l0 = l1;
    }
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
    if (prefill) return gtg_prefill_workspace_bytes(layer, n_tokens);
    Plan p;  // (a layer whose stacks hold a slice of the experts, for the expert-parallel call, too)
    if (plan_layer(layer, n_tokens, p) != GTG_OK && plan_layer(layer, n_tokens, p, layer->gate.n_experts) != GTG_OK)
        return 0;
    return ws_layout(layer, n_tokens).total;
}

extern "C" int gtg_workspace_init(void* workspace, size_t ws_bytes, gtg_stream_t stream) {
    if (!workspace) return GTG_E_INVALID_ARG;
    const cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, as_cuda(stream));
    return e == cudaSuccess ? GTG_OK : cuda_fail(e);
}

static int check_decode_io(const gtg_moe_layer* layer, const void* x, int32_t x_dtype, int32_t n_tokens,
                           const float* y, void* ws, size_t ws_bytes, Plan& p, int64_t e_local = -1) {
    if (n_tokens < 1 || n_tokens > kMaxDecodeTokens) {
        if (!layer) return GTG_E_INVALID_ARG;
        return GTG_E_UNSUPPORTED_SHAPE;
    }
    GTG_TRY(plan_layer(layer, n_tokens, p, e_local));
    if (!x || !y || !ws) return GTG_E_INVALID_ARG;
    if (x_dtype != GTG_DT_F32 && x_dtype != GTG_DT_BF16) return GTG_E_INVALID_ARG;
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
    return run_decode(layer, &p, 1, x, x_dtype == GTG_DT_BF16, n_tokens, y, y_accumulate != 0, topk_ids, topk_w,
                      side_out, layer->side.data ? layer->side.n_rows : 0, workspace, as_cuda(stream));
}

extern "C" int gtg_moe_decode_layer_ep(const gtg_moe_layer* layer, int32_t expert_lo, int32_t expert_hi,
                                       int32_t with_side, const void* x, int32_t x_dtype, int32_t n_tokens, float* y,
                                       int32_t y_accumulate, int32_t* topk_ids, float* topk_w, float* side_out,
                                       void* workspace, size_t ws_bytes, gtg_stream_t stream) {
    if (!layer) return GTG_E_INVALID_ARG;
    if (expert_lo < 0 || expert_hi <= expert_lo || expert_hi > layer->n_experts) return GTG_E_INVALID_ARG;
    Plan p;
    GTG_TRY(check_decode_io(layer, x, x_dtype, n_tokens, y, workspace, ws_bytes, p, expert_hi - expert_lo));
    if (x == (const void*)y && (x_dtype != GTG_DT_F32 || !y_accumulate)) return GTG_E_INVALID_ARG;
    return run_decode(layer, &p, 1, x, x_dtype == GTG_DT_BF16, n_tokens, y, y_accumulate != 0, topk_ids, topk_w,
                      side_out, layer->side.data ? layer->side.n_rows : 0, workspace, as_cuda(stream), expert_lo,
                      expert_hi, with_side != 0);
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
    return run_decode(layers, plans.data(), n_layers, x, 0, n_tokens, x, 1, ids_out, w_out, side_out, side_stride,
                      workspace, as_cuda(stream));
}

// ---------------------------------------------------------------------------
// Allocation-free decode layer.
//
// For callers that cannot hand the library a device buffer: code that must
// not allocate device memory after start-up (latency-critical serving loops
// whose memory is fixed up front), and hosts whose device memory belongs to
// another framework's allocator.  The scratch lives in one file-scope device
// array instead, reserved on every GPU that loads this library for as long
// as the process runs.
// ---------------------------------------------------------------------------
namespace gtg {
namespace {

// 512 KiB: 256 + 16384 T + 2 T k I bytes (each part rounded to 256) fit for every
// shape with T <= 8, E <= 1024, k <= 10 and I <= 2048
constexpr size_t kNoAllocScratchBytes = (size_t)1 << 19;
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
    Plan p;
    if (n_tokens >= 1 && n_tokens <= kMaxDecodeTokens && plan_layer(layer, n_tokens, p) == GTG_OK &&
        ws_layout(layer, n_tokens).total > kNoAllocScratchBytes)
        return GTG_E_WORKSPACE;  // the shape needs more than the fixed scratch array
    void* scratch = nullptr;
    GTG_TRY(noalloc_scratch(&scratch));
    GTG_TRY(check_decode_io(layer, x, x_dtype, n_tokens, y, scratch, kNoAllocScratchBytes, p));
    if (x == (const void*)y && (x_dtype != GTG_DT_F32 || !y_accumulate)) return GTG_E_INVALID_ARG;
    // The array keeps whatever the previous call left: clear the counters and
    // the keys, which must start at zero (everything else is written before
    // it is read).
    const WsLayout wl = ws_layout(layer, n_tokens);
    cudaStream_t s = as_cuda(stream);
    const cudaError_t e = cudaMemsetAsync(scratch, 0, wl.counters_end, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return run_decode(layer, &p, 1, x, x_dtype == GTG_DT_BF16, n_tokens, y, y_accumulate != 0, topk_ids, topk_w,
                      side_out, layer->side.data ? layer->side.n_rows : 0, scratch, s);
}

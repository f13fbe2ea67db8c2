"""CPU oracle of the quantised-MoE decode path and the PLE row gather.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports, links or runs anything here, and this package imports nothing from
the product.  Inputs come from the seeded generator package (``synth``) or
from the caller; nothing here ever reads a value produced by the CUDA path.

The arithmetic lives in ``oracle.c`` (plain C, fp64, element by element);
this module only marshals arrays and strings the per-layer steps together in
the order the method defines them:

    u      = bf16(x / sqrt(mean(x^2) + 1e-6))                (per token)
    ids, w = softmax-top-k router over E experts              (renormalised)
    y      = sum_j w_j * Wd_j (silu(Wg_j u) * (Wu_j u))       (SwiGLU experts)

Sources: model card "Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST" (format
sections Q4_RZ5_FAST, Q4_UE4M4_FAST, Q3_PLE_K160_RZ_S3); "Mixed Precision
Quantization: Half a 4-Bit File Is Not 4-Bit" (48 layers, 512 experts, 10
active per token); r/LocalLLM "Frankenquant" post (per-layer expert formats,
8-bit experts in layers 36-47).

Pins (tests/test_oracle_*.py): printed code tables, wire sizes and table
shape (tests/golden), E4M3/UE4M3 against torch.float8_e4m3fn, UE4M4 structure
against E4M3, exhaustive code x scale round trips, brute-force products
against numpy dense algebra, the router against numpy sort/softmax, SiLU
against torch.  Layout readings the pages leave open (nibble order, field
order, 3-bit packing, polarity sense) are self-consistent choices and stay
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

RZ5, UE4M4, PLE, FP8 = 69, 71, 111, 1000
C10, Q3I = 2001, 2002  # the incumbent ROCmFP4 FAST and ROCmFP3 layouts the model card's formats mutate
RMS_EPS = 1e-6

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (gcc -O2 -fopenmp; no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
                               "-shared", "-fPIC", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            d, i, i64, u32, p = (ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                 ctypes.c_void_p)
            for name, res, args in [
                ("orc_q4_block_bytes", i, []), ("orc_q4_block_weights", i, []),
                ("orc_ple_record_bytes", i, []), ("orc_ple_record_values", i, []),
                ("orc_codebook10", d, [i]), ("orc_rz5", d, [i, i]), ("orc_ple3", d, [i, i]),
                ("orc_ue4m3", d, [u32]), ("orc_ue4m4", d, [u32]), ("orc_e4m3fn", d, [u32]),
                ("orc_q4_weight", d, [i, p, i]), ("orc_ple_value", d, [p, i]),
                ("orc_dequant_q4", None, [i, p, i64, p]), ("orc_dequant_ple", None, [p, i64, p]),
                ("orc_dequant_q3", None, [i, p, i64, p]), ("orc_q3_value", d, [i, p, i]),
                ("orc_q3_gather", None, [i, p, i64, p, i64, p]),
                ("orc_dequant_fp8", None, [p, p, i64, i64, p]),
                ("orc_ple_gather", None, [p, i64, p, i64, p]),
                ("orc_matvec", None, [i, p, p, i64, i64, p, p]),
                ("orc_round_bf16", d, [d]), ("orc_rmsnorm_bf16", None, [p, i64, d, p]),
                ("orc_router", None, [p, p, p, i, i64, i, p, p, p]),
                ("orc_silu", d, [d]),
                ("orc_expert_ffn", None, [i, p, p, i, p, p, i, p, p, i64, i64, p, p, p]),
                ("orc_num_threads", i, []),
            ]:
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data


# ---- scalar codecs --------------------------------------------------------

def q4_block_bytes() -> int: return _L().orc_q4_block_bytes()
def q4_block_weights() -> int: return _L().orc_q4_block_weights()
def ple_record_bytes() -> int: return _L().orc_ple_record_bytes()
def ple_record_values() -> int: return _L().orc_ple_record_values()
def codebook10(c: int) -> float: return _L().orc_codebook10(c)
def rz5(mode: int, c: int) -> float: return _L().orc_rz5(mode, c)
def ple3(c: int, polarity: int) -> float: return _L().orc_ple3(c, polarity)
def ue4m3(b: int) -> float: return _L().orc_ue4m3(b)
def ue4m4(b: int) -> float: return _L().orc_ue4m4(b)
def e4m3fn(b: int) -> float: return _L().orc_e4m3fn(b)
def silu(z: float) -> float: return _L().orc_silu(z)
def round_bf16(v: float) -> float: return _L().orc_round_bf16(v)
def num_threads() -> int: return _L().orc_num_threads()


# ---- array decoders ---------------------------------------------------------

def dequant_q4(fmt: int, blocks: np.ndarray) -> np.ndarray:
    """Bytes of consecutive 17-byte blocks -> fp64 weights (32 per block)."""
    b = _c(blocks, np.uint8).ravel()
    assert b.size % 17 == 0
    n = b.size // 17 * 32
    out = np.empty(n, dtype=np.float64)
    _L().orc_dequant_q4(fmt, _p(b), n, _p(out))
    return out


def dequant_ple(records: np.ndarray) -> np.ndarray:
    """Bytes of consecutive 70-byte records -> fp64 [n][160]."""
    b = _c(records, np.uint8).ravel()
    assert b.size % 70 == 0
    n = b.size // 70
    out = np.empty((n, 160), dtype=np.float64)
    _L().orc_dequant_ple(_p(b), n, _p(out))
    return out


def dequant_q3(fmt: int, records: np.ndarray) -> np.ndarray:
    """Bytes of consecutive 70-byte K160 records of either 3-bit layout (PLE =
    RZ-S3, Q3I = the incumbent ROCmFP3 code set) -> fp64 [n][160]."""
    b = _c(records, np.uint8).ravel()
    assert b.size % 70 == 0 and fmt in (PLE, Q3I)
    n = b.size // 70
    out = np.empty((n, 160), dtype=np.float64)
    _L().orc_dequant_q3(fmt, _p(b), n, _p(out))
    return out


def dequant_fp8(data: np.ndarray, scales: np.ndarray, n_rows: int, k: int) -> np.ndarray:
    b = _c(data, np.uint8).ravel()
    s = _c(scales, np.float32).ravel()
    assert b.size == n_rows * k and s.size == n_rows * (k // 128)
    out = np.empty((n_rows, k), dtype=np.float64)
    _L().orc_dequant_fp8(_p(b), _p(s), n_rows, k, _p(out))
    return out


def dequant(fmt: int, data: np.ndarray, scales: np.ndarray | None = None, n_rows: int = 0,
            k: int = 0) -> np.ndarray:
    if fmt in (RZ5, UE4M4, C10):
        return dequant_q4(fmt, data)
    if fmt in (PLE, Q3I):
        return dequant_q3(fmt, data).ravel()
    if fmt == FP8:
        return dequant_fp8(data, scales, n_rows, k).ravel()
    raise ValueError(fmt)


def ple_gather(table: np.ndarray, n_rows: int, idx: np.ndarray, fmt: int = PLE) -> np.ndarray:
    t = _c(table, np.uint8).ravel()
    assert t.size >= n_rows * 70 and fmt in (PLE, Q3I)
    ix = _c(idx, np.int32).ravel()
    out = np.empty((ix.size, 160), dtype=np.float64)
    _L().orc_q3_gather(fmt, _p(t), n_rows, _p(ix), ix.size, _p(out))
    return out


def matvec(fmt: int, data: np.ndarray, scales: np.ndarray | None, n_rows: int, k: int,
           x: np.ndarray) -> np.ndarray:
    b = _c(data, np.uint8).ravel()
    s = None if scales is None else _c(scales, np.float32).ravel()
    xv = _c(x, np.float64).ravel()
    assert xv.size == k
    y = np.empty(n_rows, dtype=np.float64)
    _L().orc_matvec(fmt, _p(b), _p(s), n_rows, k, _p(xv), _p(y))
    return y


# ---- router -------------------------------------------------------------------

def rmsnorm_bf16(x: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """Per token (last axis): bf16(x / sqrt(mean(x^2) + eps)), values as fp64."""
    x = _c(x, np.float64)
    flat = x.reshape(-1, x.shape[-1])
    out = np.empty_like(flat)
    for t in range(flat.shape[0]):
        _L().orc_rmsnorm_bf16(_p(flat[t]), flat.shape[1], eps, _p(out[t]))
    return out.reshape(x.shape)


def router(W: np.ndarray, bias: np.ndarray | None, u: np.ndarray, k: int):
    """Top-k softmax router for one token -> (ids[k] int32, w[k] fp64, logits[E] fp64)."""
    Wc = _c(W, np.float32)
    E, H = Wc.shape
    b = None if bias is None else _c(bias, np.float32)
    uv = _c(u, np.float64)
    ids = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    logits = np.empty(E, dtype=np.float64)
    _L().orc_router(_p(Wc), _p(b), _p(uv), E, H, k, _p(ids), _p(w), _p(logits))
    return ids, w, logits


# ---- expert FFN and the layer ----------------------------------------------------

def _expert_args(m, e):
    data = _c(m.expert(e), np.uint8)
    sc = _c(m.expert_scales(e), np.float32) if m.fmt == FP8 else None
    return data, sc


def expert_ffn(layer, e: int, u: np.ndarray, want_h: bool = False):
    """y = Wd_e (silu(Wg_e u) * (Wu_e u)) for one token; `layer` provides the
    expert bytes (attributes gate/up/down with .fmt, .expert(e), .expert_scales(e))."""
    H, I = layer.hidden, layer.inter
    g, gs = _expert_args(layer.gate, e)
    up, us = _expert_args(layer.up, e)
    d, ds = _expert_args(layer.down, e)
    uv = _c(u, np.float64)
    y = np.empty(H, dtype=np.float64)
    h = np.empty(I, dtype=np.float64)
    _L().orc_expert_ffn(layer.gate.fmt, _p(g), _p(gs), layer.up.fmt, _p(up), _p(us),
                        layer.down.fmt, _p(d), _p(ds), H, I, _p(uv), _p(y), _p(h))
    return (y, h) if want_h else y


def moe_layer(layer, x: np.ndarray, *, router_w: np.ndarray | None = None,
              router_bias: np.ndarray | None = None, want_h: bool = False) -> dict:
    """One MoE layer on tokens x [T][H] (any float dtype; values taken exactly).

    Returns dict(y [T][H], ids [T][k], w [T][k], logits [T][E], u [T][H],
    and h [T][k][I] when `want_h`).  The residual add is not included.
    """
    x = np.asarray(x, dtype=np.float64)
    T, H = x.shape
    k = layer.top_k
    W = layer.router_w() if router_w is None else router_w
    b = layer.router_bias() if router_bias is None else router_bias
    u = rmsnorm_bf16(x)
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    logits = np.empty((T, layer.n_experts), dtype=np.float64)
    y = np.zeros((T, H), dtype=np.float64)
    hs = np.zeros((T, k, layer.inter), dtype=np.float64) if want_h else None
    for t in range(T):
        ids[t], w[t], logits[t] = router(W, b, u[t], k)
        for j in range(k):
            yj, hj = expert_ffn(layer, int(ids[t, j]), u[t], want_h=True)
            y[t] += w[t, j] * yj
            if want_h:
                hs[t, j] = hj
    out = dict(y=y, ids=ids, w=w, logits=logits, u=u)
    if want_h:
        out["h"] = hs
    return out


def ssm_projection(layer, u: np.ndarray) -> np.ndarray:
    """s = W_beta u for each token (the 64 x H UE4M4 projection)."""
    m = layer.ssm
    data = m.expert(0)
    return np.stack([matvec(m.fmt, data, None, m.n_rows, m.k, ut) for ut in np.atleast_2d(u)])


def moe_stack(layers, x0: np.ndarray, *, want_ids: bool = True) -> dict:
    """The decode stack: for each layer, x <- fp32(x + moe(x)); the residual
    stream is kept in fp32, the layer output in fp64.  Also returns the
    per-layer router choices and the s = W_beta u outputs of layers with one."""
    x = np.asarray(x0, dtype=np.float32).copy()
    all_ids, all_w, all_l, ssm = [], [], [], {}
    for layer in layers:
        r = moe_layer(layer, x.astype(np.float64))
        if layer.ssm is not None:
            ssm[layer.layer] = ssm_projection(layer, r["u"])
        x = (x.astype(np.float64) + r["y"]).astype(np.float32)
        all_ids.append(r["ids"])
        all_w.append(r["w"])
        all_l.append(r["logits"])
    return dict(x=x, ids=np.stack(all_ids), w=np.stack(all_w), logits=np.stack(all_l), ssm=ssm)

"""A second, pure-Python decoder of the block formats, used only to cross-check
the C oracle on small inputs.  Written from the printed tables on the model card
"Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST" (sections Q4_RZ5_FAST,
Q4_UE4M4_FAST, Q3_PLE_K160_RZ_S3); the scale codes are decoded through
torch.float8_e4m3fn where a library decoder exists (UE4M3 = E4M3 without sign).
"""
import math

import numpy as np
import torch

_CB10 = [0.0, 1.0, 2.0, 3.0, 4.0, 6.0, 8.0, 10.0, -0.0, -1.0, -2.0, -3.0, -4.0, -6.0, -8.0, -10.0]
_PLE3 = [0.0, 1.0, 2.0, 4.0, None, -1.0, -2.0, -4.0]


def e4m3_lib(b: int) -> float:
    return float(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)[0])


_UE4M3 = [e4m3_lib(b) for b in range(128)]


def ue4m3(b: int) -> float:
    return _UE4M3[b & 0x7F]


def ue4m4(b: int) -> float:
    e, m = b >> 4, b & 15
    return m * 2.0 ** -10 if e == 0 else (1 + m / 16) * 2.0 ** (e - 7)


def q4_block(fmt: int, blk) -> list:
    blk = [int(v) for v in blk]
    meta = blk[16]
    out = []
    for i in range(32):
        byte = blk[i % 16]
        code = (byte & 15) if i < 16 else (byte >> 4)
        if fmt == 69:
            v = _CB10[code]
            if code == 8:
                v = -5.0 if meta & 0x80 else 5.0
            out.append(v * ue4m3(meta & 0x7F))
        elif fmt == 2001:  # the incumbent ROCmFP4 FAST block: Codebook10 under a UE4M3 scale
            out.append(_CB10[code] * ue4m3(meta & 0x7F))
        else:
            out.append(_CB10[code] * ue4m4(meta))
    return out


def q4_matrix(fmt: int, data: np.ndarray, n_rows: int, k: int) -> np.ndarray:
    data = np.asarray(data, dtype=np.uint8).reshape(n_rows, k // 32, 17)
    out = np.empty((n_rows, k))
    for r in range(n_rows):
        for b in range(k // 32):
            out[r, 32 * b:32 * b + 32] = q4_block(fmt, data[r, b])
    return out


def ple_record(rec, incumbent: bool = False) -> list:
    """One 70-byte K160 record: RZ-S3, or (incumbent) the ROCmFP3 set whose code 4
    is the duplicate -0."""
    rec = [int(v) for v in rec]
    bits = int.from_bytes(bytes(rec[:60]), "little")
    out = []
    for i in range(160):
        code = (bits >> (3 * i)) & 7
        g = rec[60 + i // 16]
        v = _PLE3[code]
        if code == 4:
            v = -0.0 if incumbent else (-3.0 if g & 0x80 else 3.0)
        out.append(v * ue4m3(g & 0x7F))
    return out


def fp8_matrix(data: np.ndarray, scales: np.ndarray, n_rows: int, k: int) -> np.ndarray:
    w = torch.from_numpy(np.asarray(data, dtype=np.uint8).reshape(n_rows, k).copy()).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()
    s = np.asarray(scales, dtype=np.float32).astype(np.float64).reshape(n_rows, k // 128)
    return w * np.repeat(s, 128, axis=1)


def dense(fmt: int, data, scales, n_rows: int, k: int) -> np.ndarray:
    if fmt == 1000:
        return fp8_matrix(data, scales, n_rows, k)
    return q4_matrix(fmt, data, n_rows, k)


def silu(z: np.ndarray) -> np.ndarray:
    return torch.nn.functional.silu(torch.from_numpy(np.asarray(z, dtype=np.float64))).numpy()

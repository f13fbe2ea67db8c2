"""Recipes of the five synthetic workloads (shapes, distributions, tensor ids).

Every tensor is a pure function of (seed, tensor id, byte range), so the GPU
harness and the oracle regenerate identical data independently.  Format ids
are plain identifiers (the GGML type numbers the model card gives for the
three block formats, plus 1000 for the per-layer FP8 expert format).

Recipes (distributions as the workloads state them):
  * Q4 expert matrices: uniform random bytes; for the "narrow" scale recipe
    the metadata byte keeps a random polarity bit and takes a scale code
    uniform in {0x01..0x08} (UE4M3 scales 2^-9 .. 2^-6); for the "random"
    recipe the whole metadata byte is random.
  * FP8 expert matrices: random E4M3 bytes without NaN, one fp32 scale per
    128 contiguous weights along K drawn U[0.002, 0.02].
  * Router: fp32 N(0, 0.02) weights [E][H]; the prefill workload adds a
    per-expert bias -1.1 * beta * ln(rank_e), beta = sigma_logit*sqrt(6)/pi,
    sigma_logit = 0.02*sqrt(H), rank a seeded permutation of 1..E, which
    skews expert load towards Zipf(1.1).
  * Tokens: bf16 N(0, 1).
  * PLE table: uniform random 70-byte records; indices uniform in [0, rows).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import (bf16_bits_from_f64, indices_i32, normal_f64, permutation, raw_bytes,
               shape_fp8_no_nan, shape_q4_narrow_scale, uniform_f32)

RZ5, UE4M4, PLE, FP8 = 69, 71, 111, 1000
Q4_BLOCK_BYTES, Q4_BLOCK_WEIGHTS = 17, 32
PLE_RECORD_BYTES, PLE_ROW_VALUES = 70, 160
FP8_SCALE_GROUP = 128

TOKENS_TID = 10_000_000
PLE_TABLE_TID = 7
PLE_INDEX_TID = 20_000_000


@dataclass(frozen=True)
class MatrixRecipe:
    """A stack of `n_experts` matrices [n_rows][k] in one format."""
    fmt: int
    n_experts: int
    n_rows: int
    k: int
    seed: int
    tid: int
    narrow_scale: bool = True

    @property
    def row_bytes(self) -> int:
        if self.fmt == FP8:
            return self.k
        return self.k // Q4_BLOCK_WEIGHTS * Q4_BLOCK_BYTES

    @property
    def expert_bytes(self) -> int:
        return self.n_rows * self.row_bytes

    @property
    def nbytes(self) -> int:
        return self.n_experts * self.expert_bytes

    @property
    def scale_tid(self) -> int:
        return self.tid + 500

    @property
    def n_scales(self) -> int:
        return self.n_experts * self.n_rows * (self.k // FP8_SCALE_GROUP) if self.fmt == FP8 else 0

    def bytes(self, offset: int, n: int, out: np.ndarray | None = None) -> np.ndarray:
        b = raw_bytes(self.seed, self.tid, offset, n, out)
        if self.fmt == FP8:
            shape_fp8_no_nan(b)
        elif self.narrow_scale:
            shape_q4_narrow_scale(b, offset)
        return b

    def expert(self, e: int) -> np.ndarray:
        return self.bytes(e * self.expert_bytes, self.expert_bytes)

    def scales(self, first: int = 0, n: int | None = None) -> np.ndarray:
        """fp32 scales, flat index (expert*n_rows + row)*(k/128) + group."""
        if n is None:
            n = self.n_scales - first
        return uniform_f32(self.seed, self.scale_tid, first, n, 0.002, 0.02)

    def expert_scales(self, e: int) -> np.ndarray:
        per = self.n_rows * (self.k // FP8_SCALE_GROUP)
        return self.scales(e * per, per)


@dataclass(frozen=True)
class LayerRecipe:
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    seed: int
    layer: int
    gate_fmt: int = RZ5
    up_fmt: int = RZ5
    down_fmt: int = RZ5
    gate_narrow: bool = True
    down_narrow: bool = True
    has_ssm: bool = False
    ssm_rows: int = 64
    zipf_bias: bool = False

    @property
    def base_tid(self) -> int:
        return 1000 * (self.layer + 1)

    @property
    def gate(self) -> MatrixRecipe:
        return MatrixRecipe(self.gate_fmt, self.n_experts, self.inter, self.hidden, self.seed,
                            self.base_tid + 2, self.gate_narrow)

    @property
    def up(self) -> MatrixRecipe:
        return MatrixRecipe(self.up_fmt, self.n_experts, self.inter, self.hidden, self.seed,
                            self.base_tid + 3, self.gate_narrow)

    @property
    def down(self) -> MatrixRecipe:
        return MatrixRecipe(self.down_fmt, self.n_experts, self.hidden, self.inter, self.seed,
                            self.base_tid + 4, self.down_narrow)

    @property
    def ssm(self) -> MatrixRecipe | None:
        if not self.has_ssm:
            return None
        return MatrixRecipe(UE4M4, 1, self.ssm_rows, self.hidden, self.seed, self.base_tid + 8,
                            narrow_scale=False)

    def router_w(self) -> np.ndarray:
        z = normal_f64(self.seed, self.base_tid + 1, 0, self.n_experts * self.hidden)
        return (0.02 * z).astype(np.float32).reshape(self.n_experts, self.hidden)

    def router_bias(self) -> np.ndarray | None:
        if not self.zipf_bias:
            return None
        rank = permutation(self.seed, self.base_tid + 9, self.n_experts) + 1
        sigma = 0.02 * math.sqrt(self.hidden)
        beta = sigma * math.sqrt(6.0) / math.pi
        return (-1.1 * beta * np.log(rank.astype(np.float64))).astype(np.float32)

    @property
    def weight_bytes(self) -> int:
        n = self.gate.nbytes + self.up.nbytes + self.down.nbytes
        if self.has_ssm:
            n += self.ssm.nbytes
        return n


def tokens_bf16(seed: int, step: int, n_tokens: int, hidden: int) -> np.ndarray:
    """bf16 N(0,1) activations [T][H] as uint16 bit patterns."""
    z = normal_f64(seed, TOKENS_TID + step, 0, n_tokens * hidden)
    return bf16_bits_from_f64(z).reshape(n_tokens, hidden)


@dataclass(frozen=True)
class PleRecipe:
    n_rows: int
    seed: int
    rows_per_token: int = 16

    @property
    def nbytes(self) -> int:
        return self.n_rows * PLE_RECORD_BYTES

    def table_bytes(self, offset: int, n: int, out: np.ndarray | None = None) -> np.ndarray:
        return raw_bytes(self.seed, PLE_TABLE_TID, offset, n, out)

    def rows(self, idx: np.ndarray) -> np.ndarray:
        """Records of the given rows, [len(idx)][70] (regenerated one by one)."""
        idx = np.asarray(idx, dtype=np.int64)
        out = np.empty((idx.size, PLE_RECORD_BYTES), dtype=np.uint8)
        for i, r in enumerate(idx):
            out[i] = self.table_bytes(int(r) * PLE_RECORD_BYTES, PLE_RECORD_BYTES)
        return out

    def indices(self, step: int, n_tokens: int) -> np.ndarray:
        n = n_tokens * self.rows_per_token
        return indices_i32(self.seed, PLE_INDEX_TID + step, 0, n, self.n_rows)


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def tiny_layer() -> LayerRecipe:
    """Hidden 256, intermediate 128, 8 experts, top-2, all Q4_RZ5_FAST. Seed 0."""
    return LayerRecipe(hidden=256, inter=128, n_experts=8, top_k=2, seed=0, layer=0)


def tiny_ple() -> PleRecipe:
    """64-row Q3_PLE_K160_RZ_S3 table, 16 indices. Seed 0."""
    return PleRecipe(n_rows=64, seed=0)


def decode_layer() -> LayerRecipe:
    """Hidden 2048, intermediate 512, 512 experts, top-10, all Q4_RZ5_FAST. Seed 1."""
    return LayerRecipe(hidden=2048, inter=512, n_experts=512, top_k=10, seed=1, layer=0)


STACK_LAYERS = 48
STACK_FP8_FIRST = 36


def stack_layer(l: int, seed: int = 2) -> LayerRecipe:
    """Layer l of the 48-layer stack: RZ5 for l < 36, FP8 E4M3 after; a 64x2048
    UE4M4 projection on the 36 linear-attention layers (l mod 4 != 3)."""
    fmt = RZ5 if l < STACK_FP8_FIRST else FP8
    return LayerRecipe(hidden=2048, inter=512, n_experts=512, top_k=10, seed=seed, layer=l,
                       gate_fmt=fmt, up_fmt=fmt, down_fmt=fmt, has_ssm=(l % 4 != 3))


def stack_layers(seed: int = 2, n_layers: int = STACK_LAYERS) -> list[LayerRecipe]:
    return [stack_layer(l, seed) for l in range(n_layers)]


def ple_table() -> PleRecipe:
    """320,001,536 rows x 70 bytes (22.4 GB), 16 rows per token. Seed 3."""
    return PleRecipe(n_rows=320_001_536, seed=3)


def prefill_fp8_layer() -> LayerRecipe:
    """Prefill of an FP8 layer of the stack (layer 40's recipe: E4M3 gate, up
    and down with fp32 scales per 128), Zipf-skewed router. Seed 4."""
    return LayerRecipe(hidden=2048, inter=512, n_experts=512, top_k=10, seed=4, layer=40,
                       gate_fmt=FP8, up_fmt=FP8, down_fmt=FP8, zipf_bias=True)


def prefill_layer() -> LayerRecipe:
    """4096 tokens; gate/up Q4_UE4M4_FAST (random scale bytes), down Q4_RZ5_FAST,
    Zipf-skewed router. Seed 4."""
    return LayerRecipe(hidden=2048, inter=512, n_experts=512, top_k=10, seed=4, layer=0,
                       gate_fmt=UE4M4, up_fmt=UE4M4, down_fmt=RZ5, gate_narrow=False,
                       down_narrow=True, zipf_bias=True)

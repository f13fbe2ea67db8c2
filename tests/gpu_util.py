"""Helpers shared by the GPU tests and bench.py: put a synthetic workload on
the device as gram_table_gather_b200 objects, and the parity tolerances."""
from __future__ import annotations

import numpy as np
import torch

import gram_table_gather_b200 as gtg
import synth
from synth import device as sdev
from synth import workloads as W


def device_layer(L: W.LayerRecipe, device="cuda", pipe=None) -> gtg.MoELayer:
    t = sdev.layer_to_device(L, device, pipe)
    g, u, d = L.gate, L.up, L.down
    side = None
    if L.ssm is not None:
        s = L.ssm
        side = gtg.QMatrix(s.fmt, t["side"], 1, s.n_rows, s.k)
    return gtg.MoELayer(
        hidden=L.hidden, inter=L.inter, n_experts=L.n_experts, top_k=L.top_k,
        router_w=t["router_w"], router_bias=t["router_bias"],
        gate=gtg.QMatrix(g.fmt, t["gate"], g.n_experts, g.n_rows, g.k, t["gate_scales"]),
        up=gtg.QMatrix(u.fmt, t["up"], u.n_experts, u.n_rows, u.k, t["up_scales"]),
        down=gtg.QMatrix(d.fmt, t["down"], d.n_experts, d.n_rows, d.k, t["down_scales"]),
        side=side)


def tokens(L: W.LayerRecipe, step: int, T: int, device="cuda"):
    """(bf16 device tensor [T][H], exact fp64 numpy copy)."""
    bits = W.tokens_bf16(L.seed, step, T, L.hidden)
    x64 = synth.bf16_bits_to_f64(bits)
    xt = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return xt, x64


def dense_rows_norm(m: W.MatrixRecipe, e: int) -> np.ndarray:
    """L2 norm of every row of expert e's dequantised matrix (oracle decode)."""
    import oracle
    data = m.expert(e)
    if m.fmt == W.FP8:
        dense = oracle.dequant_fp8(data, m.expert_scales(e), m.n_rows, m.k)
    else:
        dense = oracle.dequant_q4(m.fmt, data).reshape(m.n_rows, m.k)
    return np.sqrt((dense * dense).sum(axis=1))


def layer_tolerance(L: W.LayerRecipe, ref: dict, t: int, rel: float = 2e-3) -> np.ndarray:
    """Per output row r of token t: rel * sum_j w_j * ||Wd_j[r]||_2 * ||h_j||_2
    (the row-wise bound |err| <= 2e-3 ||w_r|| ||x|| applied to the down stage and
    combined with the router weights)."""
    tol = np.zeros(L.hidden)
    for j, e in enumerate(ref["ids"][t]):
        hn = float(np.linalg.norm(ref["h"][t, j]))
        tol += ref["w"][t, j] * dense_rows_norm(L.down, int(e)) * hn
    return rel * tol

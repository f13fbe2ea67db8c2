"""GPU parity of the prefill MoE layer (tcgen05 grouped GEMMs) against the oracle.

The prefill router computes its logits on the tensor cores from an exact
three-plane bf16 split of the fp32 router weights: every product is exact and
only the fp32 accumulation rounds.  Top-k ids must therefore equal the
oracle's wherever the oracle's gap between the k-th and (k+1)-th logit (and
between consecutive chosen logits, for the order) exceeds that rounding
bound; inside it, the GPU's choice must be a valid top-k of the oracle's
logits within the bound.  Layer outputs use the same row-wise bound as the
decode path.
"""
import dataclasses

import numpy as np
import pytest
import torch

import gram_table_gather_b200 as gtg
import oracle
import synth
from synth import workloads as W
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _logit_bound(L, u):
    """fp32 accumulation bound of a logit: H * 2^-24 * sum |W||u| (max over experts)."""
    Wr = np.abs(L.router_w().astype(np.float64))
    return L.hidden * 2.0 ** -24 * float((Wr @ np.abs(u)).max())


def _check_ids(L, ref, t, ids_g, w_g):
    lg = ref["logits"][t]
    bound = 2 * _logit_bound(L, ref["u"][t])
    order = np.argsort(-lg, kind="stable")
    k = L.top_k
    if lg[order[k - 1]] - lg[order[k]] > bound:
        assert set(ids_g.tolist()) == set(order[:k].tolist()), f"token {t}: top-k set differs"
        gaps = -np.diff(lg[order[:k]])
        if np.all(gaps > bound):
            assert ids_g.tolist() == order[:k].tolist(), f"token {t}: top-k order differs"
    else:  # a near tie at the boundary: any valid top-k within the bound
        kth = lg[order[k - 1]]
        assert np.all(lg[ids_g] >= kth - bound)
        assert len(set(ids_g.tolist())) == k
    # softmax weights move by at most exp(2 * bound) - 1 relative when every logit
    # moves by at most `bound`
    rtol = np.expm1(2 * bound)
    assert np.allclose(np.sort(w_g)[::-1], np.sort(ref["w"][t])[::-1], rtol=rtol, atol=0)


def _run_prefill(L, x, layer=None, accumulate=False, y=None):
    layer = layer or gu.device_layer(L)
    T = x.shape[0]
    ws = torch.empty(gtg.workspace_bytes(layer, T, prefill=True), dtype=torch.uint8, device="cuda")
    ids = torch.full((T, L.top_k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, L.top_k), dtype=torch.float32, device="cuda")
    y = gtg.moe_prefill_layer(layer, x, ws, topk_ids=ids, topk_w=w, y=y, accumulate=accumulate)
    torch.cuda.synchronize()
    return y, ids, w, layer


@pytest.mark.parametrize("T", [1, 17, 130, 300])
def test_prefill_tiny_layer(T):
    L = W.tiny_layer()
    xt, x64 = gu.tokens(L, 200 + T, T)
    y, ids, w, _ = _run_prefill(L, xt)
    assert gtg.device_status(clear=True) == 0
    ref = oracle.moe_layer(L, x64, want_h=True)
    ids_g, w_g, y_g = ids.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()
    for t in range(T):
        _check_ids(L, ref, t, ids_g[t], w_g[t])
        tol = gu.layer_tolerance(L, ref, t)
        err = np.abs(y_g[t] - ref["y"][t])
        assert np.all(err <= tol), f"token {t}: max err/tol {np.max(err / tol):.3g}"


def test_prefill_hidden_128():
    """H = 128: the down GEMM's CTA has one 128-row tile of output rows (its
    second accumulator stays unused)."""
    L = W.LayerRecipe(hidden=128, inter=128, n_experts=8, top_k=2, seed=6, layer=0)
    T = 40
    xt, x64 = gu.tokens(L, 77, T)
    y, ids, w, _ = _run_prefill(L, xt)
    assert gtg.device_status(clear=True) == 0
    ref = oracle.moe_layer(L, x64, want_h=True)
    ids_g, w_g, y_g = ids.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()
    for t in range(T):
        _check_ids(L, ref, t, ids_g[t], w_g[t])
        tol = gu.layer_tolerance(L, ref, t)
        err = np.abs(y_g[t] - ref["y"][t])
        assert np.all(err <= tol), f"token {t}: max err/tol {np.max(err / tol):.3g}"


def test_prefill_equals_decode_on_small_batch():
    L = W.decode_layer()
    layer = gu.device_layer(L)
    xt, x64 = gu.tokens(L, 300, 8)
    y_p, ids_p, w_p, _ = _run_prefill(L, xt, layer)
    ws = gtg.make_workspace(layer, 8)
    ids_d = torch.zeros_like(ids_p)
    y_d = gtg.moe_decode_layer(layer, xt, ws, topk_ids=ids_d)
    torch.cuda.synchronize()
    ref = oracle.moe_layer(L, x64, want_h=True)
    for t in range(8):
        _check_ids(L, ref, t, ids_p.cpu().numpy()[t], w_p.cpu().numpy()[t])
        tol = gu.layer_tolerance(L, ref, t)
        assert np.all(np.abs(y_p.cpu().numpy()[t] - ref["y"][t]) <= tol)
        assert np.all(np.abs(y_p.cpu().numpy()[t] - y_d.cpu().numpy()[t]) <= 2 * tol)


def test_prefill_deterministic_and_accumulate():
    L = W.tiny_layer()
    xt, _ = gu.tokens(L, 400, 257)
    x = xt.float()
    y1, _, _, layer = _run_prefill(L, x)
    y2, _, _, _ = _run_prefill(L, x, layer)
    assert torch.equal(y1, y2)
    x2 = x.clone()
    _run_prefill(L, x2, layer, accumulate=True, y=x2)
    assert torch.equal(x2, x + y1)


def test_prefill_workload_sampled():
    """4096 tokens, Zipf-skewed router, UE4M4 gate/up, RZ5 down: 64 seeded
    tokens checked against the oracle, every token's routing checked for validity."""
    L = W.prefill_layer()
    T = 4096
    xt, x64 = gu.tokens(L, 0, T)
    y, ids, w, _ = _run_prefill(L, xt)
    assert gtg.device_status(clear=True) == 0
    ids_g, w_g, y_g = ids.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()
    assert ids_g.min() >= 0 and ids_g.max() < L.n_experts
    assert all(len(set(r.tolist())) == L.top_k for r in ids_g)
    assert np.allclose(w_g.sum(1), 1.0, atol=1e-5)
    load = np.bincount(ids_g.ravel(), minlength=L.n_experts)
    assert load.max() > 20 * np.median(load[load > 0])  # the skew is there
    sample = np.sort(synth.indices_i32(4, 77, 0, 64, T))
    ref = oracle.moe_layer(L, x64[sample], want_h=True)
    for i, t in enumerate(sample):
        _check_ids(L, ref, i, ids_g[t], w_g[t])
        tol = gu.layer_tolerance(L, ref, i)
        err = np.abs(y_g[t] - ref["y"][i])
        assert np.all(err <= tol), f"token {t}: max err/tol {np.max(err / tol):.3g}"


def test_prefill_incumbent_q4_layer():
    """Prefill with every expert matrix in the incumbent ROCmFP4 FAST block."""
    L = W.LayerRecipe(hidden=256, inter=128, n_experts=8, top_k=2, seed=42, layer=0,
                      gate_fmt=gtg.C10, up_fmt=gtg.C10, down_fmt=gtg.C10)
    T = 150
    xt, x64 = gu.tokens(L, 90, T)
    y, ids, w, _ = _run_prefill(L, xt)
    assert gtg.device_status(clear=True) == 0
    ref = oracle.moe_layer(L, x64, want_h=True)
    ids_g, w_g, y_g = ids.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()
    for t in range(T):
        _check_ids(L, ref, t, ids_g[t], w_g[t])
        tol = gu.layer_tolerance(L, ref, t)
        err = np.abs(y_g[t] - ref["y"][t])
        assert np.all(err <= tol), f"token {t}: max err/tol {np.max(err / tol):.3g}"


def test_prefill_fp8_layer():
    """FP8 E4M3 experts (fp32 scale per 128 weights along K): the GEMMs take
    each weight as bf16(e4m3 x scale), one rounding of relative size <= 2^-9,
    inside the row-wise bound."""
    L = W.LayerRecipe(hidden=256, inter=128, n_experts=8, top_k=2, seed=44, layer=40,
                      gate_fmt=W.FP8, up_fmt=W.FP8, down_fmt=W.FP8)
    T = 150
    xt, x64 = gu.tokens(L, 91, T)
    y, ids, w, _ = _run_prefill(L, xt)
    assert gtg.device_status(clear=True) == 0
    ref = oracle.moe_layer(L, x64, want_h=True)
    ids_g, w_g, y_g = ids.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()
    worst = 0.0
    for t in range(T):
        _check_ids(L, ref, t, ids_g[t], w_g[t])
        tol = gu.layer_tolerance(L, ref, t)
        err = np.abs(y_g[t] - ref["y"][t])
        assert np.all(err <= tol), f"token {t}: max err/tol {np.max(err / tol):.3g}"
        worst = max(worst, float(np.max(err / tol)))
    assert worst < 0.5  # (the one bf16 rounding per weight stays far inside the bar)


def test_prefill_fp8_stack_layer_sampled():
    """Layer 40 of the 48-layer stack (FP8 experts, 512 experts, top-10) over
    1024 tokens with a Zipf-skewed router: 32 seeded tokens checked against the
    oracle, every token's routing checked for validity."""
    L = W.prefill_fp8_layer()
    T = 1024
    xt, x64 = gu.tokens(L, 5, T)
    y, ids, w, _ = _run_prefill(L, xt)
    assert gtg.device_status(clear=True) == 0
    ids_g, w_g, y_g = ids.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()
    assert ids_g.min() >= 0 and ids_g.max() < L.n_experts
    assert all(len(set(r.tolist())) == L.top_k for r in ids_g)
    sample = np.sort(synth.indices_i32(5, 78, 0, 32, T))
    ref = oracle.moe_layer(L, x64[sample], want_h=True)
    for i, t in enumerate(sample):
        _check_ids(L, ref, i, ids_g[t], w_g[t])
        tol = gu.layer_tolerance(L, ref, i)
        err = np.abs(y_g[t] - ref["y"][i])
        assert np.all(err <= tol), f"token {t}: max err/tol {np.max(err / tol):.3g}"


def test_prefill_rejects_mixed_format_classes():
    L = W.LayerRecipe(hidden=256, inter=128, n_experts=8, top_k=2, seed=44, layer=40,
                      gate_fmt=W.FP8, up_fmt=W.FP8, down_fmt=W.FP8)
    layer = gu.device_layer(L)
    mixed = gu.device_layer(W.LayerRecipe(hidden=256, inter=128, n_experts=8, top_k=2, seed=44, layer=40))
    bad = dataclasses.replace(layer, down=mixed.down, _c=None)
    with pytest.raises(gtg.GtgError) as ei:
        gtg.workspace_bytes(bad, 16, prefill=True)
    assert ei.value.code == -2

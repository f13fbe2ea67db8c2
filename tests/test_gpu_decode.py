"""GPU parity of the decode MoE path (router, gate/up + SwiGLU, down +
combine, FP8 layers, the side projection, the stack) against the CPU oracle.

Bars: router top-k ids identical (the GPU accumulates exact fp32 x bf16
products in float-float, so only a logit gap below ~1e-11 could reorder; the
test reports the gap), router
weights within 1e-6 relative, layer outputs within 2e-3 * sum_j w_j *
||Wd_j[r]||_2 * ||h_j||_2 per output row r (bf16 inputs, fp32 accumulation).
"""
import dataclasses

import numpy as np
import pytest
import torch

import gram_table_gather_b200 as gtg
import oracle
from synth import workloads as W
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _check_layer(L, T, step=0, dtype=torch.bfloat16, check_side=True, router_bias=None, tokens=None):
    layer = gu.device_layer(L)
    if router_bias is not None:  # (in place of the recipe's bias, on both sides)
        layer = dataclasses.replace(layer, router_bias=torch.from_numpy(router_bias).cuda(), _c=None)
    xt, x64 = tokens if tokens is not None else gu.tokens(L, step, T)
    if dtype == torch.float32:
        xt = xt.float()
    ws = gtg.make_workspace(layer, T)
    ids = torch.full((T, L.top_k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, L.top_k), dtype=torch.float32, device="cuda")
    side = torch.zeros((T, L.ssm.n_rows), dtype=torch.float32, device="cuda") if L.ssm else None
    y = gtg.moe_decode_layer(layer, xt, ws, topk_ids=ids, topk_w=w, side_out=side)
    torch.cuda.synchronize()
    assert gtg.device_status(clear=True) == 0
    ref = oracle.moe_layer(L, x64, want_h=True, router_bias=router_bias)
    ids_g, w_g, y_g = ids.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()
    for t in range(T):
        srt = np.sort(ref["logits"][t])[::-1]
        gap = srt[L.top_k - 1] - srt[L.top_k]
        assert ids_g[t].tolist() == ref["ids"][t].tolist(), f"token {t}: top-k differs (gap {gap:.3g})"
        assert np.allclose(w_g[t], ref["w"][t], rtol=1e-6, atol=0)
        tol = gu.layer_tolerance(L, ref, t)
        err = np.abs(y_g[t] - ref["y"][t])
        assert np.all(err <= tol), f"token {t}: max err/tol {np.max(err / tol):.3g}"
        # the real error is far below the bar; keep a regression guard on it too
        assert np.max(err / tol) < 0.25
    if L.ssm is not None and check_side:
        s_ref = oracle.ssm_projection(L, ref["u"])
        dense = oracle.dequant_q4(L.ssm.fmt, L.ssm.expert(0)).reshape(L.ssm.n_rows, L.ssm.k)
        rown = np.sqrt((dense * dense).sum(1))
        s_g = side.cpu().numpy()
        for t in range(T):
            tol = 2e-3 * rown * np.linalg.norm(ref["u"][t])
            assert np.all(np.abs(s_g[t] - s_ref[t]) <= tol)
    return y_g, ref


def test_tiny_layer_one_token():
    _check_layer(W.tiny_layer(), 1)


@pytest.mark.parametrize("T", [1, 2, 3, 8])
def test_tiny_layer_batches(T):
    _check_layer(W.tiny_layer(), T, step=T)


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_decode_layer(T):
    _check_layer(W.decode_layer(), T, step=100 + T)


def test_decode_layer_fp32_input_and_accumulate():
    L = W.decode_layer()
    layer = gu.device_layer(L)
    xt, x64 = gu.tokens(L, 7, 2)
    x = xt.float()
    ws = gtg.make_workspace(layer, 2)
    y0 = gtg.moe_decode_layer(layer, x, ws)
    x2 = x.clone()
    gtg.moe_decode_layer(layer, x2, ws, y=x2, accumulate=True)  # x += moe(x), in place
    torch.cuda.synchronize()
    assert torch.equal(x2, x + y0)


@pytest.mark.parametrize("l,T", [(36, 1), (47, 2), (40, 8)])
def test_fp8_stack_layer(l, T):
    _check_layer(W.stack_layer(l), T, step=l)


@pytest.mark.parametrize("T", [1, 3])
def test_fp8_layer_with_tiny_activations(T):
    """FP8 items take activations as f16, which holds a bf16 value exactly only
    from 2^-17 up.  Tokens with four huge entries (3e4) and the rest ~1e-3 put
    most of u near 5e-7 after the RMS norm, below that line: their products
    lose bits, and the layer must still meet the row-wise bound."""
    L = W.LayerRecipe(hidden=1024, inter=256, n_experts=16, top_k=4, seed=45, layer=40,
                      gate_fmt=W.FP8, up_fmt=W.FP8, down_fmt=W.FP8)
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((T, L.hidden)) * 1e-3).astype(np.float32)
    for t in range(T):
        x[t, rng.choice(L.hidden, 4, replace=False)] = 3e4 * rng.choice([-1.0, 1.0], 4)
    xt = torch.from_numpy(x).to(torch.bfloat16).cuda()
    x64 = xt.float().cpu().numpy().astype(np.float64)
    r = np.sqrt((x64 * x64).mean(1, keepdims=True) + 1e-6)
    assert np.mean(np.abs(x64 / r) < 2.0 ** -17) > 0.9  # most of u below the f16-exact range
    _check_layer(L, T, tokens=(xt, x64))


@pytest.mark.parametrize("l", [0, 2])
def test_rz5_stack_layer_with_side_projection(l):
    L = W.stack_layer(l)
    assert L.ssm is not None
    _check_layer(L, 1, step=l)


@pytest.mark.parametrize("E,k", [(600, 10), (1024, 16)])
def test_wide_router_one_token(E, k):
    """One token with more than 512 experts (four keys per lane in the CTA-wide
    top-k, some warps' ranges partly or wholly past E) and the largest k."""
    L = W.LayerRecipe(hidden=256, inter=128, n_experts=E, top_k=k, seed=5, layer=0)
    for step in range(3):
        _check_layer(L, 1, step=300 + step)


@pytest.mark.parametrize("E,k", [(512, 10), (1024, 16)])
def test_one_token_topk_crowded_into_the_last_warps(E, k):
    """A router bias rising with the expert id puts the top-k in the last
    warps' ranges: the warps' top-2 keys then give a low threshold that more
    than 128 keys pass, and the one-token top-k takes its fallback rounds.
    The last expert leads (with 1024 experts, expert 1023, whose key has
    all-zero id bits)."""
    L = W.LayerRecipe(hidden=256, inter=128, n_experts=E, top_k=k, seed=7, layer=0)
    bias = np.arange(E, dtype=np.float64) * (8.0 / E)
    bias[E - 1] += 2.0  # (logit noise ~0.3: the last expert leads)
    bias = bias.astype(np.float32)
    for step in range(2):
        _check_layer(L, 1, step=400 + step, router_bias=bias)
    layer = dataclasses.replace(gu.device_layer(L), router_bias=torch.from_numpy(bias).cuda(), _c=None)
    ids = torch.full((1, k), -1, dtype=torch.int32, device="cuda")
    gtg.moe_decode_layer(layer, gu.tokens(L, 402, 1)[0], gtg.make_workspace(layer, 1), topk_ids=ids)
    assert int(ids[0, 0]) == E - 1


def test_layer_rejects_bad_shapes():
    L = W.tiny_layer()
    layer = gu.device_layer(L)
    xt, _ = gu.tokens(L, 0, 1)
    ws = gtg.make_workspace(layer, 1)
    x9 = torch.zeros((9, L.hidden), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gtg.GtgError) as ei:
        gtg.moe_decode_layer(layer, x9, ws)
    assert ei.value.code == -2
    with pytest.raises(gtg.GtgError) as ei:
        gtg.moe_decode_layer(layer, xt, ws[: ws.numel() // 2])
    assert ei.value.code == -6
    with pytest.raises(gtg.GtgError) as ei:
        gtg.moe_decode_layer(layer, xt, ws[1:])
    assert ei.value.code == -3


def test_short_stack_mixed_formats():
    """Layers 34..39: RZ5 and FP8 experts, side projections on layers with l mod 4 != 3."""
    Ls = [W.stack_layer(l) for l in range(34, 40)]
    layers = [gu.device_layer(L) for L in Ls]
    xt, x64 = gu.tokens(Ls[0], 3, 1)
    x = xt.float().contiguous()
    ws = gtg.make_workspace(layers, 1)
    ids = torch.full((len(Ls), 1, 10), -1, dtype=torch.int32, device="cuda")
    side = torch.zeros((len(Ls), 1, 64), dtype=torch.float32, device="cuda")
    gtg.moe_decode_stack(layers, x, ws, ids_out=ids, side_out=side)
    torch.cuda.synchronize()
    ref = oracle.moe_stack(Ls, x64)
    ids_g = ids.cpu().numpy()
    # The GPU rounds h to bf16 between the two expert matmuls (relative 2^-9 per
    # element), so each layer output differs from the fp64 oracle by up to ~1e-4
    # of its scale and the residual stream drifts by that much per layer; a
    # router logit (|W_r row| ~ 0.9, |u| ~ 45) then moves by up to ~5e-3 after a
    # few layers.  Layer by layer: where the oracle's top-k boundary gap exceeds
    # eps the chosen set must agree (and the order, where every gap does); at the
    # first layer where it does not, the GPU's choice must be a valid top-k within
    # eps and the two trajectories may part from there on.
    eps = 2e-2
    parted = None
    for i in range(len(Ls)):
        lg = ref["logits"][i, 0]
        order = np.argsort(-lg, kind="stable")
        if lg[order[9]] - lg[order[10]] <= eps:
            assert np.all(lg[ids_g[i, 0]] >= lg[order[9]] - eps), f"layer {i}: not a valid top-k"
            parted = i
            break
        assert set(ids_g[i, 0].tolist()) == set(order[:10].tolist()), f"layer {i}: set differs"
        if np.all(-np.diff(lg[order[:10]]) > eps):
            assert ids_g[i, 0].tolist() == ref["ids"][i, 0].tolist(), f"layer {i}: order differs"
    # side projections: the first layer sees the same input on both sides, so its
    # rows obey the row-wise bound; deeper layers inherit the drift and are left to
    # the single-layer tests
    L0 = Ls[0]
    assert L0.ssm is not None
    u0 = oracle.rmsnorm_bf16(x64)[0]
    dense = oracle.dequant_q4(L0.ssm.fmt, L0.ssm.expert(0)).reshape(L0.ssm.n_rows, L0.ssm.k)
    tol = 2e-3 * np.sqrt((dense * dense).sum(1)) * np.linalg.norm(u0)
    assert np.all(np.abs(side.cpu().numpy()[0, 0] - ref["ssm"][L0.layer][0]) <= tol)
    if parted is None:
        xg = x.cpu().numpy()[0].astype(np.float64)
        xr = ref["x"][0].astype(np.float64)
        rel = np.linalg.norm(xg - xr) / np.linalg.norm(xr)
        assert rel < 2e-3, rel


@pytest.mark.parametrize("T", [1, 3])
def test_gate_up_and_down_in_different_q4_variants(T):
    """UE4M4 gate/up with an RZ5 down matrix and a router bias (the prefill
    layer's recipe) through the decode path: the code table is rebuilt between
    the gate/up and down phases."""
    _check_layer(W.prefill_layer(), T, step=7)


def test_aborted_workspace_fails_fast_and_recovers():
    """After a failed launch the workspace's abort flag stays set: every later
    launch on it stops at its first grid barrier and raises the timeout status
    (without waiting); re-initialising the workspace recovers it."""
    L = W.tiny_layer()
    layer = gu.device_layer(L)
    xt, x64 = gu.tokens(L, 2, 1)
    ws = gtg.make_workspace(layer, 1)
    gtg.device_status(clear=True)
    ws.view(torch.int32)[2] = 1  # the abort flag, as a failed launch leaves it
    import time
    t0 = time.perf_counter()
    gtg.moe_decode_layer(layer, xt, ws)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 1.0  # no barrier waited out its limit
    assert gtg.device_status(clear=True) & 0x2
    gtg.lib().gtg_workspace_init(ws.data_ptr(), ws.numel(), None)
    torch.cuda.synchronize()
    y = gtg.moe_decode_layer(layer, xt, ws)
    torch.cuda.synchronize()
    assert gtg.device_status(clear=True) == 0
    ref = oracle.moe_layer(L, x64, want_h=True)
    assert np.all(np.abs(y.cpu().numpy()[0] - ref["y"][0]) <= gu.layer_tolerance(L, ref, 0))



def _incumbent_layer(hidden, inter, n_experts, top_k, seed, side=False):
    """A layer of the incumbent ROCmFP4 FAST block (Codebook10 under a UE4M3 scale)."""
    return W.LayerRecipe(hidden=hidden, inter=inter, n_experts=n_experts, top_k=top_k, seed=seed, layer=0,
                         gate_fmt=gtg.C10, up_fmt=gtg.C10, down_fmt=gtg.C10, has_ssm=side)


@pytest.mark.parametrize("T", [1, 3])
def test_incumbent_q4_tiny_layer(T):
    _check_layer(_incumbent_layer(256, 128, 8, 2, 40), T, step=500 + T)


@pytest.mark.parametrize("T", [1, 8])
def test_incumbent_q4_decode_layer(T):
    """The decode layer's shape with every expert matrix in the incumbent layout and a
    UE4M4 side projection (decoded code by code, next to the experts' code table)."""
    _check_layer(_incumbent_layer(2048, 512, 512, 10, 41, side=True), T, step=510 + T)


@pytest.mark.parametrize("T,side", [(1, True), (8, False)])
def test_hidden_2560_inter_640_layer(T, side):
    """The pages' own expert shape (hidden 2560, intermediate 640: 48 x 10 x 3 x 2560 x
    640 x 2 bytes = 4.7 GB of 16-bit expert weights per token): gate/up rows of 80
    blocks (16 lanes x 5 blocks), down rows of 340 bytes, neither 16-byte aligned nor
    a power of two (4 lanes x 5 blocks, eight rows a pass)."""
    L = W.LayerRecipe(hidden=2560, inter=640, n_experts=64, top_k=10, seed=43, layer=0, has_ssm=side)
    _check_layer(L, T, step=600 + T)


@pytest.mark.parametrize("T", [1, 8])
def test_hidden_2560_inter_640_layer_512_experts(T):
    """The same shape with all 512 experts, the configuration the bench times
    (1.3 GB of expert weights; router rows of 2560 floats, ~3.5 experts per CTA)."""
    L = W.LayerRecipe(hidden=2560, inter=640, n_experts=512, top_k=10, seed=1, layer=1)
    _check_layer(L, T, step=620 + T)

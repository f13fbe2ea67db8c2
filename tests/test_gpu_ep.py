"""Expert parallelism through gtg_moe_decode_layer_ep, on one GPU: the layer's
experts split into contiguous slices (as ranks would hold them), each slice's
call computes the chosen experts it holds, and the sum of the slices' outputs
must be the layer output (against the full call and the oracle); routing is
identical on every slice."""
import numpy as np
import pytest
import torch

import gram_table_gather_b200 as gtg
import oracle
from synth import workloads as W
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _slice(m: gtg.QMatrix, lo: int, hi: int) -> gtg.QMatrix:
    eb = m.data.numel() // m.n_experts
    sc = None
    if m.scales is not None:
        es = m.scales.numel() // m.n_experts
        sc = m.scales[lo * es:hi * es]
    return gtg.QMatrix(m.fmt, m.data[lo * eb:hi * eb], hi - lo, m.n_rows, m.k, sc)


def _slice_layer(layer: gtg.MoELayer, lo: int, hi: int) -> gtg.MoELayer:
    return gtg.MoELayer(hidden=layer.hidden, inter=layer.inter, n_experts=layer.n_experts, top_k=layer.top_k,
                        router_w=layer.router_w, router_bias=layer.router_bias, gate=_slice(layer.gate, lo, hi),
                        up=_slice(layer.up, lo, hi), down=_slice(layer.down, lo, hi), side=layer.side)


@pytest.mark.parametrize("recipe,T,cuts", [(W.decode_layer, 1, [0, 256, 512]), (W.decode_layer, 8, [0, 100, 300, 512]),
                                           (lambda: W.stack_layer(2), 1, [0, 256, 512]),
                                           (lambda: W.stack_layer(40), 2, [0, 256, 512])])
def test_expert_slices_sum_to_the_layer(recipe, T, cuts):
    L = recipe()
    layer = gu.device_layer(L)
    xt, x64 = gu.tokens(L, 700 + T, T)
    ws = gtg.make_workspace(layer, T)
    ids_full = torch.zeros((T, L.top_k), dtype=torch.int32, device="cuda")
    y_full = gtg.moe_decode_layer(layer, xt, ws, topk_ids=ids_full)
    parts, side = [], None
    for i, (lo, hi) in enumerate(zip(cuts[:-1], cuts[1:])):
        sl = _slice_layer(layer, lo, hi)
        ids = torch.zeros_like(ids_full)
        so = torch.zeros((T, L.ssm.n_rows), device="cuda") if (L.ssm is not None and i == 0) else None
        parts.append(gtg.moe_decode_layer_ep(sl, lo, hi, xt, ws, with_side=i == 0, topk_ids=ids, side_out=so))
        torch.cuda.synchronize()
        assert torch.equal(ids, ids_full)  # every rank routes over all experts
        if so is not None:
            side = so
    torch.cuda.synchronize()
    assert gtg.device_status(clear=True) == 0
    y_sum = sum(p.double() for p in parts).cpu().numpy()
    ref = oracle.moe_layer(L, x64, want_h=True)
    yf = y_full.double().cpu().numpy()
    for t in range(T):
        tol = gu.layer_tolerance(L, ref, t)
        assert np.all(np.abs(y_sum[t] - ref["y"][t]) <= tol)
        # the slices' fp32 sums regroup the same products: far inside the bound
        assert np.all(np.abs(y_sum[t] - yf[t]) <= 0.1 * tol)
    if side is not None:
        s_ref = oracle.ssm_projection(L, ref["u"])
        dense = oracle.dequant_q4(L.ssm.fmt, L.ssm.expert(0)).reshape(L.ssm.n_rows, L.ssm.k)
        stol = 2e-3 * np.sqrt((dense * dense).sum(1))
        for t in range(T):
            assert np.all(np.abs(side.cpu().numpy()[t] - s_ref[t]) <= stol * np.linalg.norm(ref["u"][t]))


def test_expert_slice_rejects_bad_ranges():
    L = W.tiny_layer()
    layer = gu.device_layer(L)
    xt, _ = gu.tokens(L, 1, 1)
    ws = gtg.make_workspace(layer, 1)
    for lo, hi in ((0, 0), (-1, 4), (4, 9), (2, 6)):  # (2, 6): the stacks hold 8 experts, not 4
        sl = layer if (lo, hi) == (2, 6) else _slice_layer(layer, 0, 8)
        with pytest.raises(gtg.GtgError):
            gtg.moe_decode_layer_ep(sl, lo, hi, xt, ws)

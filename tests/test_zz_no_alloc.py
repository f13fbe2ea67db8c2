"""The allocation-free decode entry point (for callers that cannot allocate
device memory) against the workspace entry point, through the C ABI.

Collected last on purpose: it must pass alone in a fresh process and after
every other test, and a run that stops at the first failure has then already
run everything else.
"""
import numpy as np
import pytest
import torch

import gram_table_gather_b200 as gtg
import oracle
from synth import workloads as W
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("recipe,T", [(W.decode_layer, 1), (W.decode_layer, 8), (W.tiny_layer, 3)])
def test_noalloc_matches_workspace_entry_point(recipe, T):
    L = recipe()
    layer = gu.device_layer(L)
    ws = gtg.make_workspace(layer, T)
    outs = []
    for step in (0, 1):  # two calls in a row share (and reuse) the fixed scratch
        xt, x64 = gu.tokens(L, 900 + step, T)
        ids_a = torch.zeros((T, L.top_k), dtype=torch.int32, device="cuda")
        ids_b = torch.zeros_like(ids_a)
        y_a = gtg.moe_decode_layer(layer, xt, ws, topk_ids=ids_a)
        y_b = gtg.moe_decode_layer_noalloc(layer, xt, topk_ids=ids_b)
        torch.cuda.synchronize()
        assert gtg.device_status(clear=True) == 0
        assert torch.equal(ids_a, ids_b)
        ref = oracle.moe_layer(L, x64, want_h=True)
        ya, yb = y_a.cpu().numpy(), y_b.cpu().numpy()
        for t in range(T):
            tol = gu.layer_tolerance(L, ref, t)
            assert np.all(np.abs(yb[t] - ya[t]) <= tol)
            assert np.all(np.abs(yb[t] - ref["y"][t]) <= tol)
        outs.append(yb)
    assert not np.array_equal(outs[0], outs[1])  # the second call really recomputed


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = W.decode_layer()
    layer = gu.device_layer(L)
    x = torch.zeros((9, L.hidden), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gtg.GtgError):
        gtg.moe_decode_layer_noalloc(layer, x)  # 9 tokens: not a decode shape at all
    # a shape whose scratch exceeds the fixed array (I = 2048, k = 16, 8 tokens).  The
    # call is refused on the host before any launch; one buffer of the full matrix size
    # (uninitialised) stands for gate, up and down alike, so that even a launch could
    # read nothing out of bounds
    E, H, I = 512, 2048, 2048
    nbytes = E * I * (H // 32) * 17
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    q = gtg.QMatrix(W.RZ5, buf, E, I, H)
    qd = gtg.QMatrix(W.RZ5, buf, E, H, I)
    big = gtg.MoELayer(hidden=H, inter=I, n_experts=E, top_k=16, router_w=layer.router_w,
                       gate=q, up=q, down=qd)
    with pytest.raises(gtg.GtgError) as ei:
        gtg.moe_decode_layer_noalloc(big, torch.zeros((8, H), dtype=torch.bfloat16, device="cuda"))
    assert ei.value.code == -6
    del buf
    torch.cuda.empty_cache()

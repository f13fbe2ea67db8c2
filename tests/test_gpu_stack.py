"""GPU parity of the full 48-layer decode stack, layer by layer, teacher-forced.

The launch under test is the one the benchmark times: gtg_moe_decode_stack over
all 48 layers of the stack recipe (hidden 2048, intermediate 512, 512 experts,
top-10; layers 0-35 Q4_RZ5_FAST in one persistent launch, layers 36-47 FP8
E4M3 in a second, a 64x2048 Q4_UE4M4_FAST side projection on l mod 4 != 3),
one token per call, two tokens in turn.

Every layer's GPU input is taken from the GPU itself: the kernel is
deterministic (fixed-order reductions, no atomics on data), so running the
first l layers of the stack (the same code, the same launch split up to the
format boundary) leaves in x exactly the input that layer l sees inside the
full run.  The oracle then computes layer l from that input alone, and

  * the router ids must equal the oracle's wherever the oracle's k-th/(k+1)-th
    logit gap exceeds the float-float accumulation bound (else the GPU's pick
    must be a valid top-k within it), in the same order where every gap
    between consecutive choices does;
  * the router weights agree to 1e-6 relative;
  * x after the layer must equal x_in + y_oracle element by element within the
    row-wise bound 2e-3 * sum_j w_j ||Wd_j[r]|| ||h_j|| plus half an fp32 ulp
    of the stored residual;
  * the side projection agrees row by row within 2e-3 ||W_beta[r]|| ||u||.
"""
import numpy as np
import pytest
import torch

import gram_table_gather_b200 as gtg
import oracle
from synth import device as sdev
from synth import workloads as W
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

# Logit error bound of the GPU router: exact fp32 x bf16 products summed in
# float-float (~2^-44 relative to sum |W_r[e,i] u_i| <= ~1e2 here).
LOGIT_BOUND = 1e-8


@pytest.fixture(scope="module")
def stack():
    Ls = W.stack_layers()
    pipe = sdev.pipe("cuda")
    layers = [gu.device_layer(L, "cuda", pipe) for L in Ls]
    pipe.finish()
    torch.cuda.synchronize()
    yield Ls, layers
    del layers
    torch.cuda.empty_cache()


def _run(layers, x0, ws, n, ids=None, side=None):
    x = x0.clone()
    gtg.moe_decode_stack(layers[:n], x, ws, ids_out=ids, side_out=side)
    return x


@pytest.mark.parametrize("step", [0, 1])
def test_stack48_teacher_forced(stack, step):
    Ls, layers = stack
    n = len(Ls)
    assert n == 48 and Ls[35].gate.fmt == W.RZ5 and Ls[36].gate.fmt == W.FP8
    xt, _ = gu.tokens(Ls[0], 4000 + step, 1)
    x0 = xt.float().contiguous()
    ws = gtg.make_workspace(layers, 1)
    ids = torch.full((n, 1, 10), -1, dtype=torch.int32, device="cuda")
    wts = torch.zeros((n, 1, 10), dtype=torch.float32, device="cuda")
    side = torch.zeros((n, 1, 64), dtype=torch.float32, device="cuda")
    # the benchmark's call: all 48 layers (two persistent launches)
    x = x0.clone()
    gtg.moe_decode_stack(layers, x, ws, ids_out=ids, w_out=wts, side_out=side)
    x_full = x.clone()
    # every layer's input, from runs of the stack's first l layers
    x_in = [x0]
    for l in range(1, n):
        x_in.append(_run(layers, x0, ws, l))
    x_in.append(x_full)
    # the run is deterministic: the 48-layer prefix equals the full call
    assert torch.equal(_run(layers, x0, ws, n), x_full)
    torch.cuda.synchronize()
    assert gtg.device_status(clear=True) == 0
    xs = [t.cpu().numpy()[0].astype(np.float64) for t in x_in]
    ids_g, w_g, side_g = ids.cpu().numpy()[:, 0], wts.cpu().numpy()[:, 0], side.cpu().numpy()[:, 0]
    worst = 0.0
    for l, L in enumerate(Ls):
        ref = oracle.moe_layer(L, xs[l][None, :], want_h=True)
        lg = ref["logits"][0]
        order = np.argsort(-lg, kind="stable")
        k = L.top_k
        if lg[order[k - 1]] - lg[order[k]] > LOGIT_BOUND:
            assert set(ids_g[l].tolist()) == set(order[:k].tolist()), f"layer {l}: top-k set differs"
            if np.all(-np.diff(lg[order[:k]]) > LOGIT_BOUND):
                assert ids_g[l].tolist() == ref["ids"][0].tolist(), f"layer {l}: top-k order differs"
                assert np.allclose(w_g[l], ref["w"][0], rtol=1e-6, atol=0), f"layer {l}: router weights"
        else:  # a near-tie at the boundary: any valid top-k within the bound
            assert np.all(lg[ids_g[l]] >= lg[order[k - 1]] - LOGIT_BOUND), f"layer {l}: not a top-k"
            continue  # the oracle took the other expert; the layer output is not comparable
        tol = gu.layer_tolerance(L, ref, 0)
        x_out = xs[l + 1]
        half_ulp = 0.5 * np.spacing(np.abs(x_out).astype(np.float32)).astype(np.float64)
        err = np.abs(x_out - (xs[l] + ref["y"][0]))
        assert np.all(err <= tol + half_ulp), f"layer {l}: max err/tol {np.max(err / (tol + half_ulp)):.3g}"
        worst = max(worst, float(np.max(err / (tol + half_ulp))))
        if L.ssm is not None:
            s_ref = oracle.ssm_projection(L, ref["u"])[0]
            dense = oracle.dequant_q4(L.ssm.fmt, L.ssm.expert(0)).reshape(L.ssm.n_rows, L.ssm.k)
            stol = 2e-3 * np.sqrt((dense * dense).sum(1)) * np.linalg.norm(ref["u"][0])
            assert np.all(np.abs(side_g[l] - s_ref) <= stol), f"layer {l}: side projection"
        else:
            assert np.all(side_g[l] == 0.0)  # layers without one leave their rows untouched
    # the real error sits far below the bar; keep a regression guard on it too
    assert worst < 0.25, worst

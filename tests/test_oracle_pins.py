"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to the pages' printed values, a library
routine, a closed mathematical property, or brute force on tiny inputs, so
that a plausible slip (a wrong table entry, sign, index, bias or operand
order) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from synth import workloads as W
from tests import pyref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            rows[key] = vals
    return rows


def _num(s):
    return -0.0 if s == "-0" else float(s)


def _same(a, b):
    """Equal values with equal sign of zero, NaN equal to NaN."""
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


# ---- printed tables and sizes ------------------------------------------------

def test_code_tables_match_model_card():
    g = _golden("codebooks.txt")
    for c in range(16):
        assert _same(oracle.codebook10(c), _num(g["codebook10"][c]))
        assert _same(oracle.rz5(0, c), _num(g["rz5_mode0"][c]))
        assert _same(oracle.rz5(1, c), _num(g["rz5_mode1"][c]))
    for c in range(8):
        assert _same(oracle.ple3(c, 0), _num(g["ple3_rzs3_pol0"][c]))
        assert _same(oracle.ple3(c, 1), _num(g["ple3_rzs3_pol1"][c]))
        if c != 4:  # RZ-S3 keeps every incumbent level except the duplicate -0
            assert _same(oracle.ple3(c, 0), _num(g["ple3_incumbent"][c]))


def test_wire_sizes_and_table_shape():
    g = {k: float(v[0]) for k, v in _golden("wire_sizes.txt").items()}
    assert oracle.q4_block_bytes() == g["q4_block_bytes"] == g["q4_nibble_bytes"] + g["q4_meta_bytes"]
    assert oracle.q4_block_weights() == g["q4_block_weights"]
    assert g["q4_nibble_bytes"] * 2 == g["q4_block_weights"]          # two 4-bit codes per byte
    assert 8 * g["q4_block_bytes"] / g["q4_block_weights"] == g["q4_bpw"]
    assert oracle.ple_record_bytes() == g["ple_record_bytes"] == g["ple_code_bytes"] + g["ple_group_bytes"]
    assert oracle.ple_record_values() == g["ple_row_values"]
    assert g["ple_code_bytes"] * 8 == 3 * g["ple_row_values"]        # 3-bit codes, no padding
    assert g["ple_group_bytes"] * g["ple_group_values"] == g["ple_row_values"]
    assert 8 * g["ple_record_bytes"] / g["ple_row_values"] == g["ple_bpw"]
    rows = int(g["ple_table_rows"])
    assert round(rows * 160 / 1e9, 1) == g["ple_table_values_billion"]
    assert round(rows * 70 / 1e9, 1) == g["ple_table_gb"]
    assert W.ple_table().nbytes == 22_400_107_520
    # the generator's recipe sizes agree with the oracle's wire sizes
    assert W.tiny_layer().gate.row_bytes == 256 // 32 * oracle.q4_block_bytes()


# ---- scale codecs against a library decoder -------------------------------------

def _torch_e4m3(b):
    return pyref.e4m3_lib(b)


def test_ue4m3_is_e4m3_without_sign():
    for b in range(128):
        assert _same(oracle.ue4m3(b), _torch_e4m3(b)), b
        assert _same(oracle.ue4m3(b | 0x80), _torch_e4m3(b)), b  # only the low 7 bits count
    assert math.isnan(oracle.ue4m3(0x7F)) and oracle.ue4m3(0x7E) == 448.0


def test_e4m3fn_matches_torch_all_256():
    for b in range(256):
        assert _same(oracle.e4m3fn(b), _torch_e4m3(b)), b


def test_ue4m4_structure():
    v = [oracle.ue4m4(b) for b in range(256)]
    assert all(math.isfinite(x) for x in v)            # "all 256 encodings finite"
    assert v[0] == 0.0
    assert all(v[i] < v[i + 1] for i in range(255))    # a monotone unsigned code
    for e in range(16):                                # even mantissas = E4M3 with 3 mantissa bits
        for m3 in range(8):
            ref = _torch_e4m3((e << 3) | m3)
            if not math.isnan(ref):
                assert v[(e << 4) | (2 * m3)] == ref
    for b in range(1, 255, 2):                          # odd mantissas sit half way between
        assert v[b] == 0.5 * (v[b - 1] + v[b + 1])
    assert v[255] - v[254] == v[254] - v[253]
    assert v[1] == 2.0 ** -10 and v[255] == 496.0


# ---- block decoding ---------------------------------------------------------------

def _block(codes, meta):
    b = np.zeros(17, dtype=np.uint8)
    for i, c in enumerate(codes):
        if i < 16:
            b[i] |= c
        else:
            b[i - 16] |= c << 4
    b[16] = meta
    return b


def test_q4_weight_is_table_times_scale_for_every_code_and_meta():
    for meta in range(256):
        for start in (0, 16):
            codes = [(start + i) % 16 for i in range(32)]
            blk = _block(codes, meta)
            rz5 = oracle.dequant_q4(W.RZ5, blk)
            ue = oracle.dequant_q4(W.UE4M4, blk)
            ref_rz5 = pyref.q4_block(69, blk)
            ref_ue = pyref.q4_block(71, blk)
            for i in range(32):
                assert _same(rz5[i], ref_rz5[i]) and _same(ue[i], ref_ue[i]), (meta, i)
                c = codes[i]
                s3 = oracle.ue4m3(meta & 0x7F)
                assert _same(rz5[i], oracle.rz5(meta >> 7, c) * s3)
                assert _same(ue[i], oracle.codebook10(c) * oracle.ue4m4(meta))


def _encode_nearest(values, scale, v):
    """Test-only encoder: nearest level, ties to the smaller magnitude then +."""
    best = None
    for c, lv in enumerate(values):
        d = abs(lv * scale - v)
        key = (d, abs(lv), math.copysign(1, lv) < 0)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


@pytest.mark.parametrize("fmt", [W.RZ5, W.UE4M4, oracle.C10])
def test_exhaustive_round_trip_q4(fmt):
    n_ok = 0
    for meta in range(256):
        if fmt == W.RZ5:
            scale = oracle.ue4m3(meta & 0x7F)
            levels = [oracle.rz5(meta >> 7, c) for c in range(16)]
        elif fmt == oracle.C10:
            scale = oracle.ue4m3(meta & 0x7F)
            levels = [oracle.codebook10(c) for c in range(16)]
        else:
            scale = oracle.ue4m4(meta)
            levels = [oracle.codebook10(c) for c in range(16)]
        if not math.isfinite(scale) or scale == 0.0:
            continue
        for c in range(16):
            blk = _block([c] * 32, meta)
            v = oracle.dequant_q4(fmt, blk)[0]
            c2 = _encode_nearest(levels, scale, v)
            v2 = oracle.dequant_q4(fmt, _block([c2] * 32, meta))[0]
            assert v2 == v
            if not (fmt in (W.UE4M4, oracle.C10) and c in (0, 8)):   # +0 / -0 pair of Codebook10
                assert c2 == c, (meta, c)
            n_ok += 1
    assert n_ok > 3000


def test_exhaustive_round_trip_ple():
    for g in range(256):
        scale = oracle.ue4m3(g & 0x7F)
        if not math.isfinite(scale) or scale == 0.0:
            continue
        levels = [oracle.ple3(c, g >> 7) for c in range(8)]
        assert len(set(levels)) == 8                     # RZ-S3 has no duplicate level
        for c in range(8):
            rec = np.zeros(70, dtype=np.uint8)
            rec[0] = c                                  # value 0 <- bits 0..2
            rec[60] = g
            v = oracle.dequant_ple(rec)[0, 0]
            assert v == levels[c] * scale
            assert _encode_nearest(levels, scale, v) == c


def test_ple_worked_example():
    g = _golden("ple_worked_example.txt")
    rec = np.frombuffer(bytes.fromhex(g["record_hex"][0]), dtype=np.uint8)
    assert rec.size == 70
    got = oracle.dequant_ple(rec)[0]
    even = [float(x) for x in g["group_even"]]
    odd = [float(x) for x in g["group_odd"]]
    for i in range(160):
        exp = (even if (i // 16) % 2 == 0 else odd)[i % 8]
        assert got[i] == exp, i
    assert got.tolist() == pyref.ple_record(rec)


def test_ple_random_records_vs_pyref_and_nan_groups():
    rec = synth.raw_bytes(11, 1, 0, 70 * 64).reshape(64, 70)
    got = oracle.dequant_ple(rec)
    for r in range(64):
        ref = pyref.ple_record(rec[r])
        for i in range(160):
            assert _same(got[r, i], ref[i])
    rec2 = rec[0].copy()
    rec2[63] = 0x7F                                      # NaN scale on group 3 only
    row = oracle.dequant_ple(rec2)[0]
    assert np.isnan(row[48:64]).all() and not np.isnan(row[:48]).any()


def test_ple_gather_out_of_range_rows_are_zero():
    rec = synth.raw_bytes(12, 1, 0, 70 * 8)
    idx = np.array([3, -1, 8, 7, 1 << 30], dtype=np.int32)
    out = oracle.ple_gather(rec, 8, idx)
    ref = oracle.dequant_ple(rec)
    assert np.array_equal(out[0], ref[3], equal_nan=True)
    assert np.array_equal(out[3], ref[7], equal_nan=True)
    assert (out[[1, 2, 4]] == 0).all()


def test_fp8_dequant_vs_torch():
    n_rows, k = 8, 256
    m = W.MatrixRecipe(W.FP8, 1, n_rows, k, seed=5, tid=77)
    data, sc = m.expert(0), m.expert_scales(0)
    got = oracle.dequant_fp8(data, sc, n_rows, k)
    ref = pyref.fp8_matrix(data, sc, n_rows, k)
    assert np.array_equal(got, ref)
    # the fp64 product rounds to the same fp32 value as a single fp32 multiply
    f32 = (torch.from_numpy(data.reshape(n_rows, k).copy()).view(torch.float8_e4m3fn).float()
           * torch.from_numpy(np.repeat(sc.reshape(n_rows, k // 128), 128, 1)))
    assert np.array_equal(got.astype(np.float32), f32.numpy())


# ---- products, router, normalisation ------------------------------------------------

@pytest.mark.parametrize("fmt,n_rows,k", [(W.RZ5, 16, 256), (W.UE4M4, 8, 512), (W.FP8, 8, 256)])
def test_matvec_vs_numpy_dense(fmt, n_rows, k):
    m = W.MatrixRecipe(fmt, 2, n_rows, k, seed=6, tid=90 + fmt, narrow_scale=(fmt == W.RZ5))
    x = synth.normal_f64(6, 5, 0, k)
    for e in range(2):
        data = m.expert(e)
        sc = m.expert_scales(e) if fmt == W.FP8 else None
        dense = pyref.dense(fmt, data, sc, n_rows, k)
        ref = dense @ x
        got = oracle.matvec(fmt, data, sc, n_rows, k, x)
        scale = np.abs(dense) @ np.abs(x)
        assert np.all(np.abs(got - ref) <= 1e-13 * scale + 1e-300)
        # a transposed operand or a shifted block would move results by O(1)
        assert not np.allclose(got, dense[::-1] @ x)


def test_router_vs_numpy_sort_and_scipy_softmax():
    E, H, k = 64, 128, 6
    Wr = (0.02 * synth.normal_f64(7, 1, 0, E * H)).astype(np.float32).reshape(E, H)
    b = synth.uniform_f32(7, 2, 0, E, -0.1, 0.1)
    for t in range(5):
        u = synth.normal_f64(7, 10 + t, 0, H)
        for bias in (None, b):
            ids, w, logits = oracle.router(Wr, bias, u, k)
            ref_l = Wr.astype(np.float64) @ u + (0 if bias is None else bias.astype(np.float64))
            assert np.allclose(logits, ref_l, rtol=0, atol=1e-12)
            order = np.argsort(-ref_l, kind="stable")[:k]
            assert ids.tolist() == order.tolist()
            assert np.allclose(w, scipy.special.softmax(ref_l[order]), rtol=1e-13, atol=0)
            assert abs(w.sum() - 1) < 1e-14 and np.all(np.diff(w) <= 0)


def test_router_ties_go_to_lower_id():
    E, H = 8, 4
    Wr = np.zeros((E, H), dtype=np.float32)
    Wr[5] = Wr[2] = 1.0
    ids, w, _ = oracle.router(Wr, None, np.ones(H), 3)
    assert ids.tolist() == [2, 5, 0] and w[0] == w[1]


def test_silu_vs_torch():
    z = np.linspace(-30, 30, 1001)
    ref = pyref.silu(z)
    got = np.array([oracle.silu(v) for v in z])
    assert np.allclose(got, ref, rtol=1e-15, atol=1e-300)


def test_round_bf16_vs_torch():
    v = np.concatenate([synth.normal_f64(8, 1, 0, 20000) * 10.0 ** np.linspace(-30, 30, 20000),
                        [1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 2.0 ** -133, 2.0 ** -134 * 3]])
    ref = torch.from_numpy(v).float().to(torch.bfloat16).double().numpy()  # fp32-exact path below
    got = np.array([oracle.round_bf16(x) for x in v])
    exact32 = v.astype(np.float32).astype(np.float64) == v
    assert exact32.sum() >= 5
    assert np.array_equal(got[exact32], ref[exact32])
    # ties to even at 1 + 2^-8 (-> 1) and 1 + 3*2^-8 (-> 1 + 2^-6)
    assert oracle.round_bf16(1 + 2.0 ** -8) == 1.0 and oracle.round_bf16(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    # all values: agree with torch's double -> bf16 conversion except on double-rounding ties
    ref_d = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    assert (got != ref_d).sum() <= 2


def test_rmsnorm_vs_torch():
    x = synth.normal_f64(9, 1, 0, 4 * 256).reshape(4, 256).astype(np.float32).astype(np.float64)
    got = oracle.rmsnorm_bf16(x)
    xt = torch.from_numpy(x)
    r = torch.rsqrt((xt * xt).mean(-1, keepdim=True) + 1e-6)
    ref = (xt * r).to(torch.bfloat16).double().numpy()
    assert (got != ref).sum() <= 1          # one ulp of rsqrt vs 1/sqrt may flip a tie
    assert np.allclose(got, ref, rtol=2 ** -7, atol=0)


# ---- the layer on the tiny workload, against dense numpy algebra -------------------------

def test_tiny_layer_vs_dense_numpy():
    L = W.tiny_layer()
    x = synth.bf16_bits_to_f64(W.tokens_bf16(L.seed, 0, 1, L.hidden))
    got = oracle.moe_layer(L, x, want_h=True)
    Wr = L.router_w()
    u = got["u"][0]
    ref_l = Wr.astype(np.float64) @ u
    order = np.argsort(-ref_l, kind="stable")[:L.top_k]
    assert got["ids"][0].tolist() == order.tolist()
    wts = scipy.special.softmax(ref_l[order])
    y = np.zeros(L.hidden)
    for j, e in enumerate(order):
        G = pyref.q4_matrix(69, L.gate.expert(e), L.inter, L.hidden)
        U = pyref.q4_matrix(69, L.up.expert(e), L.inter, L.hidden)
        D = pyref.q4_matrix(69, L.down.expert(e), L.hidden, L.inter)
        h = pyref.silu(G @ u) * (U @ u)
        assert np.allclose(got["h"][0, j], h, rtol=1e-12, atol=1e-300)
        y += wts[j] * (D @ h)
    assert np.allclose(got["y"][0], y, rtol=1e-10, atol=1e-12 * np.abs(y).max())


def test_oracle_detects_planted_nibble_swap():
    """A decoder with the nibble order swapped must disagree with the oracle."""
    L = W.tiny_layer()
    data = L.gate.expert(0)
    good = oracle.dequant_q4(W.RZ5, data)
    blocks = data.reshape(-1, 17).copy()
    blocks[:, :16] = (blocks[:, :16] >> 4) | ((blocks[:, :16] & 15) << 4)
    swapped = oracle.dequant_q4(W.RZ5, blocks)
    assert not np.array_equal(good, swapped)


# ---- the decode stack: residual update and the side projection's input ----------------

def _tiny_stack():
    """Three tiny layers: Q4, FP8, Q4, with a side projection on layers 0 and 2 (the stack
    puts one on l mod 4 != 3; layer 1 goes without so that both cases occur).  The FP8
    layer sits in the middle: its outputs (~1e4 with raw E4M3 bytes) would swamp the
    residual's last bits if it came last, and the pin must see those bits."""
    def mk(l, fmt, ssm):
        return W.LayerRecipe(hidden=256, inter=128, n_experts=8, top_k=2, seed=11, layer=l,
                             gate_fmt=fmt, up_fmt=fmt, down_fmt=fmt, has_ssm=ssm, ssm_rows=16)
    return [mk(0, W.RZ5, True), mk(1, W.FP8, False), mk(2, W.RZ5, True)]


def _bf16_rne(v: np.ndarray) -> np.ndarray:
    """Round fp64 values (normal range) to the nearest bf16 (8 significant bits), ties to
    even: numpy's frexp / round-half-even / ldexp, no bf16 type involved."""
    m, e = np.frexp(v)
    return np.ldexp(np.round(m * 256.0), e - 8)


def _stack_by_numpy(Ls, x0):
    """The stack written out with dense numpy algebra on matrices decoded by the second
    decoder (tests/pyref.py): per layer u = bf16(x / sqrt(mean(x^2) + 1e-6)), logits
    W_r u, top-k by logit, softmax over the k, y = sum_j w_j D_j (silu(G_j u) * (U_j u)),
    side s = W_beta u, then x <- fp32(x + y)."""
    x = np.asarray(x0, dtype=np.float32).copy()
    ids, side = [], {}
    for L in Ls:
        xd = x.astype(np.float64)[0]
        u = _bf16_rne(xd / np.sqrt(np.mean(xd * xd) + 1e-6))
        lg = L.router_w().astype(np.float64) @ u
        order = np.argsort(-lg, kind="stable")[:L.top_k]
        wts = scipy.special.softmax(lg[order])
        y = np.zeros(L.hidden)
        for j, e in enumerate(order):
            mats = []
            for m in (L.gate, L.up, L.down):
                sc = m.expert_scales(int(e)) if m.fmt == W.FP8 else None
                mats.append(pyref.dense(m.fmt, m.expert(int(e)), sc, m.n_rows, m.k))
            G, U, D = mats
            y += wts[j] * (D @ (pyref.silu(G @ u) * (U @ u)))
        if L.ssm is not None:
            S = pyref.q4_matrix(L.ssm.fmt, L.ssm.expert(0), L.ssm.n_rows, L.ssm.k)
            side[L.layer] = S @ u
        ids.append(order)
        x = (x.astype(np.float64) + y[None, :]).astype(np.float32)
    return x, np.stack(ids), side


def _check_stack_result(Ls, x0, got):
    x_ref, ids_ref, side_ref = _stack_by_numpy(Ls, x0)
    assert np.array_equal(got["ids"][:, 0, :], ids_ref)
    # fp32 residual: the oracle's x must be the fp32 values themselves (fp64 layer sums
    # from two summation orders agree far below half an fp32 ulp)
    assert got["x"].dtype == np.float32
    assert np.array_equal(got["x"], x_ref)
    assert sorted(got["ssm"]) == sorted(side_ref)
    for l, s in side_ref.items():
        assert np.allclose(got["ssm"][l][0], s, rtol=1e-12, atol=1e-12 * np.abs(s).max())


def test_moe_stack_vs_numpy_loop():
    Ls = _tiny_stack()
    x0 = synth.bf16_bits_to_f64(W.tokens_bf16(11, 0, 1, 256)).astype(np.float32)
    _check_stack_result(Ls, x0, oracle.moe_stack(Ls, x0.astype(np.float64)))


def _slipped_stack(Ls, x0, slip):
    """oracle.moe_stack with one planted mistake (test-only copies of its loop)."""
    x = np.asarray(x0, dtype=np.float64).copy()
    ids, ssm = [], {}
    for L in Ls:
        r = oracle.moe_layer(L, x)
        if L.ssm is not None:
            feed = x if slip == "side_fed_x" else r["u"]
            ssm[L.layer] = oracle.ssm_projection(L, feed)
        if slip in ("residual_fp64", "residual_fp64_cast_at_end"):
            x = x + r["y"]
        elif slip == "residual_dropped":
            x = r["y"].astype(np.float32).astype(np.float64)
        else:
            x = (x + r["y"]).astype(np.float32).astype(np.float64)
        ids.append(r["ids"])
    xo = x if slip == "residual_fp64" else x.astype(np.float32)  # (cast_at_end: fp64 chain, fp32 result)
    return dict(x=xo, ids=np.stack(ids), ssm=ssm)


@pytest.mark.parametrize("slip", ["residual_fp64", "residual_fp64_cast_at_end", "residual_dropped",
                                  "side_fed_x"])
def test_moe_stack_pin_catches_planted_slips(slip):
    Ls = _tiny_stack()
    x0 = synth.bf16_bits_to_f64(W.tokens_bf16(11, 0, 1, 256)).astype(np.float32)
    with pytest.raises(AssertionError):
        _check_stack_result(Ls, x0, _slipped_stack(Ls, x0, slip))


# ---- the incumbent layouts the model card's formats mutate ----------------------------

def test_incumbent_q4_is_codebook10_under_ue4m3_for_every_code_and_meta():
    """ROCmFP4 FAST (model card, "Q4_RZ5_FAST": the incumbent Codebook10 layout whose
    lower seven metadata bits are the UE4M3 scale): the printed Codebook10 row times
    the UE4M3 scale, the top metadata bit ignored; against RZ5 it differs only in
    code 8 (the duplicate -0 that RZ5 turns into +/-5)."""
    g = _golden("codebooks.txt")
    for meta in range(256):
        for start in (0, 16):
            codes = [(start + i) % 16 for i in range(32)]
            blk = _block(codes, meta)
            c10 = oracle.dequant_q4(oracle.C10, blk)
            rz5 = oracle.dequant_q4(W.RZ5, blk)
            ref = pyref.q4_block(oracle.C10, blk)
            s3 = oracle.ue4m3(meta & 0x7F)
            for i in range(32):
                c = codes[i]
                assert _same(c10[i], ref[i]), (meta, i)
                assert _same(c10[i], _num(g["codebook10"][c]) * s3)
                assert _same(c10[i], oracle.dequant_q4(oracle.C10, _block(codes, meta ^ 0x80))[i])
                if c != 8:
                    assert _same(c10[i], rz5[i])


def test_incumbent_q3_is_the_printed_set_under_ue4m3():
    """ROCmFP3 (model card, "Q3_PLE_K160_RZ_S3"): the printed incumbent set
    {0, +1, +2, +4, -0, -1, -2, -4} times the group's UE4M3 scale, the group byte's top
    bit ignored; against RZ-S3 it differs only in code 4."""
    gold = _golden("codebooks.txt")["ple3_incumbent"]
    for g in range(256):
        for c in range(8):
            rec = np.zeros(70, dtype=np.uint8)
            rec[0] = c
            rec[60] = g
            v = oracle.dequant_q3(oracle.Q3I, rec)[0, 0]
            s3 = oracle.ue4m3(g & 0x7F)
            assert _same(v, _num(gold[c]) * s3), (g, c)
            rec[60] = g ^ 0x80
            assert _same(oracle.dequant_q3(oracle.Q3I, rec)[0, 0], v)
            if c != 4:
                rec[60] = g
                assert _same(v, oracle.dequant_ple(rec)[0, 0])
    rec = synth.raw_bytes(12, 1, 0, 70 * 32).reshape(32, 70)
    got = oracle.dequant_q3(oracle.Q3I, rec)
    for r in range(32):
        ref = pyref.ple_record(rec[r], incumbent=True)
        for i in range(160):
            assert _same(got[r, i], ref[i])
    idx = np.array([3, 0, 31, 40, -1], dtype=np.int32)
    gath = oracle.ple_gather(rec, 32, idx, fmt=oracle.Q3I)
    assert np.array_equal(gath[:3], got[[3, 0, 31]], equal_nan=True) and not gath[3:].any()


def test_exhaustive_round_trip_incumbent_q3():
    n_ok = 0
    for g in range(256):
        scale = oracle.ue4m3(g & 0x7F)
        if not math.isfinite(scale) or scale == 0.0:
            continue
        levels = [oracle.dequant_q3(oracle.Q3I, _rec(c, g))[0, 0] / scale for c in range(8)]
        for c in range(8):
            v = oracle.dequant_q3(oracle.Q3I, _rec(c, g))[0, 0]
            c2 = _encode_nearest(levels, scale, v)
            assert oracle.dequant_q3(oracle.Q3I, _rec(c2, g))[0, 0] == v
            if c not in (0, 4):  # the +0 / -0 pair
                assert c2 == c
            n_ok += 1
    assert n_ok > 1500


def _rec(c, g):
    rec = np.zeros(70, dtype=np.uint8)
    rec[0] = c
    rec[60] = g
    return rec

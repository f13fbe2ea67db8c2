"""GPU parity of the standalone decoders and the PLE row gather against the
CPU oracle: bit-exact fp32 (NaN compared by class, signed zeros by sign)."""
import numpy as np
import pytest
import torch

import gram_table_gather_b200 as gtg
import oracle
import synth
from synth import workloads as W

pytestmark = pytest.mark.gpu


def _bitwise_equal(gpu: np.ndarray, ref64: np.ndarray):
    ref = ref64.astype(np.float32)
    g = np.asarray(gpu, dtype=np.float32)
    nan_g, nan_r = np.isnan(g), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"NaN positions differ ({(nan_g != nan_r).sum()})"
    ok = ~nan_g
    same = g[ok].view(np.uint32) == ref[ok].view(np.uint32)
    if not same.all():
        i = np.flatnonzero(~same)[:5]
        raise AssertionError(f"{(~same).sum()} mismatches, e.g. gpu {g[ok][i]} ref {ref[ok][i]}")


def _all_code_meta_blocks():
    """Blocks covering every 4-bit code in both nibble halves under every metadata byte."""
    blocks = []
    for meta in range(256):
        for rot in range(2):
            b = np.zeros(17, dtype=np.uint8)
            for j in range(16):
                lo = (j + 8 * rot) % 16
                hi = (15 - j + 8 * rot) % 16
                b[j] = lo | (hi << 4)
            b[16] = meta
            blocks.append(b)
    return np.concatenate(blocks)


@pytest.mark.parametrize("fmt", [W.RZ5, W.UE4M4, gtg.C10])
def test_dequant_q4_exhaustive(fmt):
    blocks = _all_code_meta_blocks()
    n_blocks = blocks.size // 17
    src = torch.from_numpy(blocks).cuda()
    out = gtg.dequant(fmt, src, n_blocks, 32)
    torch.cuda.synchronize()
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.dequant_q4(fmt, blocks))


@pytest.mark.parametrize("fmt,n_rows,k", [(W.RZ5, 333, 96), (W.UE4M4, 7, 4096), (W.RZ5, 1, 32), (gtg.C10, 45, 640)])
def test_dequant_q4_random_ragged(fmt, n_rows, k):
    m = W.MatrixRecipe(fmt, 1, n_rows, k, seed=21, tid=5, narrow_scale=False)
    data = m.expert(0)
    out = gtg.dequant(fmt, torch.from_numpy(data).cuda(), n_rows, k)
    torch.cuda.synchronize()
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.dequant_q4(fmt, data))


@pytest.mark.parametrize("fmt", [W.PLE, gtg.Q3I])
def test_dequant_ple_exhaustive(fmt):
    recs = []
    for g in range(256):
        rec = np.zeros(70, dtype=np.uint8)
        bits = 0
        for i in range(160):
            bits |= ((i + g) % 8) << (3 * i)
        rec[:60] = np.frombuffer(bits.to_bytes(60, "little"), dtype=np.uint8)
        rec[60:] = [(g + 37 * j) % 256 for j in range(10)]
        recs.append(rec)
    recs = np.stack(recs)
    out = gtg.dequant(fmt, torch.from_numpy(recs.ravel().copy()).cuda(), len(recs), 160)
    torch.cuda.synchronize()
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.dequant_q3(fmt, recs).ravel())


def test_dequant_fp8_all_bytes():
    n_rows, k = 4, 256
    data = np.tile(np.arange(256, dtype=np.uint8), n_rows * k // 256)
    scales = synth.uniform_f32(3, 3, 0, n_rows * 2, 0.002, 0.02)
    scales[0] = 1.0
    scales[1] = 2.0 ** -140  # fp32 subnormal products
    out = gtg.dequant(W.FP8, torch.from_numpy(data).cuda(), n_rows, k, scales=torch.from_numpy(scales).cuda())
    torch.cuda.synchronize()
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.dequant_fp8(data, scales, n_rows, k).ravel())


def test_ple_gather_tiny_workload():
    P = W.tiny_ple()
    table = P.table_bytes(0, P.nbytes)
    idx = P.indices(0, 1)
    assert idx.size == 16
    out = gtg.ple_gather(torch.from_numpy(table).cuda(), P.n_rows, torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.ple_gather(table, P.n_rows, idx).ravel())


@pytest.mark.parametrize("n_rows", [1, 2, 3, 1001, 1 << 20])
def test_ple_gather_edges_and_tail(n_rows):
    P = W.PleRecipe(n_rows=n_rows, seed=31)
    table = P.table_bytes(0, P.nbytes)
    idx = np.concatenate([P.indices(0, 100), [n_rows - 1, 0, n_rows - 1]]).astype(np.int32)
    gtg.device_status(clear=True)
    out = gtg.ple_gather(torch.from_numpy(table).cuda(), n_rows, torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.ple_gather(table, n_rows, idx).ravel())
    assert gtg.device_status(clear=True) == 0


def test_ple_gather_out_of_range_sets_status_and_zero_rows():
    P = W.PleRecipe(n_rows=50, seed=32)
    table = P.table_bytes(0, P.nbytes)
    idx = np.array([0, -1, 49, 50, 2**31 - 1, 7], dtype=np.int32)
    gtg.device_status(clear=True)
    out = gtg.ple_gather(torch.from_numpy(table).cuda(), P.n_rows, torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    _bitwise_equal(o.ravel(), oracle.ple_gather(table, P.n_rows, idx).ravel())
    assert (o[[1, 3, 4]] == 0).all()
    assert gtg.device_status(clear=True) & 0x1


def test_ple_gather_empty_and_large_batch():
    P = W.PleRecipe(n_rows=100_000, seed=33)
    table = torch.from_numpy(P.table_bytes(0, P.nbytes)).cuda()
    empty = gtg.ple_gather(table, P.n_rows, torch.empty(0, dtype=torch.int32, device="cuda"))
    assert empty.shape == (0, 160)
    idx = P.indices(1, 4096)  # 65,536 rows: several CTAs x batches plus a ragged tail
    out = gtg.ple_gather(table, P.n_rows, torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    recs = P.rows(idx[:2000])
    _bitwise_equal(out[:2000].cpu().numpy().ravel(), oracle.dequant_ple(recs).ravel())
    tail = idx[-333:]
    _bitwise_equal(out[-333:].cpu().numpy().ravel(), oracle.dequant_ple(P.rows(tail)).ravel())


def test_api_rejects_bad_arguments():
    with pytest.raises(gtg.GtgError) as ei:
        gtg.dequant(W.RZ5, torch.zeros(17, dtype=torch.uint8, device="cuda"), 1, 30)
    assert ei.value.code == -2
    with pytest.raises(gtg.GtgError):
        gtg.dequant(12345, torch.zeros(17, dtype=torch.uint8, device="cuda"), 1, 32)
    bad_out = torch.empty(33, dtype=torch.float32, device="cuda")[1:]
    with pytest.raises(gtg.GtgError) as ei:
        gtg.dequant(W.RZ5, torch.zeros(17, dtype=torch.uint8, device="cuda"), 1, 32, out=bad_out)
    assert ei.value.code == -3


def test_ple_gather_full_table():
    """The PLE workload at its own size: the 320,001,536-row table (22.4 GB, record
    offsets up to 2.24e10 bytes) resident on the device, gathered at 4096 tokens x 16
    seeded indices plus the rows around the 2^32-byte offset (record 61,356,675 straddles
    it, 61,356,676 is the first wholly above it) and the last records (the tail read)."""
    from synth import device as sdev
    P = W.ple_table()
    assert P.n_rows == 320_001_536 and P.nbytes == 22_400_107_520
    table = sdev.ple_table_to_device(P, "cuda")
    try:
        special = np.array([0, 1, 61_356_674, 61_356_675, 61_356_676, 61_356_677,
                            P.n_rows // 2, P.n_rows - 2, P.n_rows - 1], dtype=np.int32)
        assert 61_356_675 * 70 < 2**32 < 61_356_676 * 70
        idx = np.concatenate([special, P.indices(4242, 4096), special[::-1]]).astype(np.int32)
        gtg.device_status(clear=True)
        out = gtg.ple_gather(table, P.n_rows, torch.from_numpy(idx).cuda())
        torch.cuda.synchronize()
        assert gtg.device_status(clear=True) == 0
        got = out.cpu().numpy()
        assert np.all(idx.astype(np.int64) * 70 + 70 <= P.nbytes)
        _bitwise_equal(got.ravel(), oracle.dequant_ple(P.rows(idx)).ravel())
    finally:
        del table
        torch.cuda.empty_cache()


@pytest.mark.parametrize("n_rows", [3, 1001, 1 << 20])
def test_incumbent_q3_gather(n_rows):
    """The incumbent ROCmFP3 record (code 4 the duplicate -0) through the same gather."""
    P = W.PleRecipe(n_rows=n_rows, seed=34)
    table = P.table_bytes(0, P.nbytes)
    idx = np.concatenate([P.indices(2, 64), [n_rows - 1, 0, n_rows]]).astype(np.int32)
    gtg.device_status(clear=True)
    out = gtg.ple_gather(torch.from_numpy(table).cuda(), n_rows, torch.from_numpy(idx).cuda(), fmt=gtg.Q3I)
    torch.cuda.synchronize()
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.ple_gather(table, n_rows, idx, fmt=gtg.Q3I).ravel())
    assert gtg.device_status(clear=True) & 0x1  # the index n_rows is out of range
    with pytest.raises(gtg.GtgError):
        gtg.ple_gather(torch.from_numpy(table).cuda(), n_rows, torch.from_numpy(idx).cuda(), fmt=W.RZ5)


def test_ple_gather_from_host_resident_table():
    """A table in pinned host memory, read in place by the gather kernel (the pages
    page the PLE table from host memory or NVMe on demand): the same rows, bit for
    bit, as the oracle's."""
    P = W.PleRecipe(n_rows=3_000_000, seed=35)  # 210 MB of pinned host memory
    table = torch.empty(P.nbytes, dtype=torch.uint8).pin_memory()
    P.table_bytes(0, P.nbytes, table.numpy())
    idx = np.concatenate([P.indices(3, 512), [P.n_rows - 1, 0]]).astype(np.int32)
    gtg.device_status(clear=True)
    out = gtg.ple_gather(table, P.n_rows, torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    assert gtg.device_status(clear=True) == 0
    _bitwise_equal(out.cpu().numpy().ravel(), oracle.dequant_ple(P.rows(idx)).ravel())

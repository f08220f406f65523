"""Host-side checks of the seeded input generators and of the algorithmic
FLOP / byte accounting used by the benchmark."""
import os

import numpy as np
import torch

import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_benchmark_table.txt")


def test_byte_accounting_reproduces_pages_table():
    """DeepGEMM page 2 "性能实测": 206 TFLOPS <-> 1688 GB/s at M=64 N=2112 K=7168
    fixes the byte count (operands + scales + BF16 output)."""
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    for layout, M, N, K, tflops, gbps in rows:
        M, N, K = int(M), int(N), int(K)
        prob = W.Problem("dense", M, N, K, 1, None, None, 0, None, None)
        t = prob.flops() / (float(tflops) * 1e12)
        assert abs(prob.bytes() / t / 1e9 - float(gbps)) < 1.0


def test_generators_are_deterministic():
    p1 = W.make_dense(64, 256, 384, seed=5, outliers=True)
    p2 = W.make_dense(64, 256, 384, seed=5, outliers=True)
    assert np.array_equal(p1.a, p2.a) and np.array_equal(p1.b, p2.b)
    assert np.array_equal(p1.sfa, p2.sfa) and np.array_equal(p1.sfb, p2.sfb)
    p3 = W.make_dense(64, 256, 384, seed=6, outliers=True)
    assert not np.array_equal(p1.a, p3.a)


def test_quantised_blocks_reach_full_range():
    p = W.make_dense(8, 200, 256, seed=1)
    deq = torch.from_numpy(p.a).view(torch.float8_e4m3fn).float().numpy()
    amax_rows = np.abs(deq.reshape(8, 2, 128)).max(axis=2)
    assert np.all(amax_rows == 448.0)                   # each row block hits the E4M3 max
    assert p.sfa.shape == (2, 8) and p.sfb.shape == (1, 2, 2)
    assert p.b.shape == (1, 200, 256)


def test_contiguous_structure():
    p = W.make_contiguous([130, 0, 5], N=64, K=128, seed=1)
    assert p.M == 256 + 0 + 128
    mi = p.m_indices
    assert (mi[:130] == 0).all() and (mi[130:256] == -1).all()
    assert (mi[256:261] == 2).all() and (mi[261:] == -1).all()
    assert (p.a[mi < 0] == W.NAN_BYTE).all()
    assert np.isnan(p.sfa[:, mi < 0]).all() and np.isfinite(p.sfa[:, mi >= 0]).all()
    for blk in range(p.M // 128):                         # one group per 128-row block
        ids = set(mi[blk * 128:(blk + 1) * 128].tolist()) - {-1}
        assert len(ids) <= 1


def test_contiguous_gap_blocks():
    """gaps[g] whole 128-row padding blocks follow group g (a caller's buffer
    with unused blocks); without gaps the generator is unchanged."""
    p = W.make_contiguous([200, 100, 300], N=64, K=128, seed=1, gaps=[2, 0, 1])
    mi = p.m_indices
    assert p.M == (256 + 256) + 128 + (384 + 128)
    assert (mi[:200] == 0).all() and (mi[200:512] == -1).all()       # 56 rows + 2 whole blocks
    assert (mi[512:612] == 1).all() and (mi[612:640] == -1).all()
    assert (mi[640:940] == 2).all() and (mi[940:] == -1).all()
    assert (p.a[mi < 0] == W.NAN_BYTE).all() and np.isnan(p.sfa[:, mi < 0]).all()
    q, r = W.make_contiguous([200, 100, 300], N=64, K=128, seed=1), \
        W.make_contiguous([200, 100, 300], N=64, K=128, seed=1, gaps=[0, 0, 0])
    assert np.array_equal(q.a, r.a) and np.array_equal(q.m_indices, r.m_indices)
    assert np.array_equal(q.b, p.b) and np.array_equal(p.a[mi == 2], q.a[q.m_indices == 2])
    h = W.make_bf16_contiguous([5, 130], N=64, K=64, seed=3, gaps=[3, 1])
    assert h.M == 128 * 4 + 256 + 128 and (h.m_indices[128:512] == -1).all()
    assert (h.m_indices[512:642] == 1).all() and (h.m_indices[642:] == -1).all()


def test_masked_structure():
    p = W.make_masked_uniform(16, 256, N=128, K=128, seed=5)
    assert p.masked_m.min() >= 0 and p.masked_m.max() <= 256
    for g in range(16):
        m = p.masked_m[g]
        assert (p.a[g, m:] == W.NAN_BYTE).all()
        assert np.isnan(p.sfa[g, :, m:256]).all()
        assert np.isfinite(p.sfa[g, :, :m]).all()


def test_workload_table_shapes():
    w = W.WORKLOADS
    assert (w["dense_decode_m64"]["M"], w["dense_decode_m64"]["N"], w["dense_decode_m64"]["K"]) == (64, 2112, 7168)
    assert (w["dense_large"]["M"], w["dense_large"]["N"], w["dense_large"]["K"]) == (4096, 7168, 16384)
    assert w["contiguous_g4"]["G"] == 4 and w["masked_g16"]["Mmax"] == 256

"""GPU parity of the K-grouped GEMM (groups contiguous along K) against the
oracle, through the C ABI.

Same tolerance as the other layouts (per element |D - D_ref| <= 1e-2 *
max(1, |D_ref|), relative Frobenius <= 2e-3); integer operands with
power-of-two scales match bit for bit.  D is pre-filled with a sentinel: every
element of every group (zeros for an empty group) must be written.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_fp32_b200 as dg
import oracle
import workloads as W
from gpu_util import SENTINEL, DeviceProblem, compare, to_f64, valid_mask

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.fixture(autouse=True, scope="module")
def _clean_status():
    from moe_grouped_gemm_fp32_b200 import build
    build.build()
    oracle.build()
    dg.dg_get_device_status(clear=True)
    yield
    assert dg.dg_get_device_status(clear=True) == 0, "a kernel recorded an error"


def _run(prob):
    dp = DeviceProblem(prob)
    dp.fill_sentinel()
    d = dp.run()
    torch.cuda.synchronize()
    bits = d.view(torch.int16).cpu().numpy()
    assert not (bits == np.int16(SENTINEL)).any(), "an output element was not written"
    return dp, to_f64(d)


@pytest.mark.parametrize("ks,M,N", [
    ([128], 128, 256),                       # one group = dense
    ([256, 0, 512, 128], 200, 2112),         # empty group, token tail, weight-block tail
    ([1024, 384], 300, 512),                 # CTA-pair tiles with a row tail
    ([128] * 9, 64, 144),                    # many small groups, narrow N with a weight tail
    ([0, 0, 640], 1, 256),                   # one token row
    ([384, 896], 513, 7168),                 # wide N, pair tiles with 224/256 columns
])
def test_k_grouped_matches_oracle(ks, M, N):
    prob = W.make_k_grouped(ks, M, N, seed=sum(ks) + M + N)
    dp, d = _run(prob)
    ref = oracle.solve(prob)
    compare(d, ref, valid_mask(prob))
    for g, kg in enumerate(ks):
        if kg == 0:
            assert (d[g] == 0).all(), f"empty group {g} not zero"


def test_k_grouped_maximum_group_count():
    """G = 1024 groups along K (the prefix table's capacity), about three in
    four of them empty: empty groups give zeros, the others their own K range."""
    rng = np.random.default_rng(4096)
    ks = np.where(rng.random(1024) < 0.25, 128, 0).astype(np.int32)
    ks[-1] = 256
    prob = W.make_k_grouped(ks, 128, 128, seed=4097)
    dp, d = _run(prob)
    compare(d, oracle.solve(prob), valid_mask(prob))
    assert (d[ks == 0] == 0).all()


def test_k_grouped_exact_integers():
    """Integer operands in {-1, 0, 1} with power-of-two scales: every partial
    sum and the BF16 output are exact, so D must match bit for bit."""
    rng = np.random.default_rng(44)
    ks = np.array([256, 128, 384], np.int32)
    M, N, K = 260, 384, int(ks.sum())
    KB, NB = K // 128, (N + 127) // 128
    one = {-1: 0xB8, 0: 0x00, 1: 0x38}
    ai = rng.integers(-1, 2, size=(M, K))
    bi = rng.integers(-1, 2, size=(N, K))
    enc = np.vectorize(one.get)
    a, b = enc(ai).astype(np.uint8), enc(bi).astype(np.uint8)
    sa = np.ldexp(1.0, rng.integers(-2, 3, size=(M, KB))).astype(np.float32)
    sb = np.ldexp(1.0, rng.integers(-2, 3, size=(NB, KB))).astype(np.float32)
    ld = W.tma_aligned(M)
    prob = W.Problem("k_grouped", M, N, K, len(ks), a, W.sfa_mn_major(sa, ld), ld, b[None], sb[None], ks=ks)
    dp, d = _run(prob)
    ref = oracle.solve(prob)
    assert np.array_equal(d, torch.from_numpy(ref).to(torch.bfloat16).double().numpy())


def test_k_grouped_graph_replay_with_new_sizes():
    """The group sizes are read on the device: a captured call replays with
    new sizes (same total K) and gives the new result."""
    p1 = W.make_k_grouped([256, 256, 128], 256, 512, seed=61)
    dp = DeviceProblem(p1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dp.run(s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dp.run()
    new_ks = np.array([0, 384, 256], np.int32)
    dp.ks.copy_(torch.from_numpy(new_ks))
    dp.fill_sentinel()
    g.replay()
    torch.cuda.synchronize()
    p2 = W.Problem("k_grouped", p1.M, p1.N, p1.K, p1.G, p1.a, p1.sfa, p1.ld_sfa, p1.b, p1.sfb, ks=new_ks)
    compare(to_f64(dp.d), oracle.solve(p2), valid_mask(p2))


def test_k_grouped_bad_sizes_are_reported():
    prob = W.make_k_grouped([256, 128], 128, 256, seed=71)
    dp = DeviceProblem(prob)
    dp.ks.copy_(torch.tensor([200, 184], dtype=torch.int32))   # not multiples of 128
    dp.run()
    torch.cuda.synchronize()
    code = dg.dg_get_device_status(clear=True)
    assert code & 0xFF == 1 and (code >> 8) & 0xFF == 10
    dp.ks.copy_(torch.tensor([256, 256], dtype=torch.int32))   # adds up past K
    dp.run()
    torch.cuda.synchronize()
    code = dg.dg_get_device_status(clear=True)
    assert code & 0xFF == 1 and (code >> 8) & 0xFF == 10


def test_k_grouped_validation():
    L = dg.lib()
    a = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((2, 128), dtype=torch.float32, device="cuda")
    b = torch.zeros((256, 256), dtype=torch.uint8, device="cuda")
    sfb = torch.zeros((2, 2), dtype=torch.float32, device="cuda")
    d = torch.zeros((2, 128, 256), dtype=torch.bfloat16, device="cuda")
    ks = torch.tensor([128, 128], dtype=torch.int32, device="cuda")
    args = lambda **kw: [kw.get("a", a.data_ptr()), sfa.data_ptr(), 128, b.data_ptr(), sfb.data_ptr(),
                         d.data_ptr(), kw.get("ks", ks.data_ptr()), kw.get("G", 2), 128,
                         kw.get("N", 256), kw.get("K", 256), None]
    assert L.dg_k_grouped_fp8_gemm_nt_contiguous(*args(ks=None)) == 1
    assert L.dg_k_grouped_fp8_gemm_nt_contiguous(*args(G=0)) == 1
    assert L.dg_k_grouped_fp8_gemm_nt_contiguous(*args(G=1025)) == 3
    assert L.dg_k_grouped_fp8_gemm_nt_contiguous(*args(K=200)) == 3
    assert L.dg_k_grouped_fp8_gemm_nt_contiguous(*args(N=200)) == 3
    assert L.dg_k_grouped_fp8_gemm_nt_contiguous(*args(a=a.data_ptr() + 8)) == 2
    torch.cuda.synchronize()
    assert (d == 0).all()


def test_k_grouped_full_size_sampled():
    prob = W.make_workload("kgrouped_g4")
    dp, d = _run(prob)
    rng = np.random.default_rng(9)
    n = 6000
    g, r, c = rng.integers(0, prob.G, n), rng.integers(0, prob.M, n), rng.integers(0, prob.N, n)
    ref = oracle.points(prob, g, r, c)
    got = d[g, r, c]
    err = np.abs(got - ref)
    assert (err <= 1e-2 * np.maximum(1.0, np.abs(ref))).all()
    assert np.linalg.norm(got - ref) <= 2e-3 * np.linalg.norm(ref)

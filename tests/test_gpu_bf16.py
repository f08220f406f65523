"""GPU parity of the BF16 GEMMs (dense, contiguous, masked) against the
oracle, through the C ABI.

Tolerance: per element |D - D_ref| <= 1e-2 * max(1, |D_ref|) and relative
Frobenius error <= 2e-3 (BF16 output rounding is 2^-9 relative; FP32
accumulation over K <= 16384 adds far less).  Integer operands whose sums are
exact in FP32 match bit for bit.  D is pre-filled with a sentinel so rows the
method must not write (masked) can be checked bit for bit.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_fp32_b200 as dg
import oracle
import workloads as W
from gpu_util import SENTINEL, compare

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


def _t(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _run(prob):
    a, b = _t(prob.a), _t(prob.b)
    d = torch.empty(prob.d_shape(), dtype=torch.bfloat16, device="cuda")
    d.view(torch.int16).fill_(SENTINEL)
    if prob.layout == "dense":
        dg.dg_bf16_gemm_nt(a, b[0], d)
    elif prob.layout == "contiguous":
        dg.dg_m_grouped_bf16_gemm_nt_contiguous(a, b, d, torch.from_numpy(prob.m_indices).cuda())
    else:
        dg.dg_m_grouped_bf16_gemm_nt_masked(a, b, d, torch.from_numpy(prob.masked_m).cuda())
    torch.cuda.synchronize()
    return d


def _ref(prob):
    return oracle.gemm_bf16(prob.layout, prob.a, prob.b[0] if prob.layout == "dense" else prob.b,
                            prob.M, prob.N, prob.K, G=prob.G, m_indices=prob.m_indices,
                            masked_m=prob.masked_m)


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (1, 8, 8), (257, 264, 1000), (64, 2112, 7168),
                                   (300, 520, 136), (640, 7168, 256)])
def test_dense_matches_oracle(M, N, K):
    prob = W.make_bf16_dense(M, N, K, seed=M + N + K)
    d = _run(prob).double().cpu().numpy()
    compare(d, _ref(prob), np.ones(prob.d_shape(), bool))


@pytest.mark.parametrize("M,N,K", [(100, 264, 1000), (128, 2112, 512), (33, 128, 4096), (64, 384, 256)])
def test_dense_split_k_shapes(M, N, K):
    """M <= 128 with few weight tiles: K split over a cluster of CTAs, partials
    reduced through distributed shared memory (N tail, K tail, short K)."""
    prob = W.make_bf16_dense(M, N, K, seed=M * 7 + N + K)
    d = _run(prob).double().cpu().numpy()
    compare(d, _ref(prob), np.ones(prob.d_shape(), bool))


def test_dense_split_k_exact_integers():
    """Integer operands: the split partial sums are exact in FP32, so the
    rank-order reduction must give the exact result bit for bit."""
    rng = np.random.default_rng(8)
    M, N, K = 64, 256, 2048
    ai, bi = rng.integers(-3, 4, size=(M, K)), rng.integers(-3, 4, size=(N, K))
    prob = W.BF16Problem("dense", M, N, K, 1, W._bf16_bits(ai.astype(np.float32)),
                         W._bf16_bits(bi.astype(np.float32))[None])
    d = _run(prob).cpu()
    exact = torch.from_numpy((ai @ bi.T).astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(d.view(torch.int16), exact.view(torch.int16))


def test_dense_exact_integers():
    rng = np.random.default_rng(5)
    M, N, K = 200, 384, 320
    ai, bi = rng.integers(-6, 7, size=(M, K)), rng.integers(-6, 7, size=(N, K))
    a = W._bf16_bits(ai.astype(np.float32))
    b = W._bf16_bits(bi.astype(np.float32))
    prob = W.BF16Problem("dense", M, N, K, 1, a, b[None])
    d = _run(prob).cpu()
    exact = torch.from_numpy((ai @ bi.T).astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(d.view(torch.int16), exact.view(torch.int16))


@pytest.mark.parametrize("counts,N,K", [([130, 200, 5, 300, 129], 384, 512), ([1] * 7, 256, 128),
                                        ([0, 700, 0], 2112, 1024)])
def test_contiguous_matches_oracle(counts, N, K):
    prob = W.make_bf16_contiguous(counts, N, K, seed=sum(counts) + N)
    d = _run(prob).double().cpu().numpy()
    valid = np.broadcast_to((prob.m_indices >= 0)[:, None], prob.d_shape())
    compare(d, _ref(prob), valid)


def _bf16_child(kind, args, pairs):
    """Runs one BF16 problem in a child process with DG_BF16_PAIRS forcing CTA
    pairs (1) or single-CTA tiles (0); returns the launch log."""
    import os, subprocess, sys
    make = {"dense": "W.make_bf16_dense(*%r, seed=21)",
            "contiguous": "W.make_bf16_contiguous(*%r[:3], seed=22, gaps=%r[3])"}[kind]
    code = ("import sys; sys.path[:0] = [%r, %r]\n"
            "import numpy as np, test_gpu_bf16 as T, workloads as W\n"
            "from gpu_util import compare\n"
            "import oracle; oracle.build()\n"
            "p = " + make + "\n"
            "d = T._run(p).double().cpu().numpy()\n"
            "valid = np.ones(p.d_shape(), bool) if p.layout == 'dense' else "
            "np.broadcast_to((p.m_indices >= 0)[:, None], p.d_shape())\n"
            "compare(d, T._ref(p), valid)\n"
            "import moe_grouped_gemm_fp32_b200 as dg; assert dg.dg_get_device_status(clear=True) == 0\n"
            "print('OK')\n") % ((os.path.dirname(os.path.dirname(__file__)), os.path.dirname(__file__))
                                  + ((args,) if kind == "dense" else (args, args)))
    env = dict(os.environ, DG_BF16_PAIRS="1" if pairs else "0", DG_VERBOSE="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr
    return r.stderr


@pytest.mark.parametrize("kind,args", [("dense", (512, 448, 512)), ("dense", (300, 520, 136)),
                                       ("dense", (1024, 7168, 256)),
                                       ("contiguous", ([130, 200, 5, 300, 129], 448, 384, None)),
                                       ("contiguous", ([200, 100, 300], 256, 256, [2, 0, 0])),
                                       ("contiguous", ([5, 130], 384, 128, [3, 1]))])
@pytest.mark.parametrize("pairs", [True, False])
def test_cta_pairs_and_single_tiles(kind, args, pairs):
    """Both tile kinds of the dense and contiguous BF16 layouts, each forced in
    a child process: 256-row CTA-pair tiles (second passes where a pair's two
    blocks belong to different groups; pairs of padding blocks with no work)
    and 128-row single-CTA tiles."""
    log = _bf16_child(kind, args, pairs)
    assert ("ctas/mma=2" if pairs else "ctas/mma=1") in log


@pytest.mark.parametrize("masked_m,Mmax,N,K", [([0, 1, 64, 200, 130], 200, 384, 512),
                                               ([256] * 3, 256, 4096, 256), ([5, 0], 8, 136, 64)])
def test_masked_matches_oracle_and_leaves_rows(masked_m, Mmax, N, K):
    prob = W.make_bf16_masked(masked_m, Mmax, N, K, seed=Mmax + N)
    d = _run(prob)
    bits = d.view(torch.int16).cpu().numpy()
    rows = np.arange(Mmax)[None, :] < prob.masked_m[:, None]
    valid = np.broadcast_to(rows[:, :, None], prob.d_shape())
    compare(d.double().cpu().numpy(), _ref(prob), valid)
    assert (bits[~valid] == np.int16(SENTINEL)).all(), "rows past masked_m were written"


def test_masked_maximum_group_count():
    """G = 1024, the masked call's largest group count; every seventh group empty."""
    counts = np.random.default_rng(1024).integers(0, 65, size=1024)
    counts[::7] = 0
    test_masked_matches_oracle_and_leaves_rows(counts.tolist(), 64, 128, 128)


def test_masked_graph_replay_with_new_counts():
    prob = W.make_bf16_masked([40, 0, 128], 128, 256, 384, seed=9)
    a, b = _t(prob.a), _t(prob.b)
    mm = torch.from_numpy(prob.masked_m).cuda()
    d = torch.zeros(prob.d_shape(), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dg.dg_m_grouped_bf16_gemm_nt_masked(a, b, d, mm, s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dg.dg_m_grouped_bf16_gemm_nt_masked(a, b, d, mm)
    new = np.array([7, 0, 100], np.int32)      # within the rows that hold data
    mm.copy_(torch.from_numpy(new))
    d.zero_()
    g.replay()
    torch.cuda.synchronize()
    p2 = W.BF16Problem("masked", prob.M, prob.N, prob.K, prob.G, prob.a, prob.b, masked_m=new)
    rows = np.arange(prob.M)[None, :] < new[:, None]
    valid = np.broadcast_to(rows[:, :, None], prob.d_shape())
    got = d.double().cpu().numpy()
    compare(got, _ref(p2), valid)
    assert (got[~valid] == 0).all()


def test_bf16_validation():
    L = dg.lib()
    x = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    p = x.data_ptr()
    assert L.dg_bf16_gemm_nt(p, p, p, 128, 128, 12, None) == 3      # K % 8
    assert L.dg_bf16_gemm_nt(p, p, p, 128, 12, 128, None) == 3      # N % 8
    assert L.dg_bf16_gemm_nt(p + 2, p, p, 128, 128, 128, None) == 2
    assert L.dg_bf16_gemm_nt(None, p, p, 128, 128, 128, None) == 1
    assert L.dg_bf16_gemm_nt(p, p, p, 0, 128, 128, None) == 0
    mi = torch.zeros(128, dtype=torch.int32, device="cuda")
    assert L.dg_m_grouped_bf16_gemm_nt_contiguous(p, p, p, mi.data_ptr(), 100, 128, 128, 1, None) == 3
    assert L.dg_m_grouped_bf16_gemm_nt_masked(p, p, p, mi.data_ptr(), 1025, 8, 128, 128, None) == 3


@pytest.mark.parametrize("name", ["bf16_dense_large", "bf16_contiguous_g4", "bf16_masked_g16",
                                  "bf16_dense_decode_m64"])
def test_full_size_sampled_rows(name):
    prob = W.make_bf16_workload(name)
    d = _run(prob).double().cpu().numpy()
    rng = np.random.default_rng(3)
    if prob.layout == "masked":
        g = [int(x) for x in np.flatnonzero(prob.masked_m)[:4]]
        for gg in g:
            rows = np.sort(rng.choice(int(prob.masked_m[gg]), size=min(8, int(prob.masked_m[gg])), replace=False))
            ref = oracle.gemm_bf16("dense", prob.a[gg, rows], prob.b[gg], len(rows), prob.N, prob.K)
            compare(d[gg, rows], ref, np.ones(ref.shape, bool))
        return
    valid = np.arange(prob.M) if prob.layout == "dense" else np.flatnonzero(prob.m_indices >= 0)
    rows = np.sort(rng.choice(valid, size=24, replace=False))
    for r in rows:
        g = 0 if prob.layout == "dense" else int(prob.m_indices[r])
        ref = oracle.gemm_bf16("dense", prob.a[r:r + 1], prob.b[g], 1, prob.N, prob.K)
        compare(d[r:r + 1], ref, np.ones(ref.shape, bool))

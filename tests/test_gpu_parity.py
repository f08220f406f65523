"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Tolerance (the workload definition's): per element |D - D_ref| <= 1e-2 *
max(1, |D_ref|) and relative Frobenius error <= 2e-3 over valid rows.
Integer-valued cases with power-of-two scales must match bit for bit.
Padding rows hold NaN bytes and NaN scales (a leak shows as NaN); D is
pre-filled with a sentinel so that rows the method must not write can be
checked bit for bit.
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
    dg.dg_get_device_status(clear=True)
    yield
    assert dg.dg_get_device_status(clear=True) == 0, "a kernel recorded an error"


def _run_full(prob, sentinel=True):
    dp = DeviceProblem(prob)
    if sentinel:
        dp.fill_sentinel()
    d = to_f64(dp.run())
    torch.cuda.synchronize()
    ref = oracle.solve(prob)
    margins = compare(d, ref, valid_mask(prob))
    return dp, d, ref, margins


# ------------------------------------------------------------------ dense
def test_dense_tiny():
    _run_full(W.make_workload("dense_tiny"))


@pytest.mark.parametrize("M", [1, 63, 64, 65, 127, 128, 129, 200, 256, 257, 300])
def test_dense_m_sweep_with_n_tail(M):
    # N = 2112 = 16.5 weight blocks: a half-filled last block; K = 1024 (8 K-blocks)
    _run_full(W.make_dense(M, 2112, 1024, seed=100 + M, outliers=True))


@pytest.mark.parametrize("M,K", [(64, 4096), (128, 4096), (16, 7168)])
def test_dense_small_m_split_k(M, K):
    # enough K-blocks for an 8-CTA split-K cluster
    _run_full(W.make_dense(M, 2112, K, seed=7 + M, outliers=True))


def test_split_k_needs_four_k_blocks_per_cta():
    """The split-K factor of swap-mode tiles leaves every CTA at least four
    K-blocks: K = 512 (4 K-blocks) runs unsplit, K = 1024 splits at most in two,
    K = 7168 splits; each result matches the oracle (child process, DG_VERBOSE
    reports the launch)."""
    import os, re, subprocess, sys
    code = ("import sys; sys.path[:0] = [%r, %r]\n"
            "import workloads as W, oracle\n"
            "from gpu_util import DeviceProblem, compare, to_f64, valid_mask\n"
            "for i, (M, N, K) in enumerate([(128, 256, 512), (64, 2112, 1024), (64, 2112, 7168)]):\n"
            "    p = W.make_dense(M, N, K, seed=40 + i, outliers=True)\n"
            "    d = to_f64(DeviceProblem(p).run())\n"
            "    compare(d, oracle.solve(p), valid_mask(p))\n"
            "    print('OK', K, flush=True)\n"
            % (os.path.dirname(os.path.dirname(__file__)), os.path.dirname(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, DG_VERBOSE="1"),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.count("OK") == 3, r.stdout + r.stderr
    split = {int(k): int(s) for k, s in re.findall(r"K=(\d+) G=1 .*? split=(\d+)", r.stderr)}
    assert split[512] == 1 and split[1024] <= 2 and split[7168] >= 2, split


@pytest.mark.parametrize("M,N", [(512, 256), (384, 384), (1024, 1152)])
def test_dense_normal_mode(M, N):
    _run_full(W.make_dense(M, N, 1024, seed=M + N))


def test_dense_wide_tile_n_128():
    _run_full(W.make_dense(512, 128, 512, seed=3))


def _exact_dense(M, N, K, seed):
    """Operands in {-1,0,1} (sparse), power-of-two scales: every partial sum
    and every output is exact in FP32 and representable in BF16."""
    rng = np.random.default_rng(seed)
    KB, NB = K // 128, (N + 127) // 128
    ai = rng.choice([-1, 0, 0, 0, 0, 0, 0, 1], size=(M, K))
    bi = rng.choice([-1, 0, 0, 0, 0, 0, 0, 1], size=(N, K))
    to8 = lambda v: torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sa = np.ldexp(1.0, rng.integers(-1, 2, size=(M, KB))).astype(np.float32)
    sb = np.ldexp(1.0, rng.integers(-1, 1, size=(NB, KB))).astype(np.float32)
    ld = W.tma_aligned(M)
    return W.Problem("dense", M, N, K, 1, to8(ai), W.sfa_mn_major(sa, ld), ld, to8(bi)[None], sb[None])


@pytest.mark.parametrize("M", [32, 64, 128, 300])
def test_dense_integer_cases_bit_exact(M):
    prob = _exact_dense(M, 384, 512, seed=M)
    ref = oracle.solve(prob)
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16)
    assert torch.equal(ref_bf16.double(), torch.from_numpy(ref)), "case not BF16-exact"
    d = DeviceProblem(prob).run().cpu()
    assert torch.equal(d.view(torch.int16), ref_bf16.view(torch.int16))


def test_dense_deterministic():
    prob = W.make_dense(64, 2112, 4096, seed=11, outliers=True)
    dp = DeviceProblem(prob)
    d1 = dp.run().clone()
    d2 = dp.run().clone()
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))


# ------------------------------------------------------------------ contiguous
@pytest.mark.parametrize("counts,N,K", [([130, 0, 700, 5], 384, 512),
                                        ([0, 0, 1, 0], 256, 256),
                                        ([128, 256], 2112, 512),
                                        # 128-row blocks 4|5 and 2|3 of different groups share a
                                        # CTA pair tile (second pass), odd block count at the end
                                        ([130, 200, 5, 300, 129], 448, 384),
                                        ([1, 1, 1, 1, 1, 1, 1], 256, 256)])
def test_contiguous(counts, N, K):
    _run_full(W.make_contiguous(counts, N, K, seed=sum(counts) + N))


@pytest.mark.parametrize("counts,N,K,gaps", [([130, 200, 5, 300, 129], 448, 384, None),
                                             ([128, 256], 2112, 512, None),
                                             # blocks 2 and 3 are both padding: a pair tile with
                                             # no work; blocks 4|5 hold groups 1|2 (second pass)
                                             ([200, 100, 300], 256, 256, [2, 0, 0]),
                                             ([5, 130], 384, 256, [3, 1])])
def test_contiguous_cta_pairs(counts, N, K, gaps):
    """The CTA-pair contiguous path (the default for N > 128 and K >= 4096),
    forced on at small K in a child process: second passes for pair tiles
    whose two 128-row blocks belong to different groups, and pair tiles whose
    two blocks are both padding (whole unused blocks of the caller's buffer)."""
    _run_contiguous_child(counts, N, K, pairs=True, gaps=gaps)


@pytest.mark.parametrize("counts,N,K", [([130, 200, 5, 300, 129], 384, 4096), ([1] * 7, 256, 4096)])
def test_contiguous_single_cta_tiles(counts, N, K):
    """The single-CTA contiguous path forced at long K in a child process."""
    _run_contiguous_child(counts, N, K, pairs=False)


def _run_contiguous_child(counts, N, K, pairs, gaps=None):
    import os, subprocess, sys
    code = ("import sys; sys.path[:0] = [%r, %r]\n"
            "import workloads as W, oracle\n"
            "from gpu_util import DeviceProblem, compare, to_f64, valid_mask\n"
            "p = W.make_contiguous(%r, %d, %d, seed=77, gaps=%r)\n"
            "dp = DeviceProblem(p); dp.fill_sentinel(); d = to_f64(dp.run())\n"
            "compare(d, oracle.solve(p), valid_mask(p)); print('OK')\n"
            % (os.path.dirname(os.path.dirname(__file__)), os.path.dirname(__file__), counts, N, K, gaps))
    env = dict(os.environ, DG_CONTIG_PAIRS="1" if pairs else "0", DG_VERBOSE="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr
    assert ("ctas/mma=2" if pairs else "ctas/mma=1") in r.stderr


def test_contiguous_long_k_default_pairs():
    """K >= 4096 takes CTA pairs by default (group boundaries inside pair tiles)."""
    _run_full(W.make_contiguous([130, 200, 5, 300, 129], 448, 4096, seed=91))


def test_contiguous_multinomial_small():
    _run_full(W.make_contiguous_multinomial(4, 2000, 256, 1024, seed=4))


def test_contiguous_equals_dense_per_group():
    prob = W.make_contiguous([200, 100, 300], 256, 512, seed=12)
    dp = DeviceProblem(prob)
    d = dp.run().clone()
    for g in range(prob.G):
        rows = np.flatnonzero(prob.m_indices == g)
        sub = W.Problem("dense", len(rows), prob.N, prob.K, 1, prob.a[rows],
                        W.sfa_mn_major(prob.sfa[:, rows].T.copy(), W.tma_aligned(len(rows))),
                        W.tma_aligned(len(rows)), prob.b[g:g + 1], prob.sfb[g:g + 1])
        dd = DeviceProblem(sub).run()
        ref = oracle.solve(sub)
        compare(to_f64(d[torch.from_numpy(rows).cuda()]), ref, np.ones_like(ref, bool))
        compare(to_f64(dd), ref, np.ones_like(ref, bool))


# ------------------------------------------------------------------ masked
@pytest.mark.parametrize("masked_m,Mmax", [([0, 256, 1, 100, 255, 64, 65, 128], 256),
                                           ([64, 0, 17, 63], 64),
                                           ([128, 5, 0, 127, 64], 128),
                                           ([0, 0, 0], 256)])
def test_masked_rows_untouched(masked_m, Mmax):
    prob = W.make_masked(masked_m, Mmax, 384, 512, seed=Mmax + len(masked_m))
    dp, d, ref, _ = _run_full(prob, sentinel=True)
    raw = dp.d.view(torch.int16).cpu().numpy()
    for g, m in enumerate(masked_m):
        assert (raw[g, m:] == np.int16(SENTINEL)).all(), f"group {g} rows >= {m} written"
        assert (raw[g, :m] != np.int16(SENTINEL)).all()


def test_masked_maximum_group_count():
    """G = 1024, the largest group count the masked call accepts (its tile table
    holds one prefix entry per group plus the total): mostly tiny groups, every
    seventh one empty, the last one full."""
    rng = np.random.default_rng(1024)
    masked_m = rng.integers(0, 65, size=1024)
    masked_m[::7] = 0
    masked_m[-1] = 64
    prob = W.make_masked(masked_m.tolist(), 64, 128, 256, seed=1025)
    dp, d, ref, _ = _run_full(prob, sentinel=True)
    raw = dp.d.view(torch.int16).cpu().numpy()
    for g, m in enumerate(masked_m):
        assert (raw[g, m:] == np.int16(SENTINEL)).all(), f"group {g} rows >= {m} written"


def test_masked_n_tail_large_k():
    _run_full(W.make_masked([200, 33, 0, 256], 256, 2112, 2048, seed=21))


def test_masked_cuda_graph_replay_reads_new_counts():
    """The masked call reads masked_m on the device only: a captured graph
    replayed after the counts change computes (and leaves untouched) the rows
    the NEW counts say."""
    prob = W.make_masked([10, 200, 0, 64], 256, 256, 512, seed=31, poison=False)
    dp = DeviceProblem(prob)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dp.run(s)                        # first call outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dp.run(s)
    new_m = np.array([256, 0, 100, 1], np.int32)
    dp.masked_m.copy_(torch.from_numpy(new_m))
    dp.fill_sentinel()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    prob2 = W.Problem("masked", prob.M, prob.N, prob.K, prob.G, prob.a, prob.sfa, prob.ld_sfa,
                      prob.b, prob.sfb, masked_m=new_m)
    compare(to_f64(dp.d), oracle.solve(prob2), valid_mask(prob2))
    raw = dp.d.view(torch.int16).cpu().numpy()
    for gi, m in enumerate(new_m):
        assert (raw[gi, m:] == np.int16(SENTINEL)).all()
    del g


def test_masked_equals_dense_per_group():
    prob = W.make_masked([77, 0, 256, 130], 256, 384, 1024, seed=41)
    d = DeviceProblem(prob).run().clone()
    for g, m in enumerate(prob.masked_m):
        if m == 0:
            continue
        sub = W.Problem("dense", int(m), prob.N, prob.K, 1, prob.a[g, :m],
                        np.ascontiguousarray(prob.sfa[g]), prob.ld_sfa, prob.b[g:g + 1], prob.sfb[g:g + 1])
        dd = DeviceProblem(sub).run()
        ref = oracle.solve(sub)
        compare(to_f64(d[g, :m]), ref, np.ones_like(ref, bool))
        compare(to_f64(dd), ref, np.ones_like(ref, bool))


def test_rejected_calls_leave_d_untouched():
    """Argument errors are reported before anything is enqueued: each call
    returns its status code and D keeps its sentinel bit for bit."""
    prob = W.make_dense(64, 256, 512, seed=5)
    dp = DeviceProblem(prob)
    dp.fill_sentinel()
    L = dg.lib()
    a, sfa, b, sfb, d = (dp.a.data_ptr(), dp.sfa.data_ptr(), dp.b.data_ptr(), dp.sfb.data_ptr(),
                         dp.d.data_ptr())
    ld = prob.ld_sfa
    assert L.dg_fp8_gemm_nt(a, sfa, ld, b, sfb, d, 64, 256, 500, None) == 3        # K % 128
    assert L.dg_fp8_gemm_nt(a, sfa, ld, b, sfb, d, 64, 200, 512, None) == 3        # N % 16
    assert L.dg_fp8_gemm_nt(a + 8, sfa, ld, b, sfb, d, 64, 256, 512, None) == 2    # misaligned A
    assert L.dg_fp8_gemm_nt(a, sfa, ld + 2, b, sfb, d, 64, 256, 512, None) == 2    # ld_sfa % 4
    assert L.dg_fp8_gemm_nt(None, sfa, ld, b, sfb, d, 64, 256, 512, None) == 1     # null A
    mm = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.dg_m_grouped_fp8_gemm_nt_masked(a, sfa, ld, b, sfb, d, mm.data_ptr(), 1025, 64, 256,
                                             512, None) == 3                           # G > 1024
    torch.cuda.synchronize()
    assert (dp.d.view(torch.int16) == SENTINEL).all(), "a rejected call wrote D"


# ------------------------------------------------------------------ full-size workloads
@pytest.mark.parametrize("name", ["dense_decode_m64", "dense_decode_m128"])
def test_full_size_decode_full_oracle(name):
    _run_full(W.make_workload(name))


@pytest.mark.parametrize("name", ["dense_large", "contiguous_g4", "masked_g16"])
def test_full_size_sampled(name):
    prob = W.make_workload(name)
    dp = DeviceProblem(prob)
    dp.fill_sentinel()
    d = to_f64(dp.run())
    rng = np.random.default_rng(2024)
    n = 6000
    mask = valid_mask(prob)
    if prob.layout == "masked":
        grp = rng.integers(0, prob.G, n)
        row = np.array([rng.integers(0, max(int(prob.masked_m[g]), 1)) for g in grp])
        keep = prob.masked_m[grp] > 0
        grp, row = grp[keep], row[keep]
    else:
        grp = np.zeros(n, np.int64)
        valid_rows = np.flatnonzero(mask[:, 0])
        row = rng.choice(valid_rows, n)
    col = rng.integers(0, prob.N, len(row))
    ref = oracle.points(prob, grp, row, col)
    got = d[grp, row, col] if prob.layout == "masked" else d[row, col]
    compare(got, ref, np.ones_like(ref, bool))
    # properties that hold at any size: no NaN in valid rows, untouched masked rows
    assert np.isfinite(d[mask]).all()
    if prob.layout == "masked":
        raw = dp.d.view(torch.int16).cpu().numpy()
        for g, m in enumerate(prob.masked_m):
            assert (raw[g, m:] == np.int16(SENTINEL)).all()

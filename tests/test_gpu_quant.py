"""GPU parity of the per-token 1x128 quantiser against the oracle.

The quantiser decides integers (E4M3 codes) from floating point, and both
sides take that decision in FP32 with a correctly rounded quotient, so codes
and scales must match bit for bit.  Covered: ragged row counts and K-block
counts that leave a warp's 8-block chunk partial, every finite BF16 value
under several scales (exact E4M3 ties, subnormal codes, signed zeros,
saturation at 448), zero blocks, the reciprocal fast path against the
all-division path, the masked layout (invalid rows never read -- they hold
NaN -- nor written), out-of-range masked counts, argument validation, CUDA
graph replay, a quantise-then-GEMM pipeline, and the full-size workloads.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_fp32_b200 as dg
import oracle
import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

SCALE_SENTINEL = -12345.0
Q_SENTINEL = 0xA5


@pytest.fixture(autouse=True, scope="module")
def _clean_status():
    from moe_grouped_gemm_fp32_b200 import build
    build.build()
    oracle.build()
    dg.dg_get_device_status(clear=True)
    yield
    dg.dg_debug_set_flags(0)
    assert dg.dg_get_device_status(clear=True) == 0, "a kernel recorded an error"


def _quant_dense(x32: np.ndarray, ld=None, exact_div=False):
    M, K = x32.shape
    ld = ld if ld is not None else W.tma_aligned(max(M, 1))
    x = torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).cuda()
    assert np.array_equal(x.float().cpu().numpy(), x32), "input must be BF16-exact"
    q = torch.full((M, K), Q_SENTINEL, dtype=torch.uint8, device="cuda")
    sfa = torch.full((K // 128, ld), SCALE_SENTINEL, dtype=torch.float32, device="cuda")
    dg.dg_debug_set_flags(2 if exact_div else 0)
    try:
        dg.dg_per_token_cast_to_fp8(x, q, sfa)
        torch.cuda.synchronize()
    finally:
        dg.dg_debug_set_flags(0)
    return q.cpu().numpy(), sfa.cpu().numpy()


def _check_dense(x32, exact_div=False):
    q, sfa = _quant_dense(x32, exact_div=exact_div)
    q_ref, sfa_ref = oracle.quantize_1x128(x32)
    M = x32.shape[0]
    bad = np.argwhere(q != q_ref)
    assert bad.size == 0, f"{len(bad)} code mismatches, first at {bad[:4].tolist()}"
    assert np.array_equal(sfa[:, :M], sfa_ref[:, :M])
    assert (sfa[:, M:] == SCALE_SENTINEL).all(), "padding scales were written"


@pytest.mark.parametrize("M,K", [(1, 128), (7, 384), (130, 1024), (33, 7168), (257, 640), (64, 1152)])
@pytest.mark.parametrize("exact_div", [False, True])
def test_dense_matches_oracle(M, K, exact_div):
    prob = W.make_activations(M, K, seed=100 + M + K)
    _check_dense(prob.x, exact_div)


def _all_finite_bf16() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    return v[np.isfinite(v)]


@pytest.mark.parametrize("amax", [448.0, 1344.0, 1.0, 3.140625, 1e-3, 2.0 ** -100, 2.0 ** -130,
                                  3.0e38, 7.0, 0.875])
def test_every_bf16_value_under_one_scale(amax):
    """Each 128-block holds the amax element first and 127 other finite BF16
    values of magnitude <= amax: all such values, both signs, so every E4M3
    tie, subnormal code and the saturation edge is exercised under that
    block scale (amax itself is rounded to BF16 first).  Scales like 7/448
    and 0.875/448 make x/s land exactly on E4M3 midpoints for many values
    (the kernel's exact tie resolution)."""
    amax = float(torch.tensor(amax, dtype=torch.float32).to(torch.bfloat16).float())
    vals = _all_finite_bf16()
    vals = vals[np.abs(vals) <= amax]
    n_blocks = (len(vals) + 126) // 127
    pad = n_blocks * 127 - len(vals)
    body = np.concatenate([vals, np.zeros(pad, np.float32)]).reshape(n_blocks, 127)
    head = np.where(np.arange(n_blocks) % 2 == 0, amax, -amax).astype(np.float32)[:, None]
    blocks = np.concatenate([head, body], axis=1).astype(np.float32)
    kb = 8
    rows = (n_blocks + kb - 1) // kb
    x = np.zeros((rows * kb, 128), np.float32)
    x[:n_blocks] = blocks
    x = x.reshape(rows, kb * 128)
    _check_dense(x, exact_div=False)
    _check_dense(x, exact_div=True)


def test_zero_blocks_and_signed_zeros():
    x = np.zeros((5, 512), np.float32)
    x[1, :128] = -0.0
    x[2, 128:256] = np.float32(2.0 ** -133)   # smallest BF16 subnormal: tiny but non-zero
    x[3, 300] = -1.5
    x[4, ::2] = 7.0
    x[4, 1::2] = -0.0
    _check_dense(x)
    q, sfa = _quant_dense(x)
    assert (q[1, :128] == 0x80).all() and (q[0] == 0).all()
    assert (sfa[:, 0] == 1.0).all()


def test_fast_path_equals_division_on_a_large_input():
    prob = W.make_activations(4096, 7168, seed=11)
    q_fast, s_fast = _quant_dense(prob.x)
    q_div, s_div = _quant_dense(prob.x, exact_div=True)
    assert np.array_equal(q_fast, q_div) and np.array_equal(s_fast, s_div)
    q_ref, s_ref = oracle.quantize_1x128(prob.x)
    assert np.array_equal(q_fast, q_ref) and np.array_equal(s_fast[:, :4096], s_ref[:, :4096])


def test_output_feeds_the_gemm():
    """Quantise on the GPU, then GEMM: equals the oracle GEMM of the oracle's
    quantisation of the same activations (bit-identical operands)."""
    M, N, K = 96, 256, 1024
    x = W.make_activations(M, K, seed=21).x
    q, sfa = _quant_dense(x)
    q_ref, sfa_ref = oracle.quantize_1x128(x)
    assert np.array_equal(q, q_ref)
    wb = W.make_dense(8, N, K, seed=22)            # weights only
    a = torch.from_numpy(q).cuda()
    sfa_t = torch.from_numpy(sfa).cuda()
    b = torch.from_numpy(wb.b[0]).cuda()
    sfb = torch.from_numpy(wb.sfb[0]).cuda()
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dg.dg_fp8_gemm_nt(a, sfa_t, b, sfb, d)
    ref = oracle.gemm_dense(q_ref, sfa_ref, sfa_ref.shape[1], wb.b[0], wb.sfb[0], M, N, K)
    got = d.float().cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= 1e-2 * np.maximum(1.0, np.abs(ref))).all()


def _quant_masked(prob, graph=False):
    G, Mmax, K = prob.x.shape
    ld = prob.ld_sfa
    x = prob.x_bf16().cuda()
    mm = torch.from_numpy(prob.masked_m).cuda()
    q = torch.full((G, Mmax, K), Q_SENTINEL, dtype=torch.uint8, device="cuda")
    sfa = torch.full((G, K // 128, ld), SCALE_SENTINEL, dtype=torch.float32, device="cuda")
    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            dg.dg_per_token_cast_to_fp8_masked(x, q, sfa, mm, s)
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            dg.dg_per_token_cast_to_fp8_masked(x, q, sfa, mm)
        q.fill_(Q_SENTINEL)
        sfa.fill_(SCALE_SENTINEL)
        g.replay()
    else:
        dg.dg_per_token_cast_to_fp8_masked(x, q, sfa, mm)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sfa.cpu().numpy()


def _check_masked(prob, q, sfa):
    for g in range(prob.G):
        m = int(min(max(prob.masked_m[g], 0), prob.M))
        if m:
            q_ref, s_ref = oracle.quantize_1x128(prob.x[g, :m])
            assert np.array_equal(q[g, :m], q_ref), f"group {g}"
            assert np.array_equal(sfa[g, :, :m], s_ref[:, :m]), f"group {g} scales"
        assert (q[g, m:] == Q_SENTINEL).all(), f"group {g}: invalid rows written"
        assert (sfa[g, :, m:] == SCALE_SENTINEL).all(), f"group {g}: invalid scales written"


@pytest.mark.parametrize("masked_m,Mmax,K", [([0, 5, 200, 77], 200, 1024), ([1] * 7, 8, 128),
                                             ([0, 0, 0], 64, 256), ([130, 3], 130, 896)])
def test_masked_matches_oracle(masked_m, Mmax, K):
    prob = W.make_activations_masked(masked_m, Mmax, K, seed=31 + Mmax)
    q, sfa = _quant_masked(prob)
    _check_masked(prob, q, sfa)


def test_masked_maximum_group_count():
    """G = 1024, the largest group count of the masked quantiser (its row-prefix
    table has one entry per group plus the total); every seventh group empty."""
    counts = np.random.default_rng(1023).integers(0, 17, size=1024)
    counts[::7] = 0
    prob = W.make_activations_masked(counts.tolist(), 16, 256, seed=1023)
    q, sfa = _quant_masked(prob)
    _check_masked(prob, q, sfa)


def test_masked_graph_replay():
    prob = W.make_activations_masked([17, 0, 64, 33], 64, 512, seed=41)
    q, sfa = _quant_masked(prob, graph=True)
    _check_masked(prob, q, sfa)


def test_masked_count_out_of_range_is_clamped_and_reported():
    prob = W.make_activations_masked([3, 9], 8, 256, seed=51, poison=False)
    prob.masked_m = np.array([-4, 9], dtype=np.int32)     # 9 > Mmax
    q, sfa = _quant_masked(prob)
    status = dg.dg_get_device_status(clear=True)
    assert status & 0xFF == 1 and (status >> 8) & 0xFF == 9
    clamped = W.QuantProblem("masked", prob.x, np.array([0, 8], np.int32))
    _check_masked(clamped, q, sfa)


def test_masked_then_masked_gemm_in_one_graph():
    """Decode step: quantise the masked activations and run the masked GEMM,
    captured together in one CUDA graph."""
    G, Mmax, N, K = 4, 64, 384, 1024
    prob = W.make_activations_masked([64, 10, 0, 37], Mmax, K, seed=61)
    wprob = W.make_masked([1] * G, 8, N, K, seed=62)       # weights only
    x = prob.x_bf16().cuda()
    mm = torch.from_numpy(prob.masked_m).cuda()
    q = torch.zeros((G, Mmax, K), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((G, K // 128, prob.ld_sfa), dtype=torch.float32, device="cuda")
    b = torch.from_numpy(wprob.b).cuda()
    sfb = torch.from_numpy(wprob.sfb).cuda()
    d = torch.zeros((G, Mmax, N), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dg.dg_per_token_cast_to_fp8_masked(x, q, sfa, mm, s)
        dg.dg_m_grouped_fp8_gemm_nt_masked(q, sfa, b, sfb, d, mm, s)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        dg.dg_per_token_cast_to_fp8_masked(x, q, sfa, mm)
        dg.dg_m_grouped_fp8_gemm_nt_masked(q, sfa, b, sfb, d, mm)
    d.zero_()
    graph.replay()
    torch.cuda.synchronize()
    got = d.float().cpu().numpy().astype(np.float64)
    for g in range(G):
        m = int(prob.masked_m[g])
        if not m:
            continue
        q_ref, s_ref = oracle.quantize_1x128(prob.x[g, :m])
        ref = oracle.gemm_dense(q_ref, s_ref, s_ref.shape[1], wprob.b[g], wprob.sfb[g], m, N, K)
        assert (np.abs(got[g, :m] - ref) <= 1e-2 * np.maximum(1.0, np.abs(ref))).all(), f"group {g}"
        assert (got[g, m:] == 0).all()


def test_validation_errors():
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((4, 256), dtype=torch.uint8, device="cuda")
    L = dg.lib()
    s = torch.zeros((2, 4), dtype=torch.float32, device="cuda")
    xp, qp, sp = x.data_ptr(), q.data_ptr(), s.data_ptr()
    assert L.dg_per_token_cast_to_fp8(xp, qp, sp, 4, 4, 200, None) == 3        # K % 128
    assert L.dg_per_token_cast_to_fp8(xp, qp, sp, 2, 4, 256, None) == 1        # ld_sfa < M
    assert L.dg_per_token_cast_to_fp8(xp, qp, sp, 6, 4, 256, None) == 2        # ld_sfa % 4
    assert L.dg_per_token_cast_to_fp8(xp + 2, qp, sp, 4, 4, 256, None) == 2    # misaligned x
    assert L.dg_per_token_cast_to_fp8(None, qp, sp, 4, 4, 256, None) == 1
    assert L.dg_per_token_cast_to_fp8(xp, qp, sp, 4, -1, 256, None) == 1
    assert L.dg_per_token_cast_to_fp8(xp, qp, sp, 4, 0, 256, None) == 0        # no-op
    mm = torch.zeros(2, dtype=torch.int32, device="cuda")
    assert L.dg_per_token_cast_to_fp8_masked(xp, qp, sp, 4, mm.data_ptr(), 0, 2, 256, None) == 1
    assert L.dg_per_token_cast_to_fp8_masked(xp, qp, sp, 4, mm.data_ptr(), 1025, 2, 256, None) == 3
    assert L.dg_per_token_cast_to_fp8_masked(xp, qp, sp, 4, None, 2, 2, 256, None) == 1
    torch.cuda.synchronize()
    assert (q == 0).all()


@pytest.mark.parametrize("name", ["quant_tokens_32768", "quant_masked_g16"])
def test_full_size_workloads(name):
    prob = W.make_quant_workload(name)
    if prob.layout == "dense":
        q, sfa = _quant_dense(prob.x)
        rng = np.random.default_rng(5)
        rows = np.sort(rng.choice(prob.M, size=512, replace=False))
        q_ref, s_ref = oracle.quantize_1x128(prob.x[rows])
        assert np.array_equal(q[rows], q_ref)
        assert np.array_equal(sfa[:, rows], s_ref[:, :len(rows)])
    else:
        q, sfa = _quant_masked(prob)
        _check_masked(prob, q, sfa)

"""GPU parity of the fused expert FFN (contiguous layout) against the oracle.

The intermediate E4M3 codes are an integer decision taken on FP32 GEMM sums,
which the oracle forms in FP64: a code may differ from the oracle's only where
the activation sits next to an E4M3 rounding boundary, and then by one step.
The test checks that (scales within 1e-4 relative, at most 0.5% of the codes
moved, each by one step at most) and compares y with the GEMM tolerance:
per element |y - y_ref| <= 1e-2 * max(1, |y_ref|), Frobenius <= 2e-3.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_fp32_b200 as dg
import oracle
import workloads as W
from gpu_util import compare

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


def _decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).float().numpy()


def _check_codes(q_gpu, s_gpu, ref):
    assert np.allclose(s_gpu, ref["s"], rtol=1e-4, atol=0)
    moved = q_gpu != ref["q"]
    assert moved.mean() <= 5e-3, f"{moved.mean():.4%} of the codes differ"
    vg, vr = _decode(q_gpu), _decode(ref["q"])
    # one E4M3 step: 2^-3 of the magnitude in the normal range, 2^-9 below 2^-6
    step = np.maximum(np.abs(vr), np.abs(vg)) * 2.0 ** -3 + 2.0 ** -9
    assert (np.abs(vg - vr)[moved] <= step[moved] + 1e-12).all(), "a code moved by more than one step"


def _device(prob):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return {"a": t(prob.a), "sfa": t(prob.sfa), "w1": t(prob.w1), "sfb1": t(prob.sfb1), "w2": t(prob.w2),
            "sfb2": t(prob.sfb2), "mi": t(prob.m_indices)}


def _run_ffn(prob):
    dv = _device(prob)
    q = torch.full((prob.M, prob.I), 0xA5, dtype=torch.uint8, device="cuda")
    s = torch.full((prob.I // 128, prob.ld_sfa), -1.0, dtype=torch.float32, device="cuda")
    y = torch.empty((prob.M, prob.H), dtype=torch.bfloat16, device="cuda")
    dg.dg_m_grouped_fp8_ffn_contiguous(dv["a"], dv["sfa"], dv["w1"], dv["sfb1"], dv["w2"], dv["sfb2"],
                                       q, s, y, dv["mi"])
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), y.double().cpu().numpy()


@pytest.mark.parametrize("counts,H,I", [([130, 0, 200, 5], 512, 256), ([1] * 3, 256, 128),
                                        ([300, 77], 1024, 512)])
def test_ffn_matches_oracle(counts, H, I):
    prob = W.make_ffn_contiguous(counts, H, I, seed=sum(counts) + H + I)
    q, s, y = _run_ffn(prob)
    rows = np.flatnonzero(prob.m_indices >= 0)
    ref = oracle.ffn_rows(prob, rows)
    _check_codes(q[rows], s[:, rows], ref)
    compare(y[rows], ref["y"], np.ones(ref["y"].shape, bool))


def test_first_stage_alone():
    prob = W.make_ffn_contiguous([129, 64], 384, 384, seed=5)
    dv = _device(prob)
    q = torch.zeros((prob.M, prob.I), dtype=torch.uint8, device="cuda")
    s = torch.zeros((prob.I // 128, prob.ld_sfa), dtype=torch.float32, device="cuda")
    dg.dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(dv["a"], dv["sfa"], dv["w1"], dv["sfb1"], q, s, dv["mi"])
    torch.cuda.synchronize()
    rows = np.flatnonzero(prob.m_indices >= 0)
    _check_codes(q.cpu().numpy()[rows], s.cpu().numpy()[:, rows], oracle.ffn_rows(prob, rows))


def test_ffn_validation():
    L = dg.lib()
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    p = z.data_ptr()
    # N not a multiple of 256
    assert L.dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(p, p, 128, p, p, p, p, 128, p, 128, 384, 128, 1, None) == 3
    # ld_s_out below M_total
    assert L.dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(p, p, 128, p, p, p, p, 64, p, 128, 256, 128, 1, None) == 1
    # I not a multiple of 128
    assert L.dg_m_grouped_fp8_ffn_contiguous(p, p, 128, p, p, p, p, p, p, 128, p, p, 128, 128, 100, 1, None) == 3


def test_ffn_full_size_sampled_rows():
    prob = W.make_ffn_workload("ffn_g4")
    q, s, y = _run_ffn(prob)
    rng = np.random.default_rng(4)
    rows = np.sort(rng.choice(np.flatnonzero(prob.m_indices >= 0), size=16, replace=False))
    ref = oracle.ffn_rows(prob, rows)
    _check_codes(q[rows], s[:, rows], ref)
    compare(y[rows], ref["y"], np.ones(ref["y"].shape, bool))

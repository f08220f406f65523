"""Shared helpers of the GPU parity tests: move a ``workloads.Problem`` to the
device, run it through the C ABI, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import moe_grouped_gemm_fp32_b200 as dg

SENTINEL = 0x7FC1          # a BF16 NaN pattern the kernels never produce
ATOL_REL = 1e-2            # per element: |D - ref| <= 1e-2 * max(1, |ref|)
FROB_REL = 2e-3            # ||D - ref||_F / ||ref||_F over valid rows


class DeviceProblem:
    def __init__(self, prob, device="cuda"):
        self.prob = prob
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(device)
        self.a = t(prob.a)
        self.sfa = t(prob.sfa)
        self.b = t(prob.b)
        self.sfb = t(prob.sfb)
        self.m_indices = t(prob.m_indices) if prob.m_indices is not None else None
        self.masked_m = t(prob.masked_m) if prob.masked_m is not None else None
        self.ks = t(prob.ks) if getattr(prob, "ks", None) is not None else None
        self.d = torch.empty(prob.d_shape(), dtype=torch.bfloat16, device=device)

    def fill_sentinel(self):
        self.d.view(torch.int16).fill_(SENTINEL)

    def run(self, stream=None):
        p = self.prob
        if p.layout == "dense":
            dg.dg_fp8_gemm_nt(self.a, self.sfa, self.b[0], self.sfb[0], self.d, stream)
        elif p.layout == "contiguous":
            dg.dg_m_grouped_fp8_gemm_nt_contiguous(self.a, self.sfa, self.b, self.sfb, self.d,
                                                   self.m_indices, stream)
        elif p.layout == "k_grouped":
            dg.dg_k_grouped_fp8_gemm_nt_contiguous(self.a, self.sfa, self.b[0], self.sfb[0], self.d,
                                                   self.ks, stream)
        else:
            dg.dg_m_grouped_fp8_gemm_nt_masked(self.a, self.sfa, self.b, self.sfb, self.d,
                                               self.masked_m, stream)
        return self.d


def valid_mask(prob) -> np.ndarray:
    """Boolean mask over D of the rows the method computes."""
    if prob.layout in ("dense", "k_grouped"):
        return np.ones(prob.d_shape(), bool)
    if prob.layout == "contiguous":
        return np.broadcast_to((prob.m_indices >= 0)[:, None], prob.d_shape())
    rows = np.arange(prob.M)[None, :] < prob.masked_m[:, None]
    return np.broadcast_to(rows[:, :, None], prob.d_shape())


def compare(d_gpu: np.ndarray, ref: np.ndarray, mask: np.ndarray):
    """Tolerance check over the masked (valid) elements; returns the margins."""
    g, r = d_gpu[mask].astype(np.float64), ref[mask]
    assert np.isfinite(r).all(), "oracle produced a non-finite valid output"
    assert np.isfinite(g).all(), "non-finite valid output (NaN padding leaked?)"
    err = np.abs(g - r)
    bound = ATOL_REL * np.maximum(1.0, np.abs(r))
    worst = float((err / bound).max()) if err.size else 0.0
    frob = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)) if err.size else 0.0
    assert worst <= 1.0, f"per-element error {worst:.3f} x bound"
    assert frob <= FROB_REL, f"relative Frobenius error {frob:.2e}"
    return worst, frob


def to_f64(d: torch.Tensor) -> np.ndarray:
    return d.float().cpu().numpy().astype(np.float64)

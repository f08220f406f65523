"""Pins of the oracle's fused expert FFN chain (GEMM1 -> SwiGLU -> per-token
quantiser -> GEMM2): silu's closed forms, the gate/up interleaving, and the
whole chain against a second statement built from the exact-fraction brute
force GEMM and math.exp."""
import math

import numpy as np

import oracle
import workloads as W
from oracle import brute


def test_silu_closed_forms():
    x = np.array([0.0, 1.0, -1.0, 40.0, -40.0, 800.0, -800.0])
    y = oracle.silu(x)
    assert y[0] == 0.0 and y[5] == 800.0 and y[6] == -0.0
    assert abs(y[1] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(y[2] + 1.0 / (1.0 + math.exp(1.0))) < 1e-15
    assert abs(y[3] - 40.0) < 1e-12 and abs(y[4]) < 1e-15


def test_ffn_chain_matches_brute_force(oracle_lib):
    prob = W.make_ffn_contiguous([3, 0, 2], H=128, I=256, seed=7)
    rows = np.flatnonzero(prob.m_indices >= 0)
    out = oracle_lib.ffn_rows(prob, rows)
    for i, r in enumerate(rows):
        g = int(prob.m_indices[r])
        kb = prob.H // 128
        sa = prob.sfa[:, r][None, :]                    # [1][KB], row-major for brute
        h = brute.gemm(prob.a[r:r + 1], sa, prob.w1[g], prob.sfb1[g], 1, 2 * prob.I, prob.H)[0]
        h = np.array([float(v) for v in h])
        assert np.allclose(out["h"][i], h, rtol=1e-13, atol=1e-13)
        gate = np.concatenate([h[256 * j:256 * j + 128] for j in range(prob.I // 128)])
        up = np.concatenate([h[256 * j + 128:256 * j + 256] for j in range(prob.I // 128)])
        act = np.array([gv / (1.0 + math.exp(-gv)) * uv for gv, uv in zip(gate, up)], np.float32)
        assert np.array_equal(out["act"][i], act)
        q, s = oracle_lib.quantize_1x128(act[None, :])
        assert np.array_equal(out["q"][i], q[0]) and np.array_equal(out["s"][:, i], s[:, 0])
        y = brute.gemm(q, s[:, :1].T, prob.w2[g], prob.sfb2[g], 1, prob.H, prob.I)[0]
        assert np.allclose(out["y"][i], [float(v) for v in y], rtol=1e-12, atol=1e-12)

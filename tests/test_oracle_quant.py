"""Pins of the oracle's per-token 1x128 quantiser and its E4M3 encoder.

The encoder is checked against torch's float8_e4m3fn cast (a library routine)
on every representable value, on every exact midpoint between neighbours
(round-half-to-even), and on random data; the quantiser against the closed
forms of its definition (amax element maps to +-448, scale = amax / 448, zero
blocks) and against an independent torch-ops statement of the same steps.
"""
import numpy as np
import pytest
import torch

import oracle


def _torch_e4m3(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _finite_values():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    return codes, vals


def test_encoder_roundtrips_every_finite_code(oracle_lib):
    codes, vals = _finite_values()
    enc = oracle_lib.e4m3_encode(vals)
    assert np.array_equal(enc, codes)


def test_encoder_ties_to_even_at_every_midpoint(oracle_lib):
    _, vals = _finite_values()
    pos = np.unique(vals[vals >= 0]).astype(np.float64)
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)      # exact in float32
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)
    for m in (mids, -mids):
        assert np.array_equal(oracle_lib.e4m3_encode(m), _torch_e4m3(m))


def test_encoder_matches_torch_on_random_values(oracle_lib):
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(50000) * 10.0 ** rng.integers(-5, 3, 50000)).astype(np.float32)
    v = np.clip(v, -448, 448)
    assert np.array_equal(oracle_lib.e4m3_encode(v), _torch_e4m3(v))


def test_quantiser_closed_forms(oracle_lib):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 384)).astype(np.float32)
    x[1, 128:256] = 0.0                                   # an all-zero block
    q, sfa = oracle_lib.quantize_1x128(x)
    assert sfa.shape == (3, 8) and q.shape == (5, 384)
    amax = np.abs(x.reshape(5, 3, 128)).max(axis=2)
    want_s = np.where(amax == 0, np.float32(1), (amax / np.float32(448)).astype(np.float32))
    assert np.array_equal(sfa[:, :5].T, want_s)
    assert (q[1, 128:256] == 0).all()
    deq = torch.from_numpy(q).view(torch.float8_e4m3fn).float().numpy().reshape(5, 3, 128)
    # the block's largest magnitude lands on +-448 (codes 0x7E / 0xFE)
    for m in range(5):
        for kb in range(3):
            if amax[m, kb] > 0:
                assert np.abs(deq[m, kb]).max() == 448.0
    # dequantised values approximate x within half an E4M3 step (relative 2^-4)
    recon = deq * sfa[:, :5].T[:, :, None]
    err = np.abs(recon - x.reshape(5, 3, 128))
    assert (err <= np.abs(x.reshape(5, 3, 128)) * 2.0 ** -4 + sfa[:, :5].T[:, :, None] * 2.0 ** -10).all()


def test_quantiser_matches_independent_torch_statement(oracle_lib):
    rng = np.random.default_rng(3)
    x = torch.from_numpy((rng.standard_normal((33, 512)) * 3).astype(np.float32)).bfloat16().float().numpy()
    q, sfa = oracle_lib.quantize_1x128(x)
    t = torch.from_numpy(x).view(33, 4, 128)
    amax = t.abs().amax(dim=2)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    qt = torch.clamp(t / s[:, :, None], -448, 448).to(torch.float8_e4m3fn).view(torch.uint8).reshape(33, 512)
    assert np.array_equal(q, qt.numpy())
    assert np.array_equal(sfa[:, :33], s.numpy().T)

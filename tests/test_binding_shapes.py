"""Host-only checks of the Python binding's marshalling (no GPU): every entry
point, called with the shapes the GPU tests and the bench use, passes its
checks and hands the C function the sizes in the order include/dg.h declares;
buffers whose shapes disagree with those sizes are refused before any C call
(the C functions see only pointers, so an undersized output would otherwise be
written past its end)."""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_fp32_b200 as dg
import workloads as W


class _FakeLib:
    """Records each call (name, args) and returns DG_SUCCESS."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("dg_"):
            raise AttributeError(name)

        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()

    def req_cpu(t, dtype, name, ndim=None):
        # the real check minus "is on a CUDA device"
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if ndim is not None and t.dim() not in ((ndim,) if isinstance(ndim, int) else ndim):
            raise ValueError(f"{name} has {t.dim()} dims")
        return 0x1000
    monkeypatch.setattr(dg, "_req", req_cpu)
    monkeypatch.setattr(dg, "lib", lambda: lib)
    monkeypatch.setattr(dg, "_stream_handle", lambda stream: None)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    return lib


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x))


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _ints(args):
    """The integer arguments of a recorded call (the pointers are 0x1000, the stream None)."""
    return [a for a in args if isinstance(a, int) and a != 0x1000]


def test_dense_and_grouped_fp8(fake):
    p = W.make_dense(65, 2112, 1024, seed=1)
    d = torch.empty(p.d_shape(), dtype=torch.bfloat16)
    dg.dg_fp8_gemm_nt(_t(p.a), _t(p.sfa), _t(p.b[0]), _t(p.sfb[0]), d)
    dg.dg_fp8_gemm_nt(_t(p.a), _t(p.sfa), _t(p.b), _t(p.sfb), d)          # [1, N, K] forms
    assert fake.calls[0][0] == "dg_fp8_gemm_nt"
    assert _ints(fake.calls[0][1]) == [p.ld_sfa, 65, 2112, 1024]

    c = W.make_contiguous([130, 0, 200], 384, 512, seed=2)
    dg.dg_m_grouped_fp8_gemm_nt_contiguous(_t(c.a), _t(c.sfa), _t(c.b), _t(c.sfb),
                                           torch.empty(c.d_shape(), dtype=torch.bfloat16),
                                           _t(c.m_indices))
    assert _ints(fake.calls[-1][1]) == [c.ld_sfa, c.M, 384, 512, 3]

    m = W.make_masked([5, 0, 64], 64, 256, 384, seed=3)
    dg.dg_m_grouped_fp8_gemm_nt_masked(_t(m.a), _t(m.sfa), _t(m.b), _t(m.sfb),
                                       torch.empty(m.d_shape(), dtype=torch.bfloat16), _t(m.masked_m))
    assert _ints(fake.calls[-1][1]) == [m.ld_sfa, 3, 64, 256, 384]

    k = W.make_k_grouped([256, 0, 128], 200, 384, seed=4)
    dg.dg_k_grouped_fp8_gemm_nt_contiguous(_t(k.a), _t(k.sfa), _t(k.b[0]), _t(k.sfb[0]),
                                           torch.empty(k.d_shape(), dtype=torch.bfloat16), _t(k.ks))
    assert _ints(fake.calls[-1][1]) == [k.ld_sfa, 3, 200, 384, 384]


def test_ffn_and_first_stage(fake):
    f = W.make_ffn_contiguous([130, 0, 5], 384, 256, seed=5)
    q = torch.empty((f.M, f.I), dtype=torch.uint8)
    s = torch.empty((f.I // 128, f.ld_sfa), dtype=torch.float32)
    y = torch.empty((f.M, f.H), dtype=torch.bfloat16)
    dg.dg_m_grouped_fp8_ffn_contiguous(_t(f.a), _t(f.sfa), _t(f.w1), _t(f.sfb1), _t(f.w2), _t(f.sfb2),
                                       q, s, y, _t(f.m_indices))
    assert _ints(fake.calls[-1][1]) == [f.ld_sfa, f.ld_sfa, f.M, 384, 256, 3]
    dg.dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(_t(f.a), _t(f.sfa), _t(f.w1), _t(f.sfb1), q, s,
                                                     _t(f.m_indices))
    assert _ints(fake.calls[-1][1]) == [f.ld_sfa, f.ld_sfa, f.M, 512, 384, 3]
    with pytest.raises(ValueError, match="y"):
        dg.dg_m_grouped_fp8_ffn_contiguous(_t(f.a), _t(f.sfa), _t(f.w1), _t(f.sfb1), _t(f.w2),
                                           _t(f.sfb2), q, s, y[:-1], _t(f.m_indices))
    with pytest.raises(ValueError, match="q_out"):
        dg.dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(_t(f.a), _t(f.sfa), _t(f.w1), _t(f.sfb1),
                                                         q[:, :128], s, _t(f.m_indices))


def test_bf16_and_quantiser(fake):
    b = W.make_bf16_dense(64, 136, 200, seed=6)
    dg.dg_bf16_gemm_nt(_bf16(b.a), _bf16(b.b[0]), torch.empty(b.d_shape(), dtype=torch.bfloat16))
    assert _ints(fake.calls[-1][1]) == [64, 136, 200]
    c = W.make_bf16_contiguous([130, 0, 7], 256, 128, seed=7)
    dg.dg_m_grouped_bf16_gemm_nt_contiguous(_bf16(c.a), _bf16(c.b),
                                            torch.empty(c.d_shape(), dtype=torch.bfloat16),
                                            _t(c.m_indices))
    assert _ints(fake.calls[-1][1]) == [c.M, 256, 128, 3]
    m = W.make_bf16_masked([5, 0], 8, 136, 64, seed=8)
    dg.dg_m_grouped_bf16_gemm_nt_masked(_bf16(m.a), _bf16(m.b),
                                        torch.empty(m.d_shape(), dtype=torch.bfloat16), _t(m.masked_m))
    assert _ints(fake.calls[-1][1]) == [2, 8, 136, 64]

    x = W.make_activations(130, 640, seed=9)
    ld = W.tma_aligned(130)
    q = torch.empty((130, 640), dtype=torch.uint8)
    sfa = torch.empty((5, ld), dtype=torch.float32)
    dg.dg_per_token_cast_to_fp8(x.x_bf16(), q, sfa)
    assert _ints(fake.calls[-1][1]) == [ld, 130, 640]
    with pytest.raises(ValueError, match="sfa"):
        dg.dg_per_token_cast_to_fp8(x.x_bf16(), q, sfa[:4])

    xm = W.make_activations_masked([3, 0], 8, 256, seed=10)
    qm = torch.empty((2, 8, 256), dtype=torch.uint8)
    sm = torch.empty((2, 2, xm.ld_sfa), dtype=torch.float32)
    dg.dg_per_token_cast_to_fp8_masked(xm.x_bf16(), qm, sm, _t(xm.masked_m))
    assert _ints(fake.calls[-1][1]) == [xm.ld_sfa, 2, 8, 256]
    with pytest.raises(ValueError, match="masked_m"):
        dg.dg_per_token_cast_to_fp8_masked(xm.x_bf16(), qm, sm, _t(xm.masked_m[:1]))


@pytest.mark.parametrize("what", ["d_rows", "d_cols", "sfa_blocks", "sfb_blocks", "b_k"])
def test_dense_mismatches_are_refused(fake, what):
    p = W.make_dense(64, 256, 512, seed=11)
    a, sfa, b, sfb = _t(p.a), _t(p.sfa), _t(p.b[0]), _t(p.sfb[0])
    d = torch.empty((64, 256), dtype=torch.bfloat16)
    if what == "d_rows":
        d = d[:63]
    elif what == "d_cols":
        d = torch.empty((64, 128), dtype=torch.bfloat16)
    elif what == "sfa_blocks":
        sfa = sfa[:3]
    elif what == "sfb_blocks":
        sfb = sfb[:1]
    else:
        b = b[:, :384].contiguous()
    with pytest.raises(ValueError):
        dg.dg_fp8_gemm_nt(a, sfa, b, sfb, d)
    assert not fake.calls, "a mismatched call reached the C library"


def test_grouped_mismatches_are_refused(fake):
    m = W.make_masked([5, 0, 64], 64, 256, 384, seed=12)
    args = [_t(m.a), _t(m.sfa), _t(m.b), _t(m.sfb), torch.empty(m.d_shape(), dtype=torch.bfloat16),
            _t(m.masked_m)]
    for i, bad in ((4, torch.empty((3, 63, 256), dtype=torch.bfloat16)),   # d rows < Mmax
                   (3, _t(m.sfb[:2])),                                        # sfb of 2 groups
                   (1, _t(m.sfa[:, :2]))):                                    # sfa of 2 K-blocks
        call = list(args)
        call[i] = bad
        with pytest.raises(ValueError):
            dg.dg_m_grouped_fp8_gemm_nt_masked(*call)
    c = W.make_contiguous([130, 7], 256, 256, seed=13)
    with pytest.raises(ValueError, match="m_indices"):
        dg.dg_m_grouped_fp8_gemm_nt_contiguous(_t(c.a), _t(c.sfa), _t(c.b), _t(c.sfb),
                                               torch.empty(c.d_shape(), dtype=torch.bfloat16),
                                               _t(c.m_indices[:128]))
    assert not fake.calls


def test_tensors_on_two_devices_are_refused(fake):
    class T:
        def __init__(self, dev):
            self.device = torch.device(dev)
    with pytest.raises(ValueError, match="one CUDA device"):
        dg._call("x", lambda *a: 0, (T("cuda:0"), T("cuda:1")), None)
    with pytest.raises(ValueError, match="current device"):       # the fixture's current device is 1
        dg._call("x", lambda *a: 0, (T("cuda:0"), T("cuda:0")), None)
    dg._call("x", lambda *a: 0, (T("cuda:1"), T("cuda:1")), None)

"""The fused expert FFN entry point that allocates nothing
(dg_m_grouped_fp8_ffn_contiguous_noalloc), called through the C ABI.

Some callers cannot allocate device memory where they run the FFN: a plugin
inside another runtime's execution step (that runtime owns the device memory),
a serving loop that freezes its memory after warm-up, a plain C program with no
device allocator.  This entry point keeps the FFN's intermediate codes and
scales in the library's fixed device array instead of caller buffers.  The
test checks it against the existing entry point (caller-allocated
intermediate) on two calls in a row, within the GEMM tolerance, and that a call
too large for the array is refused.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_grouped_gemm_fp32_b200 as dg
import workloads as W
from gpu_util import compare, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

SCRATCH_BYTES = 16 * 1024 * 1024     # DG_NOALLOC_SCRATCH_BYTES in include/dg.h


@pytest.fixture(autouse=True, scope="module")
def _clean_status():
    from moe_grouped_gemm_fp32_b200 import build
    build.build()
    dg.dg_get_device_status(clear=True)
    yield
    assert dg.dg_get_device_status(clear=True) == 0, "a kernel recorded an error"


def _device(prob):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return {"a": t(prob.a), "sfa": t(prob.sfa), "w1": t(prob.w1), "sfb1": t(prob.sfb1), "w2": t(prob.w2),
            "sfb2": t(prob.sfb2), "mi": t(prob.m_indices)}


def _with_caller_buffers(prob, dv):
    q = torch.empty((prob.M, prob.I), dtype=torch.uint8, device="cuda")
    s = torch.empty((prob.I // 128, prob.ld_sfa), dtype=torch.float32, device="cuda")
    y = torch.empty((prob.M, prob.H), dtype=torch.bfloat16, device="cuda")
    dg.dg_m_grouped_fp8_ffn_contiguous(dv["a"], dv["sfa"], dv["w1"], dv["sfb1"], dv["w2"], dv["sfb2"],
                                       q, s, y, dv["mi"])
    torch.cuda.synchronize()
    return to_f64(y)


def _no_alloc_c_call(prob, dv, y):
    """The C entry point called directly with raw device pointers."""
    L = dg.lib()
    st = L.dg_m_grouped_fp8_ffn_contiguous_noalloc(
        dv["a"].data_ptr(), dv["sfa"].data_ptr(), prob.ld_sfa, dv["w1"].data_ptr(), dv["sfb1"].data_ptr(),
        dv["w2"].data_ptr(), dv["sfb2"].data_ptr(), y.data_ptr(), dv["mi"].data_ptr(),
        prob.M, prob.H, prob.I, prob.G, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def test_no_alloc_ffn_matches_the_caller_buffer_entry_point_on_two_calls_in_a_row():
    # two different problems (group counts, sizes), the second call reusing the
    # array the first one left behind
    probs = [W.make_ffn_contiguous([130, 0, 200, 5], 512, 256, seed=11),
             W.make_ffn_contiguous([300, 77], 1024, 512, seed=12)]
    devs = [_device(p) for p in probs]
    refs = [_with_caller_buffers(p, dv) for p, dv in zip(probs, devs)]
    ys = [torch.full((p.M, p.H), float("nan"), dtype=torch.bfloat16, device="cuda") for p in probs]
    for p, dv, y in zip(probs, devs, ys):
        assert _no_alloc_c_call(p, dv, y) == 0
    torch.cuda.synchronize()
    for p, y, ref in zip(probs, ys, refs):
        rows = np.flatnonzero(p.m_indices >= 0)
        got = to_f64(y)
        compare(got[rows], ref[rows], np.ones((len(rows), p.H), bool))


def test_no_alloc_ffn_refuses_a_call_larger_than_its_array():
    # 8192 tokens x I = 2048 need 16 MiB of codes plus the scales: one block too many
    M, H, I, G = 8192, 256, 2048, 1
    need = M * I + (I // 128) * M * 4
    assert need > SCRATCH_BYTES
    a = torch.zeros((M, H), dtype=torch.uint8, device="cuda")
    y = torch.zeros((M, H), dtype=torch.bfloat16, device="cuda")
    L = dg.lib()
    st = L.dg_m_grouped_fp8_ffn_contiguous_noalloc(a.data_ptr(), a.data_ptr(), M, a.data_ptr(), a.data_ptr(),
                                                   a.data_ptr(), a.data_ptr(), y.data_ptr(), a.data_ptr(),
                                                   M, H, I, G, None)
    assert st == 3                              # DG_ERR_UNSUPPORTED_SHAPE, nothing launched
    assert int(y.view(torch.int16).abs().sum()) == 0

"""Host-only checks of the C ABI (no GPU needed): the shared library loads,
exports every function include/dg.h declares, the helpers return the
documented values, and invalid arguments are rejected before any CUDA call."""
import ctypes
import subprocess

import pytest

import moe_grouped_gemm_fp32_b200 as dg
from moe_grouped_gemm_fp32_b200 import build as dg_build


@pytest.fixture(scope="module")
def L():
    dg_build.build()
    return dg.lib()


def test_header_declares_the_three_gemms_and_helpers():
    names = dg.exported_names()
    for n in ("dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous",
              "dg_m_grouped_fp8_gemm_nt_masked", "dg_get_m_alignment_for_contiguous_layout",
              "dg_get_tma_aligned_size", "dg_get_device_status", "dg_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", dg.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in dg.exported_names():
        assert n in exported, n
        assert hasattr(L, n)
    # nothing else with the library prefix leaks out
    assert {e for e in exported if e.startswith("dg_")} == set(dg.exported_names())


def test_helpers(L):
    assert dg.dg_get_m_alignment_for_contiguous_layout() == 128
    assert dg.dg_get_tma_aligned_size(1, 4) == 4
    assert dg.dg_get_tma_aligned_size(64, 4) == 64
    assert dg.dg_get_tma_aligned_size(65, 4) == 68
    assert dg.dg_get_tma_aligned_size(17, 1) == 32
    assert dg.dg_get_tma_aligned_size(3, 2) == 8
    assert dg.dg_get_tma_aligned_size(5, 3) == 0
    assert dg.dg_status_string(6) == "a kernel wait timed out"
    assert dg.dg_status_string(0) == "success"


FAKE = 0x10000   # a 16-byte aligned non-null address; never dereferenced on these paths


def _dense(L, **kw):
    args = dict(a=FAKE, sfa=FAKE, ld=64, b=FAKE, sfb=FAKE, d=FAKE, M=64, N=256, K=512)
    args.update(kw)
    return L.dg_fp8_gemm_nt(args["a"], args["sfa"], args["ld"], args["b"], args["sfb"],
                            args["d"], args["M"], args["N"], args["K"], None)


def test_dense_validation(L):
    assert _dense(L, a=None) == 1
    assert _dense(L, d=None) == 1
    assert _dense(L, M=-1) == 1
    assert _dense(L, K=100) == 3
    assert _dense(L, K=0) == 1
    assert _dense(L, N=200) == 3
    assert _dense(L, ld=32) == 1            # ld_sfa < M
    assert _dense(L, ld=66) == 2            # ld_sfa not a multiple of 4
    assert _dense(L, a=FAKE + 8) == 2
    assert _dense(L, sfb=FAKE + 4) == 2
    # valid arguments on a host without a usable B200: refused as an unsupported device
    assert _dense(L) in (4,)


def test_grouped_validation(L):
    c = L.dg_m_grouped_fp8_gemm_nt_contiguous
    assert c(FAKE, FAKE, 256, FAKE, FAKE, FAKE, None, 256, 256, 512, 4, None) == 1   # m_indices
    assert c(FAKE, FAKE, 256, FAKE, FAKE, FAKE, FAKE, 200, 256, 512, 4, None) == 3   # M_total % 128
    assert c(FAKE, FAKE, 256, FAKE, FAKE, FAKE, FAKE, 256, 256, 512, 0, None) == 1   # G
    m = L.dg_m_grouped_fp8_gemm_nt_masked
    assert m(FAKE, FAKE, 256, FAKE, FAKE, FAKE, None, 4, 256, 256, 512, None) == 1   # masked_m
    assert m(FAKE, FAKE, 256, FAKE, FAKE, FAKE, FAKE, 2000, 256, 256, 512, None) == 3  # G > 1024
    assert m(FAKE, FAKE, 128, FAKE, FAKE, FAKE, FAKE, 4, 256, 256, 512, None) == 1   # ld < Mmax
    assert m(FAKE, FAKE, 256, FAKE, FAKE, FAKE, FAKE, 4, 256, 256, 384, None) == 4   # no device
    big = 1 << 21                                                                      # G * rows = 2^31
    assert m(FAKE, FAKE, big, FAKE, FAKE, FAKE, FAKE, 1024, big, 256, 512, None) == 3
    k = L.dg_k_grouped_fp8_gemm_nt_contiguous
    assert k(FAKE, FAKE, big, FAKE, FAKE, FAKE, FAKE, 1024, big, 256, 512, None) == 3
    assert L.dg_m_grouped_bf16_gemm_nt_masked(FAKE, FAKE, FAKE, FAKE, 1024, big, 256, 512, None) == 3


def test_no_alloc_ffn_refuses_before_any_device_work(L):
    """The fused FFN without allocation checks its fixed array's limit (16 MiB:
    codes M_total * I, 256-byte rounded, plus (I / 128) scale rows of M_total
    rounded to 4 floats) and its shape rules before touching a device."""
    f = L.dg_m_grouped_fp8_ffn_contiguous_noalloc
    args = lambda M, H, I, G: (FAKE, FAKE, max(M, 4), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, M, H, I, G, None)
    assert f(*args(-1, 256, 256, 1)) == 1                 # negative M_total
    assert f(*args(128, 256, 200, 1)) == 3                # I not a multiple of 128
    assert f(*args(8192, 256, 2048, 1)) == 3              # 16 MiB of codes plus scales: too large
    assert f(*args(7936, 256, 2048, 1)) == 4              # fits (15.5 MiB + 0.5 MiB): no device here
    assert 8192 * 2048 + 16 * 8192 * 4 > dg.NOALLOC_SCRATCH_BYTES >= 7936 * 2048 + 16 * 7936 * 4
    import re
    m = re.search(r"#define DG_NOALLOC_SCRATCH_BYTES \((\d+)u \* 1024u \* 1024u\)", open(dg.HEADER).read())
    assert m and int(m.group(1)) * 1024 * 1024 == dg.NOALLOC_SCRATCH_BYTES


def test_python_binding_rejects_cpu_tensors():
    import torch
    a = torch.zeros((64, 128), dtype=torch.uint8)
    with pytest.raises(TypeError):
        dg.dg_fp8_gemm_nt(a, torch.zeros((1, 64)), torch.zeros((128, 128), dtype=torch.uint8),
                          torch.zeros((1, 1)), torch.zeros((64, 128), dtype=torch.bfloat16))


def test_header_is_plain_c_and_links(tmp_path):
    """include/dg.h compiles as C11 (no C++ in the signatures) and every
    function it declares links against _dg.so."""
    dg_build.build()
    names = dg.exported_names()
    src = tmp_path / "use_dg.c"
    body = "\n".join(f"    (void)&{n};" for n in names)
    src.write_text('#include "dg.h"\nint main(void) {\n' + body + "\n    return 0;\n}\n")
    import os
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    lib_dir = os.path.dirname(dg.LIB_PATH)
    exe = tmp_path / "use_dg"
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe),
                        os.path.join(lib_dir, "_dg.so"), "-Wl,-rpath," + lib_dir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

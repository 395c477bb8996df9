"""Host-side checks of the C-ABI library (CPU only, no kernel launches).

The library must load, export every function include/mxq.h declares, compute
sizes the way the oracle's layout does, reject bad arguments before touching
the GPU, and pick the same path as the selective-quantisation rule.
"""

import ctypes
import os
import re

import pytest
import torch

import fp8_gemm_diffusion_b200 as mxq
import workloads
from oracle import dispatch as D
from oracle import quant as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "mxq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mxq_[a-z0-9_]+)\s*\(", src)))


def test_header_symbols_exported():
    declared = _declared_functions()
    assert len(declared) >= 15
    lib = ctypes.CDLL(mxq.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(mxq.EXPORTED) == declared


def test_version_and_status_strings():
    assert mxq.version() >> 16 == 1
    for s in range(8):
        assert mxq.status_string(s)
    assert mxq.status_string(99) == "unknown status"


@pytest.mark.parametrize("rows,k", [(1, 64), (130, 128), (4608, 3072), (0, 64), (257, 12288)])
def test_sizes_match_oracle_layout(rows, k):
    assert mxq.sf_bytes(rows, k, "nvfp4") == Q.sf_bytes(rows, k, 16)
    assert mxq.sf_bytes(rows, k, "mxfp8") == Q.sf_bytes(rows, k, 32)
    assert mxq.codes_bytes(rows, k, "nvfp4") == rows * k // 2
    assert mxq.codes_bytes(rows, k, "mxfp8") == rows * k
    assert mxq.sf_bytes(rows, k, "bf16") == 0
    ws = mxq.linear_workspace_bytes(rows, k, "nvfp4")
    assert ws >= 256 + rows * k // 2 + Q.sf_bytes(rows, k, 16) and ws % 256 == 0


A16 = 1 << 20  # a 16-byte aligned fake device address (never dereferenced)


def _st(fn, *a):
    try:
        fn(*a)
    except mxq.MxqError as e:
        return e.status
    return mxq.OK


def test_quantize_rejects_bad_arguments():
    q = lambda *a, **kw: mxq.quantize_nvfp4(*a, **kw)
    assert _st(q, None, A16, A16, A16, A16, 4, 64, 64) == mxq.ERR_INVALID_ARG
    assert _st(q, A16, A16, A16, A16, None, 4, 64, 64) == mxq.ERR_INVALID_ARG  # g_out
    if not torch.cuda.is_available():
        # a NULL amax selects g = 1 (no per-tensor scale): past the argument
        # checks, stopped only by the missing device
        assert _st(q, A16, None, A16, A16, A16, 4, 64, 64) == mxq.ERR_ARCH
    assert _st(q, A16 + 2, A16, A16, A16, A16, 4, 64, 64) == mxq.ERR_ALIGNMENT
    assert _st(q, A16, A16, A16 + 8, A16, A16, 4, 64, 64) == mxq.ERR_ALIGNMENT
    assert _st(q, A16, A16, A16, A16, A16, 4, 48, 48) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(q, A16, A16, A16, A16, A16, 4, 64, 60) == mxq.ERR_INVALID_ARG  # ld < k
    assert _st(q, A16, A16, A16, A16, A16, 4, 64, 68) == mxq.ERR_ALIGNMENT  # ld % 8
    assert _st(q, A16, A16, A16, A16, A16, -1, 64, 64) == mxq.ERR_INVALID_ARG
    m = lambda *a, **kw: mxq.quantize_mxfp8(*a, **kw)
    assert _st(m, A16, A16, A16, 4, 64, 64) == mxq.ERR_UNSUPPORTED_SHAPE  # k % 128
    assert _st(m, A16, None, A16, 4, 128, 128) == mxq.ERR_INVALID_ARG


def test_gemm_rejects_bad_arguments():
    g = lambda *a: mxq.gemm_blockscaled(*a)
    ok = ("nvfp4", 128, 128, 256, A16, A16, A16, A16, A16, A16, None, A16, 128)
    assert _st(g, 9, *ok[1:]) == mxq.ERR_INVALID_ARG
    assert _st(g, "nvfp4", 128, 128, 96, *ok[4:]) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(g, "mxfp8", 128, 128, 192, *ok[4:]) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(g, "nvfp4", 128, 128, 0, *ok[4:]) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(g, *ok[:4], None, *ok[5:]) == mxq.ERR_INVALID_ARG
    assert _st(g, *ok[:6], None, *ok[7:]) == mxq.ERR_INVALID_ARG  # NVFP4 needs g_A
    assert _st(g, *ok[:11], A16 + 16, 120) == mxq.ERR_INVALID_ARG  # ldy < N
    assert _st(g, *ok[:11], A16, 132) == mxq.ERR_ALIGNMENT
    assert _st(g, *ok[:11], A16 + 4, 128) == mxq.ERR_ALIGNMENT
    assert _st(g, "bf16", 128, 128, 12, A16, None, None, A16, None, None, None, A16, 128) \
        == mxq.ERR_UNSUPPORTED_SHAPE


def test_workspace_and_storage_checks():
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=4096, K=4096, w_bf16=A16, bias_bf16=None,
                       codes=A16, sf=A16, g_dev=A16, amax_dev=A16)
    need = mxq.linear_workspace_bytes(4096, 4096, "nvfp4")
    assert _st(mxq.linear, w, A16, 4096, A16, A16, need - 1) == mxq.ERR_WORKSPACE
    assert _st(mxq.linear, w, A16, 4096, A16, A16 + 16, need) == mxq.ERR_ALIGNMENT
    assert _st(mxq.linear, w, A16, 4096, A16, None, need) == mxq.ERR_INVALID_ARG
    need_w = mxq.weight_storage_bytes(4096, 4096, "mxfp8")
    assert _st(mxq.weight_prepare, "mxfp8", A16, 4096, 4096, None, 0, A16, need_w - 1) \
        == mxq.ERR_WORKSPACE
    assert _st(mxq.weight_prepare, "mxfp8", A16, 4096, 4000, None, 0, A16, 1 << 30) \
        == mxq.ERR_UNSUPPORTED_SHAPE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_fails_loudly():
    # no CPU fallback: a well-formed call on a machine without an sm_100 GPU
    # returns MXQ_ERR_ARCH and computes nothing
    assert _st(mxq.quantize_mxfp8, A16, A16, A16, 4, 128, 128) == mxq.ERR_ARCH
    assert _st(mxq.gemm_blockscaled, "bf16", 8, 8, 64, A16, None, None, A16, None, None, None,
               A16, 8) == mxq.ERR_ARCH
    assert mxq.get_device_error() == mxq.ERR_ARCH


def test_linear_path_follows_selection_rule():
    for B in (1, 4):
        for l in workloads.flux_linear_stack(batch=B):
            w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=l["N"], K=l["K"])
            want = mxq.BF16 if D.use_bf16(l["M"], l["K"], l["N"]) else mxq.NVFP4
            assert mxq.linear_path(w, l["M"]) == want, l
    w = mxq.mxq_weight(format=mxq.MXFP8, flags=0, N=1024, K=1024)
    assert mxq.linear_path(w, 1024) == mxq.MXFP8
    assert mxq.linear_path(w, 1023) == mxq.BF16
    assert mxq.linear_path(w, 1024, min_dim=2048) == mxq.BF16
    w.flags = mxq.WEIGHT_KEEP_BF16
    assert mxq.linear_path(w, 8192) == mxq.BF16


def test_linear_kernel_count_host_cases():
    w = mxq.mxq_weight(format=mxq.MXFP8, flags=0, N=1024, K=1024)
    assert mxq.linear_kernel_count(w, 0) == 0            # nothing launched
    assert mxq.linear_kernel_count(w, 1023) == 1         # bf16 GEMM
    assert mxq.linear_kernel_count(w, 1024) == 2         # MXFP8 quantise + GEMM
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=0, K=1024)
    assert mxq.linear_kernel_count(w, 4096) == 0
    if not torch.cuda.is_available():
        # the NVFP4 choice (one or two quantiser kernels) depends on the SM count
        w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=1024, K=1024)
        assert mxq.linear_kernel_count(w, 4096) == -1


def test_no_tensor_scale_weight_host_cases():
    # NVFP4 without a per-tensor scale: no amax pass, one quantiser + the GEMM,
    # decided without querying the device
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=mxq.WEIGHT_NO_TENSOR_SCALE, N=1024, K=1024)
    assert mxq.linear_path(w, 4096) == mxq.NVFP4
    assert mxq.linear_kernel_count(w, 4096) == 2
    assert mxq.linear_kernel_count(w, 1023) == 1         # still bf16 below the threshold
    w.flags |= mxq.WEIGHT_KEEP_BF16
    assert mxq.linear_path(w, 4096) == mxq.BF16


def test_weight_prepare_rejects_bad_flags():
    out = mxq.mxq_weight()
    # unknown bits, and the no-tensor-scale bit on a format without a per-tensor scale
    for fmt, flags in ((mxq.NVFP4, 4), (mxq.NVFP4, 1 << 20), (mxq.MXFP8, mxq.WEIGHT_NO_TENSOR_SCALE),
                       (mxq.BF16, mxq.WEIGHT_NO_TENSOR_SCALE)):
        st = mxq._weight_prepare(fmt, A16, 1024, 1024, None, flags, None, 0, mxq.ctypes.byref(out), None)
        assert st == mxq.ERR_INVALID_ARG, (fmt, flags, st)


class _FakeEvent:
    """Stands in for a torch.cuda.Event: only its handle is passed (never used)."""

    def __init__(self, handle):
        self.cuda_event = handle


def test_linear_rejects_half_an_event_pair():
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=4096, K=4096, w_bf16=A16, bias_bf16=None,
                       codes=A16, sf=A16, g_dev=A16, amax_dev=A16)
    need = mxq.linear_workspace_bytes(4096, 4096, "nvfp4")
    half = (_FakeEvent(0x1000), _FakeEvent(0))
    assert _st(mxq.linear, w, A16, 4096, A16, A16, need, None, None, half) == mxq.ERR_INVALID_ARG


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of mxq_weight and mxq_linear_opts have the C header's
    size and field offsets (a mismatch would hand the library shifted fields)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    fields = {"mxq_weight": [f[0] for f in mxq.mxq_weight._fields_],
              "mxq_linear_opts": [f[0] for f in mxq.mxq_linear_opts._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "mxq.h"', "int main(void) {"]
    for st, names in fields.items():
        lines.append(f'  printf("{st} size %zu\\n", sizeof({st}));')
        for n in names:
            lines.append(f'  printf("{st} {n} %zu\\n", offsetof({st}, {n}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(root, "include"), str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for st, cls in (("mxq_weight", mxq.mxq_weight), ("mxq_linear_opts", mxq.mxq_linear_opts)):
        assert got[(st, "size")] == ctypes.sizeof(cls), st
        for n in fields[st]:
            assert got[(st, n)] == getattr(cls, n).offset, (st, n)

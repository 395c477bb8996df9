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


_KEEP = []


def dev(nbytes: int, misalign: int = 0) -> int:
    """A device address for a buffer of `nbytes` (plus `misalign` bytes of offset).

    On a machine with a GPU this is a real allocation of that size, so that a
    call which got past its host checks by mistake could only touch valid
    memory.  Without a GPU every call returns before any launch, and a fixed
    256-byte aligned address stands in (nothing dereferences it there)."""
    if torch.cuda.is_available():
        t = torch.zeros(int(nbytes) + 256, dtype=torch.uint8, device="cuda")
        _KEEP.append(t)
        return t.data_ptr() + misalign
    return (1 << 20) + misalign


SMALL = 1 << 16  # covers every buffer of the small shapes below (4 x 64, 128 x 128 x 256)


def _st(fn, *a):
    try:
        fn(*a)
    except mxq.MxqError as e:
        return e.status
    return mxq.OK


def test_quantize_rejects_bad_arguments():
    q = lambda *a, **kw: mxq.quantize_nvfp4(*a, **kw)
    assert _st(q, None, dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), 4, 64, 64) == mxq.ERR_INVALID_ARG
    assert _st(q, dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), None, 4, 64, 64) == mxq.ERR_INVALID_ARG  # g_out
    if not torch.cuda.is_available():
        # a NULL amax selects g = 1 (no per-tensor scale): past the argument
        # checks, stopped only by the missing device
        assert _st(q, dev(SMALL), None, dev(SMALL), dev(SMALL), dev(SMALL), 4, 64, 64) == mxq.ERR_ARCH
    assert _st(q, dev(SMALL, 2), dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), 4, 64, 64) == mxq.ERR_ALIGNMENT
    assert _st(q, dev(SMALL), dev(SMALL), dev(SMALL, 8), dev(SMALL), dev(SMALL), 4, 64, 64) == mxq.ERR_ALIGNMENT
    assert _st(q, dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), 4, 48, 48) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(q, dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), 4, 64, 60) == mxq.ERR_INVALID_ARG  # ld < k
    assert _st(q, dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), 4, 64, 68) == mxq.ERR_ALIGNMENT  # ld % 8
    assert _st(q, dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), -1, 64, 64) == mxq.ERR_INVALID_ARG
    m = lambda *a, **kw: mxq.quantize_mxfp8(*a, **kw)
    assert _st(m, dev(SMALL), dev(SMALL), dev(SMALL), 4, 64, 64) == mxq.ERR_UNSUPPORTED_SHAPE  # k % 128
    assert _st(m, dev(SMALL), None, dev(SMALL), 4, 128, 128) == mxq.ERR_INVALID_ARG


def test_gemm_rejects_bad_arguments():
    g = lambda *a: mxq.gemm_blockscaled(*a)
    ok = ("nvfp4", 128, 128, 256, dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), dev(SMALL), None, dev(SMALL), 128)
    assert _st(g, 9, *ok[1:]) == mxq.ERR_INVALID_ARG
    assert _st(g, "nvfp4", 128, 128, 96, *ok[4:]) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(g, "mxfp8", 128, 128, 192, *ok[4:]) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(g, "nvfp4", 128, 128, 0, *ok[4:]) == mxq.ERR_UNSUPPORTED_SHAPE
    assert _st(g, *ok[:4], None, *ok[5:]) == mxq.ERR_INVALID_ARG
    assert _st(g, *ok[:6], None, *ok[7:]) == mxq.ERR_INVALID_ARG  # NVFP4 needs g_A
    assert _st(g, *ok[:11], dev(SMALL, 16), 120) == mxq.ERR_INVALID_ARG  # ldy < N
    assert _st(g, *ok[:11], dev(SMALL), 132) == mxq.ERR_ALIGNMENT
    assert _st(g, *ok[:11], dev(SMALL, 4), 128) == mxq.ERR_ALIGNMENT
    assert _st(g, "bf16", 128, 128, 12, dev(SMALL), None, None, dev(SMALL), None, None, None, dev(SMALL), 128) \
        == mxq.ERR_UNSUPPORTED_SHAPE


def test_workspace_and_storage_checks():
    N = K = M = 4096
    need = mxq.linear_workspace_bytes(M, K, "nvfp4")
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=N, K=K, w_bf16=dev(N * K * 2), bias_bf16=None,
                       codes=dev(N * K // 2), sf=dev(mxq.sf_bytes(N, K, "nvfp4")), g_dev=dev(4),
                       amax_dev=dev(4))
    x, y, ws = dev(M * K * 2), dev(M * N * 2), dev(need + 16)
    assert _st(mxq.linear, w, x, M, y, ws, need - 1) == mxq.ERR_WORKSPACE
    assert _st(mxq.linear, w, x, M, y, ws + 16, need) == mxq.ERR_ALIGNMENT
    assert _st(mxq.linear, w, x, M, y, None, need) == mxq.ERR_INVALID_ARG
    need_w = mxq.weight_storage_bytes(N, K, "mxfp8")
    storage = dev(need_w)
    assert _st(mxq.weight_prepare, "mxfp8", w.w_bf16, N, K, None, 0, storage, need_w - 1) \
        == mxq.ERR_WORKSPACE
    assert _st(mxq.weight_prepare, "mxfp8", w.w_bf16, N, 4000, None, 0, storage, need_w) \
        == mxq.ERR_UNSUPPORTED_SHAPE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_fails_loudly():
    # no CPU fallback: a well-formed call on a machine without an sm_100 GPU
    # returns MXQ_ERR_ARCH and computes nothing
    assert _st(mxq.quantize_mxfp8, dev(SMALL), dev(SMALL), dev(SMALL), 4, 128, 128) == mxq.ERR_ARCH
    assert _st(mxq.gemm_blockscaled, "bf16", 8, 8, 64, dev(SMALL), None, None, dev(SMALL), None, None, None,
               dev(SMALL), 8) == mxq.ERR_ARCH
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
    w16 = dev(1024 * 1024 * 2)
    # unknown bits, and the no-tensor-scale bit on a format without a per-tensor scale
    for fmt, flags in ((mxq.NVFP4, 4), (mxq.NVFP4, 1 << 20), (mxq.MXFP8, mxq.WEIGHT_NO_TENSOR_SCALE),
                       (mxq.BF16, mxq.WEIGHT_NO_TENSOR_SCALE)):
        st = mxq._weight_prepare(fmt, w16, 1024, 1024, None, flags, None, 0, mxq.ctypes.byref(out), None)
        assert st == mxq.ERR_INVALID_ARG, (fmt, flags, st)


class _FakeEvent:
    """Stands in for a torch.cuda.Event: only its handle is passed (never used)."""

    def __init__(self, handle):
        self.cuda_event = handle


def test_linear_rejects_half_an_event_pair():
    N = K = M = 4096
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=N, K=K, w_bf16=dev(N * K * 2), bias_bf16=None,
                       codes=dev(N * K // 2), sf=dev(mxq.sf_bytes(N, K, "nvfp4")), g_dev=dev(4),
                       amax_dev=dev(4))
    need = mxq.linear_workspace_bytes(M, K, "nvfp4")
    if torch.cuda.is_available():
        real = torch.cuda.Event(enable_timing=True)
        real.record()  # torch creates the event's handle on its first record
        half = (real, _FakeEvent(0))
    else:
        half = (_FakeEvent(0x1000), _FakeEvent(0))
    assert _st(mxq.linear, w, dev(M * K * 2), M, dev(M * N * 2), dev(need), need, None, None, half) \
        == mxq.ERR_INVALID_ARG


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


def test_producer_and_known_amax_options_are_checked_on_the_host():
    N = K = M = 1024
    need = mxq.linear_workspace_bytes(M, K, "nvfp4")
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=N, K=K, w_bf16=dev(N * K * 2), bias_bf16=None,
                       codes=dev(N * K // 2), sf=dev(mxq.sf_bytes(N, K, "nvfp4")), g_dev=dev(4),
                       amax_dev=dev(4))
    x, y, ws, f4 = dev(M * K * 2), dev(M * N * 2), dev(need), dev(16)

    def call(M_=M, **kw):
        return mxq._linear(mxq.ctypes.byref(w), x, M_, y, ws, need, mxq._opts(None, **kw), mxq._stream(None))

    assert call(activation=7) == mxq.ERR_INVALID_ARG
    assert call(y_amax=f4 + 2) == mxq.ERR_ALIGNMENT
    assert call(x_amax=f4 + 1) == mxq.ERR_ALIGNMENT
    assert call(y_amax=f4, x_amax=f4) == mxq.ERR_INVALID_ARG            # must not alias
    assert call(M_=128, activation=mxq.ACT_GELU) == mxq.ERR_UNSUPPORTED_SHAPE   # single-CTA GEMM
    assert call(M_=64, y_amax=f4) == mxq.ERR_UNSUPPORTED_SHAPE
    # a known amax removes the amax pass: quantiser + GEMM
    assert mxq.linear_kernel_count(w, 4096, x_amax=f4) == 2
    if not torch.cuda.is_available():
        assert call(activation=mxq.ACT_GELU, y_amax=f4) == mxq.ERR_ARCH  # past every argument check


def test_rceil_flag_and_scale_rule_checks():
    out = mxq.mxq_weight()
    w16 = dev(1024 * 1024 * 2)
    for fmt in (mxq.NVFP4, mxq.BF16):
        st = mxq._weight_prepare(fmt, w16, 1024, 1024, None, mxq.WEIGHT_MXFP8_RCEIL, None, 0,
                                 mxq.ctypes.byref(out), None)
        assert st == mxq.ERR_INVALID_ARG, fmt
    assert _st(mxq.quantize_mxfp8, dev(SMALL), dev(SMALL), dev(SMALL), 4, 128, 128, None, 2) \
        == mxq.ERR_INVALID_ARG
    if not torch.cuda.is_available():
        assert _st(mxq.quantize_mxfp8, dev(SMALL), dev(SMALL), dev(SMALL), 4, 128, 128, None,
                   mxq.SCALE_RCEIL) == mxq.ERR_ARCH


def test_attention_arguments_are_checked_on_the_host():
    H, T, d = 2, 256, 128
    need = mxq.attention_workspace_bytes(H, T, d)
    assert need >= 3 * H * T * d and need % 256 == 0
    assert mxq.attention_workspace_bytes(H, T, 64) == 0 and mxq.attention_workspace_bytes(0, T, d) == 0
    q, k, v, o = (dev(H * T * d * 2) for _ in range(4))
    ws = dev(need)

    def call(H_=H, T_=T, d_=d, ws_=ws, nbytes=need, q_=q):
        return mxq._attention_mxfp8(q_, k, v, H_, T_, d_, 0.0, o, ws_, nbytes, None)

    assert call(d_=64) == mxq.ERR_UNSUPPORTED_SHAPE
    assert call(T_=200) == mxq.ERR_UNSUPPORTED_SHAPE       # tokens % 128
    assert call(H_=-1) == mxq.ERR_INVALID_ARG
    assert call(nbytes=need - 1) == mxq.ERR_WORKSPACE
    assert call(ws_=ws + 16) == mxq.ERR_ALIGNMENT
    assert call(q_=q + 2) == mxq.ERR_ALIGNMENT
    assert call(q_=None) == mxq.ERR_INVALID_ARG
    assert call(H_=0) == mxq.OK                              # nothing to do
    if not torch.cuda.is_available():
        assert call() == mxq.ERR_ARCH                        # past every argument check

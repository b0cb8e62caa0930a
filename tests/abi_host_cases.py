"""Host-side argument validation of every C-ABI call, with fake device
addresses (a helper module, run by tests/test_abi_cpu.py in a child process).

Each call is made with one bad argument at a time and must return the status
for it; with all arguments valid it must stop at the device check.  The
addresses below are never valid device memory, so this module refuses to run
unless the process sees no CUDA device at all: CUDA_VISIBLE_DEVICES must be
set and empty, and the library must report no device before the first call.
"""
import ctypes
import os
import sys

import pytest

if os.environ.get("CUDA_VISIBLE_DEVICES", None) != "":
    raise RuntimeError("abi_host_cases.py runs only with CUDA_VISIBLE_DEVICES='' (no device visible)")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ternary_weight_linear_forward_b200 as bl  # noqa: E402

if bl.lib().bitlinear_num_sms() != 0:
    raise RuntimeError("a CUDA device is visible: refusing to pass fake device addresses")

OK, NULL, SHAPE, ALIGN, DTYPE, WS, DEVICE, CUDA, TIMEOUT, ALIAS = range(10)

# fake, never-dereferenced device addresses: 16-byte aligned and disjoint
A1, A2, A3, A4, A5, A6 = (0x10000000 * i for i in range(1, 7))


def _L():
    return bl.lib()


def P(x):
    return ctypes.c_void_p(x)


def test_forward_validation_order():
    f = _L().bitlinear_forward
    assert f(None, P(A2), 1, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == NULL
    assert f(P(A1), P(A2), 1, 1000, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == SHAPE   # K % 64
    assert f(P(A1), P(A2), 0, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == SHAPE   # M < 1
    assert f(P(A1), P(A2), 1, 1024, P(A3), P(A4), 0, P(A5), 0, None, 0, None) == SHAPE    # N < 1
    assert f(P(A1), P(A2), 1, 2 ** 19, P(A3), P(A4), 8, P(A5), 0, None, 0, None) == SHAPE  # K > max
    assert f(P(A1 + 8), P(A2), 1, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == ALIGN
    assert f(P(A1), P(A2), 1, 1024, P(A3), P(A4), 64, P(A5), 7, None, 0, None) == DTYPE
    assert f(P(A1), P(A2), 1, 1024, P(A3), P(A4), 64, P(A1), 0, None, 0, None) == ALIAS
    # prefill path needs a workspace
    assert _L().bitlinear_forward_workspace(2048, 4096, 4096) >= 2048 * 4
    assert f(P(A1), P(A2), 2048, 1024, P(A3), P(A4), 64, P(A5), 1, None, 0, None) == WS
    # everything valid: without a CUDA device the call stops at the device check
    assert f(P(A1), P(A2), 1, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == DEVICE


def test_forward_acc_validation():
    f = _L().bitlinear_forward_acc
    assert f(None, 1, 1024, P(A3), 64, P(A5), None, 0, None) == NULL
    assert f(P(A1), 1, 1040, P(A3), 64, P(A5), None, 0, None) == SHAPE
    assert f(P(A1), 1, 1024, P(A3), 64, P(A5 + 4), None, 0, None) == ALIGN
    assert f(P(A1), 1, 1024, P(A3), 64, P(A5), None, 0, None) == DEVICE


def test_quantize_weights_validation():
    f = _L().bitlinear_quantize_weights
    ws = _L().bitlinear_quantize_weights_workspace(16, 16)
    assert ws > 0
    assert f(None, 16, 16, 1e-5, P(A2), P(A3), P(A4), ws, None) == NULL
    assert f(P(A1), 16, 8, 1e-5, P(A2), P(A3), P(A4), ws, None) == SHAPE      # K % 16
    assert f(P(A1), 16, 16, -1.0, P(A2), P(A3), P(A4), ws, None) == SHAPE     # eps < 0
    assert f(P(A1), 16, 16, float("nan"), P(A2), P(A3), P(A4), ws, None) == SHAPE
    assert f(P(A1), 16, 16, 1e-5, P(A2), P(A3), P(A4), ws - 1, None) == WS
    assert f(P(A1), 16, 16, 1e-5, P(A2), P(A3), None, 0, None) == WS
    assert f(P(A1), 16, 16, 1e-5, P(A2 + 1), P(A3), P(A4), ws, None) == ALIGN
    assert f(P(A1), 16, 16, 1e-5, P(A1), P(A3), P(A4), ws, None) == ALIAS
    assert f(P(A1), 16, 16, 1e-5, P(A2), P(A3), P(A4), ws, None) == DEVICE


def test_pack_and_quant_act_validation():
    pk = _L().bitlinear_pack
    assert pk(None, 4, 16, P(A2), None) == NULL
    assert pk(P(A1), 4, 24, P(A2), None) == SHAPE
    assert pk(P(A1), 4, 16, P(A2 + 4), None) == ALIGN
    assert pk(P(A1), 4, 16, P(A1), None) == ALIAS
    assert pk(P(A1), 4, 16, P(A2), None) == DEVICE
    qa = _L().bitlinear_quant_act
    assert qa(P(A1), 0, 1, 1024, None, P(A3), None) == NULL
    assert qa(P(A1), 2, 1, 1024, P(A2), P(A3), None) == DTYPE
    assert qa(P(A1), 1, 1, 1000, P(A2), P(A3), None) == SHAPE
    assert qa(P(A1), 1, 0, 1024, P(A2), P(A3), None) == SHAPE
    assert qa(P(A1 + 2), 1, 1, 1024, P(A2), P(A3), None) == ALIGN
    assert qa(P(A1), 0, 1, 1024, P(A1 + 16), P(A3), None) == ALIAS
    assert qa(P(A1), 1, 1, 1024, P(A2), P(A3), None) == DEVICE


def test_quant_act_rms_validation():
    f = _L().bitlinear_quant_act_rms
    assert f(P(A1), None, 9, 1, 64, None, P(A2), P(A3), None) == DTYPE
    assert f(P(A1), None, 1, 1, 64, None, P(A2), P(A3), None) == NULL       # add needs b
    assert f(P(A1), None, 0, 1, 64, None, P(A2), None, None) == NULL        # x_q without gamma
    assert f(P(A1), None, 0, 1, 64, None, None, None, None) == NULL         # nothing to write
    assert f(P(A1), None, 0, 1, 60, None, P(A2), P(A3), None) == SHAPE
    assert f(P(A1), P(A4), 2, 1, 64, P(A4), P(A2), P(A3), None) == ALIAS
    assert f(P(A1), None, 0, 1, 64, None, P(A2), P(A3), None) == DEVICE


def test_device_queries_without_gpu():
    assert _L().bitlinear_num_sms() == 0
    assert _L().bitlinear_device_status(None) == DEVICE


class _Prob(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("W_p", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("y", ctypes.c_void_p), ("K", ctypes.c_int64), ("N", ctypes.c_int64)]


def test_forward_fp_batch_validation():
    f = _L().bitlinear_forward_fp_batch
    arr = (_Prob * 9)()
    for i in range(9):
        arr[i] = _Prob(A1, None, A2, A3, A4 + i * 0x100000, 1024, 64)
    pa = ctypes.cast(arr, ctypes.c_void_p)
    assert f(None, 1, 1, 0, 0, None) == NULL
    assert f(pa, 0, 1, 0, 0, None) == SHAPE
    assert f(pa, 9, 1, 0, 0, None) == SHAPE
    assert f(pa, 2, 5, 0, 0, None) == SHAPE           # M > 4
    assert f(pa, 2, 1, 3, 0, None) == DTYPE
    assert f(pa, 2, 1, 2, 0, None) == NULL            # int8 x needs gamma
    arr[1].y = A4                                      # two outputs overlap
    assert f(pa, 2, 1, 0, 0, None) == ALIAS
    arr[1].y = A4 + 0x100000
    arr[1].K = 1000
    assert f(pa, 2, 1, 0, 0, None) == SHAPE
    arr[1].K = 1024
    assert f(pa, 2, 1, 0, 0, None) == DEVICE


def test_binary_weight_calls_validation():
    f = _L().bitlinear_binarize_weights
    ws = _L().bitlinear_binarize_weights_workspace(16, 32)
    assert ws > 0
    assert f(None, 16, 32, P(A2), P(A3), P(A3 + 16), P(A4), ws, None) == NULL
    assert f(P(A1), 16, 48, P(A2), P(A3), P(A3 + 16), P(A4), ws, None) == SHAPE     # K % 32
    assert f(P(A1), 16, 32, P(A2), P(A3), P(A3 + 16), P(A4), ws - 1, None) == WS
    assert f(P(A1), 16, 32, P(A2), P(A3 + 4), P(A3 + 16), P(A4), ws, None) == ALIGN
    assert f(P(A1), 16, 32, P(A2), P(A3), P(A3), P(A4), ws, None) == ALIAS           # alpha is beta
    assert f(P(A1), 16, 32, P(A1), P(A3), P(A3 + 16), P(A4), ws, None) == ALIAS      # W_b on W
    assert f(P(A1), 16, 32, P(A2), P(A3), P(A3 + 16), P(A2), ws, None) == ALIAS      # ws on W_b
    assert f(P(A1), 16, 32, P(A2), P(A3), P(A3 + 16), P(A4), ws, None) == DEVICE
    pk = _L().bitlinear_pack_bits
    assert pk(None, 4, 32, P(A2), None) == NULL
    assert pk(P(A1), 4, 48, P(A2), None) == SHAPE
    assert pk(P(A1), 4, 32, P(A2 + 4), None) == ALIGN
    assert pk(P(A1), 4, 32, P(A1), None) == ALIAS
    assert pk(P(A1), 4, 32, P(A2), None) == DEVICE


def test_binary_forward_validation():
    f = _L().bitlinear_forward_binary
    assert f(None, P(A2), 1, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == NULL
    assert f(P(A1), P(A2), 1, 1088, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == SHAPE   # K % 128
    assert f(P(A1), P(A2), 0, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == SHAPE
    assert f(P(A1), P(A2), 1, 1024, P(A3 + 8), P(A4), 64, P(A5), 0, None, 0, None) == ALIGN
    assert f(P(A1), P(A2), 1, 1024, P(A3), P(A4), 64, P(A5), 5, None, 0, None) == DTYPE
    assert f(P(A1), P(A2), 1, 1024, P(A3), P(A4), 64, P(A3), 0, None, 0, None) == ALIAS
    # decode shapes need no workspace; the GEMM path (M > 4, or x_hat too large) does
    assert _L().bitlinear_forward_binary_workspace(4, 4096, 4096) == 0
    assert _L().bitlinear_forward_binary_workspace(4, 4096, 32768) >= 16
    assert _L().bitlinear_forward_binary_workspace(2048, 4096, 4096) >= 2048 * 4
    assert f(P(A1), P(A2), 2048, 1024, P(A3), P(A4), 64, P(A5), 1, None, 0, None) == WS
    assert f(P(A1), P(A2), 1, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == DEVICE
    g = _L().bitlinear_forward_binary_acc
    assert g(P(A1), 1, 1088, P(A3), 64, P(A5), None, 0, None) == SHAPE
    assert g(P(A1), 1, 1024, P(A3), 64, P(A5), None, 0, None) == DEVICE
    h = _L().bitlinear_forward_binary_fp
    assert h(P(A1), 3, 1, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == DTYPE
    assert h(P(A1), 0, 1, 1088, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == SHAPE
    assert _L().bitlinear_forward_binary_fp_workspace(1, 4096, 4096) == 0
    need = _L().bitlinear_forward_binary_fp_workspace(64, 4096, 4096)
    assert need >= 64 * 4096 + 64 * 4
    assert h(P(A1), 0, 64, 4096, P(A3), P(A4), 4096, P(A5), 0, P(A6), need - 1, None) == WS
    assert h(P(A1), 0, 1, 1024, P(A3), P(A4), 64, P(A5), 0, None, 0, None) == DEVICE


def test_glu_validation():
    f = _L().bitlinear_glu_forward
    ws = _L().bitlinear_glu_workspace(2, 256, 512)
    assert ws >= 2 * 256 + 2 * 2 * 512 * 4 + 2 * 512
    base = [P(A1), 2, 256, 512, P(A2), P(A3), P(A2 + 0x1000000), P(A3 + 16), P(A4), P(A3 + 32), P(A5), None,
            P(A6), ws, None]

    def call(**kw):
        a = list(base)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)
    assert call(a0=None) == NULL
    assert call(a10=None) == NULL
    assert call(a2=200) == SHAPE            # D % 64
    assert call(a3=520) == SHAPE            # F % 64
    assert call(a1=0) == SHAPE
    assert call(a12=None) == WS
    assert call(a13=ws - 1) == WS
    assert call(a10=P(A5 + 4)) == ALIGN
    assert call(a10=P(A1)) == ALIAS         # y on x
    assert call(a11=P(A5)) == ALIAS         # u on y
    assert call(a12=P(A4)) == ALIAS         # workspace on W_down
    assert call() == DEVICE


def test_grouped_validation():
    assert _L().bitlinear_quantize_weights_grouped_workspace(16, 512, 3) == 0       # K % (64 G)
    assert _L().bitlinear_quantize_weights_grouped_workspace(16, 512, 9) == 0       # G > BL_MAX_GROUPS
    wsq = _L().bitlinear_quantize_weights_grouped_workspace(16, 512, 4)
    assert wsq >= 16 * 512 * 4
    q = _L().bitlinear_quantize_weights_grouped
    assert q(None, 16, 512, 4, 1e-5, P(A2), P(A3), P(A4), wsq, None) == NULL
    assert q(P(A1), 16, 512, 3, 1e-5, P(A2), P(A3), P(A4), wsq, None) == SHAPE
    assert q(P(A1), 16, 512, 0, 1e-5, P(A2), P(A3), P(A4), wsq, None) == SHAPE
    assert q(P(A1), 16, 512, 4, 1e-5, P(A2), P(A3), P(A4), wsq - 1, None) == WS
    assert q(P(A1), 16, 512, 4, 1e-5, P(A2), P(A3 + 4), P(A4), wsq, None) == ALIGN
    assert q(P(A1), 16, 512, 4, 1e-5, P(A2), P(A1 + 16), P(A4), wsq, None) == ALIAS
    assert q(P(A1), 16, 512, 4, 1e-5, P(A2), P(A3), P(A4), wsq, None) == DEVICE
    a = _L().bitlinear_quant_act_grouped
    assert a(P(A1), 1, 2, 512, 4, None, P(A3), None) == NULL
    assert a(P(A1), 2, 2, 512, 4, P(A2), P(A3), None) == DTYPE
    assert a(P(A1), 1, 2, 448, 4, P(A2), P(A3), None) == SHAPE
    assert a(P(A1), 1, 2, 512, 4, P(A2), P(A3), None) == DEVICE
    f = _L().bitlinear_forward_grouped
    ws = _L().bitlinear_forward_grouped_workspace(3, 100, 512, 4)
    assert ws >= 4 * 300 * 4
    assert f(P(A1), P(A2), 3, 512, 4, P(A3), P(A4), 100, P(A5), 0, P(A6), ws, None) == DEVICE
    assert f(P(A1), None, 3, 512, 4, P(A3), P(A4), 100, P(A5), 0, P(A6), ws, None) == NULL
    assert f(P(A1), P(A2), 3, 512, 4, P(A3), P(A4), 100, P(A5), 3, P(A6), ws, None) == DTYPE
    assert f(P(A1), P(A2), 3, 576, 4, P(A3), P(A4), 100, P(A5), 0, P(A6), ws, None) == SHAPE
    assert f(P(A1), P(A2), 3, 512, 4, P(A3), P(A4), 100, P(A5), 0, P(A6), ws - 1, None) == WS
    assert f(P(A1), P(A2), 3, 512, 4, P(A3), P(A4), 100, P(A1), 0, P(A6), ws, None) == ALIAS
    g = _L().bitlinear_forward_grouped_acc
    assert g(P(A1), 3, 512, 4, P(A3), 100, P(A5), P(A6), ws, None) == DEVICE
    h = _L().bitlinear_forward_grouped_fp
    wsf = _L().bitlinear_forward_grouped_fp_workspace(3, 100, 512, 4)
    assert wsf > ws
    assert h(P(A1), 0, 3, 512, 4, P(A3), P(A4), 100, P(A5), 0, P(A6), wsf, None) == DEVICE
    assert h(P(A1), 0, 3, 512, 4, P(A3), P(A4), 100, P(A5), 0, P(A6), wsf - 1, None) == WS




def test_forward_path_validation():
    f = _L().bitlinear_forward_path
    p = ctypes.c_int(-1)
    assert f(4, 4096, 4096, None) == NULL
    assert f(0, 4096, 4096, ctypes.byref(p)) == SHAPE
    assert f(4, 4096, 100, ctypes.byref(p)) == SHAPE
    assert f(4, 4096, 4096, ctypes.byref(p)) == DEVICE

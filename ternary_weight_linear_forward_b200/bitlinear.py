"""Thin Python binding of libbitlinear.so (argument marshalling only).

Every function below checks dtypes, shapes and devices of torch tensors,
allocates outputs with torch (device memory is PyTorch's job here), passes raw
pointers and the current CUDA stream through the C ABI declared in
``include/bitlinear.h``, and raises ``BitLinearError`` on a nonzero status.
All arithmetic happens in the library's CUDA kernels.  There is no fallback:
if the shared library is missing or no sm_100 device is present, calls fail.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

BL_F32, BL_BF16, BL_I8 = 0, 1, 2
COMBINE = {"none": 0, "add": 1, "silu_mul": 2}
EPS_W = 1e-5

_STATUS = {0: "BL_OK", 1: "BL_ERR_NULL", 2: "BL_ERR_SHAPE", 3: "BL_ERR_ALIGN", 4: "BL_ERR_DTYPE",
           5: "BL_ERR_WORKSPACE", 6: "BL_ERR_DEVICE", 7: "BL_ERR_CUDA", 8: "BL_ERR_TIMEOUT", 9: "BL_ERR_ALIAS"}

# every symbol the header declares: (name, restype, argtypes)
_P, _I64, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "bitlinear_status_string": (ctypes.c_char_p, [_I]),
    "bitlinear_quantize_weights_workspace": (_SZ, [_I64, _I64]),
    "bitlinear_quantize_weights": (_I, [_P, _I64, _I64, _F, _P, _P, _P, _SZ, _P]),
    "bitlinear_pack": (_I, [_P, _I64, _I64, _P, _P]),
    "bitlinear_quant_act": (_I, [_P, _I, _I64, _I64, _P, _P, _P]),
    "bitlinear_forward_workspace": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_forward": (_I, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_forward_fp_workspace": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_forward_fp": (_I, [_P, _I, _I64, _I64, _P, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_forward_fp_batch": (_I, [_P, _I, _I64, _I, _I, _P]),
    "bitlinear_forward_acc": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "bitlinear_forward_noalloc": (_I, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _I, _P]),
    "bitlinear_quant_act_rms": (_I, [_P, _P, _I, _I64, _I64, _P, _P, _P, _P]),
    "bitlinear_quantize_weights_grouped_workspace": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_quantize_weights_grouped": (_I, [_P, _I64, _I64, _I64, _F, _P, _P, _P, _SZ, _P]),
    "bitlinear_quant_act_grouped": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P]),
    "bitlinear_forward_grouped_workspace": (_SZ, [_I64, _I64, _I64, _I64]),
    "bitlinear_forward_grouped": (_I, [_P, _P, _I64, _I64, _I64, _P, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_forward_grouped_acc": (_I, [_P, _I64, _I64, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "bitlinear_forward_grouped_fp_workspace": (_SZ, [_I64, _I64, _I64, _I64]),
    "bitlinear_forward_grouped_fp": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_glu_workspace": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_glu_forward": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bitlinear_binarize_weights_workspace": (_SZ, [_I64, _I64]),
    "bitlinear_binarize_weights": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    "bitlinear_pack_bits": (_I, [_P, _I64, _I64, _P, _P]),
    "bitlinear_forward_binary_workspace": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_forward_binary": (_I, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_forward_binary_acc": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "bitlinear_forward_binary_fp_workspace": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_forward_binary_fp": (_I, [_P, _I, _I64, _I64, _P, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_set_decode_engine": (_I, [_I]),
    "bitlinear_get_decode_engine": (_I, []),
    "bitlinear_forward_path": (_I, [_I64, _I64, _I64, _P]),
    "bitlinear_device_status": (_I, [_P]),
    "bitlinear_num_sms": (_I, []),
    "bitlinear_test_expire_next_wait": (_I, [_I]),
}


class BitLinearError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)} ({status_string(status)})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libbitlinear.so from the package directory (built by build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m ternary_weight_linear_forward_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().bitlinear_status_string(int(s)).decode()


def _check(fn: str, s: int):
    if s != 0:
        raise BitLinearError(fn, s)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, ndim, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_out(out, shape, dtypes, device, name="out"):
    """A caller-given output buffer: the library writes shape-many elements
    through its pointer, so the size, dtype, device and layout are checked
    here, where they are known."""
    if not isinstance(out, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if out.dtype not in dtypes:
        raise TypeError(f"{name} must be one of {dtypes}, got {out.dtype}")
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(out.shape)}")
    if out.device != device:
        raise ValueError(f"{name} must be on {device}, got {out.device}")
    if not out.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_len(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _same_device(device, **tensors):
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} must be on {device}, got {t.device}")


def _check_ws(ws, device):
    if ws is None:
        return
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or not ws.is_contiguous():
        raise TypeError("ws must be a contiguous torch.uint8 tensor")
    if ws.device != device:
        raise ValueError(f"ws must be on {device}, got {ws.device}")


FLOAT_OUT = (torch.float32, torch.bfloat16)


# --------------------------------------------------------------------------
# entry points
# --------------------------------------------------------------------------

def quantize_weights(W: torch.Tensor, eps: float = EPS_W, stream=None):
    """absmean ternarisation -> (W_t int8 [N, K], beta float32 [1]) on W's device."""
    _need(W, torch.float32, 2, "W")
    N, K = W.shape
    W_t = torch.empty((N, K), dtype=torch.int8, device=W.device)
    beta = torch.empty(4, dtype=torch.float32, device=W.device)[:1]
    nws = lib().bitlinear_quantize_weights_workspace(N, K)
    ws = torch.empty(nws, dtype=torch.uint8, device=W.device)
    _check("bitlinear_quantize_weights",
           lib().bitlinear_quantize_weights(_ptr(W), N, K, float(eps), _ptr(W_t), _ptr(beta), _ptr(ws), nws,
                                            _stream(stream)))
    return W_t, beta


def pack(W_t: torch.Tensor, stream=None) -> torch.Tensor:
    """2-bit packing, 16 trits per uint32 -> W_p int32 [N, K/16] (bit pattern of uint32)."""
    _need(W_t, torch.int8, 2, "W_t")
    N, K = W_t.shape
    W_p = torch.empty((N, K // 16 if K % 16 == 0 else 1), dtype=torch.int32, device=W_t.device)
    _check("bitlinear_pack", lib().bitlinear_pack(_ptr(W_t), N, K, _ptr(W_p), _stream(stream)))
    return W_p


def quant_act(x: torch.Tensor, out=None, stream=None):
    """Per-token absmax int8 quantiser -> (x_q int8 [M, K], gamma float32 [M])."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _need(x, x.dtype, 2, "x")
    M, K = x.shape
    if out is None:
        x_q = torch.empty((M, K), dtype=torch.int8, device=x.device)
        gamma = torch.empty(max(M, 4), dtype=torch.float32, device=x.device)[:M]
    else:
        x_q, gamma = out
        _check_out(x_q, (M, K), (torch.int8,), x.device, "x_q")
        _check_out(gamma, (M,), (torch.float32,), x.device, "gamma")
    dt = BL_BF16 if x.dtype == torch.bfloat16 else BL_F32
    _check("bitlinear_quant_act",
           lib().bitlinear_quant_act(_ptr(x), dt, M, K, _ptr(x_q), _ptr(gamma), _stream(stream)))
    return x_q, gamma


def forward_workspace(M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_forward_workspace(M, N, K))


def forward(x_q: torch.Tensor, gamma: torch.Tensor, W_p: torch.Tensor, beta: torch.Tensor,
            out_dtype=torch.float32, out=None, ws=None, stream=None) -> torch.Tensor:
    """y = BitLinear(x_q) with the fused rescale; float32 or bfloat16 output."""
    _need(x_q, torch.int8, 2, "x_q")
    _need(W_p, torch.int32, 2, "W_p")
    _need(gamma, torch.float32, 1, "gamma")
    _need(beta, torch.float32, 1, "beta")
    M, K = x_q.shape
    N = W_p.shape[0]
    if W_p.shape[1] * 16 != K:
        raise ValueError("W_p must be [N, K/16]")
    _check_len(gamma, (M,), "gamma")
    _check_len(beta, (1,), "beta")
    _same_device(x_q.device, gamma=gamma, W_p=W_p, beta=beta)
    _check_ws(ws, x_q.device)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x_q.device)
    _check_out(out, (M, N), FLOAT_OUT, x_q.device)
    dt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[out.dtype]
    nws = forward_workspace(M, N, K)
    if nws and ws is None:
        ws = torch.empty(nws, dtype=torch.uint8, device=x_q.device)
    _check("bitlinear_forward",
           lib().bitlinear_forward(_ptr(x_q), _ptr(gamma), M, K, _ptr(W_p), _ptr(beta), N, _ptr(out), dt,
                                   _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return out


def forward_fp_workspace(M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_forward_fp_workspace(M, N, K))


def forward_fp(x: torch.Tensor, W_p: torch.Tensor, beta: torch.Tensor, out_dtype=torch.float32, out=None,
               ws=None, stream=None) -> torch.Tensor:
    """quant_act + forward in one call (one kernel for M <= 4); bit-identical to the two calls."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _need(x, x.dtype, 2, "x")
    _need(W_p, torch.int32, 2, "W_p")
    _need(beta, torch.float32, 1, "beta")
    M, K = x.shape
    N = W_p.shape[0]
    if W_p.shape[1] * 16 != K:
        raise ValueError("W_p must be [N, K/16]")
    _check_len(beta, (1,), "beta")
    _same_device(x.device, W_p=W_p, beta=beta)
    _check_ws(ws, x.device)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check_out(out, (M, N), FLOAT_OUT, x.device)
    dt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[out.dtype]
    nws = int(lib().bitlinear_forward_fp_workspace(M, N, K))
    if nws and ws is None:
        ws = torch.empty(nws, dtype=torch.uint8, device=x.device)
    xdt = BL_BF16 if x.dtype == torch.bfloat16 else BL_F32
    _check("bitlinear_forward_fp",
           lib().bitlinear_forward_fp(_ptr(x), xdt, M, K, _ptr(W_p), _ptr(beta), N, _ptr(out), dt, _ptr(ws),
                                      0 if ws is None else ws.numel(), _stream(stream)))
    return out


class _Problem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("W_p", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("y", ctypes.c_void_p),
                ("K", ctypes.c_int64), ("N", ctypes.c_int64)]


class BatchPlan:
    """A forward_fp_batch call marshalled once: the problem descriptors are
    checked and packed into the C array when the plan is made, and ``run``
    only passes them to the library.  The tensors must stay alive and keep
    their storage while the plan is used (the descriptors hold pointers)."""

    def __init__(self, problems, out_dtype=torch.float32):
        self.arr, self.outs, self.m, self.xdt, self.ydt = _pack_batch(problems, out_dtype)
        self._keep = [dict(pr) for pr in problems]
        self._ptr = ctypes.cast(self.arr, ctypes.c_void_p)

    def run(self, stream=None):
        _check("bitlinear_forward_fp_batch",
               lib().bitlinear_forward_fp_batch(self._ptr, len(self.outs), self.m, self.xdt, self.ydt,
                                                _stream(stream)))
        return self.outs


def forward_fp_batch(problems, out_dtype=torch.float32, stream=None):
    """Several independent decode projections in one launch.

    ``problems``: list of dicts with keys ``x`` ([M, K] fp32/bf16, or int8 x_q
    together with ``gamma`` [M]), ``W_p``, ``beta`` and optionally ``out``.
    All share M (<= 4) and the x dtype.  Returns the list of outputs."""
    arr, outs, m, xdt, ydt = _pack_batch(problems, out_dtype)
    _check("bitlinear_forward_fp_batch",
           lib().bitlinear_forward_fp_batch(ctypes.cast(arr, ctypes.c_void_p), len(problems), m, xdt, ydt,
                                            _stream(stream)))
    return outs


def _pack_batch(problems, out_dtype):
    if not 1 <= len(problems) <= 8:
        raise ValueError("1 to 8 problems")
    arr = (_Problem * len(problems))()
    outs = []
    x0 = problems[0]["x"]
    quantised = x0.dtype == torch.int8
    for i, pr in enumerate(problems):
        x, W_p, beta = pr["x"], pr["W_p"], pr["beta"]
        if x.dtype != x0.dtype or x.shape[0] != x0.shape[0]:
            raise ValueError("problems must share M and the x dtype")
        _need(x, x.dtype, 2, "x")
        _need(W_p, torch.int32, 2, "W_p")
        _need(beta, torch.float32, 1, "beta")
        gamma = pr.get("gamma")
        if quantised:
            _need(gamma, torch.float32, 1, "gamma")
        M, K = x.shape
        N = W_p.shape[0]
        if W_p.shape[1] * 16 != K:
            raise ValueError("W_p must be [N, K/16]")
        if quantised:
            _check_len(gamma, (M,), "gamma")
        _check_len(beta, (1,), "beta")
        _same_device(x0.device, x=x, gamma=gamma if quantised else None, W_p=W_p, beta=beta)
        out = pr.get("out")
        if out is None:
            out = torch.empty((M, N), dtype=out_dtype, device=x.device)
        _check_out(out, (M, N), FLOAT_OUT, x0.device)
        outs.append(out)
        arr[i] = _Problem(x.data_ptr(), gamma.data_ptr() if quantised else None, W_p.data_ptr(), beta.data_ptr(),
                          out.data_ptr(), K, N)
    if any(o.dtype != outs[0].dtype for o in outs):
        raise ValueError("outputs must share a dtype")
    ydt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[outs[0].dtype]
    xdt = BL_I8 if quantised else BL_BF16 if x0.dtype == torch.bfloat16 else BL_F32
    return arr, outs, x0.shape[0], xdt, ydt


def forward_noalloc(x_q: torch.Tensor, gamma: torch.Tensor, W_p: torch.Tensor, beta: torch.Tensor,
                    out_dtype=torch.float32, out=None, stream=None) -> torch.Tensor:
    """forward() for callers that cannot allocate device memory: the library
    keeps the prefill scratch in a static device array (M <= 16384; the first
    call on a device should come before any stream capture; concurrent calls
    on one device race on the shared scratch).  Only ``out`` is allocated
    here, and only when it is not given."""
    _need(x_q, torch.int8, 2, "x_q")
    _need(W_p, torch.int32, 2, "W_p")
    _need(gamma, torch.float32, 1, "gamma")
    _need(beta, torch.float32, 1, "beta")
    M, K = x_q.shape
    N = W_p.shape[0]
    if W_p.shape[1] * 16 != K:
        raise ValueError("W_p must be [N, K/16]")
    _check_len(gamma, (M,), "gamma")
    _check_len(beta, (1,), "beta")
    _same_device(x_q.device, gamma=gamma, W_p=W_p, beta=beta)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x_q.device)
    _check_out(out, (M, N), FLOAT_OUT, x_q.device)
    dt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[out.dtype]
    _check("bitlinear_forward_noalloc",
           lib().bitlinear_forward_noalloc(_ptr(x_q), _ptr(gamma), M, K, _ptr(W_p), _ptr(beta), N, _ptr(out), dt,
                                           _stream(stream)))
    return out


def forward_acc(x_q: torch.Tensor, W_p: torch.Tensor, ws=None, stream=None) -> torch.Tensor:
    """int32 accumulators acc[m, n] = sum_k W_t[n, k] x_q[m, k] (same kernels as forward)."""
    _need(x_q, torch.int8, 2, "x_q")
    _need(W_p, torch.int32, 2, "W_p")
    M, K = x_q.shape
    N = W_p.shape[0]
    if W_p.shape[1] * 16 != K:
        raise ValueError("W_p must be [N, K/16]")
    _same_device(x_q.device, W_p=W_p)
    _check_ws(ws, x_q.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=x_q.device)
    nws = forward_workspace(M, N, K)
    if nws and ws is None:
        ws = torch.empty(nws, dtype=torch.uint8, device=x_q.device)
    _check("bitlinear_forward_acc",
           lib().bitlinear_forward_acc(_ptr(x_q), M, K, _ptr(W_p), N, _ptr(acc), _ptr(ws),
                                       0 if ws is None else ws.numel(), _stream(stream)))
    return acc


# --------------------------------------------------------------------------
# 1-bit weights (unite.ai page, "Mathematische Grundlagen", item 1
# "Gewichtsbinarisierung": W_b = Sign(W - mean(W)))
# --------------------------------------------------------------------------

def binarize_weights(W: torch.Tensor, stream=None):
    """Binarisation -> (W_b int8 [N, K] in {-1, +1}, alpha float32 [1], beta float32 [1])."""
    _need(W, torch.float32, 2, "W")
    N, K = W.shape
    W_b = torch.empty((N, K), dtype=torch.int8, device=W.device)
    ab = torch.empty(8, dtype=torch.float32, device=W.device)
    alpha, beta = ab[0:1], ab[4:5]  # distinct 16-byte-aligned scalars
    nws = lib().bitlinear_binarize_weights_workspace(N, K)
    ws = torch.empty(nws, dtype=torch.uint8, device=W.device)
    _check("bitlinear_binarize_weights",
           lib().bitlinear_binarize_weights(_ptr(W), N, K, _ptr(W_b), _ptr(alpha), _ptr(beta), _ptr(ws), nws,
                                            _stream(stream)))
    return W_b, alpha, beta


def pack_bits(W_b: torch.Tensor, stream=None) -> torch.Tensor:
    """1-bit packing, 32 signs per uint32 -> W_p int32 [N, K/32] (bit pattern of uint32)."""
    _need(W_b, torch.int8, 2, "W_b")
    N, K = W_b.shape
    W_p = torch.empty((N, K // 32 if K % 32 == 0 else 1), dtype=torch.int32, device=W_b.device)
    _check("bitlinear_pack_bits", lib().bitlinear_pack_bits(_ptr(W_b), N, K, _ptr(W_p), _stream(stream)))
    return W_p


def _bits_shape(W_p, K):
    if W_p.shape[1] * 32 != K:
        raise ValueError("W_p must be [N, K/32]")
    return W_p.shape[0]


def forward_binary(x_q: torch.Tensor, gamma: torch.Tensor, W_p: torch.Tensor, beta: torch.Tensor,
                   out_dtype=torch.float32, out=None, ws=None, stream=None) -> torch.Tensor:
    """y = BitLinear(x_q) with 1-bit weights and the fused rescale."""
    _need(x_q, torch.int8, 2, "x_q")
    _need(W_p, torch.int32, 2, "W_p")
    _need(gamma, torch.float32, 1, "gamma")
    _need(beta, torch.float32, 1, "beta")
    M, K = x_q.shape
    N = _bits_shape(W_p, K)
    _check_len(gamma, (M,), "gamma")
    _check_len(beta, (1,), "beta")
    _same_device(x_q.device, gamma=gamma, W_p=W_p, beta=beta)
    _check_ws(ws, x_q.device)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x_q.device)
    _check_out(out, (M, N), FLOAT_OUT, x_q.device)
    dt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[out.dtype]
    nws = int(lib().bitlinear_forward_binary_workspace(M, N, K))
    if nws and ws is None:
        ws = torch.empty(nws, dtype=torch.uint8, device=x_q.device)
    _check("bitlinear_forward_binary",
           lib().bitlinear_forward_binary(_ptr(x_q), _ptr(gamma), M, K, _ptr(W_p), _ptr(beta), N, _ptr(out), dt,
                                          _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return out


def forward_binary_acc(x_q: torch.Tensor, W_p: torch.Tensor, ws=None, stream=None) -> torch.Tensor:
    """int32 accumulators sum_k W_b[n, k] x_q[m, k] of the 1-bit forward."""
    _need(x_q, torch.int8, 2, "x_q")
    _need(W_p, torch.int32, 2, "W_p")
    M, K = x_q.shape
    N = _bits_shape(W_p, K)
    _same_device(x_q.device, W_p=W_p)
    _check_ws(ws, x_q.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=x_q.device)
    nws = int(lib().bitlinear_forward_binary_workspace(M, N, K))
    if nws and ws is None:
        ws = torch.empty(nws, dtype=torch.uint8, device=x_q.device)
    _check("bitlinear_forward_binary_acc",
           lib().bitlinear_forward_binary_acc(_ptr(x_q), M, K, _ptr(W_p), N, _ptr(acc), _ptr(ws),
                                              0 if ws is None else ws.numel(), _stream(stream)))
    return acc


def forward_binary_fp(x: torch.Tensor, W_p: torch.Tensor, beta: torch.Tensor, out_dtype=torch.float32, out=None,
                      ws=None, stream=None) -> torch.Tensor:
    """quant_act + forward_binary in one call (one kernel for M <= 4)."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _need(x, x.dtype, 2, "x")
    _need(W_p, torch.int32, 2, "W_p")
    _need(beta, torch.float32, 1, "beta")
    M, K = x.shape
    N = _bits_shape(W_p, K)
    _check_len(beta, (1,), "beta")
    _same_device(x.device, W_p=W_p, beta=beta)
    _check_ws(ws, x.device)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check_out(out, (M, N), FLOAT_OUT, x.device)
    dt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[out.dtype]
    nws = int(lib().bitlinear_forward_binary_fp_workspace(M, N, K))
    if nws and ws is None:
        ws = torch.empty(nws, dtype=torch.uint8, device=x.device)
    xdt = BL_BF16 if x.dtype == torch.bfloat16 else BL_F32
    _check("bitlinear_forward_binary_fp",
           lib().bitlinear_forward_binary_fp(_ptr(x), xdt, M, K, _ptr(W_p), _ptr(beta), N, _ptr(out), dt,
                                             _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return out


def quant_act_rms(a: torch.Tensor, b: torch.Tensor | None = None, combine: str = "none", h=None,
                  quantize: bool = True, want_h: bool = False, out=None, stream=None):
    """Fused combine (none/add/silu_mul) + RMSNorm-folded int8 quantiser.

    Returns (h or None, x_q or None, gamma or None)."""
    _need(a, torch.float32, 2, "a")
    if b is not None:
        _need(b, torch.float32, 2, "b")
    M, K = a.shape
    if b is not None:
        _check_len(b, (M, K), "b")
        _same_device(a.device, b=b)
    if want_h and h is None:
        h = torch.empty_like(a)
    if h is not None:
        _check_out(h, (M, K), (torch.float32,), a.device, "h")
    if quantize:
        if out is None:
            x_q = torch.empty((M, K), dtype=torch.int8, device=a.device)
            gamma = torch.empty(max(M, 4), dtype=torch.float32, device=a.device)[:M]
        else:
            x_q, gamma = out
            _check_out(x_q, (M, K), (torch.int8,), a.device, "x_q")
            _check_out(gamma, (M,), (torch.float32,), a.device, "gamma")
    else:
        x_q = gamma = None
    _check("bitlinear_quant_act_rms",
           lib().bitlinear_quant_act_rms(_ptr(a), _ptr(b), COMBINE[combine], M, K, _ptr(h), _ptr(x_q),
                                         _ptr(gamma), _stream(stream)))
    return h, x_q, gamma


ENGINES = {"auto": 0, "cuda_cores": 1, "tensor_cores": 2, "cuda_cores_general": 3}


def set_decode_engine(name: str):
    """Engine of later decode calls (M <= 64): 'auto', 'cuda_cores', 'tensor_cores' or
    'cuda_cores_general' (CUDA cores without the one-token streaming kernel)."""
    if name not in ENGINES:
        raise ValueError(f"unknown decode engine {name!r}")
    _check("bitlinear_set_decode_engine", lib().bitlinear_set_decode_engine(ENGINES[name]))


PATHS = {0: "cuda_cores", 1: "swap_ab", 2: "gemm"}


def forward_path(M: int, N: int, K: int) -> str:
    """The kernel family the forward runs for one [M, K] x [N, K] problem on the
    current device under the current engine: "cuda_cores", "swap_ab" or "gemm"."""
    v = ctypes.c_int(-1)
    _check("bitlinear_forward_path", lib().bitlinear_forward_path(M, N, K, ctypes.byref(v)))
    return PATHS[v.value]


def get_decode_engine() -> str:
    v = int(lib().bitlinear_get_decode_engine())
    return {i: n for n, i in ENGINES.items()}[v]


@contextlib.contextmanager
def decode_engine(name: str):
    """Run the enclosed calls with the given decode engine, then restore the previous one."""
    prev = get_decode_engine()
    set_decode_engine(name)
    try:
        yield
    finally:
        set_decode_engine(prev)


def device_status(stream=None):
    """Synchronise the stream and raise if a kernel gave up a bounded wait."""
    _check("bitlinear_device_status", lib().bitlinear_device_status(_stream(stream)))


def num_sms() -> int:
    return int(lib().bitlinear_num_sms())


# --------------------------------------------------------------------------
# convenience layer objects (still only marshalling around the C ABI)
# --------------------------------------------------------------------------

class BitLinear:
    """A prepared ternary layer: packed weights W_p [N, K/16] and scale beta [1]."""

    def __init__(self, W_p: torch.Tensor, beta: torch.Tensor):
        self.W_p, self.beta = W_p, beta
        self.N, self.K = W_p.shape[0], W_p.shape[1] * 16

    @classmethod
    def from_float(cls, W: torch.Tensor, eps: float = EPS_W):
        W_t, beta = quantize_weights(W, eps)
        return cls(pack(W_t), beta)

    def __call__(self, x: torch.Tensor, out_dtype=torch.float32, out=None) -> torch.Tensor:
        return forward_fp(x, self.W_p, self.beta, out_dtype=out_dtype, out=out)


# --------------------------------------------------------------------------
# Group quantisation along K (unite.ai page, "Gruppenquantisierung und
# -normalisierung"); group-major layouts, see include/bitlinear.h
# --------------------------------------------------------------------------

def quantize_weights_grouped(W: torch.Tensor, G: int, eps: float = EPS_W, stream=None):
    """Per-group absmean ternarisation -> (W_t int8 [G, N, K/G], beta float32 [G])."""
    _need(W, torch.float32, 2, "W")
    N, K = W.shape
    W_t = torch.empty((G, N, K // G), dtype=torch.int8, device=W.device)
    beta = torch.empty(max(G, 4), dtype=torch.float32, device=W.device)[:G]
    nws = int(lib().bitlinear_quantize_weights_grouped_workspace(N, K, G))
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=W.device)
    _check("bitlinear_quantize_weights_grouped",
           lib().bitlinear_quantize_weights_grouped(_ptr(W), N, K, G, float(eps), _ptr(W_t), _ptr(beta), _ptr(ws),
                                                    nws, _stream(stream)))
    return W_t, beta


def pack_grouped(W_t: torch.Tensor, stream=None) -> torch.Tensor:
    """2-bit packing of group-major trits [G, N, K/G] -> W_p int32 [G, N, K/(16G)]."""
    _need(W_t, torch.int8, 3, "W_t")
    G, N, Kg = W_t.shape
    return pack(W_t.view(G * N, Kg), stream=stream).view(G, N, -1)


def quant_act_grouped(x: torch.Tensor, G: int, stream=None):
    """Per-token, per-group absmax quantiser -> (x_q int8 [G, M, K/G], gamma float32 [M, G])."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _need(x, x.dtype, 2, "x")
    M, K = x.shape
    x_q = torch.empty((G, M, K // G), dtype=torch.int8, device=x.device)
    gamma = torch.empty(max(M * G, 4), dtype=torch.float32, device=x.device)[:M * G].view(M, G)
    dt = BL_BF16 if x.dtype == torch.bfloat16 else BL_F32
    _check("bitlinear_quant_act_grouped",
           lib().bitlinear_quant_act_grouped(_ptr(x), dt, M, K, G, _ptr(x_q), _ptr(gamma), _stream(stream)))
    return x_q, gamma


def _grouped_shapes(W_p, G, K):
    _need(W_p, torch.int32, 3, "W_p")
    if W_p.shape[0] != G or W_p.shape[2] * 16 * G != K:
        raise ValueError("W_p must be [G, N, K/(16G)]")
    return W_p.shape[1]


def forward_grouped(x_q: torch.Tensor, gamma: torch.Tensor, W_p: torch.Tensor, beta: torch.Tensor,
                    out_dtype=torch.float32, out=None, ws=None, stream=None) -> torch.Tensor:
    """Group-quantised forward from group-major x_q [G, M, K/G] and gamma [M, G]."""
    _need(x_q, torch.int8, 3, "x_q")
    _need(gamma, torch.float32, 2, "gamma")
    _need(beta, torch.float32, 1, "beta")
    G, M, Kg = x_q.shape
    K = G * Kg
    N = _grouped_shapes(W_p, G, K)
    _check_len(gamma, (M, G), "gamma")
    _check_len(beta, (G,), "beta")
    _same_device(x_q.device, gamma=gamma, W_p=W_p, beta=beta)
    _check_ws(ws, x_q.device)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x_q.device)
    _check_out(out, (M, N), FLOAT_OUT, x_q.device)
    dt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[out.dtype]
    nws = int(lib().bitlinear_forward_grouped_workspace(M, N, K, G))
    if ws is None:
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=x_q.device)
    _check("bitlinear_forward_grouped",
           lib().bitlinear_forward_grouped(_ptr(x_q), _ptr(gamma), M, K, G, _ptr(W_p), _ptr(beta), N, _ptr(out), dt,
                                           _ptr(ws), ws.numel(), _stream(stream)))
    return out


def forward_grouped_acc(x_q: torch.Tensor, W_p: torch.Tensor, stream=None) -> torch.Tensor:
    """Per-group int32 accumulators -> [G, M, N]."""
    _need(x_q, torch.int8, 3, "x_q")
    G, M, Kg = x_q.shape
    K = G * Kg
    N = _grouped_shapes(W_p, G, K)
    _same_device(x_q.device, W_p=W_p)
    S = (M * N + 3) // 4 * 4
    acc = torch.empty(G * S, dtype=torch.int32, device=x_q.device)
    nws = int(lib().bitlinear_forward_grouped_workspace(M, N, K, G))
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=x_q.device)
    _check("bitlinear_forward_grouped_acc",
           lib().bitlinear_forward_grouped_acc(_ptr(x_q), M, K, G, _ptr(W_p), N, _ptr(acc), _ptr(ws), nws,
                                               _stream(stream)))
    return acc.view(G, S)[:, :M * N].reshape(G, M, N)


def forward_grouped_fp(x: torch.Tensor, W_p: torch.Tensor, beta: torch.Tensor, out_dtype=torch.float32, out=None,
                       ws=None, stream=None) -> torch.Tensor:
    """quant_act_grouped + forward_grouped in one call."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _need(x, x.dtype, 2, "x")
    _need(beta, torch.float32, 1, "beta")
    M, K = x.shape
    G = beta.shape[0]
    N = _grouped_shapes(W_p, G, K)
    _same_device(x.device, W_p=W_p, beta=beta)
    _check_ws(ws, x.device)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check_out(out, (M, N), FLOAT_OUT, x.device)
    dt = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}[out.dtype]
    nws = int(lib().bitlinear_forward_grouped_fp_workspace(M, N, K, G))
    if ws is None:
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=x.device)
    xdt = BL_BF16 if x.dtype == torch.bfloat16 else BL_F32
    _check("bitlinear_forward_grouped_fp",
           lib().bitlinear_forward_grouped_fp(_ptr(x), xdt, M, K, G, _ptr(W_p), _ptr(beta), N, _ptr(out), dt,
                                              _ptr(ws), ws.numel(), _stream(stream)))
    return out


def glu_forward(x: torch.Tensor, gate, up, down, want_u: bool = False, out=None, ws=None, stream=None):
    """The MatMul-free GLU channel mixer on x [M, D]: down(SiLU(gate(x)) * up(x)),
    every BitLinear input RMS-normalised.  gate, up and down are BitLinear
    layers (or (W_p, beta) pairs).  Returns y [M, D], or (y, u) with u [M, F]."""
    _need(x, torch.float32, 2, "x")
    (Wg, bg), (Wu, bu), (Wd, bd) = [(L.W_p, L.beta) if isinstance(L, BitLinear) else L for L in (gate, up, down)]
    for t, n in ((Wg, "W_gate"), (Wu, "W_up"), (Wd, "W_down")):
        _need(t, torch.int32, 2, n)
    for t, n in ((bg, "beta_gate"), (bu, "beta_up"), (bd, "beta_down")):
        _need(t, torch.float32, 1, n)
    M, D = x.shape
    F = Wg.shape[0]
    if Wg.shape[1] * 16 != D or Wu.shape != Wg.shape or Wd.shape[0] != D or Wd.shape[1] * 16 != F:
        raise ValueError("W_gate and W_up must be [F, D/16], W_down [D, F/16]")
    for t, n in ((bg, "beta_gate"), (bu, "beta_up"), (bd, "beta_down")):
        _check_len(t, (1,), n)
    _same_device(x.device, W_gate=Wg, W_up=Wu, W_down=Wd, beta_gate=bg, beta_up=bu, beta_down=bd)
    _check_ws(ws, x.device)
    y = torch.empty((M, D), dtype=torch.float32, device=x.device) if out is None else out
    _check_out(y, (M, D), (torch.float32,), x.device)
    u = torch.empty((M, F), dtype=torch.float32, device=x.device) if want_u else None
    nws = int(lib().bitlinear_glu_workspace(M, D, F))
    if ws is None:
        ws = torch.empty(nws, dtype=torch.uint8, device=x.device)
    _check("bitlinear_glu_forward",
           lib().bitlinear_glu_forward(_ptr(x), M, D, F, _ptr(Wg), _ptr(bg), _ptr(Wu), _ptr(bu), _ptr(Wd), _ptr(bd),
                                       _ptr(y), _ptr(u), _ptr(ws), ws.numel(), _stream(stream)))
    return (y, u) if want_u else y


class DecoderBlock:
    """One ternary decoder block at batch-1 decode (seven BitLinear projections).

    h1 = x + o(v(x)) where attention over the single token returns v; out =
    h1 + down(SiLU(gate(h1)) * up(h1)); every projection input is
    RMS-normalised (gain 1) inside the fused quantiser."""

    PROJ = ("q", "k", "v", "o", "gate", "up", "down")

    def __init__(self, layers: dict):
        self.layers = layers
        self.hidden = layers["q"].K
        self.inter = layers["gate"].N
        dev = layers["q"].W_p.device
        H, F = self.hidden, self.inter
        f32 = dict(dtype=torch.float32, device=dev)
        self.buf = {
            "xq_h": torch.empty((1, H), dtype=torch.int8, device=dev),
            "g_h": torch.empty(4, **f32)[:1],
            "xq_f": torch.empty((1, F), dtype=torch.int8, device=dev),
            "g_f": torch.empty(4, **f32)[:1],
            "q": torch.empty((1, H), **f32), "k": torch.empty((1, H), **f32), "v": torch.empty((1, H), **f32),
            "o": torch.empty((1, H), **f32), "h1": torch.empty((1, H), **f32),
            "gate": torch.empty((1, F), **f32), "up": torch.empty((1, F), **f32),
            "u": torch.empty((1, F), **f32), "down": torch.empty((1, H), **f32),
            "out": torch.empty((1, H), **f32),
        }

    @classmethod
    def from_float(cls, weights: dict, eps: float = EPS_W):
        return cls({p: BitLinear.from_float(weights[p], eps) for p in cls.PROJ})

    def __call__(self, x: torch.Tensor, keep_u: bool = True) -> dict:
        b, L = self.buf, self.layers
        xh = (b["xq_h"], b["g_h"])
        xf = (b["xq_f"], b["g_f"])
        quant_act_rms(x, out=xh)
        forward_fp_batch([{"x": xh[0], "gamma": xh[1], "W_p": L[p].W_p, "beta": L[p].beta, "out": b[p]}
                          for p in ("q", "k", "v")])
        quant_act_rms(b["v"], out=xh)                     # attention over one token = v
        forward(*xh, L["o"].W_p, L["o"].beta, out=b["o"])
        quant_act_rms(x, b["o"], "add", h=b["h1"], out=xh)
        forward_fp_batch([{"x": xh[0], "gamma": xh[1], "W_p": L[p].W_p, "beta": L[p].beta, "out": b[p]}
                          for p in ("gate", "up")])
        quant_act_rms(b["gate"], b["up"], "silu_mul", h=b["u"] if keep_u else None, out=xf)
        forward(*xf, L["down"].W_p, L["down"].beta, out=b["down"])
        quant_act_rms(b["h1"], b["down"], "add", h=b["out"], quantize=False)
        return b

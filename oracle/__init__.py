"""CPU oracle for the BitLinear W1.58A8 forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library; the product path never calls it.

Each function states the passage it follows.  Sources (web pages):

* DataCamp blog "MatMul-free language models" (Dutch), section "MatMul
  vervangen door ternaire bewerkingen" -- absmean ternarisation; -1/0/+1
  multiplies become negate/zero/pass-through.  Figure item "RMS norm" --
  activations are normalised before quantisation.  Section "Kerncomponenten:
  MLGRU en GLU" -- the MatMul-free GLU (two BitLinears, SiLU, elementwise
  product, a third BitLinear): ``glu`` for any number of tokens, and the
  decoder block at batch-1 decode.
* unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle
  auf lokale Geraete" (German), section "Mathematische Grundlagen", eq. 2
  "Aktivierungsquantisierung" and eq. 3 "BitLinear-Betrieb"; item 1
  "Gewichtsbinarisierung", eq. 1 -- the 1-bit weights Sign(W - mean(W)).

Pins (tests/test_oracle_pins.py, tests/test_oracle_binary_pins.py): hand-worked
examples for the ternary, the 1-bit and the grouped weights (tests/golden/), closed
forms of the Gaussian absmean and mean statistics, invariants, brute force on
tiny inputs (every 3^8 trit half-word, every 2^16 sign pattern), reduction of
the contraction to numpy's int64 matmul; the exact |W| and signed sums are
checked against ``math.fsum`` (sticky-bit ties included).  Composite functions
are pinned by reduction to pinned parts: ``forward_grouped`` (G = 1 is the
ungrouped path, duplicated halves, zero groups, power-of-two group scales, its
binary32 error bound) and ``glu`` (zero gate, oddness in W_up and W_down,
token independence, the decoder block's MLP half).  Parity unpinned:
``silu_mul`` beyond its binary64 error bound (exp is a library routine on both
sides), and so ``glu``'s gated intermediate to the same extent.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

# ORACLE_OPENMP=1 loads the -fopenmp build of the same source (the
# benchmark's all-core CPU baseline); results are identical.
_lib = ctypes.CDLL(_build.build_omp() if os.environ.get("ORACLE_OPENMP") == "1" else _build.build())

_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i8p = np.ctypeslib.ndpointer(np.int8, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64

_lib.orc_exact_abs_sum.argtypes = [_f32p, _i64]
_lib.orc_exact_abs_sum.restype = ctypes.c_double
_lib.orc_exact_sum.argtypes = [_f32p, _i64]
_lib.orc_exact_sum.restype = ctypes.c_double
_lib.orc_mean_alpha.argtypes = [_f32p, _i64, _i64]
_lib.orc_mean_alpha.restype = ctypes.c_float
_lib.orc_binarize.argtypes = [_f32p, _i64, _i64, ctypes.c_float, _i8p]
_lib.orc_pack_bits.argtypes = [_i8p, _i64, _i64, _u32p]
_lib.orc_unpack_bits.argtypes = [_u32p, _i64, _i64, _i8p]
_lib.orc_absmean_beta.argtypes = [_f32p, _i64, _i64]
_lib.orc_absmean_beta.restype = ctypes.c_float
_lib.orc_ternarize.argtypes = [_f32p, _i64, _i64, ctypes.c_float, ctypes.c_float, _i8p]
_lib.orc_pack.argtypes = [_i8p, _i64, _i64, _u32p]
_lib.orc_unpack.argtypes = [_u32p, _i64, _i64, _i8p]
_lib.orc_unpack.restype = _i64
_lib.orc_quant_act.argtypes = [_f32p, _i64, _i64, _i8p, _f32p]
_lib.orc_ternary_acc.argtypes = [_i8p, _i64, _i64, _i8p, _i64, _i32p]
_lib.orc_rescale_f32.argtypes = [_i32p, _i64, _i64, ctypes.c_float, _f32p, _f32p]
_lib.orc_rescale_f64.argtypes = [_i32p, _i64, _i64, ctypes.c_float, _f32p, _f64p]
_lib.orc_f32_to_bf16.argtypes = [_f32p, _i64, _u16p]
_lib.orc_rms_rho.argtypes = [_f32p, _i64, ctypes.c_double]
_lib.orc_rms_rho.restype = ctypes.c_float
_lib.orc_silu_mul.argtypes = [_f32p, _f32p, _i64, _f32p]

EPS_W = np.float32(1e-5)      # divisor guard of the ternariser
Q_B = 127                     # int8 activation range [-127, 127]
GAMMA_FLOOR = np.float32(1e-5)
RMS_EPS = 1e-6                # RMSNorm epsilon of the decoder block


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def exact_abs_sum(w: np.ndarray) -> float:
    """Exact sum of |w| over binary32 values, correctly rounded to binary64."""
    w = _c(w, np.float32).ravel()
    return float(_lib.orc_exact_abs_sum(w, w.size))


def absmean_beta(W: np.ndarray) -> np.float32:
    """absmean scale, one per matrix (MatMul-free blog, "MatMul vervangen door
    ternaire bewerkingen"): beta = mean |W|, the exact mean rounded to binary64
    then binary32."""
    W = _c(W, np.float32)
    N, K = W.shape
    return np.float32(_lib.orc_absmean_beta(W, N, K))


def ternarize(W: np.ndarray, beta, eps=EPS_W) -> np.ndarray:
    """W_t = clip(round(W / (beta + eps)), -1, 1), binary32 divide, ties to even
    (MatMul-free blog, "MatMul vervangen door ternaire bewerkingen")."""
    W = _c(W, np.float32)
    N, K = W.shape
    out = np.empty((N, K), np.int8)
    _lib.orc_ternarize(W, N, K, np.float32(beta), np.float32(eps), out)
    return out


def quantize_weights(W: np.ndarray, eps=EPS_W):
    """absmean ternarisation of a full-precision matrix -> (W_t int8, beta fp32)."""
    beta = absmean_beta(W)
    return ternarize(W, beta, eps), beta


def pack(W_t: np.ndarray) -> np.ndarray:
    """2-bit codes c = w + 1, trit k = 16j + 4s + b of a row at bits 8b + 2s of word j."""
    W_t = _c(W_t, np.int8)
    N, K = W_t.shape
    assert K % 16 == 0
    out = np.empty((N, K // 16), np.uint32)
    _lib.orc_pack(W_t, N, K, out)
    return out


def unpack(W_p: np.ndarray, K: int):
    """Inverse of :func:`pack`; returns (W_t, number of invalid code-3 fields)."""
    W_p = _c(W_p, np.uint32)
    N = W_p.shape[0]
    out = np.empty((N, K), np.int8)
    bad = _lib.orc_unpack(W_p, N, K, out)
    return out, int(bad)


# ---------------------------------------------------------------------------
# 1-bit variant: unite.ai page, "Mathematische Grundlagen", item 1
# "Gewichtsbinarisierung", eq. 1.
# ---------------------------------------------------------------------------

def exact_sum(w: np.ndarray) -> float:
    """Exact signed sum over binary32 values, correctly rounded to binary64."""
    w = _c(w, np.float32).ravel()
    return float(_lib.orc_exact_sum(w, w.size))


def mean_alpha(W: np.ndarray) -> np.float32:
    """alpha = mean(W) over the whole matrix (eq. 1): the exact sum rounded to
    binary64, divided by N*K in binary64, then rounded to binary32."""
    W = _c(W, np.float32)
    N, K = W.shape
    return np.float32(_lib.orc_mean_alpha(W, N, K))


def binarize(W: np.ndarray, alpha) -> np.ndarray:
    """W_b = Sign(W - alpha) (eq. 1), Sign(d) = +1 if d > 0 else -1, with
    d = W - alpha one binary32 subtraction."""
    W = _c(W, np.float32)
    N, K = W.shape
    out = np.empty((N, K), np.int8)
    _lib.orc_binarize(W, N, K, np.float32(alpha), out)
    return out


def binarize_weights(W: np.ndarray):
    """Binarisation of a full-precision matrix -> (W_b int8 in {-1, +1}, alpha,
    beta).  beta, which the page names a scaling factor without a formula, is
    read as the same absmean scale mean |W| that the ternary weights use."""
    alpha = mean_alpha(W)
    return binarize(W, alpha), alpha, absmean_beta(W)


def pack_bits(W_b: np.ndarray) -> np.ndarray:
    """1 bit per weight: k = 32j + 4s + b of a row at bit 8b + s of word j,
    set for +1 (w > 0), clear otherwise."""
    W_b = _c(W_b, np.int8)
    N, K = W_b.shape
    assert K % 32 == 0
    out = np.empty((N, K // 32), np.uint32)
    _lib.orc_pack_bits(W_b, N, K, out)
    return out


def unpack_bits(W_p: np.ndarray, K: int) -> np.ndarray:
    """Inverse of :func:`pack_bits` (set bit -> +1, clear bit -> -1)."""
    W_p = _c(W_p, np.uint32)
    N = W_p.shape[0]
    out = np.empty((N, K), np.int8)
    _lib.orc_unpack_bits(W_p, N, K, out)
    return out


def quant_act(x: np.ndarray):
    """Per-token absmax int8 quantiser (unite.ai page, eq. 2 "Aktivierungs-
    quantisierung") with Q_b = 127: gamma = max(||x_m||_inf, 1e-5),
    s = 127 / gamma, x_hat = clip(rint(x * s), -127, 127), all binary32."""
    x = _c(x, np.float32)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    g = np.empty(M, np.float32)
    _lib.orc_quant_act(x, M, K, xq, g)
    return xq, g


def ternary_acc(x_q: np.ndarray, W_t: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k W_t[n, k] x_hat[m, k] by literal add / subtract / skip
    (MatMul-free blog: multiplying by -1, 0, 1 is negation, zero, identity)."""
    x_q = _c(x_q, np.int8)
    W_t = _c(W_t, np.int8)
    M, K = x_q.shape
    N = W_t.shape[0]
    assert W_t.shape[1] == K
    acc = np.empty((M, N), np.int32)
    _lib.orc_ternary_acc(x_q, M, K, W_t, N, acc)
    return acc


_lib_omp = None


def ternary_acc_all_cores(x_q: np.ndarray, W_t: np.ndarray) -> np.ndarray:
    """:func:`ternary_acc` computed by the -fopenmp build of the same C source,
    whose only difference is that the (m, n) pairs are shared among the
    host's cores: the same integers, in time for full-size checks."""
    global _lib_omp
    if _lib_omp is None:
        L = ctypes.CDLL(_build.build_omp())
        L.orc_ternary_acc.argtypes = [_i8p, _i64, _i64, _i8p, _i64, _i32p]
        _lib_omp = L
    x_q = _c(x_q, np.int8)
    W_t = _c(W_t, np.int8)
    M, K = x_q.shape
    N = W_t.shape[0]
    assert W_t.shape[1] == K
    acc = np.empty((M, N), np.int32)
    _lib_omp.orc_ternary_acc(x_q, M, K, W_t, N, acc)
    return acc


def rescale_f32(acc, beta, gamma) -> np.ndarray:
    """unite.ai eq. 3 "BitLinear-Betrieb": y = acc * (beta * gamma / 127),
    binary32 with f = (beta * gamma) / 127 formed first."""
    acc = _c(acc, np.int32)
    M, N = acc.shape
    y = np.empty((M, N), np.float32)
    _lib.orc_rescale_f32(acc, M, N, np.float32(beta), _c(gamma, np.float32), y)
    return y


def rescale_f64(acc, beta, gamma) -> np.ndarray:
    """The same rescale in binary64 (the reference the 1e-6 tolerance is taken against)."""
    acc = _c(acc, np.int32)
    M, N = acc.shape
    y = np.empty((M, N), np.float64)
    _lib.orc_rescale_f64(acc, M, N, np.float32(beta), _c(gamma, np.float32), y)
    return y


def to_bf16(y: np.ndarray) -> np.ndarray:
    """binary32 -> bf16 bit patterns, round to nearest, ties to even."""
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint16)
    _lib.orc_f32_to_bf16(y.ravel(), y.size, out.reshape(-1))
    return out


def forward(x: np.ndarray, W_t: np.ndarray, beta):
    """Whole BitLinear forward from fp32 activations and ternary weights.

    Returns a dict with x_q, gamma, acc, y (binary32 op order) and y64."""
    x_q, gamma = quant_act(x)
    acc = ternary_acc(x_q, W_t)
    return {"x_q": x_q, "gamma": gamma, "acc": acc,
            "y": rescale_f32(acc, beta, gamma), "y64": rescale_f64(acc, beta, gamma)}


# ---------------------------------------------------------------------------
# Decoder block at batch-1 decode (hidden 2560, intermediate 6912).
# ---------------------------------------------------------------------------

def rms_rho(x: np.ndarray) -> np.float32:
    """RMSNorm scalar with gain 1 (MatMul-free blog, figure item "RMS norm"):
    rho = 1 / sqrt(mean(x^2) + 1e-6), binary64, rounded once to binary32."""
    x = _c(x, np.float32).ravel()
    return np.float32(_lib.orc_rms_rho(x, x.size, RMS_EPS))


def quant_act_rmsnorm(x: np.ndarray):
    """Quantiser of RMSNorm(x) for one token.  absmax quantisation is invariant
    under a positive scale of the token, so Q(rho * x) has the codes of Q(x)
    and the scale gamma_eff = rho * gamma(x) (binary32 multiply)."""
    x_q, g = quant_act(x)
    rho = rms_rho(x)
    return x_q, (g * rho).astype(np.float32), rho


def silu_mul(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """SiLU(gate) * up in binary64, rounded once to binary32 (the GLU of the
    MatMul-free blog, section "Kerncomponenten: MLGRU en GLU")."""
    gate = _c(gate, np.float32).ravel()
    up = _c(up, np.float32).ravel()
    out = np.empty(gate.size, np.float32)
    _lib.orc_silu_mul(gate, up, gate.size, out)
    return out


def bitlinear_rms(x_row: np.ndarray, W_t: np.ndarray, beta):
    """One projection of the block: RMSNorm folded into the quantiser, ternary
    contraction, binary32 rescale."""
    x_q, g_eff, _ = quant_act_rmsnorm(x_row.reshape(1, -1))
    acc = ternary_acc(x_q, W_t)
    return {"x_q": x_q, "gamma": g_eff, "acc": acc, "y": rescale_f32(acc, beta, g_eff)}


def block_decode(x: np.ndarray, tern: dict) -> dict:
    """One decoder block for one token.  ``tern[p] = (W_t, beta)`` for p in
    q, k, v, o, gate, up, down.

    Attention over the single token in the context is softmax of one score,
    i.e. weight 1 on v, so the attention output equals v.  Residual adds are
    binary32.  Every BitLinear input is RMS-normalised before quantisation."""
    x = _c(x, np.float32).reshape(1, -1)
    out = {}
    q = bitlinear_rms(x, *tern["q"])          # all three share one x_hat
    k = bitlinear_rms(x, *tern["k"])
    v = bitlinear_rms(x, *tern["v"])
    out.update(q=q["y"], k=k["y"], v=v["y"], x_q_attn=q["x_q"], gamma_attn=q["gamma"])
    attn = v["y"]
    o = bitlinear_rms(attn, *tern["o"])
    h1 = (x + o["y"]).astype(np.float32)
    gate = bitlinear_rms(h1, *tern["gate"])
    up = bitlinear_rms(h1, *tern["up"])
    u = silu_mul(gate["y"], up["y"]).reshape(1, -1)
    down = bitlinear_rms(u, *tern["down"])
    h2 = (h1 + down["y"]).astype(np.float32)
    out.update(o=o["y"], h1=h1, gate=gate["y"], up=up["y"], u=u, down=down["y"], out=h2,
               x_q_o=o["x_q"], x_q_mlp=gate["x_q"], x_q_down=down["x_q"],
               acc_down=down["acc"])
    return out


# ---------------------------------------------------------------------------
# MatMul-free GLU channel mixer, any number of tokens.
# ---------------------------------------------------------------------------

def glu(x: np.ndarray, tern: dict) -> dict:
    """The MatMul-free GLU of the MatMul-free blog, section "Kerncomponenten:
    MLGRU en GLU": the input goes through two separate BitLinear layers, SiLU
    of one output is multiplied elementwise by the other, and the gated result
    goes through a third BitLinear.  Every BitLinear input is RMS-normalised
    before quantisation (figure item "RMS norm"), token by token.
    ``tern[p] = (W_t, beta)`` for p in gate, up ([F, D]) and down ([D, F])."""
    x = _c(x, np.float32)
    out = {k: [] for k in ("x_q", "gamma", "gate", "up", "u", "u_q", "gamma_u", "acc_down", "y")}
    for m in range(x.shape[0]):
        gate = bitlinear_rms(x[m], *tern["gate"])
        up = bitlinear_rms(x[m], *tern["up"])
        u = silu_mul(gate["y"], up["y"])
        down = bitlinear_rms(u, *tern["down"])
        for k, v in (("x_q", gate["x_q"][0]), ("gamma", gate["gamma"][0]), ("gate", gate["y"][0]),
                     ("up", up["y"][0]), ("u", u), ("u_q", down["x_q"][0]), ("gamma_u", down["gamma"][0]),
                     ("acc_down", down["acc"][0]), ("y", down["y"][0])):
            out[k].append(v)
    return {k: np.stack(v) for k, v in out.items()}


# ---------------------------------------------------------------------------
# Group quantisation: unite.ai page, section "Gruppenquantisierung und
# -normalisierung" -- weights and activations are divided into G groups and
# each group gets its own parameters.  Groups are G contiguous, equal blocks
# of the contraction dimension K (the split that divides both W and x).
# ---------------------------------------------------------------------------

def _groups(K: int, G: int):
    assert G >= 1 and K % G == 0
    Kg = K // G
    return [slice(g * Kg, (g + 1) * Kg) for g in range(G)]


def quantize_weights_grouped(W: np.ndarray, G: int, eps=EPS_W):
    """absmean ternarisation per column group: beta_g = mean |W[:, K_g]| and
    W_t[:, K_g] = clip(round(W[:, K_g] / (beta_g + eps)), -1, 1).
    Returns (W_t [N, K], beta [G])."""
    W = _c(W, np.float32)
    W_t = np.empty(W.shape, np.int8)
    beta = np.empty(G, np.float32)
    for g, sl in enumerate(_groups(W.shape[1], G)):
        W_t[:, sl], beta[g] = quantize_weights(W[:, sl], eps)
    return W_t, beta


def quant_act_grouped(x: np.ndarray, G: int):
    """Per-token absmax quantiser per channel group: gamma[m, g] =
    max(||x[m, K_g]||_inf, 1e-5), codes as eq. 2 with that gamma.
    Returns (x_q [M, K], gamma [M, G])."""
    x = _c(x, np.float32)
    x_q = np.empty(x.shape, np.int8)
    gamma = np.empty((x.shape[0], G), np.float32)
    for g, sl in enumerate(_groups(x.shape[1], G)):
        x_q[:, sl], gamma[:, g] = quant_act(x[:, sl])
    return x_q, gamma


def forward_grouped(x: np.ndarray, W_t: np.ndarray, beta, G: int):
    """Group-quantised forward: acc_g = sum_{k in K_g} W_t x_hat (int32) and
    y = sum over g = 0, 1, ... of (float)acc_g * ((beta_g * gamma_{m,g}) / 127),
    each term binary32 as eq. 3, added in binary32 in increasing g.
    Returns x_q, gamma, acc [G, M, N], y, the binary64 y64 and yabs64, the
    binary64 sum of the terms' magnitudes (terms of different groups can
    cancel, so binary32 evaluation is bounded relative to yabs64, not y)."""
    x_q, gamma = quant_act_grouped(x, G)
    M, N = x.shape[0], W_t.shape[0]
    acc = np.empty((G, M, N), np.int32)
    y = np.zeros((M, N), np.float32)
    y64 = np.zeros((M, N), np.float64)
    yabs64 = np.zeros((M, N), np.float64)
    for g, sl in enumerate(_groups(x.shape[1], G)):
        acc[g] = ternary_acc(x_q[:, sl], W_t[:, sl])
        t = rescale_f32(acc[g], beta[g], gamma[:, g])
        y = t if g == 0 else (y + t).astype(np.float32)
        t64 = rescale_f64(acc[g], beta[g], gamma[:, g])
        y64 += t64
        yabs64 += np.abs(t64)
    return {"x_q": x_q, "gamma": gamma, "acc": acc, "y": y, "y64": y64, "yabs64": yabs64}


def group_major(a: np.ndarray, G: int) -> np.ndarray:
    """[R, K] -> [G, R, K/G]: column group g of every row, groups one after another."""
    return np.stack([a[:, sl] for sl in _groups(a.shape[1], G)])

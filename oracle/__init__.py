"""Plain CPU oracle for the Sparse-BitNet BitLinear hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library never links, loads or calls it, and it shares no
code with the CUDA path: the arithmetic lives in ``bitnet_oracle.c`` (plain C,
written from the definitions) and this module only marshals NumPy arrays.

Definitions followed (page title and section):
  * "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", "The mechanism":
    absmean scale over the whole matrix, divide, round, clip to {-1, 0, 1};
    per-token symmetric 8-bit activations; ternary product as signed sums.
  * "Sparse-BitNet" (gist.science technical summary), section 2
    "Kerncomponenten": N:M mask from the master magnitudes, quantise then
    mask; "Training Strategie": dynamic mask, straight-through gradients.

Every function here is pinned by a test in ``tests/test_oracle_pins.py`` to
something other than itself (math.fsum, brute force, closed forms, hand-worked
fixtures in ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitnet_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no FMA contraction, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-shared", "-fPIC", _SRC, "-o", _LIB, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    F = ctypes.c_float
    lib.oracle_abs_sum.restype = ctypes.c_double
    lib.oracle_abs_sum.argtypes = [P, I64]
    lib.oracle_gamma.restype = F
    lib.oracle_gamma.argtypes = [P, I64, F]
    lib.oracle_mask_nm.restype = None
    lib.oracle_mask_nm.argtypes = [P, I64, I64, ctypes.c_int, ctypes.c_int, P]
    lib.oracle_ternary.restype = None
    lib.oracle_ternary.argtypes = [P, I64, F, P]
    lib.oracle_apply_mask.restype = None
    lib.oracle_apply_mask.argtypes = [P, P, I64, P]
    lib.oracle_pack_24.restype = ctypes.c_int
    lib.oracle_pack_24.argtypes = [P, P, I64, I64, P]
    lib.oracle_quant_act.restype = None
    lib.oracle_quant_act.argtypes = [P, I64, I64, F, P, P]
    lib.oracle_gemm_i32.restype = ctypes.c_int
    lib.oracle_gemm_i32.argtypes = [P, P, I64, I64, I64, P]
    lib.oracle_dequant.restype = None
    lib.oracle_dequant.argtypes = [P, P, F, I64, I64, P]
    lib.oracle_dgrad.restype = None
    lib.oracle_dgrad.argtypes = [P, P, F, I64, I64, I64, P, P]
    lib.oracle_set_threads.restype = None
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    _lib = lib
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> int:
    lib = _load()
    lib.oracle_set_threads(int(n))
    return lib.oracle_max_threads()


def max_threads() -> int:
    return _load().oracle_max_threads()


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns (uint16) to fp32 exactly."""
    return (u16.astype(np.uint32) << np.uint32(16)).view(np.float32)


def abs_sum(W: np.ndarray) -> float:
    """fp64 nearest to the exact sum of |W| (whole matrix)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    return float(_load().oracle_abs_sum(_p(W), W.size))


def gamma(W: np.ndarray, eps: float = 1e-5) -> np.float32:
    """Absmean scale: fp32(sum|W| / n) + eps (eps added in fp32)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    return np.float32(_load().oracle_gamma(_p(W), W.size, np.float32(eps)))


def mask_nm(W: np.ndarray, n: int = 2, m: int = 4) -> np.ndarray:
    """uint8 keep-mask, top-n |W| of each m consecutive weights per row."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    rows, k = W.shape
    assert k % m == 0
    keep = np.empty((rows, k), np.uint8)
    _load().oracle_mask_nm(_p(W), rows, k, n, m, _p(keep))
    return keep


def ternary(W: np.ndarray, g: float) -> np.ndarray:
    """clip(rint(W / g), -1, 1) for every weight (int8)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    q = np.empty(W.shape, np.int8)
    _load().oracle_ternary(_p(W), W.size, np.float32(g), _p(q))
    return q


def apply_mask(wt: np.ndarray, keep: np.ndarray) -> np.ndarray:
    wt = np.ascontiguousarray(wt, dtype=np.int8)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    out = np.empty_like(wt)
    _load().oracle_apply_mask(_p(wt), _p(keep), wt.size, _p(out))
    return out


def pack_24(wq: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """Canonical 2:4 group bytes [rows, k/4]."""
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    rows, k = wq.shape
    gb = np.empty((rows, k // 4), np.uint8)
    rc = _load().oracle_pack_24(_p(wq), _p(keep), rows, k, _p(gb))
    if rc != 0:
        raise ValueError("mask is not 2:4")
    return gb


def quant_act(X: np.ndarray, eps: float = 1e-5):
    """Per-token absmax int8: returns (Xq int8 [T,K], a fp32 [T] = max(absmax, eps))."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    T, K = X.shape
    Xq = np.empty((T, K), np.int8)
    a = np.empty((T,), np.float32)
    _load().oracle_quant_act(_p(X), T, K, np.float32(eps), _p(Xq), _p(a))
    return Xq, a


def gemm_i32(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """acc[t, n] = sum_k Xq[t, k] * Wq[n, k] (exact, int32)."""
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    T, K = Xq.shape
    N = Wq.shape[0]
    acc = np.empty((T, N), np.int32)
    if _load().oracle_gemm_i32(_p(Xq), _p(Wq), T, N, K, _p(acc)) != 0:
        raise OverflowError("int32 accumulator overflow")
    return acc


def dequant(acc: np.ndarray, a: np.ndarray, g: float) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    a = np.ascontiguousarray(a, dtype=np.float32)
    T, N = acc.shape
    Y = np.empty((T, N), np.float32)
    _load().oracle_dequant(_p(acc), _p(a), np.float32(g), T, N, _p(Y))
    return Y


def dgrad(dY: np.ndarray, Wq: np.ndarray, g: float):
    """dX = g * dY @ Wq in fp64; also returns g * |dY| @ |Wq| (error-bound scale)."""
    dY = np.ascontiguousarray(dY, dtype=np.float32)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    T, N = dY.shape
    K = Wq.shape[1]
    dX = np.empty((T, K), np.float64)
    absdX = np.empty((T, K), np.float64)
    _load().oracle_dgrad(_p(dY), _p(Wq), np.float32(g), T, N, K, _p(dX), _p(absdX))
    return dX, absdX


def pack_weights(W: np.ndarray, eps: float = 1e-5):
    """Whole weight side: (gamma, keep, Wq masked ternary, canonical group bytes)."""
    g = gamma(W, eps)
    keep = mask_nm(W, 2, 4)
    wt = ternary(W, g)
    wq = apply_mask(wt, keep)
    gb = pack_24(wq, keep)
    return g, keep, wq, gb


def forward(W: np.ndarray, X: np.ndarray, eps_w: float = 1e-5, eps_a: float = 1e-5):
    """One Sparse-BitLinear forward; returns a dict of every intermediate."""
    g, keep, wq, gb = pack_weights(W, eps_w)
    Xq, a = quant_act(X, eps_a)
    acc = gemm_i32(Xq, wq)
    Y = dequant(acc, a, g)
    return dict(gamma=g, keep=keep, wq=wq, gb=gb, xq=Xq, a=a, acc=acc, y=Y)


def forward_nm(W: np.ndarray, X: np.ndarray, n: int, m: int, eps_w: float = 1e-5, eps_a: float = 1e-5):
    """Sparse-BitLinear forward with an n:m mask (e.g. 6:8): the plain dense
    definition, with the same gamma, ternary and activation steps as forward()."""
    g = gamma(W, eps_w)
    keep = mask_nm(W, n, m)
    wq = apply_mask(ternary(W, g), keep)
    Xq, a = quant_act(X, eps_a)
    acc = gemm_i32(Xq, wq)
    Y = dequant(acc, a, g)
    return dict(gamma=g, keep=keep, wq=wq, xq=Xq, a=a, acc=acc, y=Y)


# ------------------------------------------------------------------ block epilogues fused into quantisation
#
# "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", "What this paper explains"
# item 3: the stack is LLaMA-alike (RMSNorm, SwiGLU, no biases).  The pages fix
# no precision for these steps; the readings used here (and by the kernels):
#   RMSNorm:  S_t = exact sum of x^2 over the row, rounded once to fp64;
#             ms_t = fp32(S_t / K) (fp64 division, then fp32);
#             r_t = fp32(1 / fp32(sqrt(fp32(ms_t + eps))));  x_n = fp32(x * r_t)
#             [then fp32(x_n * w_k) when a weight is given]; then the usual
#             per-token absmax int8 quantisation of x_n.
#   SwiGLU:   h = fp32(silu(g) * u), silu(g) = fp32(g / fp32(1 + exp32(-g))),
#             exp32 below; then the usual quantisation of h.

def rmsnorm(X: np.ndarray, eps: float = 1e-6, w: np.ndarray | None = None, return_r: bool = False):
    """RMSNorm of each row (the reading above); X holds fp32 values (bf16 widened).
    With return_r, also the per-row fp32 factor r = 1 / sqrt(ms + eps)."""
    import math
    X = np.ascontiguousarray(X, dtype=np.float32)
    T, K = X.shape
    out = np.empty_like(X)
    rs = np.empty((T,), np.float32)
    for t in range(T):
        sq = X[t].astype(np.float64) ** 2          # exact: squares of fp32 values fit fp64
        S = math.fsum(sq.tolist())                 # exact sum, rounded once
        ms = np.float32(S / K)
        tt = np.float32(ms + np.float32(eps))
        r = np.float32(np.float32(1.0) / np.sqrt(tt))
        xn = (X[t] * r).astype(np.float32)
        if w is not None:
            xn = (xn * np.asarray(w, np.float32)).astype(np.float32)
        out[t] = xn
        rs[t] = r
    return (out, rs) if return_r else out


def exp32(x: np.ndarray) -> np.ndarray:
    """exp in fp32 by Cody-Waite range reduction (x = n ln2 + r, ln2 split in two
    parts) and the degree-6 Taylor polynomial of e^r on |r| <= ln2 / 2, each
    step one IEEE fp32 operation (no fused multiply-add); x clamped to [-87, 88]."""
    x = np.clip(np.asarray(x, np.float32), np.float32(-87.0), np.float32(88.0)).astype(np.float32)

    def f(bits):   # constants as exact fp32 bit patterns
        return np.uint32(bits).view(np.float32)
    log2e, ln2_hi, ln2_lo = f(0x3fb8aa3b), f(0x3f317200), f(0x35bfbe8e)   # ln2_hi has 16 significant bits
    n = np.rint((x * log2e).astype(np.float32)).astype(np.float32)
    r = (x - (n * ln2_hi).astype(np.float32)).astype(np.float32)
    r = (r - (n * ln2_lo).astype(np.float32)).astype(np.float32)
    p = f(0x3ab60b61)                                                    # 1/720
    for c in (f(0x3c088889), f(0x3d2aaaab), f(0x3e2aaaab), np.float32(0.5), np.float32(1.0), np.float32(1.0)):
        p = ((p * r).astype(np.float32) + c).astype(np.float32)          # 1/120, 1/24, 1/6, 1/2, 1, 1
    scale = ((n.astype(np.int32) + 127) << 23).astype(np.int32).view(np.float32)
    return (p * scale).astype(np.float32)


def swiglu(G: np.ndarray, U: np.ndarray) -> np.ndarray:
    """h = silu(g) * u with the reading above (fp32)."""
    G = np.ascontiguousarray(G, dtype=np.float32)
    U = np.ascontiguousarray(U, dtype=np.float32)
    e = exp32(-G)
    silu = (G / (np.float32(1.0) + e).astype(np.float32)).astype(np.float32)
    return (silu * U).astype(np.float32)


def wgrad(dY: np.ndarray, X: np.ndarray) -> np.ndarray:
    """dW[n, k] = sum_t dY[t, n] X[t, k] in fp64 ("Sparse-BitNet", section 2
    "Training Strategie": gradients reach every master straight through the
    quantisers and the mask; both quantisers act as the identity backward).
    dY and X hold fp32 values (bf16 widened); products and sum in fp64."""
    return np.asarray(dY, np.float64).T @ np.asarray(X, np.float64)


def adamw(W, G, M, V, lr, b1, b2, eps, wd, c1, c2):
    """One AdamW step in fp32, each operation rounded once, in this order:
    m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) (g g);
    u = (m / c1) / (sqrt(v / c2) + eps);  w = w - lr (u + wd w).
    c1, c2 are the bias corrections 1 - b1^t, 1 - b2^t (inputs).  Returns
    (W, M, V) as new fp32 arrays."""
    f = np.float32
    W, G, M, V = (np.asarray(a, f) for a in (W, G, M, V))
    lr, b1, b2, eps, wd, c1, c2 = (f(x) for x in (lr, b1, b2, eps, wd, c1, c2))
    omb1, omb2 = f(f(1.0) - b1), f(f(1.0) - b2)
    M = (b1 * M).astype(f) + (omb1 * G).astype(f)
    M = M.astype(f)
    GG = (G * G).astype(f)
    V = ((b2 * V).astype(f) + (omb2 * GG).astype(f)).astype(f)
    mh = (M / c1).astype(f)
    vh = (V / c2).astype(f)
    den = (np.sqrt(vh).astype(f) + eps).astype(f)
    u = (mh / den).astype(f)
    W = (W - (lr * (u + (wd * W).astype(f)).astype(f)).astype(f)).astype(f)
    return W, M, V

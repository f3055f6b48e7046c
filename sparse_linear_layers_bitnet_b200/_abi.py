"""ctypes binding of libbitnet_sparse.so (the C ABI in include/bitnet_sparse.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If the
library is missing the import fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitnet_sparse.so")

BITNET_OK = 0
BITNET_ERR_INVALID_ARG = 1
BITNET_ERR_UNSUPPORTED = 2
BITNET_ERR_WORKSPACE = 3
BITNET_ERR_CUDA = 4
BITNET_ERR_TIMEOUT = 5

BITNET_F32 = 0
BITNET_BF16 = 1

# Every symbol include/bitnet_sparse.h declares.
EXPORTED = [
    "bitnet_mma_meta_bytes", "bitnet_dec_bytes",
    "bitnet_pack_workspace_size", "bitnet_pack_nm", "bitnet_pack_nm_noalloc",
    "bitnet_pack_update_workspace_size", "bitnet_pack_nm_update",
    "bitnet_pack_update_batch_workspace_size", "bitnet_pack_nm_update_batch",
    "bitnet_pack_6of8_windows", "bitnet_quant_act_lift_6of8",
    "bitnet_quant_act", "bitnet_rmsnorm_quant", "bitnet_swiglu_quant",
    "bitnet_linear_workspace_size", "bitnet_sparse_linear",
    "bitnet_quant_linear_workspace_size", "bitnet_quant_linear",
    "bitnet_decode_chain_workspace_size", "bitnet_decode_chain",
    "bitnet_dgrad_workspace_size", "bitnet_dgrad",
    "bitnet_wgrad_workspace_size", "bitnet_wgrad", "bitnet_adamw_workspace_size", "bitnet_adamw_step",
    "bitnet_adamw_batch_workspace_size", "bitnet_adamw_step_batch",
    "bitnet_wait_selftest", "bitnet_tensor_peak", "bitnet_read_device_status", "bitnet_status_string", "bitnet_last_error", "bitnet_abi_version",
]


class BitnetPackedW(ctypes.Structure):
    _fields_ = [
        ("n_out", ctypes.c_int64),
        ("k", ctypes.c_int64),
        ("n", ctypes.c_int32),
        ("m", ctypes.c_int32),
        ("gamma", ctypes.c_void_p),
        ("group_bytes", ctypes.c_void_p),
        ("mma_vals", ctypes.c_void_p),
        ("mma_meta", ctypes.c_void_p),
        ("dec_codes", ctypes.c_void_p),
    ]


class BitnetPackItem(ctypes.Structure):
    _fields_ = [
        ("W", ctypes.c_void_p),
        ("out", ctypes.POINTER(BitnetPackedW)),
        ("mask_bits", ctypes.c_void_p),
        ("w_dtype", ctypes.c_int32),
        ("gamma_known", ctypes.c_int32),
    ]


class BitnetAdamWItem(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("dW", ctypes.c_void_p), ("m", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("gamma_out", ctypes.c_void_p)]


class BitnetAdamWHparams(ctypes.Structure):
    _fields_ = [(name, ctypes.c_float) for name in
                ("lr", "beta1", "beta2", "eps", "weight_decay", "bias_correction1", "bias_correction2")]


class BitnetChainOp(ctypes.Structure):
    _fields_ = [
        ("X", ctypes.c_void_p),
        ("W", ctypes.POINTER(BitnetPackedW)),
        ("Y", ctypes.c_void_p),
        ("acc_out", ctypes.c_void_p),
        ("xq_out", ctypes.c_void_p),
        ("absmax_out", ctypes.c_void_p),
        ("wait_prev", ctypes.c_int32),
    ]


class BitnetError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m sparse_linear_layers_bitnet_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    P, I64, SZ, F, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float, ctypes.c_int
    sig = {
        "bitnet_mma_meta_bytes": (SZ, [I64, I64]),
        "bitnet_dec_bytes": (SZ, [I64, I64]),
        "bitnet_pack_workspace_size": (SZ, [I64, I64]),
        "bitnet_pack_nm": (I32, [P, ctypes.POINTER(BitnetPackedW), F, P, P, SZ, P]),
        "bitnet_pack_nm_noalloc": (I32, [P, ctypes.POINTER(BitnetPackedW), F, P, P]),
        "bitnet_pack_update_workspace_size": (SZ, [I64, I64]),
        "bitnet_pack_nm_update": (I32, [P, ctypes.POINTER(BitnetPackedW), F, P, P, SZ, P]),
        "bitnet_pack_update_batch_workspace_size": (SZ, [ctypes.POINTER(BitnetPackItem), I32]),
        "bitnet_pack_nm_update_batch": (I32, [ctypes.POINTER(BitnetPackItem), I32, F, P, SZ, P]),
        "bitnet_pack_6of8_windows": (I32, [P, I64, F, ctypes.POINTER(BitnetPackedW), P, P, SZ, P]),
        "bitnet_quant_act_lift_6of8": (I32, [P, I32, I64, I64, F, P, P, P]),
        "bitnet_quant_act": (I32, [P, I32, I64, I64, F, P, P, P]),
        "bitnet_rmsnorm_quant": (I32, [P, P, I64, I64, F, F, P, P, P, P]),
        "bitnet_swiglu_quant": (I32, [P, P, I64, I64, I64, F, P, P, P]),
        "bitnet_linear_workspace_size": (SZ, []),
        "bitnet_sparse_linear": (I32, [P, P, ctypes.POINTER(BitnetPackedW), I64, P, I32, P, P, SZ, P]),
        "bitnet_quant_linear_workspace_size": (SZ, [I64, I64]),
        "bitnet_quant_linear": (I32, [P, I32, F, ctypes.POINTER(BitnetPackedW), I64, P, I32, P, P, P, P, SZ, P]),
        "bitnet_decode_chain_workspace_size": (SZ, [I32]),
        "bitnet_decode_chain": (I32, [ctypes.POINTER(BitnetChainOp), I32, I64, I32, I32, F, P, SZ, P]),
        "bitnet_dgrad_workspace_size": (SZ, [I64, I64]),
        "bitnet_dgrad": (I32, [P, I32, ctypes.POINTER(BitnetPackedW), I64, P, I32, P, SZ, P]),
        "bitnet_wgrad_workspace_size": (SZ, []),
        "bitnet_wgrad": (I32, [P, P, I64, I64, I64, P, I32, P, SZ, P]),
        "bitnet_adamw_workspace_size": (SZ, []),
        "bitnet_adamw_step": (I32, [P, P, P, P, I64, ctypes.POINTER(BitnetAdamWHparams), F, P, P, SZ, P]),
        "bitnet_adamw_batch_workspace_size": (SZ, [I32]),
        "bitnet_adamw_step_batch": (I32, [ctypes.POINTER(BitnetAdamWItem), I32, ctypes.POINTER(BitnetAdamWHparams), F,
                                          P, SZ, P]),
        "bitnet_wait_selftest": (I32, [P, SZ, I32, P]),
        "bitnet_tensor_peak": (I32, [I32, I64, P, P, SZ, P]),
        "bitnet_read_device_status": (I32, [P, P]),
        "bitnet_status_string": (ctypes.c_char_p, [I32]),
        "bitnet_last_error": (ctypes.c_char_p, []),
        "bitnet_abi_version": (I32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != BITNET_OK:
        lib = load()
        raise BitnetError(status, where, lib.bitnet_last_error().decode(errors="replace"))


# ------------------------------------------------------------------ torch helpers

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(dt) -> int:
    torch = _torch()
    if dt == torch.float32:
        return BITNET_F32
    if dt == torch.bfloat16:
        return BITNET_BF16
    raise ValueError(f"unsupported dtype {dt}")


class PackedWeights:
    """Device buffers of one packed layer (see bitnet_packed_w in the header)."""

    def __init__(self, n_out: int, k: int, device="cuda", group_bytes=True, mma=True, dec=True,
                 n: int = 2, m: int = 4):
        torch = _torch()
        lib = load()
        self.n_out, self.k, self.n, self.m = int(n_out), int(k), int(n), int(m)
        self.gamma = torch.zeros(1, dtype=torch.float32, device=device)
        self.group_bytes = torch.empty((n_out, k // 4), dtype=torch.uint8, device=device) if group_bytes else None
        self.mma_vals = torch.empty((n_out, k // 2), dtype=torch.int8, device=device) if mma else None
        self.mma_meta = (torch.empty(lib.bitnet_mma_meta_bytes(n_out, k), dtype=torch.uint8, device=device)
                         if mma else None)
        nd = lib.bitnet_dec_bytes(n_out, k)
        self.dec_codes = torch.empty(nd, dtype=torch.uint8, device=device) if (dec and nd > 0) else None
        self._struct = None

    def struct(self) -> BitnetPackedW:
        s = BitnetPackedW()
        s.n_out, s.k, s.n, s.m = self.n_out, self.k, self.n, self.m
        s.gamma = self.gamma.data_ptr()
        s.group_bytes = self.group_bytes.data_ptr() if self.group_bytes is not None else None
        s.mma_vals = self.mma_vals.data_ptr() if self.mma_vals is not None else None
        s.mma_meta = self.mma_meta.data_ptr() if self.mma_meta is not None else None
        s.dec_codes = self.dec_codes.data_ptr() if self.dec_codes is not None else None
        self._struct = s
        return s


class Workspace:
    """A device byte buffer for the ws argument of the entry points."""

    def __init__(self, nbytes: int, device="cuda"):
        torch = _torch()
        self.nbytes = int(max(nbytes, 256))
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def bitnet_pack_nm(W, out: PackedWeights, eps: float = 1e-5, mask_bits=None, ws: Workspace | None = None,
                   stream=None):
    lib = load()
    assert W.dtype == _torch().float32 and W.is_contiguous()
    if ws is None:
        ws = Workspace(lib.bitnet_pack_workspace_size(out.n_out, out.k), W.device)
    st = out.struct()
    check(lib.bitnet_pack_nm(_ptr(W), ctypes.byref(st), ctypes.c_float(eps), _ptr(mask_bits), ws.ptr,
                             ws.nbytes, _stream(stream)), "bitnet_pack_nm")
    return out


def bitnet_pack_nm_update(W, out: PackedWeights, eps: float = 1e-5, mask_bits=None, ws: Workspace | None = None,
                          stream=None):
    """Per-step pack reusing out.gamma (the previous gamma of this matrix) as a hint."""
    lib = load()
    assert W.dtype == _torch().float32 and W.is_contiguous()
    if ws is None:
        ws = Workspace(lib.bitnet_pack_update_workspace_size(out.n_out, out.k), W.device)
    st = out.struct()
    check(lib.bitnet_pack_nm_update(_ptr(W), ctypes.byref(st), ctypes.c_float(eps), _ptr(mask_bits), ws.ptr,
                                    ws.nbytes, _stream(stream)), "bitnet_pack_nm_update")
    return out


class PackBatch:
    """A fixed list of (W, PackedWeights[, mask_bits]) for bitnet_pack_nm_update_batch
    (W: fp32 or bf16 masters).  gamma_known: every out.gamma already is the exact
    gamma of its W (as bitnet_adamw_step leaves it): one read of W, no sum.

    The descriptor array and the workspace are built once, so the same batch
    can be repacked every step (or captured in a CUDA graph) without
    rebuilding them.
    """

    def __init__(self, items, eps: float = 1e-5, device="cuda", gamma_known: bool = False):
        lib = load()
        self.n = len(items)
        self.eps = float(eps)
        self._keep = []
        arr = (BitnetPackItem * max(self.n, 1))()
        for i, it in enumerate(items):
            W, out = it[0], it[1]
            mask = it[2] if len(it) > 2 else None
            assert W.dtype in (_torch().float32, _torch().bfloat16) and W.is_contiguous()
            st = out.struct()
            self._keep.append((st, W, out, mask))
            arr[i].W = W.data_ptr()
            arr[i].w_dtype = _dtype_code(W.dtype)
            arr[i].out = ctypes.pointer(st)
            arr[i].mask_bits = mask.data_ptr() if mask is not None else None
            arr[i].gamma_known = 1 if gamma_known else 0
        self._arr = arr
        self.ws = Workspace(lib.bitnet_pack_update_batch_workspace_size(arr, self.n), device)

    def __call__(self, stream=None):
        lib = load()
        check(lib.bitnet_pack_nm_update_batch(self._arr, self.n, ctypes.c_float(self.eps), self.ws.ptr,
                                              self.ws.nbytes, _stream(stream)), "bitnet_pack_nm_update_batch")


def bitnet_pack_nm_update_batch(items, eps: float = 1e-5, stream=None) -> PackBatch:
    """Per-step pack of many matrices (each out.gamma is its hint); returns the batch for reuse."""
    b = PackBatch(items, eps, items[0][0].device if items else "cuda")
    b(stream)
    return b


def bitnet_wgrad(dY, X, dW=None, accumulate: bool = False, ws: "Workspace | None" = None, stream=None):
    """dW[n, k] (+)= sum_t dY[t, n] X[t, k] (bf16 in, fp32 out)."""
    torch = _torch()
    lib = load()
    assert dY.dtype == torch.bfloat16 and X.dtype == torch.bfloat16 and dY.is_contiguous() and X.is_contiguous()
    T, n_out = dY.shape
    assert X.shape[0] == T
    k = X.shape[1]
    if dW is None:
        dW = torch.empty((n_out, k), dtype=torch.float32, device=dY.device)
    if ws is None:
        ws = Workspace(lib.bitnet_wgrad_workspace_size(), dY.device)
    check(lib.bitnet_wgrad(_ptr(dY), _ptr(X), T, n_out, k, _ptr(dW), 1 if accumulate else 0, ws.ptr, ws.nbytes,
                           _stream(stream)), "bitnet_wgrad")
    return dW


def bitnet_adamw_step(W, dW, m, v, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.95, eps: float = 1e-8,
                      weight_decay: float = 0.0, gamma_out=None, eps_gamma: float = 1e-5,
                      ws: "Workspace | None" = None, stream=None):
    """AdamW on fp32 masters in place; writes the exact absmean gamma of the new W to gamma_out."""
    torch = _torch()
    lib = load()
    for t in (W, dW, m, v):
        assert t.dtype == torch.float32 and t.is_contiguous()
    if gamma_out is None:
        gamma_out = torch.empty(1, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = Workspace(lib.bitnet_adamw_workspace_size(), W.device)
    h = BitnetAdamWHparams(lr, beta1, beta2, eps, weight_decay, adam_bias_correction(beta1, step),
                           adam_bias_correction(beta2, step))
    check(lib.bitnet_adamw_step(_ptr(W), _ptr(dW), _ptr(m), _ptr(v), W.numel(), ctypes.byref(h),
                                ctypes.c_float(eps_gamma), _ptr(gamma_out), ws.ptr, ws.nbytes, _stream(stream)),
          "bitnet_adamw_step")
    return gamma_out


class AdamWBatch:
    """A fixed list of (W, dW, m, v, gamma_out) for bitnet_adamw_step_batch; the
    descriptors and the workspace are built once, each call runs one step."""

    def __init__(self, items, device="cuda"):
        torch = _torch()
        lib = load()
        self.n = len(items)
        arr = (BitnetAdamWItem * max(self.n, 1))()
        self._keep = []
        for i, (W, G, M, V, gamma) in enumerate(items):
            for t in (W, G, M, V, gamma):
                assert t.dtype == torch.float32 and t.is_contiguous()
            self._keep.append((W, G, M, V, gamma))
            arr[i] = BitnetAdamWItem(W.data_ptr(), G.data_ptr(), M.data_ptr(), V.data_ptr(), W.numel(),
                                     gamma.data_ptr())
        self._arr = arr
        self.ws = Workspace(max(lib.bitnet_adamw_batch_workspace_size(self.n), 16), device)

    def __call__(self, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.95, eps: float = 1e-8,
                 weight_decay: float = 0.0, eps_gamma: float = 1e-5, stream=None):
        lib = load()
        h = BitnetAdamWHparams(lr, beta1, beta2, eps, weight_decay, adam_bias_correction(beta1, step),
                               adam_bias_correction(beta2, step))
        check(lib.bitnet_adamw_step_batch(self._arr, self.n, ctypes.byref(h), ctypes.c_float(eps_gamma), self.ws.ptr,
                                          self.ws.nbytes, _stream(stream)), "bitnet_adamw_step_batch")


def adam_bias_correction(beta: float, step: int) -> float:
    """fp32(1 - beta^step), with beta^step formed by repeated fp64 multiplication."""
    import numpy as np
    p = 1.0
    for _ in range(step):
        p *= float(np.float32(beta))
    return float(np.float32(1.0 - p))


def packed_6of8(n_out: int, k: int, device="cuda", mma=True, dec=False) -> "PackedWeights":
    """Buffers of the 2:4 window layout of a [n_out, k] 6:8 matrix (width k/2*3)."""
    return PackedWeights(n_out, k // 2 * 3, device, group_bytes=True, mma=mma, dec=dec)


def bitnet_pack_6of8_windows(W, out: "PackedWeights", eps: float = 1e-5, mask_bits=None, ws=None, stream=None):
    lib = load()
    assert W.dtype == _torch().float32 and W.is_contiguous()
    if ws is None:
        ws = Workspace(lib.bitnet_pack_workspace_size(W.shape[0], W.shape[1]), W.device)
    st = out.struct()
    check(lib.bitnet_pack_6of8_windows(_ptr(W), W.shape[1], ctypes.c_float(eps), ctypes.byref(st), _ptr(mask_bits),
                                       ws.ptr, ws.nbytes, _stream(stream)), "bitnet_pack_6of8_windows")
    return out


def bitnet_quant_act_lift_6of8(X, eps: float = 1e-5, Xl=None, absmax=None, stream=None):
    torch = _torch()
    lib = load()
    assert X.is_contiguous() and X.dim() == 2
    T, K = X.shape
    if Xl is None:
        Xl = torch.empty((T, K // 2 * 3), dtype=torch.int8, device=X.device)
    if absmax is None:
        absmax = torch.empty((T,), dtype=torch.float32, device=X.device)
    check(lib.bitnet_quant_act_lift_6of8(_ptr(X), _dtype_code(X.dtype), T, K, ctypes.c_float(eps), _ptr(Xl),
                                         _ptr(absmax), _stream(stream)), "bitnet_quant_act_lift_6of8")
    return Xl, absmax


def bitnet_quant_act(X, eps: float = 1e-5, Xq=None, absmax=None, stream=None):
    torch = _torch()
    lib = load()
    assert X.is_contiguous() and X.dim() == 2
    T, K = X.shape
    if Xq is None:
        Xq = torch.empty((T, K), dtype=torch.int8, device=X.device)
    if absmax is None:
        absmax = torch.empty((T,), dtype=torch.float32, device=X.device)
    check(lib.bitnet_quant_act(_ptr(X), _dtype_code(X.dtype), T, K, ctypes.c_float(eps), _ptr(Xq), _ptr(absmax),
                               _stream(stream)), "bitnet_quant_act")
    return Xq, absmax


def bitnet_rmsnorm_quant(X, w=None, eps_norm: float = 1e-6, eps_act: float = 1e-5, Xq=None, absmax=None,
                         rinv=None, stream=None):
    """RMSNorm of each bf16 row of X (optional fp32 weight w), quantised per token to int8."""
    torch = _torch()
    lib = load()
    assert X.is_contiguous() and X.dim() == 2 and X.dtype == torch.bfloat16
    assert w is None or (w.is_contiguous() and w.dtype == torch.float32 and w.numel() == X.shape[1])
    T, K = X.shape
    if Xq is None:
        Xq = torch.empty((T, K), dtype=torch.int8, device=X.device)
    if absmax is None:
        absmax = torch.empty((T,), dtype=torch.float32, device=X.device)
    check(lib.bitnet_rmsnorm_quant(_ptr(X), _ptr(w), T, K, ctypes.c_float(eps_norm), ctypes.c_float(eps_act),
                                   _ptr(Xq), _ptr(absmax), _ptr(rinv), _stream(stream)), "bitnet_rmsnorm_quant")
    return Xq, absmax


def bitnet_swiglu_quant(GU, F: int | None = None, eps_act: float = 1e-5, Xq=None, absmax=None, stream=None):
    """silu(gate) * up of a bf16 [T, 2F] buffer (gate = columns [0, F), up = [F, 2F)), quantised per token."""
    torch = _torch()
    lib = load()
    assert GU.dim() == 2 and GU.dtype == torch.bfloat16 and GU.stride(1) == 1
    T = GU.shape[0]
    if F is None:
        F = GU.shape[1] // 2
    assert GU.shape[1] >= 2 * F
    if Xq is None:
        Xq = torch.empty((T, F), dtype=torch.int8, device=GU.device)
    if absmax is None:
        absmax = torch.empty((T,), dtype=torch.float32, device=GU.device)
    G = GU.data_ptr()
    U = G + 2 * F
    check(lib.bitnet_swiglu_quant(ctypes.c_void_p(G), ctypes.c_void_p(U), GU.stride(0), T, F, ctypes.c_float(eps_act),
                                  _ptr(Xq), _ptr(absmax), _stream(stream)), "bitnet_swiglu_quant")
    return Xq, absmax


def bitnet_sparse_linear(Xq, absmax, W: PackedWeights, Y=None, y_dtype=None, acc_out=None,
                         ws: Workspace | None = None, stream=None):
    torch = _torch()
    lib = load()
    T = Xq.shape[0]
    if y_dtype is None:
        y_dtype = torch.bfloat16
    if Y is None:
        Y = torch.empty((T, W.n_out), dtype=y_dtype, device=Xq.device)
    if ws is None:
        ws = Workspace(lib.bitnet_linear_workspace_size(), Xq.device)
    st = W.struct()
    check(lib.bitnet_sparse_linear(_ptr(Xq), _ptr(absmax), ctypes.byref(st), T, _ptr(Y), _dtype_code(Y.dtype),
                                   _ptr(acc_out), ws.ptr, ws.nbytes, _stream(stream)), "bitnet_sparse_linear")
    return Y


def bitnet_quant_linear(X, W: PackedWeights, eps: float = 1e-5, Y=None, y_dtype=None, acc_out=None, xq_out=None,
                        absmax_out=None, ws: Workspace | None = None, stream=None):
    """Fused per-token quantisation + sparse linear (one kernel for decode batches)."""
    torch = _torch()
    lib = load()
    T = X.shape[0]
    if y_dtype is None:
        y_dtype = torch.bfloat16
    if Y is None:
        Y = torch.empty((T, W.n_out), dtype=y_dtype, device=X.device)
    if ws is None:
        ws = Workspace(lib.bitnet_quant_linear_workspace_size(T, W.k), X.device)
    st = W.struct()
    check(lib.bitnet_quant_linear(_ptr(X), _dtype_code(X.dtype), ctypes.c_float(eps), ctypes.byref(st), T, _ptr(Y),
                                  _dtype_code(Y.dtype), _ptr(acc_out), _ptr(xq_out), _ptr(absmax_out), ws.ptr,
                                  ws.nbytes, _stream(stream)), "bitnet_quant_linear")
    return Y


class DecodeChain:
    """A fixed sequence of decode projections for bitnet_decode_chain.

    ops: list of dicts with keys X, W (PackedWeights), Y and optionally
    acc_out, xq_out, absmax_out, wait_prev (default 1).  The descriptor array
    is built once and kept alive with the chain, so the same call can be
    repeated (or captured in a CUDA graph) without rebuilding it.
    """

    def __init__(self, ops, x_dtype, y_dtype, eps: float = 1e-5, device="cuda"):
        lib = load()
        self.n = len(ops)
        self.T = int(ops[0]["X"].shape[0]) if ops else 0
        self.eps = float(eps)
        self.x_code, self.y_code = _dtype_code(x_dtype), _dtype_code(y_dtype)
        self._keep = []
        arr = (BitnetChainOp * max(self.n, 1))()
        for i, o in enumerate(ops):
            st = o["W"].struct()
            self._keep.append(st)
            arr[i].X = o["X"].data_ptr()
            arr[i].W = ctypes.pointer(st)
            arr[i].Y = o["Y"].data_ptr()
            arr[i].acc_out = o["acc_out"].data_ptr() if o.get("acc_out") is not None else None
            arr[i].xq_out = o["xq_out"].data_ptr() if o.get("xq_out") is not None else None
            arr[i].absmax_out = o["absmax_out"].data_ptr() if o.get("absmax_out") is not None else None
            arr[i].wait_prev = int(o.get("wait_prev", 1))
        self._arr = arr
        self.ws = Workspace(lib.bitnet_decode_chain_workspace_size(self.n), device)

    def __call__(self, stream=None):
        lib = load()
        check(lib.bitnet_decode_chain(self._arr, self.n, self.T, self.x_code, self.y_code, ctypes.c_float(self.eps),
                                      self.ws.ptr, self.ws.nbytes, _stream(stream)), "bitnet_decode_chain")


def bitnet_decode_chain(ops, eps: float = 1e-5, y_dtype=None, stream=None) -> DecodeChain:
    """Runs ops (see DecodeChain) once and returns the chain for reuse."""
    torch = _torch()
    x_dtype = ops[0]["X"].dtype if ops else torch.bfloat16
    if y_dtype is None:
        y_dtype = ops[0]["Y"].dtype if ops else torch.bfloat16
    ch = DecodeChain(ops, x_dtype, y_dtype, eps, ops[0]["X"].device if ops else "cuda")
    ch(stream)
    return ch


def bitnet_dgrad(dY, W: PackedWeights, dX=None, dx_dtype=None, ws: Workspace | None = None, stream=None):
    torch = _torch()
    lib = load()
    T = dY.shape[0]
    if dx_dtype is None:
        dx_dtype = torch.float32
    if dX is None:
        dX = torch.empty((T, W.k), dtype=dx_dtype, device=dY.device)
    if ws is None:
        ws = Workspace(lib.bitnet_dgrad_workspace_size(W.n_out, W.k), dY.device)
    st = W.struct()
    check(lib.bitnet_dgrad(_ptr(dY), _dtype_code(dY.dtype), ctypes.byref(st), T, _ptr(dX), _dtype_code(dX.dtype),
                           ws.ptr, ws.nbytes, _stream(stream)), "bitnet_dgrad")
    return dX


def bitnet_wait_selftest(limit_us: int = 50000, device="cuda", stream=None) -> int:
    """Runs both kinds of bounded wait on events that never happen (limit limit_us)
    and returns the device status code that follows (BITNET_ERR_TIMEOUT expected)."""
    lib = load()
    ws = Workspace(lib.bitnet_decode_chain_workspace_size(1), device)
    check(lib.bitnet_wait_selftest(ws.ptr, ws.nbytes, int(limit_us), _stream(stream)), "bitnet_wait_selftest")
    return lib.bitnet_read_device_status(ws.ptr, _stream(stream))


def bitnet_tensor_peak(kind: int, iters: int, ws: Workspace, stream=None) -> float:
    """Launches the tensor-core ceiling loop (kind 0 sparse int8, 1 dense int8,
    2 bf16) and returns the dense-equivalent operations of the launch."""
    ops = ctypes.c_double(0.0)
    check(load().bitnet_tensor_peak(int(kind), int(iters), ctypes.byref(ops), ws.ptr, ws.nbytes, _stream(stream)),
          "bitnet_tensor_peak")
    return ops.value


def bitnet_read_device_status(ws: Workspace, stream=None) -> int:
    return load().bitnet_read_device_status(ws.ptr, _stream(stream))

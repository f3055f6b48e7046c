"""Host-side checks of the C-ABI library (no GPU needed, no compute calls).

The library must load on a machine without a GPU, export every symbol that
include/bitnet_sparse.h declares, report its buffer sizes, and reject bad
arguments on the host before any launch.  Every call below fails validation,
so none reaches a CUDA call.
"""
import ctypes
import os
import re
import subprocess

import pytest

from sparse_linear_layers_bitnet_b200 import _abi
from sparse_linear_layers_bitnet_b200 import build as nvbuild
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bitnet_sparse.h")


@pytest.fixture(scope="module")
def lib():
    nvbuild.build()
    return _abi.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(bitnet_[a-z_0-9]+)\s*\(", src))
    return sorted(names)


def test_header_and_binding_agree():
    assert sorted(_abi.EXPORTED) == declared_functions()


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (bitnet_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_library_links_no_torch_and_no_oracle():
    out = subprocess.run(["ldd", _abi.LIB_PATH], capture_output=True, text=True).stdout
    assert "torch" not in out and "oracle" not in out and "libcudart" not in out


def test_sizes(lib):
    assert lib.bitnet_abi_version() == 1
    # metadata: ceil(k/128) * ceil(n_out/128) blocks of 128 rows x 16 bytes
    assert lib.bitnet_mma_meta_bytes(256, 256) == 2 * 2 * 2048
    assert lib.bitnet_mma_meta_bytes(200, 352) == 3 * 2 * 2048
    assert lib.bitnet_mma_meta_bytes(8640, 3200) == 25 * 68 * 2048
    # decode layout: 0.25 byte per weight, tiles of 16 x 64
    assert lib.bitnet_dec_bytes(2560, 6912) == 2560 * 6912 // 4
    assert lib.bitnet_dec_bytes(200, 256) == 0
    assert lib.bitnet_pack_workspace_size(3200, 3200) >= 256 + 2048
    assert lib.bitnet_linear_workspace_size() >= 4
    assert lib.bitnet_dgrad_workspace_size(3200, 8640) >= 3200 * 8640 * 2


def _fake(addr=4096):
    return ctypes.c_void_p(addr)   # never dereferenced: every call below fails validation


def _pw(n_out=256, k=256, n=2, m=4, gamma=True, gb=True, mma=False, dec=False):
    s = _abi.BitnetPackedW()
    s.n_out, s.k, s.n, s.m = n_out, k, n, m
    s.gamma = 4096 if gamma else None
    s.group_bytes = 8192 if gb else None
    s.mma_vals = 16384 if mma else None
    s.mma_meta = 32768 if mma else None
    s.dec_codes = 65536 if dec else None
    return s


def test_pack_rejects_bad_arguments(lib):
    st = _pw()
    ws_n = lib.bitnet_pack_workspace_size(256, 256)
    assert lib.bitnet_pack_nm(None, ctypes.byref(st), 1e-5, None, _fake(), ws_n, None) == _abi.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(st), 1e-5, None, None, ws_n, None) == _abi.BITNET_ERR_WORKSPACE
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(st), 1e-5, None, _fake(), 16, None) == _abi.BITNET_ERR_WORKSPACE
    bad = _pw(n=6, m=8)
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(bad), 1e-5, None, _fake(), ws_n, None) == _abi.BITNET_ERR_UNSUPPORTED
    bad = _pw(n=3, m=5, gb=False)
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(bad), 1e-5, None, _fake(), ws_n, None) == _abi.BITNET_ERR_UNSUPPORTED
    bad = _pw(k=250)
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(bad), 1e-5, None, _fake(), ws_n, None) == _abi.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_pack_nm(_fake(4100), ctypes.byref(_pw()), 1e-5, None, _fake(), ws_n, None) == _abi.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(_pw()), -1.0, None, _fake(), ws_n, None) == _abi.BITNET_ERR_INVALID_ARG
    bad = _pw(gamma=False)
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(bad), 1e-5, None, _fake(), ws_n, None) == _abi.BITNET_ERR_INVALID_ARG
    bad = _pw(gb=False, dec=True)
    assert lib.bitnet_pack_nm(_fake(), ctypes.byref(bad), 1e-5, None, _fake(), ws_n, None) == _abi.BITNET_ERR_INVALID_ARG
    assert b"required" in lib.bitnet_last_error() or b"derived" in lib.bitnet_last_error()


def test_pack_noalloc_rejects_oversized_matrix_on_host(lib):
    # between the 2^34-weight limit and 2^40: refused before any device call
    bad = _pw(n_out=1 << 18, k=1 << 17)
    assert lib.bitnet_pack_nm_noalloc(_fake(), ctypes.byref(bad), 1e-5, None, None) == _abi.BITNET_ERR_UNSUPPORTED
    assert b"2^34" in lib.bitnet_last_error()


def test_quant_rejects_bad_arguments(lib):
    f = lib.bitnet_quant_act
    assert f(None, 0, 4, 256, 1e-5, _fake(), _fake(), None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(_fake(), 0, 4, 250, 1e-5, _fake(), _fake(), None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(_fake(), 7, 4, 256, 1e-5, _fake(), _fake(), None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(_fake(), 0, 4, 256, 0.0, _fake(), _fake(), None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(_fake(4104), 0, 4, 256, 1e-5, _fake(), _fake(), None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(_fake(), 0, -1, 256, 1e-5, _fake(), _fake(), None) == _abi.BITNET_ERR_INVALID_ARG


def test_block_quant_rejects_bad_arguments(lib):
    f = lib.bitnet_rmsnorm_quant
    ok = _abi.BITNET_OK
    bad = _abi.BITNET_ERR_INVALID_ARG
    assert f(None, None, 4, 256, 1e-6, 1e-5, _fake(), _fake(), None, None) == bad          # null X
    assert f(_fake(), None, 4, 252, 1e-6, 1e-5, _fake(), _fake(), None, None) == bad       # K % 8
    assert f(_fake(), None, 4, 65544, 1e-6, 1e-5, _fake(), _fake(), None, None) == bad     # K too large
    assert f(_fake(), None, 4, 256, 0.0, 1e-5, _fake(), _fake(), None, None) == bad        # eps_norm
    assert f(_fake(), None, 4, 256, 1e-6, -1.0, _fake(), _fake(), None, None) == bad       # eps_act
    assert f(_fake(4104), None, 4, 256, 1e-6, 1e-5, _fake(), _fake(), None, None) == bad   # X alignment
    assert f(_fake(), _fake(4098), 4, 256, 1e-6, 1e-5, _fake(), _fake(), None, None) == bad   # w alignment
    assert f(_fake(), None, -1, 256, 1e-6, 1e-5, _fake(), _fake(), None, None) == bad
    assert f(None, None, 0, 256, 1e-6, 1e-5, None, None, None, None) == ok                 # empty batch
    g = lib.bitnet_swiglu_quant
    assert g(None, _fake(), 512, 4, 256, 1e-5, _fake(), _fake(), None) == bad               # null G
    assert g(_fake(), _fake(), 512, 4, 252, 1e-5, _fake(), _fake(), None) == bad            # F % 8
    assert g(_fake(), _fake(), 100, 4, 256, 1e-5, _fake(), _fake(), None) == bad            # ld < F
    assert g(_fake(), _fake(), 1 << 17, 4, 51208, 1e-5, _fake(), _fake(), None) == bad      # F beyond shared memory
    assert g(_fake(), _fake(), 512, 4, 256, 0.0, _fake(), _fake(), None) == bad             # eps
    assert g(_fake(4097), _fake(), 512, 4, 256, 1e-5, _fake(), _fake(), None) == bad        # G alignment
    assert g(_fake(), _fake(), 512, 4, 256, 1e-5, _fake(4104), _fake(), None) == bad        # Xq alignment
    assert g(None, None, 512, 0, 256, 1e-5, None, None, None) == ok                         # empty batch


def test_train_step_entries_reject_bad_arguments(lib):
    bad = _abi.BITNET_ERR_INVALID_ARG
    ws = _fake()
    f = lib.bitnet_wgrad
    assert f(_fake(), _fake(), 64, 250, 256, _fake(), 0, ws, 1 << 20, None) == bad        # n_out % 8
    assert f(_fake(), _fake(), 64, 256, 252, _fake(), 0, ws, 1 << 20, None) == bad        # k % 8
    assert f(_fake(), _fake(), -1, 256, 256, _fake(), 0, ws, 1 << 20, None) == bad        # T < 0
    assert f(_fake(), _fake(), 64, 256, 256, None, 0, ws, 1 << 20, None) == bad           # null dW
    assert f(None, _fake(), 64, 256, 256, _fake(), 0, ws, 1 << 20, None) == bad           # null dY
    assert f(_fake(4104), _fake(), 64, 256, 256, _fake(), 0, ws, 1 << 20, None) == bad    # dY alignment
    assert f(_fake(), _fake(), 64, 256, 256, _fake(), 0, None, 0, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(None, None, 0, 256, 256, _fake(), 1, ws, 1 << 20, None) == _abi.BITNET_OK    # empty, accumulate
    g = lib.bitnet_adamw_step
    h = _abi.BitnetAdamWHparams(1e-3, 0.9, 0.95, 1e-8, 0.1, 0.1, 0.05)
    ok_args = (_fake(), _fake(), _fake(), _fake(), 1024, ctypes.byref(h), 1e-5, _fake(), ws, 1 << 20, None)
    assert g(_fake(), _fake(), _fake(), _fake(), 1022, ctypes.byref(h), 1e-5, _fake(), ws, 1 << 20, None) == bad
    assert g(None, *ok_args[1:]) == bad
    assert g(*ok_args[:7], None, *ok_args[8:]) == bad                                       # null gamma_out
    assert g(_fake(4104), *ok_args[1:]) == bad                                              # W alignment
    assert g(*ok_args[:8], None, 0, None) == _abi.BITNET_ERR_WORKSPACE
    for field, value in (("beta1", 1.0), ("beta2", -0.1), ("eps", 0.0), ("bias_correction1", 0.0), ("lr", -1.0)):
        hb = _abi.BitnetAdamWHparams(1e-3, 0.9, 0.95, 1e-8, 0.1, 0.1, 0.05)
        setattr(hb, field, value)
        assert g(*ok_args[:5], ctypes.byref(hb), *ok_args[6:]) == bad, field
    assert g(*ok_args[:5], None, *ok_args[6:]) == bad                                      # null hyper-parameters


def test_adamw_batch_rejects_bad_arguments(lib):
    bad = _abi.BITNET_ERR_INVALID_ARG
    h = _abi.BitnetAdamWHparams(1e-3, 0.9, 0.95, 1e-8, 0.1, 0.1, 0.05)
    items = (_abi.BitnetAdamWItem * 2)()
    for it in items:
        it.W, it.dW, it.m, it.v, it.n, it.gamma_out = 4096, 4096, 4096, 4096, 1024, 4096
    ws, n = _fake(), lib.bitnet_adamw_batch_workspace_size(2)
    assert n == 2 * lib.bitnet_adamw_workspace_size()
    assert lib.bitnet_adamw_step_batch(items, 0, ctypes.byref(h), 1e-5, None, 0, None) == _abi.BITNET_OK
    assert lib.bitnet_adamw_step_batch(items, -1, ctypes.byref(h), 1e-5, ws, n, None) == bad
    assert lib.bitnet_adamw_step_batch(items, 2, None, 1e-5, ws, n, None) == bad
    assert lib.bitnet_adamw_step_batch(items, 2, ctypes.byref(h), 1e-5, ws, n - 1, None) == _abi.BITNET_ERR_WORKSPACE
    items[1].n = 1022
    assert lib.bitnet_adamw_step_batch(items, 2, ctypes.byref(h), 1e-5, ws, n, None) == bad      # n % 4
    items[1].n = 1024
    items[1].v = 4100
    assert lib.bitnet_adamw_step_batch(items, 2, ctypes.byref(h), 1e-5, ws, n, None) == bad      # alignment
    items[1].v = 4096
    items[0].gamma_out = None
    assert lib.bitnet_adamw_step_batch(items, 2, ctypes.byref(h), 1e-5, ws, n, None) == bad      # null gamma


def test_wait_selftest_rejects_bad_arguments(lib):
    n = lib.bitnet_decode_chain_workspace_size(1)
    assert lib.bitnet_wait_selftest(None, n, 1000, None) == _abi.BITNET_ERR_WORKSPACE
    assert lib.bitnet_wait_selftest(_fake(), n - 1, 1000, None) == _abi.BITNET_ERR_WORKSPACE
    assert lib.bitnet_wait_selftest(_fake(4104), n, 1000, None) == _abi.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_wait_selftest(_fake(), n, 0, None) == _abi.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_wait_selftest(_fake(), n, 2000001, None) == _abi.BITNET_ERR_INVALID_ARG


def test_linear_rejects_bad_arguments(lib):
    f = lib.bitnet_sparse_linear
    ws = lib.bitnet_linear_workspace_size()
    st = _pw(gb=False, mma=False)
    # T > 8 needs the tensor-core layouts
    assert f(_fake(), _fake(), ctypes.byref(st), 64, _fake(), 0, None, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    st = _pw(k=272, mma=True)   # k % 32 != 0 on the tensor-core path
    assert f(_fake(), _fake(), ctypes.byref(st), 64, _fake(), 0, None, _fake(), ws, None) == _abi.BITNET_ERR_UNSUPPORTED
    st = _pw(mma=True)
    assert f(_fake(), _fake(), ctypes.byref(st), 64, _fake(), 0, None, None, ws, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(_fake(), _fake(), ctypes.byref(st), 64, _fake(), 0, None, _fake(), 0, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(_fake(), _fake(), ctypes.byref(st), 64, _fake(), 9, None, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    st = _pw(n=1, m=4, mma=True)
    assert f(_fake(), _fake(), ctypes.byref(st), 64, _fake(), 0, None, _fake(), ws, None) == _abi.BITNET_ERR_UNSUPPORTED
    assert f(None, _fake(), ctypes.byref(_pw()), 4, _fake(), 0, None, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG


def _chain(ops_specs):
    arr = (_abi.BitnetChainOp * max(len(ops_specs), 1))()
    keep = []
    for i, (st, x, y, wait) in enumerate(ops_specs):
        keep.append(st)
        arr[i].X = x
        arr[i].W = ctypes.pointer(st) if st is not None else None
        arr[i].Y = y
        arr[i].wait_prev = wait
    return arr, keep


def test_decode_chain_rejects_bad_arguments(lib):
    f = lib.bitnet_decode_chain
    ws = lib.bitnet_decode_chain_workspace_size(2)
    assert ws >= 256 + 8
    good = _pw(n_out=256, k=256, dec=True)
    arr, keep = _chain([(good, 4096, 8192, 1), (good, 4096, 8192, 1)])
    bf = _abi.BITNET_BF16
    assert f(arr, -1, 1, bf, bf, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(arr, 2, 9, bf, bf, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG    # T > 8
    assert f(arr, 2, 1, 7, bf, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG     # x dtype
    assert f(arr, 2, 1, bf, bf, 0.0, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG    # eps
    assert f(None, 2, 1, bf, bf, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(arr, 2, 1, bf, bf, 1e-5, None, ws, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(arr, 2, 1, bf, bf, 1e-5, _fake(), ws - 4, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(arr, 2, 1, bf, bf, 1e-5, _fake(4100), ws, None) == _abi.BITNET_ERR_INVALID_ARG   # ws alignment
    # nothing to do: no ops or no tokens
    assert f(arr, 0, 1, bf, bf, 1e-5, None, 0, None) == _abi.BITNET_OK
    assert f(arr, 2, 0, bf, bf, 1e-5, None, 0, None) == _abi.BITNET_OK
    bad_cases = [
        ((None, 4096, 8192, 1), _abi.BITNET_ERR_INVALID_ARG),                        # null W
        ((_pw(dec=False), 4096, 8192, 1), _abi.BITNET_ERR_INVALID_ARG),               # no decode layout
        ((_pw(n_out=256, k=288, dec=True), 4096, 8192, 1), _abi.BITNET_ERR_UNSUPPORTED),   # k % 64
        ((_pw(n_out=200, k=256, dec=True), 4096, 8192, 1), _abi.BITNET_ERR_UNSUPPORTED),   # n_out % 16
        ((_pw(n=1, m=4, dec=True), 4096, 8192, 1), _abi.BITNET_ERR_UNSUPPORTED),      # 2:4 only
        ((good, None, 8192, 1), _abi.BITNET_ERR_INVALID_ARG),                         # null X
        ((good, 4100, 8192, 1), _abi.BITNET_ERR_INVALID_ARG),                         # X alignment
        ((good, 4096, 8192, 2), _abi.BITNET_ERR_INVALID_ARG),                         # wait_prev
    ]
    for spec, want in bad_cases:
        arr2, keep2 = _chain([(good, 4096, 8192, 1), spec])
        assert f(arr2, 2, 1, bf, bf, 1e-5, _fake(), ws, None) == want, spec


def test_pack_update_batch_rejects_bad_arguments(lib):
    f = lib.bitnet_pack_nm_update_batch
    good = _pw(n_out=256, k=256, mma=True)
    arr = (_abi.BitnetPackItem * 2)()
    for i in range(2):
        arr[i].W = 4096
        arr[i].out = ctypes.pointer(good)
    ws = lib.bitnet_pack_update_batch_workspace_size(arr, 2)
    assert ws >= 2 * (256 + 2048) + 2 * 16384 * 4
    assert f(arr, -1, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(arr, 0, 1e-5, None, 0, None) == _abi.BITNET_OK
    assert f(None, 2, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(arr, 2, -1.0, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(arr, 2, 1e-5, None, ws, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(arr, 2, 1e-5, _fake(), ws - 4, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(arr, 2, 1e-5, _fake(4100), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    cases = [
        (_pw(n_out=256, k=264, mma=True), 4096, _abi.BITNET_ERR_UNSUPPORTED),    # k % 16
        (_pw(n_out=256, k=256, n=1, m=4), 4096, _abi.BITNET_ERR_UNSUPPORTED),    # 2:4 only
        (_pw(n_out=256, k=256, gamma=False), 4096, _abi.BITNET_ERR_INVALID_ARG),
        (good, None, _abi.BITNET_ERR_INVALID_ARG),                              # null W
        (good, 4100, _abi.BITNET_ERR_INVALID_ARG),                              # W alignment
        (_pw(n_out=200, k=256, dec=True), 4096, _abi.BITNET_ERR_INVALID_ARG),    # dec needs n_out % 16
    ]
    for st, w, want in cases:
        arr[1].W = w
        arr[1].out = ctypes.pointer(st)
        assert f(arr, 2, 1e-5, _fake(), ws, None) == want, (st.n_out, st.k, w)
    arr[1].W = 4096
    arr[1].out = ctypes.pointer(good)
    arr[1].w_dtype = 5
    assert f(arr, 2, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG       # bad master dtype
    arr[1].w_dtype = _abi.BITNET_BF16
    half = _pw(n_out=256, k=256)
    half.mma_vals = 16384                                                       # vals without meta
    arr[1].W = 4096
    arr[1].out = ctypes.pointer(half)
    assert f(arr, 2, 1e-5, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG


def test_dgrad_rejects_bad_arguments(lib):
    f = lib.bitnet_dgrad
    ws = lib.bitnet_dgrad_workspace_size(256, 256)
    st = _pw()
    assert f(_fake(), _abi.BITNET_F32, ctypes.byref(st), 64, _fake(), 0, _fake(), ws, None) == _abi.BITNET_ERR_UNSUPPORTED
    assert f(_fake(), _abi.BITNET_BF16, ctypes.byref(st), 64, _fake(), 0, _fake(), 100, None) == _abi.BITNET_ERR_WORKSPACE
    assert f(_fake(), _abi.BITNET_BF16, ctypes.byref(_pw(gb=False)), 64, _fake(), 0, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG
    assert f(_fake(), _abi.BITNET_BF16, ctypes.byref(_pw(n_out=250)), 64, _fake(), 0, _fake(), ws, None) == _abi.BITNET_ERR_INVALID_ARG


def test_status_strings(lib):
    for s in range(6):
        assert lib.bitnet_status_string(s)
    assert lib.bitnet_read_device_status(None, None) == _abi.BITNET_ERR_INVALID_ARG

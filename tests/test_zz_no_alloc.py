"""The allocation-free pack entry point against the workspace one (GPU).

bitnet_pack_nm_noalloc serves callers that cannot allocate device memory at
the call site (fixed memory pools, embedded runtimes, latency-critical paths):
its scratch lives in a fixed array inside the library.  It must give exactly
what bitnet_pack_nm gives, also when it is called twice in a row on different
matrices (the shared scratch is cleared by every call).  This file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

from sparse_linear_layers_bitnet_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _outputs(pw, mask):
    return {
        "gamma": pw.gamma.cpu().numpy().copy(),
        "group_bytes": pw.group_bytes.cpu().numpy().copy(),
        "mma_vals": pw.mma_vals.cpu().numpy().copy(),
        "mma_meta": pw.mma_meta.cpu().numpy().copy(),
        "dec_codes": pw.dec_codes.cpu().numpy().copy() if pw.dec_codes is not None else None,
        "mask": mask.cpu().numpy().copy(),
    }


def _reference(bn, W, n_out, k):
    pw = bn.PackedWeights(n_out, k)
    mask = torch.zeros(n_out * k // 8, dtype=torch.uint8, device="cuda")
    bn.bitnet_pack_nm(W, pw, 1e-5, mask_bits=mask)
    torch.cuda.synchronize()
    return _outputs(pw, mask)


def _noalloc(bn, lib, W, n_out, k):
    pw = bn.PackedWeights(n_out, k)
    mask = torch.zeros(n_out * k // 8, dtype=torch.uint8, device="cuda")
    st = pw.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.bitnet_pack_nm_noalloc(ctypes.c_void_p(W.data_ptr()), ctypes.byref(st), ctypes.c_float(1e-5),
                                    ctypes.c_void_p(mask.data_ptr()), stream)
    assert rc == 0, lib.bitnet_last_error()
    torch.cuda.synchronize()
    return _outputs(pw, mask)


def test_noalloc_pack_matches_workspace_pack_twice(cuda_device):
    import sparse_linear_layers_bitnet_b200 as bn
    lib = bn.load()
    cases = [(384, 1024, 3), (200, 352, 4)]   # two different matrices, one call each, in a row
    mats = [torch.from_numpy(synth.master_weights(n, k, 0.02, seed=s)).cuda() for n, k, s in cases]
    refs = [_reference(bn, W, n, k) for W, (n, k, _) in zip(mats, cases)]
    got = [_noalloc(bn, lib, W, n, k) for W, (n, k, _) in zip(mats, cases)]
    for r, g in zip(refs, got):
        for key in r:
            if r[key] is None:
                assert g[key] is None
            else:
                assert np.array_equal(r[key], g[key]), key


def test_noalloc_rejects_oversized_matrix(cuda_device):
    import sparse_linear_layers_bitnet_b200 as bn
    lib = bn.load()
    # 2^35 weights (just above the 2^34 limit) and 2^41: both refused before any pointer is used
    for n_out, k in ((1 << 18, 1 << 17), (1 << 21, 1 << 20)):
        st = bn.BitnetPackedW()
        st.n_out, st.k, st.n, st.m = n_out, k, 2, 4
        st.gamma = 4096
        rc = lib.bitnet_pack_nm_noalloc(ctypes.c_void_p(4096), ctypes.byref(st), ctypes.c_float(1e-5), None, None)
        assert rc == bn._abi.BITNET_ERR_UNSUPPORTED
        assert b"2^34" in lib.bitnet_last_error()

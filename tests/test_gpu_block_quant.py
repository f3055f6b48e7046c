"""GPU parity of the block epilogues fused into per-token quantisation
(RMSNorm -> int8, SwiGLU -> int8) against oracle.rmsnorm / oracle.swiglu
followed by oracle.quant_act: codes, absmax and the norm factor bit-exact.

"BitNet b1.58: Ternary Weights for 1.58-bit LLMs", "What this paper explains"
(LLaMA-alike blocks: RMSNorm, SwiGLU) and "The mechanism" (per-token absmax
int8 activations).
"""
import numpy as np
import pytest

import oracle
from sparse_linear_layers_bitnet_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def bn(cuda_device):
    import sparse_linear_layers_bitnet_b200 as m
    m.load()
    return m


def bf16_dev(a_f32):
    bits = synth.to_bf16_bits(a_f32)
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16), synth.bf16_bits_to_f32(bits)


def _rare_rows(X, rng):
    """Rows that leave the 128-bit window of the exact sum of squares."""
    T, K = X.shape
    if T > 0:
        X[0] = 0.0                                             # eps clamps
    if T > 1:
        X[1] = rng.standard_normal(K) * 1e-20                  # tiny squares (bins)
    if T > 2:
        X[2] = rng.standard_normal(K) * 3e4                    # huge squares (bins)
    if T > 3:
        sub = rng.integers(1, 128, K).astype(np.uint32) << 16  # bf16 subnormals
        X[3] = (sub.view(np.float32) * np.where(rng.random(K) < 0.5, -1, 1)).astype(np.float32)
    if T > 4:                                                  # mixed: window, bins and zeros in one row
        X[4, ::3] = 2e3
        X[4, 1::3] = 1e-25
        X[4, 2::7] = 0.0
    sign = np.where(rng.random(K) < 0.5, -1.0, 1.0)
    if T > 5:
        X[5] = rng.uniform(512.0, 1020.0, K) * sign            # top of the window: largest exact chunk sums
    if T > 6:
        X[6] = rng.uniform(1.0, 2.0, K) * 2.0 ** -29 * sign    # bottom of the window: smallest chunk sums
    return X


# K covers every register-cache width (chunks per thread 1, 2, 3, 4, 6, 8) and the
# re-reading kernel beyond them (K = 65536)
@pytest.mark.parametrize("T,K,weighted", [(1, 2560, False), (7, 3200, True), (64, 8192, False), (3, 8, True),
                                          (9, 1000, False), (5, 65536, True), (130, 2048, True), (6, 6144, True),
                                          (5, 12288, False), (6, 16384, True), (4, 16392, True)])
def test_rmsnorm_quant_parity(bn, T, K, weighted):
    rng = np.random.default_rng(T * 7 + K)
    X = synth.activations(T, K, seed=T + K, outlier_p=0.01)
    X = _rare_rows(X, rng)
    Xd, X32 = bf16_dev(X)
    w = (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32) if weighted else None
    xn, r_ref = oracle.rmsnorm(X32, 1e-6, w, return_r=True)
    xq_ref, a_ref = oracle.quant_act(xn, 1e-5)
    rinv = torch.full((T,), -1.0, dtype=torch.float32, device="cuda")
    wd = torch.from_numpy(w).cuda() if weighted else None
    Xq, a = bn.bitnet_rmsnorm_quant(Xd, wd, 1e-6, 1e-5, rinv=rinv)
    torch.cuda.synchronize()
    assert np.array_equal(rinv.cpu().numpy().view(np.uint32), r_ref.view(np.uint32))
    assert np.array_equal(a.cpu().numpy(), a_ref)
    assert np.array_equal(Xq.cpu().numpy(), xq_ref)


def test_rmsnorm_quant_unaligned_weight(bn):
    """A weight vector without 16-byte alignment takes the kernel that reads it
    one float at a time; same results."""
    T, K = 6, 3200
    rng = np.random.default_rng(11)
    X = _rare_rows(synth.activations(T, K, seed=12, outlier_p=0.01), rng)
    Xd, X32 = bf16_dev(X)
    w = (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    wbuf = torch.zeros(K + 1, dtype=torch.float32, device="cuda")
    wbuf[1:] = torch.from_numpy(w).cuda()
    xn, r_ref = oracle.rmsnorm(X32, 1e-6, w, return_r=True)
    xq_ref, a_ref = oracle.quant_act(xn, 1e-5)
    rinv = torch.empty((T,), dtype=torch.float32, device="cuda")
    Xq, a = bn.bitnet_rmsnorm_quant(Xd, wbuf[1:], 1e-6, 1e-5, rinv=rinv)
    torch.cuda.synchronize()
    assert np.array_equal(rinv.cpu().numpy(), r_ref)
    assert np.array_equal(a.cpu().numpy(), a_ref)
    assert np.array_equal(Xq.cpu().numpy(), xq_ref)


def _tie_rows():
    """Rows whose mean square lies exactly on, or a hair above, a rounding tie
    of fp32.  K = 8192 (a power of two, so S / K is exact):
    3584 x 4.0 and 2 x 2^-5 and j x 2^-4 give S = 57344 + j 2^-8 + 2^-9, so
    ms = m + 2^-22 with m = 7 + j 2^-21: halfway between two fp32 values.
    Extra elements d then decide the rounding (the fp64 ulp of S is 2^-37):
      d = 2^-19          S + 2^-38 is an fp64 tie and rounds back to S: ms on the tie;
      d = 2^-19, 2^-60   S + 2^-38 + 2^-120 rounds up in fp64: ms above the tie.
    Only a sum that keeps the 2^-120 term (a bin far below the window) until
    the single rounding gets the third row right."""
    K = 8192
    for j in range(0, 400, 2):   # even j: the tie rounds down; pick one where r tells the two apart
        m = np.float32(7.0 + j * 2.0 ** -21)
        up = np.nextafter(m, np.float32(8.0))
        r_m = np.float32(np.float32(1.0) / np.sqrt(m))
        r_up = np.float32(np.float32(1.0) / np.sqrt(up))
        if r_m != r_up:
            break
    rows = []
    for extra in ([], [2.0 ** -19], [2.0 ** -19, 2.0 ** -60], [2.0 ** -60]):
        x = np.zeros(K, np.float32)
        x[0:2 * 3584:2] = 4.0
        x[1], x[4001] = 2.0 ** -5, 2.0 ** -5
        x[3:3 + 2 * j:2] = 2.0 ** -4
        for q, v in enumerate(extra):
            x[8191 - 37 * q] = v
        rows.append(x)
    return np.stack(rows), j


def test_rmsnorm_quant_exact_sum_at_ties(bn):
    X, j = _tie_rows()
    Xd, X32 = bf16_dev(X)
    assert np.array_equal(X32, X)                      # every value is exact in bf16
    eps = 1e-30                                        # below half an ulp of ms: ms + eps == ms
    xn, r_ref = oracle.rmsnorm(X32, eps, None, return_r=True)
    assert r_ref[0] == r_ref[1] == r_ref[3] != r_ref[2]   # the rows discriminate an exact sum
    xq_ref, a_ref = oracle.quant_act(xn, 1e-5)
    rinv = torch.empty((X.shape[0],), dtype=torch.float32, device="cuda")
    Xq, a = bn.bitnet_rmsnorm_quant(Xd, None, eps, 1e-5, rinv=rinv)
    torch.cuda.synchronize()
    assert np.array_equal(rinv.cpu().numpy(), r_ref)
    assert np.array_equal(Xq.cpu().numpy(), xq_ref)
    assert np.array_equal(a.cpu().numpy(), a_ref)


def _gate_values(T, F, rng):
    G = (rng.standard_normal((T, F)) * 2.0).astype(np.float32)
    U = rng.standard_normal((T, F)).astype(np.float32)
    if T > 0:
        G[0, :8] = [-100.0, 100.0, -87.5, 88.5, 0.0, -0.0, 1e-30, -1e-38]   # clamps, zeros, tiny
    if T > 1:
        U[1] = 0.0                                                        # all-zero h: eps clamps
    if T > 2:
        G[2] = rng.standard_normal(F) * 40.0                              # saturated gates
    return G, U


# F covers every register-cache width (chunks per thread 1, 2, 3, 4, 6, 8) and the
# kernel that keeps h in shared memory only (F beyond 16384)
@pytest.mark.parametrize("T,F", [(1, 6912), (7, 8640), (33, 8192), (2, 8), (3, 1000), (300, 2048), (1, 51200),
                                 (4, 3072), (5, 5120), (3, 16384), (2, 16392)])
def test_swiglu_quant_parity(bn, T, F):
    rng = np.random.default_rng(T * 13 + F)
    G, U = _gate_values(T, F, rng)
    GU = np.concatenate([G, U], axis=1)
    GUd, GU32 = bf16_dev(GU)
    h = oracle.swiglu(GU32[:, :F], GU32[:, F:])
    xq_ref, a_ref = oracle.quant_act(h, 1e-5)
    Xq, a = bn.bitnet_swiglu_quant(GUd, F, 1e-5)
    torch.cuda.synchronize()
    assert np.array_equal(a.cpu().numpy(), a_ref)
    assert np.array_equal(Xq.cpu().numpy(), xq_ref)


@pytest.mark.parametrize("extra", [64, 3])
def test_swiglu_quant_strided_rows(bn, extra):
    """Gate and up halves inside a wider row (row stride > 2F; a stride that is
    not a multiple of 8 takes the kernel with 2-byte loads)."""
    T, F = 5, 1024
    rng = np.random.default_rng(5)
    G, U = _gate_values(T, F, rng)
    pad = rng.standard_normal((T, extra)).astype(np.float32)
    GU = np.concatenate([G, U, pad], axis=1)
    GUd, GU32 = bf16_dev(GU)
    h = oracle.swiglu(GU32[:, :F], GU32[:, F:2 * F])
    xq_ref, a_ref = oracle.quant_act(h, 1e-5)
    Xq, a = bn.bitnet_swiglu_quant(GUd[:, :2 * F], F, 1e-5)
    torch.cuda.synchronize()
    assert np.array_equal(a.cpu().numpy(), a_ref)
    assert np.array_equal(Xq.cpu().numpy(), xq_ref)


def test_block_quant_empty_batch(bn):
    X = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    Xq, a = bn.bitnet_rmsnorm_quant(X)
    GU = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    Xq2, a2 = bn.bitnet_swiglu_quant(GU)
    torch.cuda.synchronize()
    assert Xq.shape == (0, 256) and Xq2.shape == (0, 256) and a.numel() == 0 and a2.numel() == 0

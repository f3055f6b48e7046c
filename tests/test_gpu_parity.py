"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bar (element by element, same seeded inputs):
  * bit-exact: gamma, mask bits, canonical group bytes, tensor-core values and
    metadata (decoded back), decode-layout codes (decoded back), int8
    activation codes, absmax, int32 accumulators;
  * fp32 outputs within 1e-5 relative (the kernels follow the oracle's order of
    fp32 operations, so they are in fact identical);
  * bf16 outputs equal to bf16(oracle fp32);
  * STE gradient within the fp32-summation bound 2 * n_out * 2^-24 * sum|terms|
    (plus one bf16 rounding when dX is bf16).
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


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def bf16_dev(a_f32):
    bits = synth.to_bf16_bits(a_f32)
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16), synth.bf16_bits_to_f32(bits)


# ------------------------------------------------------------------ layout decoders (test side)

def decode_mma(vals, meta, n_out, k):
    """tensor-core layout -> (dense Wq int8, keep mask)."""
    vals = vals.reshape(n_out, k // 2).astype(np.int8)
    rows_pad = (n_out + 127) // 128 * 128
    kb = (k + 127) // 128
    E = meta.reshape(kb, rows_pad, 16)
    g = np.arange(k // 4)
    nib = (E[g // 32][:, :n_out, :][np.arange(len(g)), :, (g % 32) // 2] >> (4 * (g % 2))[:, None]) & 0xF
    nib = nib.T   # [n_out, groups]
    i0, i1 = nib & 3, nib >> 2
    wq = np.zeros((n_out, k), np.int8)
    keep = np.zeros((n_out, k), np.uint8)
    r = np.arange(n_out)[:, None]
    wq[r, 4 * g[None, :] + i0] = vals[:, 0::2]
    wq[r, 4 * g[None, :] + i1] = vals[:, 1::2]
    keep[r, 4 * g[None, :] + i0] = 1
    keep[r, 4 * g[None, :] + i1] = 1
    return wq, keep, E, rows_pad


def decode_dec(dec, n_out, k):
    """decode (GEMV) layout -> canonical group bytes."""
    rt, kt = n_out // 16, k // 64
    w = dec.view(np.uint32).reshape(rt, kt, 32, 2)
    gb = np.zeros((n_out, k // 4), np.uint32)
    for lane in range(32):
        gid, tq = lane >> 2, lane & 3
        cw = w[:, :, lane, 0]
        for r in range(4):
            for j in range(4):
                row = gid + 8 * (r & 1)
                col = 4 * tq + j + 16 * (r >> 1)
                code = (cw >> (8 * j + 2 * r)) & 3
                shift = 4 if (col & 1) == 0 else 6
                rows = np.arange(rt)[:, None] * 16 + row
                grp = np.arange(kt)[None, :] * 16 + (col >> 1)
                gb[rows, grp] |= code << shift
        mw = w[:, :, lane, 1]
        row = gid + 8 * (lane & 1)
        gs = 8 * ((lane >> 1) & 1)
        for q in range(8):
            rows = np.arange(rt)[:, None] * 16 + row
            grp = np.arange(kt)[None, :] * 16 + gs + q
            gb[rows, grp] |= (mw >> (4 * q)) & 0xF
    return gb.astype(np.uint8)


def mask_bits_to_keep(bits, n_out, k):
    return np.unpackbits(bits.reshape(n_out, k // 8), axis=1, bitorder="little")


# ------------------------------------------------------------------ pack

PACK_SHAPES = [(256, 256), (200, 352), (384, 1024), (16, 64), (3200, 8640), (11008, 512)]


@pytest.mark.parametrize("n_out,k", PACK_SHAPES)
def test_pack_parity(bn, n_out, k):
    W = synth.master_weights(n_out, k, 0.02, seed=n_out + k)
    g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
    pw = bn.PackedWeights(n_out, k)
    mask = torch.zeros(n_out * k // 8, dtype=torch.uint8, device="cuda")
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5, mask_bits=mask)
    torch.cuda.synchronize()
    assert pw.gamma.item() == float(g)
    assert np.array_equal(pw.group_bytes.cpu().numpy(), gb)
    assert np.array_equal(mask_bits_to_keep(mask.cpu().numpy(), n_out, k), keep)
    dwq, dkeep, E, rows_pad = decode_mma(pw.mma_vals.cpu().numpy(), pw.mma_meta.cpu().numpy(), n_out, k)
    assert np.array_equal(dwq, wq) and np.array_equal(dkeep, keep)
    # padding rows and padding k of the metadata blocks select positions (0, 1)
    assert np.all(E[:, n_out:, :] == 0x44)
    if k % 128:
        valid_bytes = ((k // 4) % 32 + 1) // 2
        assert np.all(E[-1, :n_out, valid_bytes:] == 0x44)
    if pw.dec_codes is not None:
        assert np.array_equal(decode_dec(pw.dec_codes.cpu().numpy(), n_out, k), gb)


def test_pack_adversarial_values(bn):
    r = np.random.default_rng(3)
    W = (r.normal(0, 1, (64, 256)) * 10.0 ** r.integers(-40, 30, (64, 256))).astype(np.float32)
    W[0, :8] = [0.25, 0.25, 0.25, 0.25, 0.0, -0.0, 0.0, -0.0]
    W[1, :] = 0.0
    W[2, :8] = [1e-45, -1e-45, 3e38, -3e38, 1.2e-38, 0.5, -0.5, 1e-30]
    g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
    pw = bn.PackedWeights(64, 256)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    torch.cuda.synchronize()
    assert pw.gamma.item() == float(g)
    assert np.array_equal(pw.group_bytes.cpu().numpy(), gb)


def test_pack_threshold_boundaries(bn):
    # Make gamma exactly 1: with m = fp32(mean |W|) in [0.5, 1], eps = 1 - m is
    # exact (Sterbenz) and m + eps = 1.  Then W/gamma = W, so +-0.5 must code 0
    # (ties to even) and the next float above 0.5 must code +-1.
    nxt = float(np.nextafter(np.float32(0.5), np.float32(1)))
    W = np.full((16, 64), 0.75, np.float32)
    W[0, 0:4] = [0.5, nxt, 0.4, 0.3]
    W[0, 4:8] = [-0.5, -nxt, 0.1, 0.2]
    W[1, 0:4] = [1.5, -1.5, 0.25, 0.3]
    W[1, 4:8] = [float(np.nextafter(np.float32(0.5), np.float32(0))), 0.5, 0.1, 0.0]
    m = oracle.gamma(W, 0.0)
    eps = float(np.float32(1.0) - m)
    g, keep, wq, gb = oracle.pack_weights(W, eps)
    assert g == np.float32(1.0)
    assert wq[0, :8].tolist() == [0, 1, 0, 0, 0, -1, 0, 0]
    assert wq[1, :8].tolist() == [1, -1, 0, 0, 0, 0, 0, 0]
    pw = bn.PackedWeights(16, 64)
    bn.bitnet_pack_nm(dev_f32(W), pw, eps)
    torch.cuda.synchronize()
    assert pw.gamma.item() == 1.0
    assert np.array_equal(pw.group_bytes.cpu().numpy(), gb)


def test_pack_all_zero_matrix(bn):
    W = np.zeros((32, 128), np.float32)
    g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
    pw = bn.PackedWeights(32, 128)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    torch.cuda.synchronize()
    assert pw.gamma.item() == float(g) == np.float32(1e-5)
    assert np.array_equal(pw.group_bytes.cpu().numpy(), gb)


@pytest.mark.parametrize("n,m", [(1, 4), (3, 4), (6, 8), (4, 8), (2, 8)])
def test_mask_general_nm(bn, n, m):
    W = synth.master_weights(64, 256, 0.02, seed=7)
    W[0, :8] = 0.125
    keep = oracle.mask_nm(W, n, m)
    pw = bn.PackedWeights(64, 256, group_bytes=False, mma=False, dec=False, n=n, m=m)
    mask = torch.zeros(64 * 256 // 8, dtype=torch.uint8, device="cuda")
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5, mask_bits=mask)
    torch.cuda.synchronize()
    assert pw.gamma.item() == float(oracle.gamma(W, 1e-5))
    assert np.array_equal(mask_bits_to_keep(mask.cpu().numpy(), 64, 256), keep)


# ------------------------------------------------------------------ activations

@pytest.mark.parametrize("T,K,dtype", [(1, 2560, "bf16"), (17, 4096, "bf16"), (64, 11008, "bf16"),
                                      (16, 256, "f32"), (5, 6912, "f32"), (2, 20000, "f32"), (3, 40000, "bf16")])
def test_quant_act_parity(bn, T, K, dtype):
    X = synth.activations(T, K, seed=T + K, outlier_p=0.01)
    X[0, :] = 0.0   # eps clamp row
    if dtype == "bf16":
        Xd, X32 = bf16_dev(X)
    else:
        Xd, X32 = dev_f32(X), X
    xq_ref, a_ref = oracle.quant_act(X32, 1e-5)
    Xq, a = bn.bitnet_quant_act(Xd, 1e-5)
    torch.cuda.synchronize()
    assert np.array_equal(Xq.cpu().numpy(), xq_ref)
    assert np.array_equal(a.cpu().numpy(), a_ref)


# Hundreds to thousands of token groups (more CTAs than fit on the GPU at
# once), ragged last groups (T not a multiple of the tokens per CTA), every
# group size (8, 4, 2, 1 tokens per CTA), rows past the register cache, and
# per-row scales spread over six decades so that a token quantised with another
# token's scale fails.
@pytest.mark.parametrize("T,K,dtype", [(4099, 4096, "bf16"), (2501, 3200, "bf16"), (701, 11008, "bf16"),
                                      (3003, 1024, "f32"), (1201, 4096, "f32"), (333, 40000, "bf16"),
                                      (4096, 11008, "bf16")])
def test_quant_act_many_groups_per_cta(bn, T, K, dtype):
    X = synth.activations(T, K, seed=3 * T + K, outlier_p=0.01)
    X *= (10.0 ** synth.rng(T).uniform(-3.0, 3.0, size=(T, 1))).astype(np.float32)
    X[0, :] = 0.0
    X[T - 1, :] = 0.0   # eps clamp in the ragged last group
    if dtype == "bf16":
        Xd, X32 = bf16_dev(X)
    else:
        Xd, X32 = dev_f32(X), X
    xq_ref, a_ref = oracle.quant_act(X32, 1e-5)
    Xq, a = bn.bitnet_quant_act(Xd, 1e-5)
    torch.cuda.synchronize()
    assert np.array_equal(a.cpu().numpy(), a_ref)
    assert np.array_equal(Xq.cpu().numpy(), xq_ref)


# ------------------------------------------------------------------ sparse linear

def _linear_case(bn, n_out, k, T, seed, dec=True, y_dtype="f32"):
    W = synth.master_weights(n_out, k, 0.02, seed=seed)
    X = synth.activations(T, k, seed=seed + 1, outlier_p=0.01)
    Xd, X32 = bf16_dev(X)
    ref = oracle.forward(W, X32, 1e-5, 1e-5)
    pw = bn.PackedWeights(n_out, k, dec=dec)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    Xq, a = bn.bitnet_quant_act(Xd, 1e-5)
    acc = torch.full((T, n_out), -7, dtype=torch.int32, device="cuda")
    ydt = torch.float32 if y_dtype == "f32" else torch.bfloat16
    Y = bn.bitnet_sparse_linear(Xq, a, pw, y_dtype=ydt, acc_out=acc)
    torch.cuda.synchronize()
    return ref, acc.cpu().numpy(), Y


def _check_outputs(ref, acc, Y):
    assert np.array_equal(acc, ref["acc"])
    if Y.dtype == torch.float32:
        y = Y.cpu().numpy()
        assert np.allclose(y, ref["y"], rtol=1e-5, atol=0)
    else:
        yb = Y.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(yb, synth.to_bf16_bits(ref["y"]))


@pytest.mark.parametrize("T", [1, 2, 4, 7, 8])
@pytest.mark.parametrize("n_out,k", [(3840, 2560), (2560, 6912), (208, 256)])
def test_gemv_decode_layout(bn, T, n_out, k):
    ref, acc, Y = _linear_case(bn, n_out, k, T, seed=100 + T)
    _check_outputs(ref, acc, Y)


@pytest.mark.parametrize("T", [1, 8])
@pytest.mark.parametrize("n_out,k", [(2560, 2560), (200, 264)])
def test_gemv_group_bytes(bn, T, n_out, k):
    ref, acc, Y = _linear_case(bn, n_out, k, T, seed=200 + T, dec=False, y_dtype="bf16")
    _check_outputs(ref, acc, Y)


@pytest.mark.parametrize("T", [9, 16, 17, 32, 33, 100, 128, 129, 256, 300])
def test_gemm_parity_tiles_and_tails(bn, T):
    ref, acc, Y = _linear_case(bn, 256, 256, T, seed=300 + T)
    _check_outputs(ref, acc, Y)


@pytest.mark.parametrize("n_out,k,T", [(200, 352, 40), (384, 1024, 513), (128, 8640, 64), (1000, 2560, 257)])
def test_gemm_parity_ragged(bn, n_out, k, T):
    ref, acc, Y = _linear_case(bn, n_out, k, T, seed=n_out + k + T, y_dtype="bf16")
    _check_outputs(ref, acc, Y)


@pytest.mark.parametrize("T,k,n_out", [(4096, 4096, 11008), (4096, 11008, 4096)])
def test_gemm_full_size_sampled(bn, T, k, n_out):
    """Prefill shapes at full size, launched as the benchmark does; the oracle
    checks sampled tokens x sampled output features, and every output is
    checked against the exact-integer invariant |acc| <= 127 * (#non-zero Wq)."""
    W = synth.master_weights(n_out, k, 0.02, seed=11)
    X = synth.activations(T, k, seed=12, outlier_p=0.01)
    Xd, X32 = bf16_dev(X)
    g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
    pw = bn.PackedWeights(n_out, k, dec=False)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    Xq, a = bn.bitnet_quant_act(Xd, 1e-5)
    acc = torch.empty((T, n_out), dtype=torch.int32, device="cuda")
    Y = bn.bitnet_sparse_linear(Xq, a, pw, y_dtype=torch.bfloat16, acc_out=acc)
    torch.cuda.synchronize()
    assert pw.gamma.item() == float(g)
    r = np.random.default_rng(0)
    ts = np.unique(np.concatenate([r.choice(T, 40, replace=False), [0, T - 1]]))
    ns = np.unique(np.concatenate([r.choice(n_out, 300, replace=False), [0, n_out - 1]]))
    xq_ref, a_ref = oracle.quant_act(X32[ts], 1e-5)
    assert np.array_equal(Xq.cpu().numpy()[ts], xq_ref)
    acc_ref = oracle.gemm_i32(xq_ref, wq[ns])
    acc_h = acc.cpu().numpy()
    assert np.array_equal(acc_h[np.ix_(ts, ns)], acc_ref)
    y_ref = oracle.dequant(acc_ref, a_ref, g)
    yb = Y.view(torch.int16).cpu().numpy().view(np.uint16)[np.ix_(ts, ns)]
    assert np.array_equal(yb, synth.to_bf16_bits(y_ref))
    nnz = (wq != 0).sum(1)
    assert np.all(np.abs(acc_h) <= 127 * nnz[None, :])


def test_linear_empty_batch(bn):
    pw = bn.PackedWeights(256, 256)
    W = synth.master_weights(256, 256, 0.02, 1)
    bn.bitnet_pack_nm(dev_f32(W), pw)
    Xq = torch.empty((0, 256), dtype=torch.int8, device="cuda")
    a = torch.empty((0,), dtype=torch.float32, device="cuda")
    Y = bn.bitnet_sparse_linear(Xq, a, pw, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert Y.shape == (0, 256)


# ------------------------------------------------------------------ STE input gradient

# T > 128 forms the ternary tiles in shared memory from the group bytes: ragged
# n_out (contraction tail), k not a multiple of 64 (column tail, unaligned
# group-byte rows) and ragged T included
@pytest.mark.parametrize("T,n_out,k,dx", [(128, 256, 256, "f32"), (200, 264, 384, "f32"), (300, 512, 1000, "bf16"),
                                          (512, 3200, 640, "f32"), (129, 72, 136, "f32"), (700, 1000, 2600, "bf16"),
                                          (2048, 9600, 3200, "bf16")])
def test_dgrad_parity(bn, T, n_out, k, dx):
    W = synth.master_weights(n_out, k, 0.02, seed=T + k)
    g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
    pw = bn.PackedWeights(n_out, k, mma=False, dec=False)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    dYd, dY32 = bf16_dev(synth.activations(T, n_out, seed=T))
    dX = bn.bitnet_dgrad(dYd, pw, dx_dtype=torch.float32 if dx == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    ref, absref = oracle.dgrad(dY32, wq, g)
    got = dX.float().cpu().numpy().astype(np.float64)
    tol = 2 * n_out * 2.0 ** -24 * absref + 1e-30
    if dx == "bf16":
        tol = tol + np.abs(ref) * 2.0 ** -8
    assert np.all(np.abs(got - ref) <= tol)


def test_bounded_waits_time_out_cleanly(bn):
    """Both kinds of bounded wait (mbarrier phase, grid counter) run out on
    events that never happen: the status word reports the timeout, the kernel
    ends, and the context keeps working (a pack and a quantisation afterwards
    are exact, and their own status is clear)."""
    import time
    t0 = time.time()
    assert bn.bitnet_wait_selftest(limit_us=50000) == 5          # BITNET_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    W = synth.master_weights(256, 256, 0.02, seed=3)
    pw = bn.PackedWeights(256, 256)
    ws = bn.Workspace(bn.load().bitnet_pack_workspace_size(256, 256))
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5, ws=ws)
    X = synth.activations(4, 256, seed=4)
    Xq, a = bn.bitnet_quant_act(dev_f32(X), 1e-5)
    torch.cuda.synchronize()
    g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
    assert pw.gamma.item() == float(g) and np.array_equal(pw.group_bytes.cpu().numpy(), gb)
    assert np.array_equal(Xq.cpu().numpy(), oracle.quant_act(X, 1e-5)[0])
    assert bn.bitnet_read_device_status(ws) == 0


def test_device_status_clear_after_runs(bn):
    ws = bn.Workspace(256)
    ref, acc, Y = _linear_case(bn, 256, 256, 64, seed=5)
    assert bn.bitnet_read_device_status(ws) == 0


# ------------------------------------------------------------------ fused quantisation + linear

@pytest.mark.parametrize("T,x_dtype", [(1, "bf16"), (3, "bf16"), (8, "bf16"), (2, "f32"), (8, "f32")])
@pytest.mark.parametrize("n_out,k", [(3840, 2560), (2560, 6912), (208, 320)])
def test_quant_linear_fused_decode(bn, T, x_dtype, n_out, k):
    W = synth.master_weights(n_out, k, 0.02, seed=400 + T)
    X = synth.activations(T, k, seed=401 + T, outlier_p=0.01)
    if x_dtype == "bf16":
        Xd, X32 = bf16_dev(X)
    else:
        Xd, X32 = dev_f32(X), X
    ref = oracle.forward(W, X32, 1e-5, 1e-5)
    pw = bn.PackedWeights(n_out, k, mma=False)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    acc = torch.full((T, n_out), -7, dtype=torch.int32, device="cuda")
    xq = torch.zeros((T, k), dtype=torch.int8, device="cuda")
    am = torch.zeros((T,), dtype=torch.float32, device="cuda")
    Y = bn.bitnet_quant_linear(Xd, pw, 1e-5, y_dtype=torch.float32, acc_out=acc, xq_out=xq, absmax_out=am)
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), ref["xq"])
    assert np.array_equal(am.cpu().numpy(), ref["a"])
    _check_outputs(ref, acc.cpu().numpy(), Y)


@pytest.mark.parametrize("T,x_dtype", [(1, "bf16"), (8, "bf16"), (5, "f32")])
@pytest.mark.parametrize("n_out,k", [(6912, 2560), (6928, 192), (9616, 128), (640, 64), (4752, 6912)])
def test_quant_linear_streamed_row_tiles(bn, T, x_dtype, n_out, k):
    """bitnet_quant_linear at T <= 8 runs the decode chain with one projection:
    row tiles per CTA from 1 to 5 with ragged shares (6928 and 9616 rows),
    k = 64 (one record per row tile, fewer records than warps) and odd k-tile
    counts (k = 192)."""
    W = synth.master_weights(n_out, k, 0.02, seed=420 + T)
    X = synth.activations(T, k, seed=421 + T, outlier_p=0.01)
    if x_dtype == "bf16":
        Xd, X32 = bf16_dev(X)
    else:
        Xd, X32 = dev_f32(X), X
    ref = oracle.forward(W, X32, 1e-5, 1e-5)
    pw = bn.PackedWeights(n_out, k, mma=False)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    acc = torch.full((T, n_out), -7, dtype=torch.int32, device="cuda")
    xq = torch.zeros((T, k), dtype=torch.int8, device="cuda")
    am = torch.zeros((T,), dtype=torch.float32, device="cuda")
    ws = bn.Workspace(bn.load().bitnet_quant_linear_workspace_size(T, k))
    Y = bn.bitnet_quant_linear(Xd, pw, 1e-5, y_dtype=torch.bfloat16, acc_out=acc, xq_out=xq, absmax_out=am, ws=ws)
    torch.cuda.synchronize()
    assert bn.bitnet_read_device_status(ws) == 0
    assert np.array_equal(xq.cpu().numpy(), ref["xq"])
    assert np.array_equal(am.cpu().numpy(), ref["a"])
    _check_outputs(ref, acc.cpu().numpy(), Y)


@pytest.mark.parametrize("T", [16, 100])
def test_quant_linear_unfused_path(bn, T):
    n_out, k = 384, 1024
    W = synth.master_weights(n_out, k, 0.02, seed=500 + T)
    Xd, X32 = bf16_dev(synth.activations(T, k, seed=501 + T))
    ref = oracle.forward(W, X32, 1e-5, 1e-5)
    pw = bn.PackedWeights(n_out, k)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    acc = torch.empty((T, n_out), dtype=torch.int32, device="cuda")
    Y = bn.bitnet_quant_linear(Xd, pw, 1e-5, y_dtype=torch.bfloat16, acc_out=acc)
    torch.cuda.synchronize()
    _check_outputs(ref, acc.cpu().numpy(), Y)


def test_quant_linear_chain_in_graph(bn):
    """Consecutive fused kernels (programmatic dependent launch) inside a CUDA
    graph: each layer consumes the previous layer's output."""
    T, h = 2, 512
    layers = 6
    Ws = [synth.master_weights(h, h, 0.02, seed=600 + l) for l in range(layers)]
    pws = []
    for W in Ws:
        pw = bn.PackedWeights(h, h, mma=False)
        bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
        pws.append(pw)
    x0 = synth.activations(T, h, seed=700)
    xs = [dev_f32(x0)] + [torch.empty((T, h), dtype=torch.float32, device="cuda") for _ in range(layers)]
    ws = bn.Workspace(bn.load().bitnet_quant_linear_workspace_size(T, h))

    def run():
        for l in range(layers):
            bn.bitnet_quant_linear(xs[l], pws[l], 1e-5, Y=xs[l + 1], ws=ws)

    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for x in xs[1:]:
        x.zero_()
    g.replay()
    torch.cuda.synchronize()
    x = x0
    for l in range(layers):
        x = oracle.forward(Ws[l], x, 1e-5, 1e-5)["y"]
        assert np.array_equal(xs[l + 1].cpu().numpy(), x), l


# ------------------------------------------------------------------ 6:8 through 2:4 windows

def windows_to_dense(gbw, n_out, k):
    """Window-layout group bytes [n_out, 3k/8] -> dense int8 [n_out, k] and keep.
    Window w of block b covers positions 8b + 2w .. 8b + 2w + 3; every kept
    position must appear in exactly one window slot."""
    gbw = gbw.reshape(n_out, k // 8, 3).astype(np.int64)
    wq = np.zeros((n_out, k), np.int8)
    seen = np.zeros((n_out, k), np.int32)
    code_val = np.array([0, 1, 0, -1], np.int8)
    rows = np.arange(n_out)[:, None]
    for w in range(3):
        b = gbw[:, :, w]
        i0, i1, c0, c1 = b & 3, (b >> 2) & 3, (b >> 4) & 3, b >> 6
        assert (i0 < i1).all()
        base = 8 * np.arange(k // 8)[None, :] + 2 * w
        for idx, c in ((i0, c0), (i1, c1)):
            pos = base + idx
            wq[rows, pos] = code_val[c]
            np.add.at(seen, (np.broadcast_to(rows, pos.shape), pos), 1)
    return wq, seen


@pytest.mark.parametrize("n_out,k", [(256, 512), (200, 384), (128, 1024), (48, 64)])
def test_pack_6of8_windows(bn, n_out, k):
    """gamma, the 6:8 keep bits and the window layouts against the oracle's
    dense 6:8 masked ternary matrix; every kept position sits in exactly one
    window slot; the tensor-core layout and the decode layout decode to the
    same window matrix."""
    W = synth.master_weights(n_out, k, 0.02, seed=3000 + n_out + k)
    W[0, :8] = 0.01                                            # an all-tie block
    W[1, 8:16] = [0.3, -0.3, 0.3, -0.3, 0.0, -0.0, 0.3, 0.3]   # ties and signed zeros
    ref = oracle.forward_nm(W, synth.activations(1, k, seed=1), 6, 8)
    dec = n_out % 16 == 0 and k % 128 == 0
    pw = bn.packed_6of8(n_out, k, dec=dec)
    mask = torch.zeros(n_out * k // 8, dtype=torch.uint8, device="cuda")
    bn.bitnet_pack_6of8_windows(dev_f32(W), pw, 1e-5, mask_bits=mask)
    torch.cuda.synchronize()
    assert pw.gamma.item() == float(ref["gamma"])
    assert np.array_equal(mask_bits_to_keep(mask.cpu().numpy(), n_out, k), ref["keep"])
    gbw = pw.group_bytes.cpu().numpy()
    wq, seen = windows_to_dense(gbw, n_out, k)
    assert np.array_equal(seen, ref["keep"].astype(np.int32))
    assert np.array_equal(wq, ref["wq"])
    kw = k // 2 * 3
    mwq, mkeep, _, _ = decode_mma(pw.mma_vals.cpu().numpy(), pw.mma_meta.cpu().numpy(), n_out, kw)
    g2 = gbw.reshape(n_out, kw // 4).astype(np.int64)
    cval = np.array([0, 1, 0, -1], np.int8)
    dense_w = np.zeros((n_out, kw), np.int8)
    r = np.arange(n_out)[:, None]
    gi = 4 * np.arange(kw // 4)[None, :]
    dense_w[r, gi + (g2 & 3)] = cval[(g2 >> 4) & 3]
    dense_w[r, gi + ((g2 >> 2) & 3)] = cval[g2 >> 6]
    assert np.array_equal(mwq, dense_w)
    if dec:
        assert np.array_equal(decode_dec(pw.dec_codes.cpu().numpy(), n_out, kw), g2.astype(np.uint32))


@pytest.mark.parametrize("T,x_dtype", [(1, "bf16"), (5, "f32"), (8, "bf16"), (64, "bf16"), (300, "bf16")])
@pytest.mark.parametrize("n_out,k", [(256, 1024), (2560, 2560)])
def test_6of8_forward(bn, T, x_dtype, n_out, k):
    """Lifted activations + the 2:4 GEMV (T <= 8) or tensor-core GEMM (T > 8)
    on the window layout reproduce the oracle's dense 6:8 product: int32
    accumulators bit-exact, outputs to 1e-5 / exact bf16."""
    W = synth.master_weights(n_out, k, 0.02, seed=3100 + T)
    X = synth.activations(T, k, seed=3101 + T, outlier_p=0.01)
    if x_dtype == "bf16":
        Xd, X32 = bf16_dev(X)
    else:
        Xd, X32 = dev_f32(X), X
    ref = oracle.forward_nm(W, X32, 6, 8)
    pw = bn.packed_6of8(n_out, k, dec=True)
    bn.bitnet_pack_6of8_windows(dev_f32(W), pw, 1e-5)
    Xl, am = bn.bitnet_quant_act_lift_6of8(Xd, 1e-5)
    acc = torch.full((T, n_out), -7, dtype=torch.int32, device="cuda")
    Y = bn.bitnet_sparse_linear(Xl, am, pw, y_dtype=torch.float32, acc_out=acc)
    torch.cuda.synchronize()
    xq = ref["xq"]
    # block b, window w, position j -> code of column 8b + 2w + j
    lifted = np.stack([xq.reshape(T, -1, 8)[:, :, 2 * w:2 * w + 4] for w in range(3)], axis=2).reshape(T, -1)
    assert np.array_equal(Xl.cpu().numpy(), lifted)
    assert np.array_equal(am.cpu().numpy(), ref["a"])
    _check_outputs(ref, acc.cpu().numpy(), Y)


# ------------------------------------------------------------------ decode chain (one persistent launch)

def _packed_dec(bn, n_out, k, seed):
    W = synth.master_weights(n_out, k, 0.02, seed=seed)
    pw = bn.PackedWeights(n_out, k, group_bytes=True, mma=False, dec=True)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    return W, pw


@pytest.mark.parametrize("T", [1, 3, 8])
def test_decode_chain_layers(bn, T):
    """A chain of layers: each op reads the previous op's Y (wait_prev = 1).
    Every op is checked against the oracle on the input the GPU actually had."""
    dims = [512, 768, 512, 2560, 64, 6912, 2560]
    Ws, pws = [], []
    for i in range(len(dims) - 1):
        W, pw = _packed_dec(bn, dims[i + 1], dims[i], seed=800 + i)
        Ws.append(W)
        pws.append(pw)
    x0 = synth.activations(T, dims[0], seed=900 + T, outlier_p=0.01)
    xs = [dev_f32(x0)] + [torch.empty((T, d), dtype=torch.float32, device="cuda") for d in dims[1:]]
    accs = [torch.full((T, d), -7, dtype=torch.int32, device="cuda") for d in dims[1:]]
    ops = [dict(X=xs[i], W=pws[i], Y=xs[i + 1], acc_out=accs[i], wait_prev=1) for i in range(len(pws))]
    ch = bn.bitnet_decode_chain(ops, 1e-5)
    torch.cuda.synchronize()
    assert bn.bitnet_read_device_status(ch.ws) == 0
    for i in range(len(pws)):
        ref = oracle.forward(Ws[i], xs[i].cpu().numpy(), 1e-5, 1e-5)
        _check_outputs(ref, accs[i].cpu().numpy(), xs[i + 1])
    # the same chain again (counters are cleared by every call)
    y_first = xs[-1].clone()
    for x in xs[1:]:
        x.zero_()
    ch()
    torch.cuda.synchronize()
    assert torch.equal(xs[-1], y_first)


@pytest.mark.parametrize("T", [1, 5])
def test_decode_chain_independent_and_ragged(bn, T):
    """Independent ops (wait_prev 0 and 1 mixed), bf16 in and out, row counts
    from one tile (most CTAs idle) to several tiles per CTA, k = 64 (one k-tile
    per row tile, fewer records than warps) and odd k-tile counts."""
    shapes = [(16, 64), (9616, 128), (48, 192), (2560, 6912), (4752, 2560), (640, 64), (13824, 2560)]
    ops, refs = [], []
    for i, (n_out, k) in enumerate(shapes):
        W, pw = _packed_dec(bn, n_out, k, seed=1000 + i)
        Xd, X32 = bf16_dev(synth.activations(T, k, seed=1100 + i, outlier_p=0.01))
        Y = torch.empty((T, n_out), dtype=torch.bfloat16, device="cuda")
        acc = torch.full((T, n_out), -7, dtype=torch.int32, device="cuda")
        xq = torch.zeros((T, k), dtype=torch.int8, device="cuda")
        am = torch.zeros((T,), dtype=torch.float32, device="cuda")
        ops.append(dict(X=Xd, W=pw, Y=Y, acc_out=acc, xq_out=xq, absmax_out=am, wait_prev=i % 2))
        refs.append(oracle.forward(W, X32, 1e-5, 1e-5))
    ch = bn.bitnet_decode_chain(ops, 1e-5)
    torch.cuda.synchronize()
    assert bn.bitnet_read_device_status(ch.ws) == 0
    for o, ref in zip(ops, refs):
        assert np.array_equal(o["xq_out"].cpu().numpy(), ref["xq"])
        assert np.array_equal(o["absmax_out"].cpu().numpy(), ref["a"])
        _check_outputs(ref, o["acc_out"].cpu().numpy(), o["Y"])


@pytest.mark.parametrize("T,x_dtype", [(1, "bf16"), (2, "f32"), (3, "bf16"), (5, "bf16"), (8, "f32")])
def test_decode_chain_all_independent(bn, T, x_dtype):
    """A chain with no waits at all runs the pipelined kernel: weight shares of
    consecutive projections share ring stages, the quantiser warps run ahead in
    up to four int8 buffers and the epilogue trails.  40 projections cycle every
    buffer many times; shapes from one row tile (most CTAs idle) to several per
    CTA, k = 64 and odd k-tile counts; every fourth op also copies out its int8
    activations and scales."""
    base = [(16, 64), (3840, 2560), (208, 192), (2560, 6912), (640, 64), (1040, 320), (6928, 192), (96, 2560)]
    shapes = [base[i % len(base)] for i in range(40)]
    packed = {}
    ops, refs = [], []
    for i, (n_out, k) in enumerate(shapes):
        if (n_out, k) not in packed:
            packed[(n_out, k)] = _packed_dec(bn, n_out, k, seed=1500 + len(packed))
        W, pw = packed[(n_out, k)]
        X = synth.activations(T, k, seed=1600 + i, outlier_p=0.01)
        if x_dtype == "bf16":
            Xd, X32 = bf16_dev(X)
        else:
            Xd, X32 = dev_f32(X), X
        Y = torch.empty((T, n_out), dtype=torch.bfloat16 if i % 2 else torch.float32, device="cuda")
        acc = torch.full((T, n_out), -7, dtype=torch.int32, device="cuda")
        o = dict(X=Xd, W=pw, Y=Y, acc_out=acc, wait_prev=0)
        if i % 4 == 0:
            o["xq_out"] = torch.zeros((T, k), dtype=torch.int8, device="cuda")
            o["absmax_out"] = torch.zeros((T,), dtype=torch.float32, device="cuda")
        ops.append(o)
        refs.append(oracle.forward(W, X32, 1e-5, 1e-5))
    # one y dtype per chain: split into the float32 and the bf16 halves
    for half in (0, 1):
        sub = [(o, r) for i, (o, r) in enumerate(zip(ops, refs)) if i % 2 == half]
        ch = bn.bitnet_decode_chain([o for o, _ in sub], 1e-5)
        torch.cuda.synchronize()
        assert bn.bitnet_read_device_status(ch.ws) == 0
        for o, ref in sub:
            if "xq_out" in o:
                assert np.array_equal(o["xq_out"].cpu().numpy(), ref["xq"])
                assert np.array_equal(o["absmax_out"].cpu().numpy(), ref["a"])
            _check_outputs(ref, o["acc_out"].cpu().numpy(), o["Y"])
        # again, outputs cleared: the chain is repeatable
        for o, _ in sub:
            o["acc_out"].fill_(-7)
        ch()
        torch.cuda.synchronize()
        for o, ref in sub:
            _check_outputs(ref, o["acc_out"].cpu().numpy(), o["Y"])


def test_decode_chain_independent_split_launches(bn):
    """130 independent projections: more than one launch takes, each launch the
    pipelined kernel; captured in a CUDA graph and replayed."""
    T, h = 1, 256
    ops, refs = [], []
    W, pw = _packed_dec(bn, h, h, seed=1700)
    for i in range(130):
        Xd, X32 = bf16_dev(synth.activations(T, h, seed=1800 + i))
        ops.append(dict(X=Xd, W=pw, Y=torch.empty((T, h), dtype=torch.bfloat16, device="cuda"), wait_prev=0))
        refs.append(oracle.forward(W, X32, 1e-5, 1e-5))
    ch = bn.DecodeChain(ops, torch.bfloat16, torch.bfloat16, 1e-5)
    ch()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ch()
    for o in ops:
        o["Y"].zero_()
    g.replay()
    torch.cuda.synchronize()
    assert bn.bitnet_read_device_status(ch.ws) == 0
    for o, ref in zip(ops, refs):
        yb = o["Y"].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(yb, synth.to_bf16_bits(ref["y"]))
    del g


def test_decode_chain_split_launches_and_graph(bn):
    """More ops than one launch takes (130 > 128): the library splits the chain;
    captured in a CUDA graph and replayed."""
    T, h = 2, 256
    n_ops = 130
    Ws, pws = [], []
    for i in range(n_ops):
        # master std 0.13 keeps the layer gain near 1 (0.8 std * sqrt(0.35 h)), so
        # the activations neither vanish nor blow up over 130 layers
        W = synth.master_weights(h, h, 0.13, seed=1200 + i)
        pw = bn.PackedWeights(h, h, group_bytes=True, mma=False, dec=True)
        bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
        Ws.append(W)
        pws.append(pw)
    x0 = synth.activations(T, h, seed=1300)
    xs = [dev_f32(x0)] + [torch.empty((T, h), dtype=torch.float32, device="cuda") for _ in range(n_ops)]
    ops = [dict(X=xs[i], W=pws[i], Y=xs[i + 1], wait_prev=1) for i in range(n_ops)]
    ch = bn.DecodeChain(ops, torch.float32, torch.float32, 1e-5)
    ch()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ch()
    for x in xs[1:]:
        x.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert bn.bitnet_read_device_status(ch.ws) == 0
    x = x0
    for i in range(n_ops):
        x = oracle.forward(Ws[i], x, 1e-5, 1e-5)["y"]
        assert np.array_equal(xs[i + 1].cpu().numpy(), x), i
    del g


# ------------------------------------------------------------------ per-step pack with the previous gamma as hint

def _pack_outputs(pw, mask):
    return [pw.gamma.cpu().numpy().copy(), pw.group_bytes.cpu().numpy().copy(), pw.mma_vals.cpu().numpy().copy(),
            pw.mma_meta.cpu().numpy().copy(), mask.cpu().numpy().copy(),
            pw.dec_codes.cpu().numpy().copy() if pw.dec_codes is not None else None]


@pytest.mark.parametrize("n_out,k", [(256, 512), (200, 352), (3200, 3200)])
def test_pack_update_matches_pack_over_steps(bn, n_out, k):
    """Random-walk steps W += N(0, 1e-4) (patch mode), a large jump (full
    second pass), and the first call without a hint: every step bit-identical
    to bitnet_pack_nm and to the oracle."""
    W = synth.master_weights(n_out, k, 0.02, seed=900)
    Wd = dev_f32(W)
    upd = bn.PackedWeights(n_out, k)          # gamma starts at 0: no hint on the first call
    mask_u = torch.zeros(n_out * k // 8, dtype=torch.uint8, device="cuda")
    ws = bn.Workspace(bn.load().bitnet_pack_update_workspace_size(n_out, k))
    for step in range(6):
        if step > 0:
            scale = 1e-4 if step != 4 else 5e-3   # step 4 moves gamma far outside the band
            W = synth.random_walk_step(W, scale, seed=step)
            Wd.copy_(dev_f32(W))
        bn.bitnet_pack_nm_update(Wd, upd, 1e-5, mask_bits=mask_u, ws=ws)
        ref = bn.PackedWeights(n_out, k)
        mask_r = torch.zeros_like(mask_u)
        bn.bitnet_pack_nm(Wd, ref, 1e-5, mask_bits=mask_r)
        torch.cuda.synchronize()
        for a, b in zip(_pack_outputs(upd, mask_u), _pack_outputs(ref, mask_r)):
            assert (a is None and b is None) or np.array_equal(a, b), step
        g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
        assert upd.gamma.item() == float(g) and np.array_equal(upd.group_bytes.cpu().numpy(), gb)


def test_pack_update_batch_matches_single(bn):
    """The batched per-step pack over mixed shapes (metadata padding for
    n_out % 128 != 0 and k % 128 != 0, decode layout, mask bits, a one-chunk
    matrix), over random-walk steps, a jump that leaves the band for one matrix
    only, and the first call without hints: every matrix bit-identical to
    bitnet_pack_nm, and the gamma and group bytes to the oracle."""
    shapes = [(256, 512), (200, 352), (96, 64), (1000, 1360), (3200, 3200), (640, 2560)]
    Ws = [synth.master_weights(n, k, 0.02, seed=950 + i) for i, (n, k) in enumerate(shapes)]
    Wd = [dev_f32(W) for W in Ws]
    outs, masks = [], []
    for (n, k) in shapes:
        dec = n % 16 == 0 and k % 64 == 0
        outs.append(bn.PackedWeights(n, k, dec=dec))      # gamma 0: no hint on the first call
        masks.append(torch.zeros(n * k // 8, dtype=torch.uint8, device="cuda"))
    batch = bn.PackBatch([(Wd[i], outs[i], masks[i]) for i in range(len(shapes))], 1e-5)
    for step in range(5):
        if step > 0:
            for i in range(len(shapes)):
                scale = 5e-3 if (step == 3 and i == 4) else 1e-4   # step 3: matrix 4 jumps out of the band
                Ws[i] = synth.random_walk_step(Ws[i], scale, seed=100 * step + i)
                Wd[i].copy_(dev_f32(Ws[i]))
        batch()
        torch.cuda.synchronize()
        assert bn.bitnet_read_device_status(batch.ws) == 0
        for i, (n, k) in enumerate(shapes):
            ref = bn.PackedWeights(n, k, dec=outs[i].dec_codes is not None)
            mask_r = torch.zeros_like(masks[i])
            bn.bitnet_pack_nm(Wd[i], ref, 1e-5, mask_bits=mask_r)
            torch.cuda.synchronize()
            for a, b in zip(_pack_outputs(outs[i], masks[i]), _pack_outputs(ref, mask_r)):
                assert (a is None and b is None) or np.array_equal(a, b), (step, i)
            if n * k <= 1 << 20:
                g, keep, wq, gb = oracle.pack_weights(Ws[i], 1e-5)
                assert outs[i].gamma.item() == float(g) and np.array_equal(outs[i].group_bytes.cpu().numpy(), gb)


def test_pack_update_batch_bf16_masters(bn):
    """bf16 masters, mixed with fp32 ones in one batch: every matrix bit-identical
    to bitnet_pack_nm of its values widened to fp32, and to the oracle, over
    random-walk steps (rounded back to bf16 after every step)."""
    shapes = [(256, 512), (200, 352), (640, 2560), (3200, 3200)]
    bf = [True, False, True, True]
    Ws32 = [synth.master_weights(n, k, 0.02, seed=970 + i) for i, (n, k) in enumerate(shapes)]
    Wd, Wnp = [], []
    for i, W in enumerate(Ws32):
        if bf[i]:
            d, w32 = bf16_dev(W)
        else:
            d, w32 = dev_f32(W), W
        Wd.append(d)
        Wnp.append(w32)
    outs = [bn.PackedWeights(n, k, dec=(n % 16 == 0 and k % 64 == 0)) for (n, k) in shapes]
    batch = bn.PackBatch([(Wd[i], outs[i]) for i in range(len(shapes))], 1e-5)
    for step in range(4):
        if step > 0:
            for i in range(len(shapes)):
                Wn = synth.random_walk_step(Wnp[i], 1e-4, seed=200 * step + i)
                if bf[i]:
                    d, Wn = bf16_dev(Wn)
                    Wd[i].copy_(d)
                else:
                    Wd[i].copy_(dev_f32(Wn))
                Wnp[i] = Wn
        batch()
        torch.cuda.synchronize()
        for i, (n, k) in enumerate(shapes):
            ref = bn.PackedWeights(n, k, dec=outs[i].dec_codes is not None)
            bn.bitnet_pack_nm(dev_f32(Wnp[i]), ref, 1e-5)
            torch.cuda.synchronize()
            mask_dummy = torch.zeros(1, dtype=torch.uint8, device="cuda")
            for a, b in zip(_pack_outputs(outs[i], mask_dummy), _pack_outputs(ref, mask_dummy)):
                assert (a is None and b is None) or np.array_equal(a, b), (step, i)
            if n * k <= 1 << 20:
                g, keep, wq, gb = oracle.pack_weights(Wnp[i], 1e-5)
                assert outs[i].gamma.item() == float(g) and np.array_equal(outs[i].group_bytes.cpu().numpy(), gb)


def test_pack_update_batch_many_launch_groups(bn):
    """More matrices than one launch takes (70 > 64)."""
    n_items = 70
    Ws = [synth.master_weights(64, 128, 0.02, seed=2000 + i) for i in range(n_items)]
    Wd = [dev_f32(W) for W in Ws]
    outs = [bn.PackedWeights(64, 128) for _ in range(n_items)]
    batch = bn.bitnet_pack_nm_update_batch([(Wd[i], outs[i]) for i in range(n_items)], 1e-5)
    batch()
    torch.cuda.synchronize()
    for i in range(n_items):
        g, keep, wq, gb = oracle.pack_weights(Ws[i], 1e-5)
        assert outs[i].gamma.item() == float(g), i
        assert np.array_equal(outs[i].group_bytes.cpu().numpy(), gb), i
        dwq, dkeep, _, _ = decode_mma(outs[i].mma_vals.cpu().numpy(), outs[i].mma_meta.cpu().numpy(), 64, 128)
        assert np.array_equal(dwq, wq), i


def test_pack_update_small_list_falls_back(bn):
    """A list with room for one entry overflows; the device then runs the full
    second pass and the result is still exact."""
    n_out, k = 512, 512
    W = synth.master_weights(n_out, k, 0.02, seed=901)
    pw = bn.PackedWeights(n_out, k)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    W2 = synth.random_walk_step(W, 1e-4, seed=3)
    tiny = bn.Workspace(bn.load().bitnet_pack_workspace_size(n_out, k) + 4)
    bn.bitnet_pack_nm_update(dev_f32(W2), pw, 1e-5, ws=tiny)
    torch.cuda.synchronize()
    g, keep, wq, gb = oracle.pack_weights(W2, 1e-5)
    assert pw.gamma.item() == float(g)
    assert np.array_equal(pw.group_bytes.cpu().numpy(), gb)
    dwq, dkeep, _, _ = decode_mma(pw.mma_vals.cpu().numpy(), pw.mma_meta.cpu().numpy(), n_out, k)
    assert np.array_equal(dwq, wq)


@pytest.mark.parametrize("n_out,k,T", [(200, 352, 300), (136, 256, 500), (128, 8640, 229), (2560, 2560, 448),
                                       (256, 1024, 1000)])
def test_gemm_pair_kernel_ragged(bn, n_out, k, T):
    """T > 128 runs the persistent CTA-pair kernel: ragged last 256-row pair
    (including a second CTA entirely past n_out), ragged 224-token tiles,
    k % 128 != 0, several tiles per pair."""
    ref, acc, Y = _linear_case(bn, n_out, k, T, seed=n_out * 7 + T)
    _check_outputs(ref, acc, Y)


@pytest.mark.parametrize("n_out,k,T", [(4096, 256, 896), (2048, 256, 1344), (256, 512, 160), (3200, 320, 2048),
                                       (1040, 448, 700)])
def test_gemm_pair_tile_widths(bn, n_out, k, T):
    """Larger pair-kernel shapes: many tiles per CTA pair and a ragged last
    token tile, at both token-tile widths (224 for T = 896, 1344; 192 for
    T = 160, 700, 2048, where it leaves fewer padded columns)."""
    ref, acc, Y = _linear_case(bn, n_out, k, T, seed=n_out + T, y_dtype="bf16")
    _check_outputs(ref, acc, Y)


@pytest.mark.parametrize("T,n_out,k", [(512, 256, 8192), (256, 512, 256)])
def test_dgrad_pair_tile_widths(bn, T, n_out, k):
    """dgrad through the pair kernel: wide output (k = 8192, many tiles per
    pair) and a single tile."""
    W = synth.master_weights(n_out, k, 0.02, seed=T + n_out)
    g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
    pw = bn.PackedWeights(n_out, k, mma=False, dec=False)
    bn.bitnet_pack_nm(dev_f32(W), pw, 1e-5)
    dYd, dY32 = bf16_dev(synth.activations(T, n_out, seed=T + 1))
    dX = bn.bitnet_dgrad(dYd, pw, dx_dtype=torch.float32)
    torch.cuda.synchronize()
    ref, absref = oracle.dgrad(dY32, wq, g)
    tol = 2 * n_out * 2.0 ** -24 * absref + 1e-30
    assert np.all(np.abs(dX.cpu().numpy().astype(np.float64) - ref) <= tol)

"""GPU parity of the training-step pieces around the hot path: the dense
weight gradient (straight-through to every master), the AdamW step of the fp32
masters with the exact next gamma, and the pack that reads that gamma instead
of summing |W| ("Sparse-BitNet" (gist.science), section 2 "Training
Strategie"; "BitNet b1.58 ...", section "The mechanism").

Bar: AdamW (W, m, v) and gamma bit-exact (each step one IEEE fp32 operation on
both sides); the pack with a known gamma bit-identical to bitnet_pack_nm and to
the oracle; dW within the fp32-summation bound (T + 2) 2^-24 sum_t |dY X|.
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


@pytest.mark.parametrize("n_out,k,T", [(256, 512, 64), (200, 264, 100), (1000, 2560, 300), (512, 256, 1),
                                       (136, 72, 513), (3200, 3200, 2048)])
@pytest.mark.parametrize("accumulate", [False, True])
def test_wgrad_parity(bn, n_out, k, T, accumulate):
    r = np.random.default_rng(n_out + k + T)
    dYd, dY = bf16_dev(r.normal(size=(T, n_out)).astype(np.float32))
    Xd, X = bf16_dev((r.normal(size=(T, k)) * np.where(r.random((T, k)) < 0.01, 20.0, 1.0)).astype(np.float32))
    ref = oracle.wgrad(dY, X)
    bound = (T + 2) * 2.0 ** -24 * oracle.wgrad(np.abs(dY), np.abs(X)) + 1e-30
    dW0 = r.normal(size=(n_out, k)).astype(np.float32) if accumulate else np.full((n_out, k), np.nan, np.float32)
    dW = torch.from_numpy(dW0).cuda()
    bn.bitnet_wgrad(dYd, Xd, dW=dW, accumulate=accumulate)
    torch.cuda.synchronize()
    got = dW.cpu().numpy().astype(np.float64)
    if accumulate:
        ref = ref + dW0
        bound = bound + 2.0 ** -24 * (np.abs(dW0) + np.abs(ref))
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= bound)


def test_wgrad_empty_batch(bn):
    dW = torch.full((64, 128), 3.0, device="cuda")
    bn.bitnet_wgrad(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"),
                    torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"), dW=dW)
    torch.cuda.synchronize()
    assert not dW.any()
    dW.fill_(3.0)
    bn.bitnet_wgrad(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"),
                    torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"), dW=dW, accumulate=True)
    torch.cuda.synchronize()
    assert bool((dW == 3.0).all())


def _masters(n_out, k, seed, rare=False):
    W = synth.master_weights(n_out, k, 0.02, seed=seed)
    if rare:   # magnitudes outside the fast window and exact zeros (exact-sum bins)
        W.reshape(-1)[::97] = 0.0
        W.reshape(-1)[5::131] = 3.5e-30
        W.reshape(-1)[7::257] = 12.0
    return W


@pytest.mark.parametrize("n_out,k,rare", [(256, 512, False), (200, 352, True), (3200, 3200, False), (96, 64, True)])
def test_adamw_step_parity(bn, n_out, k, rare):
    r = np.random.default_rng(n_out * 7 + k)
    W = _masters(n_out, k, 400 + n_out, rare)
    n = W.size
    M = np.zeros(n, np.float32)
    V = np.zeros(n, np.float32)
    Wd, Md, Vd = (torch.from_numpy(a.reshape(-1).copy()).cuda() for a in (W, M, V))
    gamma = torch.zeros(1, device="cuda")
    Wn = W.reshape(-1).copy()
    for step in range(1, 4):
        G = (r.normal(size=n) * 1e-3 * 2.0 ** r.integers(-8, 4, size=n)).astype(np.float32)
        c1, c2 = bn.adam_bias_correction(0.9, step), bn.adam_bias_correction(0.95, step)
        bn.bitnet_adamw_step(Wd, torch.from_numpy(G).cuda(), Md, Vd, step, lr=1e-3, beta1=0.9, beta2=0.95,
                             eps=1e-8, weight_decay=0.1, gamma_out=gamma, eps_gamma=1e-5)
        Wn, M, V = oracle.adamw(Wn, G, M, V, 1e-3, 0.9, 0.95, 1e-8, 0.1, c1, c2)
        torch.cuda.synchronize()
        assert np.array_equal(Wd.cpu().numpy().view(np.uint32), Wn.view(np.uint32)), step
        assert np.array_equal(Md.cpu().numpy().view(np.uint32), M.view(np.uint32)), step
        assert np.array_equal(Vd.cpu().numpy().view(np.uint32), V.view(np.uint32)), step
        assert gamma.item() == float(oracle.gamma(Wn.reshape(n_out, k), 1e-5)), step


def test_pack_with_known_gamma(bn):
    """AdamW leaves the exact gamma in out.gamma; the batched pack with
    gamma_known reads W once, keeps that gamma and writes every layout exactly
    as bitnet_pack_nm (and the oracle) does for the updated masters."""
    shapes = [(256, 512), (200, 352), (3200, 3200), (640, 2560)]
    r = np.random.default_rng(5)
    Ws = [torch.from_numpy(_masters(n, k, 600 + i)).cuda() for i, (n, k) in enumerate(shapes)]
    Ms = [torch.zeros_like(W) for W in Ws]
    Vs = [torch.zeros_like(W) for W in Ws]
    outs = [bn.PackedWeights(n, k, dec=(n % 16 == 0 and k % 64 == 0)) for n, k in shapes]
    masks = [torch.zeros(n * k // 8, dtype=torch.uint8, device="cuda") for n, k in shapes]
    for W, o in zip(Ws, outs):
        bn.bitnet_pack_nm(W, o, 1e-5)
    batch = bn.PackBatch([(Ws[i], outs[i], masks[i]) for i in range(len(shapes))], 1e-5, gamma_known=True)
    for step in range(1, 4):
        for i, W in enumerate(Ws):
            G = torch.from_numpy((r.normal(size=W.shape) * 1e-3).astype(np.float32)).cuda()
            bn.bitnet_adamw_step(W, G, Ms[i], Vs[i], step, lr=1e-3, weight_decay=0.1, gamma_out=outs[i].gamma)
        batch()
        torch.cuda.synchronize()
        for i, (n, k) in enumerate(shapes):
            ref = bn.PackedWeights(n, k, dec=outs[i].dec_codes is not None)
            mask_r = torch.zeros_like(masks[i])
            bn.bitnet_pack_nm(Ws[i], ref, 1e-5, mask_bits=mask_r)
            torch.cuda.synchronize()
            a = [outs[i].gamma, outs[i].group_bytes, outs[i].mma_vals, outs[i].mma_meta, masks[i]]
            b = [ref.gamma, ref.group_bytes, ref.mma_vals, ref.mma_meta, mask_r]
            if outs[i].dec_codes is not None:
                a.append(outs[i].dec_codes)
                b.append(ref.dec_codes)
            for x, y in zip(a, b):
                assert torch.equal(x, y), (step, i)
            if n * k <= 1 << 20:
                g, keep, wq, gb = oracle.pack_weights(Ws[i].cpu().numpy(), 1e-5)
                assert outs[i].gamma.item() == float(g) and np.array_equal(outs[i].group_bytes.cpu().numpy(), gb)


def test_adamw_batch_matches_single_calls(bn):
    """The one-launch AdamW over a list of matrices (mixed sizes: one chunk,
    many chunks, rare magnitudes) leaves W, m, v and every gamma bit-identical
    to one bitnet_adamw_step per matrix, over three steps; gamma also equals
    the oracle's."""
    shapes = [(256, 512, False), (96, 64, True), (3200, 3200, False), (200, 352, True), (640, 2560, False)]
    r = np.random.default_rng(21)
    Wb, Ws = [], []
    for i, (n, k, rare) in enumerate(shapes):
        W = _masters(n, k, 700 + i, rare).reshape(-1)
        Wb.append(torch.from_numpy(W.copy()).cuda())
        Ws.append(torch.from_numpy(W.copy()).cuda())
    Mb = [torch.zeros_like(w) for w in Wb]
    Vb = [torch.zeros_like(w) for w in Wb]
    Ms = [torch.zeros_like(w) for w in Ws]
    Vs = [torch.zeros_like(w) for w in Ws]
    gb = torch.zeros(len(shapes), device="cuda")
    gs = torch.zeros(len(shapes), device="cuda")
    Gs = [torch.empty_like(w) for w in Wb]
    batch = bn.AdamWBatch([(Wb[i], Gs[i], Mb[i], Vb[i], gb[i:i + 1]) for i in range(len(shapes))])
    for step in range(1, 4):
        for G in Gs:
            G.copy_(torch.from_numpy((r.normal(size=G.numel()) * 1e-3).astype(np.float32)))
        batch(step, lr=1e-3, weight_decay=0.1)
        for i in range(len(shapes)):
            bn.bitnet_adamw_step(Ws[i], Gs[i], Ms[i], Vs[i], step, lr=1e-3, weight_decay=0.1, gamma_out=gs[i:i + 1])
        torch.cuda.synchronize()
        for i in range(len(shapes)):
            assert torch.equal(Wb[i], Ws[i]) and torch.equal(Mb[i], Ms[i]) and torch.equal(Vb[i], Vs[i]), (step, i)
        assert torch.equal(gb, gs), step
        for i, (n, k, _) in enumerate(shapes):
            if n * k <= 1 << 20:
                assert gb[i].item() == float(oracle.gamma(Wb[i].cpu().numpy().reshape(n, k), 1e-5)), (step, i)

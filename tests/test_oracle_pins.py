"""Pins of the CPU oracle to things other than itself (CPU only).

Each function of ``oracle/`` is checked against an independent route to the
same defined value: math.fsum for the exact absolute sum, brute-force sorting
for the top-N mask, hand-worked fixtures in tests/golden/, NumPy integer and
fp64 matrix products, closed forms for Gaussian weights, and invariants the
pages state (codes in {-1,0,1}, at most N non-zeros per group of M, symmetric
activation codes with no zero-point).
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from sparse_linear_layers_bitnet_b200 import synth
from tests.conftest import ROOT, load_golden
import os


# ---------------------------------------------------------------- abs sum / gamma

def _fsum_abs(W):
    return math.fsum(abs(float(v)) for v in np.asarray(W, np.float32).ravel())


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_abs_sum_matches_fsum_gaussian(seed):
    W = synth.master_weights(64, 96, 0.02, seed)
    assert oracle.abs_sum(W) == _fsum_abs(W)


def test_abs_sum_matches_fsum_wide_exponents():
    r = np.random.default_rng(5)
    parts = [
        r.normal(0, 1, 500) * np.float32(1e30),
        r.normal(0, 1, 500) * np.float32(1e-30),
        r.normal(0, 1, 500) * np.float32(1e-3),
        np.array([0.0, -0.0, 1e-45, -1e-45, 1.17549435e-38, 3.4e38, -3.4e38, 2.0 ** -149]),
        r.normal(0, 1, 500) * np.float32(1e-40),     # subnormal fp32
    ]
    W = np.concatenate([np.asarray(p, np.float32) for p in parts]).astype(np.float32)
    r.shuffle(W)
    assert oracle.abs_sum(W) == _fsum_abs(W)


def test_abs_sum_rounding_tie_cases():
    # 2^53 + 1 (in units) is a tie between 2^53 and 2^53 + 2; exact-then-round
    # must give the even neighbour; fsum agrees.
    W = np.array([2.0 ** 52, 2.0 ** 52, 1.0], np.float32)
    assert oracle.abs_sum(W) == _fsum_abs(W) == 2.0 ** 53
    W = np.array([2.0 ** 52, 2.0 ** 52, 1.0, 1.0, 1.0], np.float32)
    assert oracle.abs_sum(W) == _fsum_abs(W) == 2.0 ** 53 + 4
    W = np.array([2.0 ** 60] + [1.0] * 300, np.float32)
    assert oracle.abs_sum(W) == _fsum_abs(W)


@pytest.mark.parametrize("eps", [0.0, 1e-5])
def test_gamma_from_fsum(eps):
    W = synth.master_weights(32, 64, 0.02, 7)
    expect = np.float32(np.float32(_fsum_abs(W) / W.size) + np.float32(eps))
    assert oracle.gamma(W, eps) == expect


def test_gamma_is_order_independent():
    W = synth.master_weights(16, 256, 0.02, 3)
    perm = np.random.default_rng(0).permutation(W.size)
    assert oracle.gamma(W) == oracle.gamma(W.ravel()[perm].reshape(W.shape))


# ---------------------------------------------------------------- mask

def _brute_mask(W, n, m):
    keep = np.zeros(W.shape, np.uint8)
    for r in range(W.shape[0]):
        for g in range(W.shape[1] // m):
            vals = [abs(float(W[r, g * m + p])) for p in range(m)]
            order = sorted(range(m), key=lambda p: (-vals[p], p))
            for p in order[:n]:
                keep[r, g * m + p] = 1
    return keep


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (3, 4), (6, 8), (4, 8)])
def test_mask_matches_sorting_brute_force(n, m):
    W = synth.master_weights(24, 64, 0.02, 11)
    # plant exact ties and signed zeros
    W[0, :m] = 0.25
    W[1, :m] = 0.0
    W[1, 1] = -0.0
    W[2, :4] = [-0.5, 0.5, 0.25, -0.25]
    assert np.array_equal(oracle.mask_nm(W, n, m), _brute_mask(W, n, m))


def test_mask_all_permutations_of_distinct_magnitudes():
    mags = [0.1, 0.2, 0.3, 0.4]
    rows = []
    for perm in itertools.permutations(range(4)):
        rows.append([mags[p] * (1 if i % 2 else -1) for i, p in enumerate(perm)])
    W = np.array(rows, np.float32)
    keep = oracle.mask_nm(W, 2, 4)
    for i, perm in enumerate(itertools.permutations(range(4))):
        # kept positions hold the two largest magnitudes (0.3 and 0.4)
        kept = {p for p in range(4) if keep[i, p]}
        assert kept == {j for j in range(4) if perm[j] >= 2}


def test_mask_ties_lower_index():
    W = np.array([[0.25, 0.25, 0.25, 0.25],
                  [0.0, -0.0, 0.0, -0.0],
                  [0.1, 0.3, 0.3, 0.3],
                  [0.3, 0.1, 0.1, 0.3]], np.float32)
    keep = oracle.mask_nm(W, 2, 4)
    assert keep.tolist() == [[1, 1, 0, 0], [1, 1, 0, 0], [0, 1, 1, 0], [1, 0, 0, 1]]


# ---------------------------------------------------------------- ternary

def _hexf(s):
    return np.float32(float.fromhex(s))


def test_ternary_boundaries_golden():
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", "ternary_boundaries.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                g, w, c = line.split()
                rows.append((_hexf(g), _hexf(w), int(c)))
    for g, w, c in rows:
        assert oracle.ternary(np.array([w], np.float32), g)[0] == c, (g, w, c)


def test_ternary_matches_numpy_rint_clip():
    W = synth.master_weights(64, 64, 0.02, 4)
    g = oracle.gamma(W)
    ref = np.clip(np.rint(W / np.float32(g)), -1, 1).astype(np.int8)   # numpy float32 IEEE ops
    assert np.array_equal(oracle.ternary(W, g), ref)


def test_gaussian_zero_fraction_closed_form():
    # W ~ N(0, s): gamma -> s*sqrt(2/pi) (+eps); a weight is coded 0 when
    # |W| <= gamma/2, so P(zero) = 2*Phi(c) - 1 with c = gamma / (2 s).
    # Among the 2 kept of 4 (top-2 by |W|), the zero fraction is
    # [P(X(3) <= c) + P(X(4) <= c)] / 2 = 2 F^3 (1 - F) + F^4, F = P(zero).
    s, eps = 0.02, 1e-5
    W = synth.master_weights(1024, 1024, s, 21)
    g = float(oracle.gamma(W, eps))
    c = (s * math.sqrt(2 / math.pi) + eps) / (2 * s)
    F = math.erf(c / math.sqrt(2))
    wt = oracle.ternary(W, g)
    n = W.size
    dense_zero = float(np.mean(wt == 0))
    assert abs(dense_zero - F) < 5 * math.sqrt(F * (1 - F) / n)
    assert abs(F - 0.3101) < 1e-3
    keep = oracle.mask_nm(W, 2, 4)
    kept_zero = float(np.mean(wt[keep == 1] == 0))
    Fk = 2 * F ** 3 * (1 - F) + F ** 4
    assert abs(kept_zero - Fk) < 6 * math.sqrt(Fk * (1 - Fk) / (n / 2))


# ---------------------------------------------------------------- pack

def _decode_group_bytes(gb, k):
    rows = gb.shape[0]
    wq = np.zeros((rows, k), np.int8)
    keep = np.zeros((rows, k), np.uint8)
    val = {0: 0, 1: 1, 3: -1}
    for r in range(rows):
        for g in range(k // 4):
            b = int(gb[r, g])
            i0, i1, c0, c1 = b & 3, (b >> 2) & 3, (b >> 4) & 3, (b >> 6) & 3
            assert i0 < i1 and c0 != 2 and c1 != 2
            keep[r, 4 * g + i0] = keep[r, 4 * g + i1] = 1
            wq[r, 4 * g + i0] = val[c0]
            wq[r, 4 * g + i1] = val[c1]
    return wq, keep


def test_pack_round_trip_and_invariants():
    W = synth.master_weights(40, 128, 0.02, 9)
    g, keep, wq, gb = oracle.pack_weights(W)
    assert set(np.unique(wq)).issubset({-1, 0, 1})
    assert np.all(keep.reshape(40, -1, 4).sum(-1) == 2)
    assert np.all((wq != 0).reshape(40, -1, 4).sum(-1) <= 2)
    dwq, dkeep = _decode_group_bytes(gb, 128)
    assert np.array_equal(dwq, wq) and np.array_equal(dkeep, keep)


# ---------------------------------------------------------------- golden forward

def test_apply_mask_zeroes_exactly_the_dropped_entries():
    # hand example: codes of every sign, a kept zero code and dropped non-zero codes
    wt = np.array([[1, -1, 0, 1, -1, -1, 1, 0]], np.int8)
    keep = np.array([[1, 0, 1, 0, 0, 1, 1, 0]], np.uint8)
    assert oracle.apply_mask(wt, keep).tolist() == [[1, 0, 0, 0, 0, -1, 1, 0]]


def test_bf16_widening_known_bit_patterns():
    # bf16 is the top half of the fp32 pattern: values fixed by the IEEE format
    u = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x0001, 0x7F7F, 0x3EAB], np.uint16)
    got = oracle.bf16_to_f32(u)
    assert got[0] == 1.0 and got[1] == -2.0 and got[2] == 0.0
    assert got[3] == 0.0 and np.signbit(got[3])
    assert got[4] == np.float32(2.0 ** -133)                           # smallest bf16 subnormal
    assert got[5] == np.float32((2 - 2.0 ** -7) * 2.0 ** 127)          # largest finite bf16
    assert got[6] == np.float32((1 + 0x2B / 128) * 2.0 ** -2)          # 0.333984375


def test_worked_example():
    G = load_golden("worked_2x8.txt")
    f = lambda k: np.array([float(v) for v in G[k]], np.float32)
    i = lambda k: np.array([int(v) for v in G[k]])
    W = f("W").reshape(2, 8)
    X = f("X").reshape(2, 8)
    eps_w, eps_a = float(G["eps_w"][0]), float(G["eps_a"][0])
    out = oracle.forward(W, X, eps_w, eps_a)
    assert out["gamma"] == np.float32(float(G["gamma"][0]))
    assert out["keep"].ravel().tolist() == i("keep").tolist()
    assert out["wq"].ravel().tolist() == i("wq").tolist()
    assert out["gb"].ravel().tolist() == i("group_bytes").tolist()
    assert out["xq"].ravel().tolist() == i("xq").tolist()
    assert np.array_equal(out["a"], f("a"))
    assert out["acc"].ravel().tolist() == i("acc").tolist()
    y_exact = np.array([float(v) for v in G["y_num"]]) / float(G["y_den"][0])
    assert np.allclose(out["y"].ravel(), y_exact, rtol=1e-6, atol=0)
    dY = f("dY").reshape(1, 2)
    dX, _ = oracle.dgrad(dY, out["wq"], out["gamma"])
    assert np.array_equal(dX.ravel(), np.array([float(v) for v in G["dX"]]))


# ---------------------------------------------------------------- activations

def test_quant_act_invariants():
    X = synth.activations(33, 200, 3, outlier_p=0.01)
    Xq, a = oracle.quant_act(X)
    assert Xq.dtype == np.int8 and np.all(np.abs(Xq.astype(int)) <= 127)
    assert np.all(np.abs(Xq.astype(int)).max(1) == 127)       # the absmax element maps to 127
    assert np.array_equal(a, np.maximum(np.abs(X).max(1), np.float32(1e-5)))
    Xn, an = oracle.quant_act(-X)
    assert np.array_equal(Xn, -Xq) and np.array_equal(an, a)   # symmetric, no zero-point
    # codes are monotone in x within a token
    for t in range(4):
        o = np.argsort(X[t], kind="stable")
        assert np.all(np.diff(Xq[t][o].astype(int)) >= 0)


def test_quant_act_zero_row_uses_eps():
    X = np.zeros((2, 16), np.float32)
    X[1, 3] = 1e-7
    Xq, a = oracle.quant_act(X, 1e-5)
    assert np.all(Xq[0] == 0) and a[0] == np.float32(1e-5)
    assert a[1] == np.float32(1e-5) and Xq[1, 3] == round(1e-7 * 127 / 1e-5)


# ---------------------------------------------------------------- products

def test_gemm_i32_matches_numpy_int64():
    r = np.random.default_rng(2)
    Xq = r.integers(-127, 128, size=(17, 96)).astype(np.int8)
    Wq = r.integers(-1, 2, size=(40, 96)).astype(np.int8)
    ref = Xq.astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(oracle.gemm_i32(Xq, Wq), ref)


def test_gemm_i32_extreme_accumulator():
    K = 4096
    Xq = np.full((2, K), 127, np.int8)
    Xq[1] = -127
    Wq = np.zeros((1, K), np.int8)
    Wq[0, ::2] = 1        # 2:4-feasible: half the weights non-zero
    assert oracle.gemm_i32(Xq, Wq).ravel().tolist() == [127 * K // 2, -127 * K // 2]


def test_forward_matches_dense_masked_brute_force():
    W = synth.master_weights(48, 64, 0.02, 13)
    X = synth.activations(5, 64, 14)
    out = oracle.forward(W, X)
    # brute force: dense fp64 product of dequantised operands
    yb = (out["xq"].astype(np.float64) * out["a"][:, None] / 127.0) @ \
         (out["wq"].astype(np.float64) * float(out["gamma"])).T
    assert np.allclose(out["y"], yb, rtol=2e-6, atol=1e-7)
    # and the method approximates the full-precision product of the masked weights
    yfp = X.astype(np.float64) @ (out["wq"] * float(out["gamma"])).T
    bound = (np.abs(out["wq"]).astype(np.float64) * float(out["gamma"])).sum(1)[None, :] \
        * (out["a"][:, None] / 127.0) * 0.5 + 1e-6
    assert np.all(np.abs(out["y"] - yfp) <= bound)


def test_forward_6of8_matches_python_brute_force():
    """The 6:8 forward of the oracle against pure-Python loops: top-6 of every
    8 by (|w| desc, position asc), codes clip(rint(w / gamma)), integer sums."""
    W = synth.master_weights(6, 32, 0.02, 31)
    W[0, :8] = 0.01                      # an all-tie block: positions 0..5 kept
    X = synth.activations(3, 32, 32)
    out = oracle.forward_nm(W, X, 6, 8)
    g = float(out["gamma"])
    keep = _brute_mask(W, 6, 8)
    assert np.array_equal(out["keep"], keep)
    assert keep[0, :8].tolist() == [1, 1, 1, 1, 1, 1, 0, 0]
    xq = out["xq"].astype(np.int64)
    for r in range(W.shape[0]):
        for t in range(X.shape[0]):
            acc = 0
            for c in range(W.shape[1]):
                if keep[r, c]:
                    q = int(np.clip(np.rint(np.float32(W[r, c]) / np.float32(g)), -1, 1))
                    acc += q * int(xq[t, c])
            assert acc == int(out["acc"][t, r])
    assert (keep.reshape(6, -1, 8).sum(2) == 6).all()


def test_dgrad_matches_numpy_fp64():
    r = np.random.default_rng(8)
    dY = r.normal(size=(6, 40)).astype(np.float32)
    Wq = r.integers(-1, 2, size=(40, 24)).astype(np.int8)
    dX, absdX = oracle.dgrad(dY, Wq, np.float32(0.0173))
    ref = (dY.astype(np.float64) @ Wq.astype(np.float64)) * float(np.float32(0.0173))
    assert np.allclose(dX, ref, rtol=1e-12, atol=1e-12)
    assert np.all(absdX >= np.abs(dX) - 1e-12)


def test_quant_act_ties_golden():
    G = load_golden("quant_ties.txt")
    X = np.array([float(v) for v in G["X"]], np.float32).reshape(2, 8)
    Xq, a = oracle.quant_act(X)
    assert Xq.ravel().tolist() == [int(v) for v in G["xq"]]
    assert a.tolist() == [float(v) for v in G["a"]]


# ------------------------------------------------------------------ block epilogues (RMSNorm, SwiGLU)

def test_exp32_within_5_ulp_of_exp_and_exact_at_zero():
    x = np.linspace(-87.0, 88.0, 350001).astype(np.float32)
    e = oracle.exp32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    assert np.all(np.abs(e - ref) <= 5 * 2.0 ** -24 * ref)
    assert oracle.exp32(np.zeros(3, np.float32)).tolist() == [1.0, 1.0, 1.0]
    # at the reduction boundaries (x near n ln 2 for every n) the same bound holds
    xs = (np.arange(-125, 127, dtype=np.float64) * math.log(2.0)).astype(np.float32)
    xs = xs[(xs >= -87.0) & (xs <= 88.0)]
    e2 = oracle.exp32(xs).astype(np.float64)
    ref2 = np.exp(xs.astype(np.float64))
    assert np.all(np.abs(e2 - ref2) <= 5 * 2.0 ** -24 * ref2)


def test_swiglu_matches_fp64_and_limits():
    r = np.random.default_rng(41)
    G = (r.normal(size=(3, 2000)) * 6).astype(np.float32)
    U = r.normal(size=(3, 2000)).astype(np.float32)
    h = oracle.swiglu(G, U).astype(np.float64)
    g64, u64 = G.astype(np.float64), U.astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64)) * u64
    assert np.all(np.abs(h - ref) <= 1e-6 * np.abs(ref) + 1e-30)
    z = oracle.swiglu(np.zeros((1, 4), np.float32), np.ones((1, 4), np.float32))
    assert z.tolist() == [[0.0, 0.0, 0.0, 0.0]]                      # silu(0) = 0
    big = oracle.swiglu(np.full((1, 2), 60.0, np.float32), np.ones((1, 2), np.float32))
    assert big.tolist() == [[60.0, 60.0]]                            # silu(g) = g for large g in fp32


def test_rmsnorm_closed_forms_and_fp64():
    import fractions
    # constant row c: mean of squares is c^2 exactly
    for c in (0.5, 3.0, 1.0 / 1024):
        X = np.full((1, 3200), c, np.float32)
        xn = oracle.rmsnorm(X, 1e-6)
        ms = np.float32(c * c)
        r = np.float32(np.float32(1.0) / np.sqrt(np.float32(ms + np.float32(1e-6))))
        assert np.all(xn == np.float32(np.float32(c) * r))
    # the exact sum: fsum of the squares equals the rational sum rounded once
    r = np.random.default_rng(42)
    X = (r.normal(size=(1, 257)) * 2.0 ** r.integers(-20, 10, size=(1, 257))).astype(np.float32)
    exact = sum(fractions.Fraction(float(v)) ** 2 for v in X[0])
    S = math.fsum((X[0].astype(np.float64) ** 2).tolist())
    assert S == float(exact)
    # against fp64 arithmetic on random rows
    X = r.normal(size=(4, 3200)).astype(np.float32)
    xn = oracle.rmsnorm(X, 1e-6).astype(np.float64)
    ref = X / np.sqrt((X.astype(np.float64) ** 2).mean(1, keepdims=True) + 1e-6)
    assert np.all(np.abs(xn - ref) <= 4 * 2.0 ** -24 * np.abs(ref))
    # a weight scales the normalised row element by element
    w = r.normal(size=3200).astype(np.float32)
    xw = oracle.rmsnorm(X, 1e-6, w)
    assert np.array_equal(xw, (oracle.rmsnorm(X, 1e-6) * w).astype(np.float32))


def test_wgrad_brute_force_and_one_hot():
    r = np.random.default_rng(7)
    T, N, K = 5, 3, 4
    dY = r.normal(size=(T, N)).astype(np.float32)
    X = r.normal(size=(T, K)).astype(np.float32)
    dW = oracle.wgrad(dY, X)
    for n in range(N):                      # brute force, one product at a time
        for k in range(K):
            s = math.fsum(float(dY[t, n]) * float(X[t, k]) for t in range(T))
            assert abs(dW[n, k] - s) <= 1e-12 * max(1.0, abs(s))
    # a one-hot output gradient picks one input row into one gradient row
    e = np.zeros((T, N), np.float32)
    e[2, 1] = 1.0
    dW1 = oracle.wgrad(e, X)
    assert np.array_equal(dW1[1], X[2].astype(np.float64)) and not dW1[[0, 2]].any()


def test_adamw_closed_forms():
    f = np.float32
    r = np.random.default_rng(3)
    W = r.normal(size=4096).astype(f)
    G = (r.normal(size=4096) * 2.0 ** r.integers(-10, 4, size=4096)).astype(f)
    z = np.zeros_like(W)
    b1, b2 = 0.9, 0.95
    # first step from zero moments: m / c1 = g and v / c2 = g^2 up to rounding, so the
    # update is sign(g) (|g| >> eps): w' = w - lr sign(g)
    W1, M1, V1 = oracle.adamw(W, G, z, z, 1e-3, b1, b2, 1e-12, 0.0, f(1 - b1), f(1 - b2))
    assert np.all(np.abs((W1.astype(np.float64) - W) + 1e-3 * np.sign(G)) <= 1e-3 * 1e-5 + 4 * 2.0 ** -24 * np.abs(W))
    # (1 - b1) is formed in fp32 from fp32(b1): a relative 2.4e-7 from 0.1, plus one rounding
    assert np.allclose(M1, (1 - b1) * G.astype(np.float64), rtol=4e-7, atol=0)
    assert np.allclose(V1, (1 - b2) * G.astype(np.float64) ** 2, rtol=8e-7, atol=0)
    # no gradient and no moments: pure decoupled decay w' = w (1 - lr wd)
    W2, M2, V2 = oracle.adamw(W, z, z, z, 1e-2, b1, b2, 1e-8, 0.1, f(0.5), f(0.5))
    assert not M2.any() and not V2.any()
    assert np.allclose(W2, W.astype(np.float64) * (1 - 1e-3), rtol=3e-7, atol=0)
    # a constant gradient for t steps: the bias-corrected first moment is that gradient
    g = f(0.25)
    Wt, Mt, Vt = W[:8].copy(), np.zeros(8, f), np.zeros(8, f)
    p1 = p2 = 1.0
    for t in range(1, 6):
        p1 *= b1
        p2 *= b2
        c1, c2 = f(1 - p1), f(1 - p2)
        Wn, Mt, Vt = oracle.adamw(Wt, np.full(8, g, f), Mt, Vt, 1e-3, b1, b2, 1e-12, 0.0, c1, c2)
        assert np.allclose(Mt / c1, g, rtol=1e-6) and np.allclose(np.sqrt(Vt / c2), g, rtol=1e-6)
        assert np.allclose(Wt - Wn, 1e-3, rtol=1e-4)       # |update| = lr when m_hat = sqrt(v_hat)
        Wt = Wn
    # the update does not depend on the gradient's scale (eps negligible)
    Wa, _, _ = oracle.adamw(W, G, z, z, 1e-3, b1, b2, 1e-30, 0.0, f(1 - b1), f(1 - b2))
    Wb, _, _ = oracle.adamw(W, (G * f(8.0)).astype(f), z, z, 1e-3, b1, b2, 1e-30, 0.0, f(1 - b1), f(1 - b2))
    assert np.allclose(Wa, Wb, rtol=0, atol=4 * 2.0 ** -24 * 4)

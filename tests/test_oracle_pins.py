"""Pins for the fp64 CPU oracle: values and identities the pages and the mathematics fix.

Nothing here compares the oracle with itself.  Each test checks it against
something independent: numbers printed on the pages (golden files), closed forms,
a library routine for a special case (torch scaled_dot_product_attention in
float64), or an algebraic identity whose failure a dropped term, a wrong sign,
a wrong loop index or a transposed operand would expose.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import lla_synth as S
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [line.split() for line in f if line.strip() and not line.startswith("#")]


def sdpa(q, K, V, scale):
    """Textbook attention of one query via torch (float64): returns (o, lse)."""
    qt = torch.as_tensor(q, dtype=torch.float64)[None, None, None, :]
    Kt = torch.as_tensor(K, dtype=torch.float64)[None, None]
    Vt = torch.as_tensor(V, dtype=torch.float64)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    lse = torch.logsumexp(scale * (Kt[0, 0] @ qt[0, 0, 0]), dim=0)
    return o[0, 0, 0].numpy(), float(lse)


# ---------------------------------------------------------------------------
# Eq. 4 / Figure 10 / Table 8: exact compression ratio and cache bytes
# ---------------------------------------------------------------------------
def test_rank_table_golden():
    rows = _rows("rank_table.txt")
    assert len(rows) == 6
    for T, d, rk, rv, printed in rows:
        lat, unc, num, den = oracle.cache_bytes(int(T), 1, 1, int(d), int(rk), int(rv),
                                                False, 2, 1)
        digits = len(printed.split(".")[1]) if "." in printed else 0
        assert round(num / den, digits) == float(printed)
        assert Fraction(unc, lat) == Fraction(num, den)


def test_headline_ratios_golden():
    for T, d, rsum, printed, digits in _rows("headline_ratios.txt"):
        rk = int(rsum) // 3
        rv = int(rsum) - rk
        _, _, num, den = oracle.cache_bytes(int(T), 1, 1, int(d), rk, rv, False, 2, 1)
        assert round(num / den, int(digits)) == float(printed)


def test_rho_closed_forms():
    # per head: 2*T*d/(r_k+r_v), reduced
    assert oracle.cache_bytes(4, 1, 16, 128, 16, 32, False, 2, 1)[2:] == (64, 3)
    assert oracle.cache_bytes(4, 1, 2, 64, 8, 16, False, 4, 1)[2:] == (64, 3)
    assert oracle.cache_bytes(4, 24, 16, 128, 96, 160, False, 2, 1)[2:] == (4, 1)
    assert oracle.cache_bytes(32, 8, 16, 128, 96, 160, False, 2, 1)[2:] == (32, 1)
    # LLA-2D folds the H heads into one latent: 2*T*H*d/(r_k+r_v) = 16384/192
    assert oracle.cache_bytes(4, 24, 16, 128, 64, 128, True, 2, 1)[2:] == (256, 3)


def test_capacity_bytes_exact():
    # 768 sequences x 4096 tokens, 24 layers, 16 heads, r_k+r_v = 48, bf16
    lat, unc, num, den = oracle.cache_bytes(4, 24, 16, 128, 16, 32, False, 2, 768 * 4096)
    assert lat == 768 * 4096 * 24 * 16 * 48 * 2 == 115_964_116_992
    assert unc == 768 * 4096 * 24 * 16 * 2 * 4 * 128 * 2
    assert lat * num == unc * den


def test_cache_bytes_linear_and_divided_by_rho():
    rng = np.random.default_rng(5)
    for _ in range(200):
        T, L, H = (int(v) for v in rng.integers(1, 40, 3))
        d = int(rng.choice([16, 32, 64, 128, 256]))
        rk, rv = (int(v) for v in rng.integers(1, 600, 2))
        fold = bool(rng.integers(0, 2))
        e = int(rng.choice([2, 4]))
        n = int(rng.integers(0, 10 ** 7))
        lat, unc, num, den = oracle.cache_bytes(T, L, H, d, rk, rv, fold, e, n)
        lat2, unc2, _, _ = oracle.cache_bytes(T, L, H, d, rk, rv, fold, e, 2 * n + 3)
        assert lat2 * n == lat * (2 * n + 3) and unc2 * n == unc * (2 * n + 3)
        assert lat * num == unc * den
        assert math.gcd(num, den) == 1
        Hs = 1 if fold else H
        assert Fraction(num, den) == Fraction(2 * T * H * d, Hs * (rk + rv))


def test_cache_bytes_rejects_bad_dims():
    with pytest.raises(ValueError):
        oracle.cache_bytes(0, 1, 1, 64, 8, 16, False, 2, 1)
    with pytest.raises(ValueError):
        oracle.cache_bytes(4, 1, 1, 64, 8, 16, False, 2, -1)


# ---------------------------------------------------------------------------
# Eqs. 2-3: encode and per-loop reconstruction
# ---------------------------------------------------------------------------
def test_full_rank_roundtrip_is_exact():
    T, d = 4, 8
    codec = S.orthonormal_codec(T * d, T, seed=1)
    x = np.random.default_rng(2).standard_normal((50, T * d)) * 3 + 1
    c = oracle.encode(x, codec.mu, codec.W_down)
    for t in range(T):
        xt = oracle.reconstruct(c, codec.W_up[t], codec.mu_t()[t])
        np.testing.assert_allclose(xt, x[:, t * d:(t + 1) * d], atol=1e-12, rtol=0)


def test_encode_of_mean_is_zero_and_affine():
    T, d, r = 3, 8, 5
    rng = np.random.default_rng(3)
    W_down = rng.standard_normal((T * d, r))
    mu = rng.standard_normal(T * d)
    np.testing.assert_allclose(oracle.encode(mu[None], mu, W_down), 0.0, atol=1e-14)
    x1, x2 = rng.standard_normal((2, 7, T * d))
    a = 0.3
    lhs = oracle.encode(a * x1 + (1 - a) * x2, mu, W_down)
    rhs = a * oracle.encode(x1, mu, W_down) + (1 - a) * oracle.encode(x2, mu, W_down)
    np.testing.assert_allclose(lhs, rhs, atol=1e-12)
    # one-hot tokens pick rows of W_down (checks operand orientation)
    e = np.zeros((T * d, T * d))
    np.fill_diagonal(e, 1.0)
    np.testing.assert_allclose(oracle.encode(e, np.zeros(T * d), W_down), W_down, atol=0)


def test_reconstruct_orientation_one_hot():
    r, d = 5, 7
    rng = np.random.default_rng(4)
    W_up = rng.standard_normal((r, d))
    mu = rng.standard_normal(d)
    c = np.eye(r)
    np.testing.assert_allclose(oracle.reconstruct(c, W_up, mu), W_up + mu[None], atol=0)


@pytest.mark.parametrize("r", [1, 4, 16, 40])
def test_eckart_young_calibration_residual(r):
    """Residual of the SVD codec on its own calibration set = tail singular energy."""
    w = S.shrink(S.WORKLOADS["tiny-fp32"], d=16)
    model = S.trajectory_model(11, w.T * w.d)
    x_cal = S.draw_tokens_np(model, S.N_CALIB, 12)
    codec = S.fit_codec(x_cal, r, w.T)
    c = oracle.encode(x_cal, codec.mu, codec.W_down)
    resid = 0.0
    for t in range(w.T):
        xt = oracle.reconstruct(c, codec.W_up[t], codec.mu_t()[t])
        resid += ((x_cal[:, t * w.d:(t + 1) * w.d] - xt) ** 2).sum()
    tail = (codec.sigma[r:] ** 2).sum()
    assert resid == pytest.approx(tail, rel=1e-9, abs=1e-9)


# ---------------------------------------------------------------------------
# Decode attention (reconstruct and absorb forms)
# ---------------------------------------------------------------------------
VARIANTS = ["absorb", "reconstruct"]


def _codec_pair(T, d, rk, rv, seed, perturb=0.2):
    rng = np.random.default_rng(seed)
    out = []
    for r in (rk, rv):
        W_up = rng.standard_normal((T, r, d)) / math.sqrt(r)
        mu = rng.standard_normal((T, d))
        out.append((W_up * (1 + perturb), mu))
    return out


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("scale", [1.0, 0.125, 3.0])
def test_full_rank_codec_equals_uncompressed_attention(variant, scale):
    """Full-rank orthonormal codec: decode over latents == plain attention on K/V."""
    T, d, n = 3, 8, 20
    rng = np.random.default_rng(7)
    cK, cV = S.orthonormal_codec(T * d, T, 8), S.orthonormal_codec(T * d, T, 9)
    xK = rng.standard_normal((n, T * d))
    xV = rng.standard_normal((n, T * d)) * 2
    lK, lV = oracle.encode(xK, cK.mu, cK.W_down), oracle.encode(xV, cV.mu, cV.W_down)
    for t in range(T):
        q = rng.standard_normal(d)
        o, lse = oracle.attend(variant, lK, lV, cK.W_up[t], cK.mu_t()[t], cV.W_up[t],
                               cV.mu_t()[t], q, scale)
        o_ref, lse_ref = sdpa(q, xK[:, t * d:(t + 1) * d], xV[:, t * d:(t + 1) * d], scale)
        np.testing.assert_allclose(o, o_ref, atol=1e-10, rtol=0)
        assert lse == pytest.approx(lse_ref, abs=1e-10)


def test_absorb_equals_reconstruct_low_rank():
    T, d, rk, rv, n = 4, 16, 3, 6, 33
    rng = np.random.default_rng(10)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 11)
    cK = rng.standard_normal((n, rk))
    cV = rng.standard_normal((n, rv))
    for t in range(T):
        q = rng.standard_normal(d)
        a = oracle.attend("absorb", cK, cV, WK[t], muK[t], WV[t], muV[t], q, 0.7)
        b = oracle.attend("reconstruct", cK, cV, WK[t], muK[t], WV[t], muV[t], q, 0.7)
        np.testing.assert_allclose(a[0], b[0], atol=1e-10, rtol=0)
        assert a[1] == pytest.approx(b[1], abs=1e-10)


@pytest.mark.parametrize("variant", VARIANTS)
def test_softmax_weights_sum_to_one(variant):
    """Constant values: o must equal that value exactly when sum_n p_n = 1."""
    T, d, rk, rv, n = 2, 8, 4, 5, 17
    rng = np.random.default_rng(12)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 13)
    cK = rng.standard_normal((n, rk)) * 3
    v0 = rng.standard_normal(rv)
    cV = np.tile(v0, (n, 1))
    q = rng.standard_normal(d)
    o, _ = oracle.attend(variant, cK, cV, WK[1], muK[1], WV[1], muV[1], q, 1.0)
    np.testing.assert_allclose(o, v0 @ WV[1] + muV[1], atol=1e-12)
    o0, _ = oracle.attend(variant, cK, 0 * cV, WK[1], muK[1], WV[1], muV[1], q, 1.0)
    np.testing.assert_allclose(o0, muV[1], atol=1e-14)


@pytest.mark.parametrize("variant", VARIANTS)
def test_shift_of_key_mean_is_invisible(variant):
    T, d, rk, rv, n = 2, 8, 4, 5, 9
    rng = np.random.default_rng(14)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 15)
    cK, cV = rng.standard_normal((n, rk)), rng.standard_normal((n, rv))
    q = rng.standard_normal(d)
    delta = rng.standard_normal(d)
    s = 0.9
    o1, l1 = oracle.attend(variant, cK, cV, WK[0], muK[0], WV[0], muV[0], q, s)
    o2, l2 = oracle.attend(variant, cK, cV, WK[0], muK[0] + delta, WV[0], muV[0], q, s)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    assert l2 - l1 == pytest.approx(s * q @ delta, abs=1e-12)


@pytest.mark.parametrize("variant", VARIANTS)
def test_single_token_returns_its_value(variant):
    T, d, rk, rv = 3, 8, 4, 6
    rng = np.random.default_rng(16)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 17)
    cK, cV = rng.standard_normal((1, rk)), rng.standard_normal((1, rv))
    q = rng.standard_normal(d)
    o, lse = oracle.attend(variant, cK, cV, WK[2], muK[2], WV[2], muV[2], q, 0.5)
    np.testing.assert_allclose(o, cV[0] @ WV[2] + muV[2], atol=1e-12)
    assert lse == pytest.approx(0.5 * q @ (cK[0] @ WK[2] + muK[2]), abs=1e-12)


@pytest.mark.parametrize("variant", VARIANTS)
def test_identity_codec_is_textbook_attention(variant):
    """T = 1, r = d, W_down = I, mu = 0: the latents are K and V themselves."""
    d, n = 8, 25
    rng = np.random.default_rng(18)
    K, V, q = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal(d)
    I, z = np.eye(d), np.zeros(d)
    cK, cV = oracle.encode(K, z, I), oracle.encode(V, z, I)
    o, lse = oracle.attend(variant, cK, cV, I, z, I, z, q, 1 / math.sqrt(d))
    o_ref, lse_ref = sdpa(q, K, V, 1 / math.sqrt(d))
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    assert lse == pytest.approx(lse_ref, abs=1e-12)


@pytest.mark.parametrize("variant", VARIANTS)
def test_large_logits_select_the_best_token(variant):
    """Very large scale: softmax becomes argmax and stays finite (max subtraction)."""
    d, n = 8, 40
    rng = np.random.default_rng(19)
    I, z = np.eye(d), np.zeros(d)
    K, V, q = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal(d)
    o, lse = oracle.attend(variant, K, V, I, z, I, z, q, 1e4)
    best = int(np.argmax(K @ q))
    assert np.all(np.isfinite(o)) and math.isfinite(lse)
    np.testing.assert_allclose(o, V[best], atol=1e-9)
    assert lse == pytest.approx(1e4 * K[best] @ q, rel=1e-12)


@pytest.mark.parametrize("variant", VARIANTS)
def test_empty_context(variant):
    d = 8
    o, lse = oracle.attend(variant, np.zeros((0, 3)), np.zeros((0, 4)), np.ones((3, d)),
                           np.ones(d), np.ones((4, d)), np.ones(d), np.ones(d), 1.0)
    assert np.all(o == 0) and lse == -math.inf


def _ragged_layer(T, H, d, lens, rk, rv, fold2d, seed, gap=3):
    rng = np.random.default_rng(seed)
    starts = S.slot_starts(np.asarray(lens), gap=gap)
    n_slots = int(starts[-1] + lens[-1] + gap)
    Hs = 1 if fold2d else H
    c_K = rng.standard_normal((Hs, n_slots, rk))
    c_V = rng.standard_normal((Hs, n_slots, rv))
    if fold2d:
        WK = rng.standard_normal((T, rk, H * d)) / math.sqrt(rk)
        WV = rng.standard_normal((T, rv, H * d)) / math.sqrt(rv)
        mK, mV = rng.standard_normal((T, H * d)), rng.standard_normal((T, H * d))
    else:
        WK = rng.standard_normal((H, T, rk, d)) / math.sqrt(rk)
        WV = rng.standard_normal((H, T, rv, d)) / math.sqrt(rv)
        mK, mV = rng.standard_normal((H, T, d)), rng.standard_normal((H, T, d))
    return starts, c_K, c_V, WK, mK, WV, mV


@pytest.mark.parametrize("fold2d", [False, True])
def test_decode_layer_matches_masked_dense_attention(fold2d):
    """Ragged batch: per-sequence slicing checked against dense reconstruct + SDPA."""
    T, H, d, rk, rv = 3, 2, 8, 4, 6
    lens = np.array([5, 1, 0, 9], dtype=np.int32)
    starts, c_K, c_V, WK, mK, WV, mV = _ragged_layer(T, H, d, lens, rk, rv, fold2d, 20)
    B, Tq, t0, s = len(lens), 2, 1, 0.8
    q = np.random.default_rng(21).standard_normal((B, Tq, H, d))
    for variant in VARIANTS:
        o, lse = oracle.decode_layer(variant, q, c_K, c_V, starts, lens, WK, mK, WV, mV,
                                     t0, s, fold2d=fold2d, threads=2)
        for b in range(B):
            sl = slice(int(starts[b]), int(starts[b] + lens[b]))
            for tq in range(Tq):
                t = t0 + tq
                for h in range(H):
                    if fold2d:
                        cols = slice(h * d, (h + 1) * d)
                        Kh = c_K[0, sl] @ WK[t][:, cols] + mK[t][cols]
                        Vh = c_V[0, sl] @ WV[t][:, cols] + mV[t][cols]
                    else:
                        Kh = c_K[h, sl] @ WK[h, t] + mK[h, t]
                        Vh = c_V[h, sl] @ WV[h, t] + mV[h, t]
                    if lens[b] == 0:
                        assert np.all(o[b, tq, h] == 0) and lse[b, tq, h] == -np.inf
                        continue
                    o_ref, lse_ref = sdpa(q[b, tq, h], Kh, Vh, s)
                    np.testing.assert_allclose(o[b, tq, h], o_ref, atol=1e-11)
                    assert lse[b, tq, h] == pytest.approx(lse_ref, abs=1e-11)


def test_fold2d_with_one_head_equals_per_head():
    T, H, d, rk, rv = 3, 1, 8, 4, 6
    lens = np.array([7, 3], dtype=np.int32)
    starts, c_K, c_V, WK, mK, WV, mV = _ragged_layer(T, H, d, lens, rk, rv, True, 22)
    q = np.random.default_rng(23).standard_normal((2, 3, H, d))
    a = oracle.decode_layer("absorb", q, c_K, c_V, starts, lens, WK, mK, WV, mV, 0, 1.0,
                            fold2d=True, threads=1)
    b = oracle.decode_layer("absorb", q, c_K, c_V, starts, lens, WK[None], mK[None],
                            WV[None], mV[None], 0, 1.0, fold2d=False, threads=1)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("variant", VARIANTS)
def test_fold2d_full_rank_reproduces_each_head(variant):
    """LLA-2D full-rank codec over x in [T][H][d] order: head h's output equals plain
    attention on head h's own original K/V (pins the head column slicing)."""
    T, H, d, n = 2, 3, 4, 11
    W = T * H * d
    rng = np.random.default_rng(24)
    cK, cV = S.orthonormal_codec(W, T, 25), S.orthonormal_codec(W, T, 26)
    xK, xV = rng.standard_normal((n, W)), rng.standard_normal((n, W))
    lK, lV = oracle.encode(xK, cK.mu, cK.W_down), oracle.encode(xV, cV.mu, cV.W_down)
    q = rng.standard_normal((1, T, H, d))
    o, lse = oracle.decode_layer(variant, q, lK[None], lV[None], [0], [n], cK.W_up,
                                 cK.mu_t(), cV.W_up, cV.mu_t(), 0, 1.0, fold2d=True,
                                 threads=1)
    xK4, xV4 = xK.reshape(n, T, H, d), xV.reshape(n, T, H, d)
    for t in range(T):
        for h in range(H):
            o_ref, lse_ref = sdpa(q[0, t, h], xK4[:, t, h], xV4[:, t, h], 1.0)
            np.testing.assert_allclose(o[0, t, h], o_ref, atol=1e-10)
            assert lse[0, t, h] == pytest.approx(lse_ref, abs=1e-10)


# ---------------------------------------------------------------------------
# The input generator's stated statistics (pins the recipe, not the oracle)
# ---------------------------------------------------------------------------
def test_trajectory_model_energy_split():
    m = S.trajectory_model(30, 512)
    e = (m.A ** 2).sum(axis=1) / 512
    assert e.sum() == pytest.approx(1.0, abs=1e-12)
    assert e[0] == pytest.approx(S.TOP_ENERGY, abs=1e-12)
    np.testing.assert_allclose(m.A @ m.A.T, np.diag(e * 512), atol=1e-9)
    assert np.all(np.diff(e[1:]) < 0)


def test_latent_draw_statistics():
    std = np.array([3.0, 1.0, 0.25])
    z = S.draw_latents(200_000, std, 31, "cpu", torch.float32).double().numpy()
    np.testing.assert_allclose(z.std(axis=0), std, rtol=0.01)
    np.testing.assert_allclose(z.mean(axis=0), 0, atol=0.02)


# ---------------------------------------------------------------------------
# Hybrid form ("Hybrid Latent Attention for Looped Language Models", abstract):
# exact K/V for the window tokens, latents for the older ones, one softmax
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n,w", [(20, 5), (0, 7), (13, 0), (1, 1)])
def test_hybrid_full_rank_equals_attention_over_all_tokens(n, w):
    """A full-rank orthonormal codec rebuilds the older tokens exactly, so the hybrid
    result is textbook attention over all n + w original tokens (torch SDPA)."""
    T, d = 3, 8
    rng = np.random.default_rng(31 + n + 7 * w)
    cK, cV = S.orthonormal_codec(T * d, T, 18), S.orthonormal_codec(T * d, T, 19)
    xK = rng.standard_normal((n + w, T * d))
    xV = rng.standard_normal((n + w, T * d)) * 1.5
    lK = oracle.encode(xK[:n], cK.mu, cK.W_down) if n else np.zeros((0, T * d))
    lV = oracle.encode(xV[:n], cV.mu, cV.W_down) if n else np.zeros((0, T * d))
    for t in range(T):
        q = rng.standard_normal(d)
        sl = slice(t * d, (t + 1) * d)
        o, lse = oracle.attend_hybrid(lK, lV, cK.W_up[t], cK.mu_t()[t], cV.W_up[t], cV.mu_t()[t],
                                      xK[n:, sl], xV[n:, sl], q, 0.7)
        o_ref, lse_ref = sdpa(q, xK[:, sl], xV[:, sl], 0.7)
        np.testing.assert_allclose(o, o_ref, atol=1e-10, rtol=0)
        assert lse == pytest.approx(lse_ref, abs=1e-10)


def test_hybrid_window_order_is_irrelevant_and_empty_is_neutral():
    """The window is a set: its row order does not matter; and with no window the hybrid
    form is the latent-only decode attention (absorbed form, written separately)."""
    T, d, rk, rv, n, w = 4, 16, 3, 6, 17, 9
    rng = np.random.default_rng(40)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 41)
    cK, cV = rng.standard_normal((n, rk)), rng.standard_normal((n, rv))
    kw, vw = rng.standard_normal((w, d)), rng.standard_normal((w, d))
    perm = rng.permutation(w)
    for t in range(T):
        q = rng.standard_normal(d)
        a = oracle.attend_hybrid(cK, cV, WK[t], muK[t], WV[t], muV[t], kw, vw, q, 0.5)
        b = oracle.attend_hybrid(cK, cV, WK[t], muK[t], WV[t], muV[t], kw[perm], vw[perm], q, 0.5)
        np.testing.assert_allclose(a[0], b[0], atol=1e-12, rtol=0)
        assert a[1] == pytest.approx(b[1], abs=1e-12)
        e = oracle.attend_hybrid(cK, cV, WK[t], muK[t], WV[t], muV[t], kw[:0], vw[:0], q, 0.5)
        ref = oracle.attend("absorb", cK, cV, WK[t], muK[t], WV[t], muV[t], q, 0.5)
        np.testing.assert_allclose(e[0], ref[0], atol=1e-12, rtol=0)
        assert e[1] == pytest.approx(ref[1], abs=1e-12)


@pytest.mark.parametrize("fold2d", [False, True])
def test_decode_layer_hybrid_matches_dense_attention_over_both_parts(fold2d):
    """Ragged batch with ragged windows (one sequence with no latents, one with no
    window, one with neither): each unit against SDPA over [rebuilt older tokens; window]."""
    T, H, d, rk, rv = 3, 2, 8, 4, 6
    lens = np.array([5, 0, 4, 0], dtype=np.int32)
    wins = np.array([3, 2, 0, 0], dtype=np.int32)
    starts, c_K, c_V, WK, mK, WV, mV = _ragged_layer(T, H, d, lens, rk, rv, fold2d, 24)
    B, Tq, t0, s, wmax = len(lens), 2, 1, 0.6, 4
    rng = np.random.default_rng(25)
    q = rng.standard_normal((B, Tq, H, d))
    win_k = rng.standard_normal((B, H, T, wmax, d))
    win_v = rng.standard_normal((B, H, T, wmax, d))
    o, lse = oracle.decode_layer("absorb", q, c_K, c_V, starts, lens, WK, mK, WV, mV, t0, s,
                                 fold2d=fold2d, threads=2, window=(win_k, win_v, wins))
    for b in range(B):
        sl = slice(int(starts[b]), int(starts[b] + lens[b]))
        for tq in range(Tq):
            t = t0 + tq
            for h in range(H):
                if fold2d:
                    cols = slice(h * d, (h + 1) * d)
                    Kh = c_K[0, sl] @ WK[t][:, cols] + mK[t][cols]
                    Vh = c_V[0, sl] @ WV[t][:, cols] + mV[t][cols]
                else:
                    Kh = c_K[h, sl] @ WK[h, t] + mK[h, t]
                    Vh = c_V[h, sl] @ WV[h, t] + mV[h, t]
                Kh = np.concatenate([Kh, win_k[b, h, t, :wins[b]]])
                Vh = np.concatenate([Vh, win_v[b, h, t, :wins[b]]])
                if Kh.shape[0] == 0:
                    assert np.all(o[b, tq, h] == 0) and lse[b, tq, h] == -np.inf
                    continue
                o_ref, lse_ref = sdpa(q[b, tq, h], Kh, Vh, s)
                np.testing.assert_allclose(o[b, tq, h], o_ref, atol=1e-11)
                assert lse[b, tq, h] == pytest.approx(lse_ref, abs=1e-11)


# ---------------------------------------------------------------------------
# Faithful read with rotary embedding (RoPE after reconstruction: LLA paper, Pith
# verdict record, key_machinery and domain assumptions; RoFormer arXiv:2104.09864)
# ---------------------------------------------------------------------------
def _complex_pairs(x, style):
    d = x.shape[-1]
    if style == oracle.ROPE_HALF:
        return x[..., :d // 2] + 1j * x[..., d // 2:]
    return x[..., 0::2] + 1j * x[..., 1::2]


@pytest.mark.parametrize("style", [oracle.ROPE_HALF, oracle.ROPE_INTERLEAVED])
@pytest.mark.parametrize("q_pos,k_pos0", [(9, 0), (0, 0), (3000, 17)])
def test_rope_matches_roformer_complex_form(style, q_pos, k_pos0):
    """RoFormer writes the rotary map as complex multiplication, f(x, m) = x e^{i m theta_j}
    per component pair, so the score of query m and key n is
    Re sum_j z_q,j conj(z_k,j) e^{i (m - n) theta_j}, theta_j = base^(-2j/d).  With an
    identity codec (W_up = I, mu = 0) the latents are the keys themselves."""
    d, n, base, scale = 8, 11, 100.0, 0.7
    rng = np.random.default_rng(50 + style)
    K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    q = rng.standard_normal(d)
    I, z = np.eye(d), np.zeros(d)
    o, lse = oracle.attend_rope(K, V, I, z, I, z, q, scale, style, base, q_pos, k_pos0)
    theta = base ** (-2.0 * np.arange(d // 2) / d)
    pos = k_pos0 + np.arange(n)
    rot = np.exp(1j * (q_pos - pos)[:, None] * theta[None, :])
    scores = scale * np.real((_complex_pairs(q, style)[None, :] * np.conj(_complex_pairs(K, style)) * rot).sum(1))
    lse_ref = float(np.log(np.exp(scores - scores.max()).sum()) + scores.max())
    o_ref = np.exp(scores - lse_ref) @ V
    np.testing.assert_allclose(o, o_ref, atol=1e-11, rtol=0)
    assert lse == pytest.approx(lse_ref, abs=1e-11)


def test_rope_depends_on_relative_position_only():
    """Shifting the query and every key by the same offset leaves the result unchanged."""
    T, d, rk, rv, n = 3, 16, 4, 6, 23
    rng = np.random.default_rng(52)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 53)
    cK, cV = rng.standard_normal((n, rk)), rng.standard_normal((n, rv))
    q = rng.standard_normal(d)
    for style in (oracle.ROPE_HALF, oracle.ROPE_INTERLEAVED):
        a = oracle.attend_rope(cK, cV, WK[1], muK[1], WV[1], muV[1], q, 0.5, style, 10000.0, 40, 0)
        b = oracle.attend_rope(cK, cV, WK[1], muK[1], WV[1], muV[1], q, 0.5, style, 10000.0, 40 + 1234, 1234)
        np.testing.assert_allclose(a[0], b[0], atol=1e-10, rtol=0)
        assert a[1] == pytest.approx(b[1], abs=1e-10)
        # and the rotation matters: another query position gives another result
        c = oracle.attend_rope(cK, cV, WK[1], muK[1], WV[1], muV[1], q, 0.5, style, 10000.0, 41, 0)
        assert np.abs(c[0] - a[0]).max() > 1e-4


def test_rope_pairings_are_one_permutation_apart():
    """Interleaved pairs (2i, 2i+1) become half-split pairs (i, i + d/2) once the key and
    query components are reordered even-first; values are not rotated."""
    T, d, rk, rv, n = 2, 12, 5, 3, 14
    rng = np.random.default_rng(54)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 55)
    cK, cV = rng.standard_normal((n, rk)), rng.standard_normal((n, rv))
    q = rng.standard_normal(d)
    P = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
    a = oracle.attend_rope(cK, cV, WK[0], muK[0], WV[0], muV[0], q, 1.0, oracle.ROPE_INTERLEAVED, 500.0, 30)
    b = oracle.attend_rope(cK, cV, WK[0][:, P], muK[0][P], WV[0], muV[0], q[P], 1.0, oracle.ROPE_HALF, 500.0, 30)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12, rtol=0)
    assert a[1] == pytest.approx(b[1], abs=1e-12)


def test_rope_at_position_zero_is_the_plain_read():
    """One cached token at position 0 and the query at position 0: every angle is zero."""
    T, d, rk, rv = 2, 8, 3, 5
    rng = np.random.default_rng(56)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 57)
    cK, cV = rng.standard_normal((1, rk)), rng.standard_normal((1, rv))
    q = rng.standard_normal(d)
    for style in (oracle.ROPE_HALF, oracle.ROPE_INTERLEAVED):
        a = oracle.attend_rope(cK, cV, WK[0], muK[0], WV[0], muV[0], q, 0.9, style, 10000.0, 0, 0)
        ref = oracle.attend("reconstruct", cK, cV, WK[0], muK[0], WV[0], muV[0], q, 0.9)
        np.testing.assert_allclose(a[0], ref[0], atol=1e-13, rtol=0)
        assert a[1] == pytest.approx(ref[1], abs=1e-13)


def _rotate_complex(x, pos, base, style):
    """Rotary map in RoFormer's complex form, returned in the real layout of ``style``."""
    d = x.shape[-1]
    theta = base ** (-2.0 * np.arange(d // 2) / d)
    z = _complex_pairs(x, style) * np.exp(1j * np.asarray(pos, dtype=float)[..., None] * theta)
    out = np.empty_like(x)
    if style == oracle.ROPE_HALF:
        out[..., :d // 2], out[..., d // 2:] = z.real, z.imag
    else:
        out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


@pytest.mark.parametrize("style", [oracle.ROPE_HALF, oracle.ROPE_INTERLEAVED])
def test_decode_layer_rope_matches_dense_rotated_attention(style):
    """Ragged batch with per-sequence query positions: each unit against SDPA over the
    rebuilt keys rotated at positions 0..len-1 and the query rotated at q_pos[b]."""
    T, H, d, rk, rv = 3, 2, 8, 4, 6
    lens = np.array([5, 1, 0, 9], dtype=np.int32)
    q_pos = np.array([5, 700, 0, 12], dtype=np.int64)
    starts, c_K, c_V, WK, mK, WV, mV = _ragged_layer(T, H, d, lens, rk, rv, False, 26)
    B, Tq, t0, s, base = len(lens), 2, 1, 0.8, 1000.0
    q = np.random.default_rng(27).standard_normal((B, Tq, H, d))
    o, lse = oracle.decode_layer("reconstruct", q, c_K, c_V, starts, lens, WK, mK, WV, mV, t0, s,
                                 threads=2, rope=(q_pos, base, style))
    for b in range(B):
        sl = slice(int(starts[b]), int(starts[b] + lens[b]))
        for tq in range(Tq):
            for h in range(H):
                Kh = c_K[h, sl] @ WK[h, t0 + tq] + mK[h, t0 + tq]
                Vh = c_V[h, sl] @ WV[h, t0 + tq] + mV[h, t0 + tq]
                if lens[b] == 0:
                    assert np.all(o[b, tq, h] == 0) and lse[b, tq, h] == -np.inf
                    continue
                Kr = _rotate_complex(Kh, np.arange(lens[b]), base, style)
                qr = _rotate_complex(q[b, tq, h], q_pos[b], base, style)
                o_ref, lse_ref = sdpa(qr, Kr, Vh, s)
                np.testing.assert_allclose(o[b, tq, h], o_ref, atol=1e-11)
                assert lse[b, tq, h] == pytest.approx(lse_ref, abs=1e-11)


# ---------------------------------------------------------------------------
# Per-token reconstruction residual (LLA paper, Pith verdict record: the skeptic's
# concrete test, ||x - (x - mu) W_down W_up^T - mu|| / ||x||)
# ---------------------------------------------------------------------------
def test_residual_full_rank_codec_is_zero_and_norm_is_euclidean():
    T, d = 4, 8
    cod = S.orthonormal_codec(T * d, T, seed=60)
    x = np.random.default_rng(61).standard_normal((30, T * d)) * 2 + 0.5
    err, norm = oracle.codec_residual(x, cod.mu, cod.W_down, cod.W_up)
    np.testing.assert_allclose(err, 0.0, atol=1e-12)
    np.testing.assert_allclose(norm, np.linalg.norm(x, axis=1), rtol=1e-14)


@pytest.mark.parametrize("r", [1, 5, 16, 40])
def test_residual_energy_on_calibration_set_is_the_svd_tail(r):
    """Eckart-Young: the SVD codec's summed squared residual on its own calibration set
    equals the energy of the discarded singular values."""
    w = S.shrink(S.WORKLOADS["tiny-fp32"], d=16)
    model = S.trajectory_model(62, w.T * w.d)
    x_cal = S.draw_tokens_np(model, S.N_CALIB, 63)
    cod = S.fit_codec(x_cal, r, w.T)
    err, _ = oracle.codec_residual(x_cal, cod.mu, cod.W_down, cod.W_up)
    assert float((err ** 2).sum()) == pytest.approx(float((cod.sigma[r:] ** 2).sum()), rel=1e-9, abs=1e-9)


def test_residual_of_in_span_and_orthogonal_offsets():
    """Orthonormal rank-r codec with W_up = W_down^T: x = mu + (span vector) is rebuilt
    exactly; x = mu + v with v orthogonal to the span leaves exactly ||v||."""
    T, d, r = 3, 8, 5
    rng = np.random.default_rng(64)
    Q, _ = np.linalg.qr(rng.standard_normal((T * d, T * d)))
    Wd = Q[:, :r]
    Wu = Wd.reshape(T, d, r).transpose(0, 2, 1)
    mu = rng.standard_normal(T * d)
    a = rng.standard_normal((6, r))
    b = rng.standard_normal((6, T * d - r))
    x_in = mu + a @ Wd.T
    v = b @ Q[:, r:].T
    err_in, _ = oracle.codec_residual(x_in, mu, Wd, Wu)
    err_out, norm_out = oracle.codec_residual(mu + v, mu, Wd, Wu)
    np.testing.assert_allclose(err_in, 0.0, atol=1e-12)
    np.testing.assert_allclose(err_out, np.linalg.norm(b, axis=1), rtol=1e-12)
    np.testing.assert_allclose(norm_out, np.linalg.norm(mu + v, axis=1), rtol=1e-13)


def test_residual_with_differently_scaled_down_and_up_projections():
    """W_down = alpha Q_r and W_up,t = beta (t-block of Q_r)^T with Q_r orthonormal: for
    x = mu + a Q_r^T + v (v orthogonal to the span) the definition gives
    ||x - x_hat||^2 = (1 - alpha beta)^2 ||a||^2 + ||v||^2, which tells the two projections'
    roles apart (SVD codecs, where W_up = W_down^T, cannot)."""
    T, d, r, alpha, beta = 3, 8, 5, 2.0, 0.25
    rng = np.random.default_rng(66)
    Q, _ = np.linalg.qr(rng.standard_normal((T * d, T * d)))
    Qr = Q[:, :r]
    Wd = alpha * Qr
    Wu = beta * Qr.reshape(T, d, r).transpose(0, 2, 1)
    mu = rng.standard_normal(T * d)
    a = rng.standard_normal((9, r))
    b = rng.standard_normal((9, T * d - r))
    x = mu + a @ Qr.T + b @ Q[:, r:].T
    err, _ = oracle.codec_residual(x, mu, Wd, Wu)
    ref = np.sqrt((1 - alpha * beta) ** 2 * (a ** 2).sum(axis=1) + (b ** 2).sum(axis=1))
    np.testing.assert_allclose(err, ref, rtol=1e-12)


def test_residual_is_homogeneous_in_the_centred_vector():
    """x - x_hat is linear in y = x - mu for any codec (W_up need not be W_down^T), so
    scaling y by s scales the residual by |s|."""
    T, d, r = 4, 8, 3
    rng = np.random.default_rng(65)
    Wd = rng.standard_normal((T * d, r))
    Wu = rng.standard_normal((T, r, d))
    mu = rng.standard_normal(T * d)
    y = rng.standard_normal((7, T * d))
    e1, _ = oracle.codec_residual(mu + y, mu, Wd, Wu)
    e3, _ = oracle.codec_residual(mu - 3.0 * y, mu, Wd, Wu)
    np.testing.assert_allclose(e3, 3.0 * e1, rtol=1e-12)
    assert np.all(e1 > 0.1)


# ---------------------------------------------------------------------------
# Decoupled rotary sub-key beside the latent (LLA paper, Pith verdict record, desk-editor
# letter: the absorbed variant needs decoupled RoPE)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("style", [oracle.ROPE_HALF, oracle.ROPE_INTERLEAVED])
def test_decoupled_identity_codec_is_attention_over_concatenated_keys(style):
    """Identity codec (W_up = I, mu = 0): the result is textbook attention of the query
    [q ; rope(q_rope, q_pos)] (rotated in RoFormer's complex form) over the keys
    [k ; k_rope] (SDPA)."""
    d, d_r, n, base, q_pos = 8, 4, 13, 200.0, 37
    rng = np.random.default_rng(70 + style)
    K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    K_r = rng.standard_normal((n, d_r))
    q, q_r = rng.standard_normal(d), rng.standard_normal(d_r)
    I, z = np.eye(d), np.zeros(d)
    o, lse = oracle.attend_decoupled(K, V, I, z, I, z, K_r, q, q_r, 0.8, style, base, q_pos)
    q_full = np.concatenate([q, _rotate_complex(q_r, q_pos, base, style)])
    o_ref, lse_ref = sdpa(q_full, np.concatenate([K, K_r], axis=1), V, 0.8)
    np.testing.assert_allclose(o, o_ref, atol=1e-11, rtol=0)
    assert lse == pytest.approx(lse_ref, abs=1e-11)


def test_decoupled_rope_part_depends_on_relative_position():
    """Sub-keys stored rotated at their positions p_i: shifting every p_i and q_pos by the
    same offset leaves the result unchanged; the latent part is unaffected."""
    T, d, rk, rv, n, d_r = 2, 8, 3, 5, 9, 6
    rng = np.random.default_rng(72)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 73)
    cK, cV = rng.standard_normal((n, rk)), rng.standard_normal((n, rv))
    raw = rng.standard_normal((n, d_r))
    q, q_r = rng.standard_normal(d), rng.standard_normal(d_r)
    out = []
    for off in (0, 4321):
        stored = _rotate_complex(raw, off + np.arange(n), 10000.0, oracle.ROPE_HALF)
        out.append(oracle.attend_decoupled(cK, cV, WK[1], muK[1], WV[1], muV[1], stored, q, q_r, 0.5,
                                           oracle.ROPE_HALF, 10000.0, off + 20))
    np.testing.assert_allclose(out[0][0], out[1][0], atol=1e-10, rtol=0)
    assert out[0][1] == pytest.approx(out[1][1], abs=1e-10)


def test_decoupled_without_rope_part_is_the_plain_read():
    """d_r = 0: nothing beside the latent, the result is the plain (unrotated) read."""
    T, d, rk, rv, n = 2, 8, 3, 5, 11
    rng = np.random.default_rng(74)
    (WK, muK), (WV, muV) = _codec_pair(T, d, rk, rv, 75)
    cK, cV = rng.standard_normal((n, rk)), rng.standard_normal((n, rv))
    q = rng.standard_normal(d)
    a = oracle.attend_decoupled(cK, cV, WK[0], muK[0], WV[0], muV[0], np.zeros((n, 0)), q, np.zeros(0), 0.7,
                                oracle.ROPE_HALF, 10000.0, 5)
    ref = oracle.attend("absorb", cK, cV, WK[0], muK[0], WV[0], muV[0], q, 0.7)
    np.testing.assert_allclose(a[0], ref[0], atol=1e-12, rtol=0)
    assert a[1] == pytest.approx(ref[1], abs=1e-12)


def test_decode_layer_decoupled_matches_dense_attention():
    """Ragged batch: each unit against SDPA over [rebuilt keys | stored sub-keys] with the
    query [q ; rope(q_rope, q_pos[b])] (complex form)."""
    T, H, d, rk, rv, d_r = 3, 2, 8, 4, 6, 4
    lens = np.array([5, 1, 0, 9], dtype=np.int32)
    q_pos = np.array([5, 900, 0, 9])
    starts, c_K, c_V, WK, mK, WV, mV = _ragged_layer(T, H, d, lens, rk, rv, False, 28)
    rng = np.random.default_rng(29)
    B, Tq, t0, s, base = len(lens), 2, 1, 0.8, 1000.0
    k_rope = rng.standard_normal((H, c_K.shape[1], d_r))
    q = rng.standard_normal((B, Tq, H, d))
    q_r = rng.standard_normal((B, Tq, H, d_r))
    o, lse = oracle.decode_layer("absorb", q, c_K, c_V, starts, lens, WK, mK, WV, mV, t0, s, threads=2,
                                 decoupled=(k_rope, q_r, q_pos, base, oracle.ROPE_INTERLEAVED))
    for b in range(B):
        sl = slice(int(starts[b]), int(starts[b] + lens[b]))
        for tq in range(Tq):
            for h in range(H):
                if lens[b] == 0:
                    assert np.all(o[b, tq, h] == 0) and lse[b, tq, h] == -np.inf
                    continue
                Kh = c_K[h, sl] @ WK[h, t0 + tq] + mK[h, t0 + tq]
                Vh = c_V[h, sl] @ WV[h, t0 + tq] + mV[h, t0 + tq]
                qf = np.concatenate([q[b, tq, h], _rotate_complex(q_r[b, tq, h], q_pos[b], base,
                                                                  oracle.ROPE_INTERLEAVED)])
                o_ref, lse_ref = sdpa(qf, np.concatenate([Kh, k_rope[h, sl]], axis=1), Vh, s)
                np.testing.assert_allclose(o[b, tq, h], o_ref, atol=1e-11)
                assert lse[b, tq, h] == pytest.approx(lse_ref, abs=1e-11)


# ---------------------------------------------------------------------------
# Codec fit (SVD initialisation; LLA review page, What carries the argument)
# ---------------------------------------------------------------------------
def test_codec_fit_recovers_planted_orthogonal_directions():
    """x = mu0 + Z A with orthogonal columns of Z and orthonormal rows of A, distinct
    weights: the right singular vectors are A's rows (up to the sign convention), the
    singular values the weights, and the mean mu0 (Z's columns sum to zero)."""
    T, d, r, n = 4, 8, 3, 40
    W = T * d
    rng = np.random.default_rng(80)
    Qa, _ = np.linalg.qr(rng.standard_normal((W, W)))
    A = Qa[:, :r].T                                   # [r, W], orthonormal rows
    Z0 = rng.standard_normal((n, r))
    Z0 -= Z0.mean(axis=0)
    Qz, _ = np.linalg.qr(Z0)                         # orthonormal, zero-mean columns
    weights = np.array([9.0, 4.0, 2.5])
    mu0 = rng.standard_normal(W)
    x = mu0 + (Qz * weights) @ A
    mu, Wd, Wu, sigma = oracle.codec_fit(x, r, T)
    np.testing.assert_allclose(mu, mu0, atol=1e-12)
    np.testing.assert_allclose(sigma[:r], weights, rtol=1e-12)
    assert np.all(sigma[r:] < 1e-10)
    for j in range(r):
        v = A[j] * np.sign(A[j][np.argmax(np.abs(A[j]))])
        np.testing.assert_allclose(Wd[:, j], v, atol=1e-10)
    np.testing.assert_allclose(Wu[2], Wd[2 * d:3 * d].T, atol=0)


def test_codec_fit_energy_and_orthonormality():
    """Orthonormal W_down; the fitted codec's residual energy on its calibration set is
    the tail of the singular values (Eckart-Young), through the pinned residual oracle."""
    w = S.shrink(S.WORKLOADS["tiny-fp32"], d=16)
    model = S.trajectory_model(81, w.T * w.d)
    x = S.draw_tokens_np(model, 100, 82)
    for r in (1, 7, 30):
        mu, Wd, Wu, sigma = oracle.codec_fit(x, r, w.T)
        np.testing.assert_allclose(Wd.T @ Wd, np.eye(r), atol=1e-12)
        err, _ = oracle.codec_residual(x, mu, Wd, Wu)
        assert float((err ** 2).sum()) == pytest.approx(float((sigma[r:] ** 2).sum()), rel=1e-9)
        assert np.all(np.diff(sigma) <= 0)


def test_codec_fit_shift_moves_only_the_mean():
    w = S.shrink(S.WORKLOADS["tiny-fp32"], d=16)
    x = S.draw_tokens_np(S.trajectory_model(83, w.T * w.d), 60, 84)
    shift = np.random.default_rng(85).standard_normal(w.T * w.d) * 5
    a = oracle.codec_fit(x, 6, w.T)
    b = oracle.codec_fit(x + shift, 6, w.T)
    np.testing.assert_allclose(b[0], a[0] + shift, atol=1e-12)
    np.testing.assert_allclose(b[1], a[1], atol=1e-9)
    np.testing.assert_allclose(b[3], a[3], rtol=1e-10, atol=1e-10 * a[3][0])  # last one is ~0 (rank n-1)


def test_decode_layer_rope_with_folded_heads():
    """LLA-2D codec with the faithful read: head h rebuilds its column slice of the folded
    up-projection, then rotates it; against dense SDPA over keys rotated in complex form."""
    T, H, d, rk, rv = 2, 3, 8, 5, 7
    lens = np.array([6, 0, 3], dtype=np.int32)
    q_pos = np.array([6, 2, 40])
    starts, c_K, c_V, WK, mK, WV, mV = _ragged_layer(T, H, d, lens, rk, rv, True, 30)
    B, Tq, t0, s, base = len(lens), 2, 0, 0.9, 300.0
    q = np.random.default_rng(31).standard_normal((B, Tq, H, d))
    o, lse = oracle.decode_layer("reconstruct", q, c_K, c_V, starts, lens, WK, mK, WV, mV, t0, s,
                                 fold2d=True, threads=2, rope=(q_pos, base, oracle.ROPE_INTERLEAVED))
    for b in range(B):
        sl = slice(int(starts[b]), int(starts[b] + lens[b]))
        for tq in range(Tq):
            for h in range(H):
                if lens[b] == 0:
                    assert np.all(o[b, tq, h] == 0) and lse[b, tq, h] == -np.inf
                    continue
                cols = slice(h * d, (h + 1) * d)
                Kh = c_K[0, sl] @ WK[t0 + tq][:, cols] + mK[t0 + tq][cols]
                Vh = c_V[0, sl] @ WV[t0 + tq][:, cols] + mV[t0 + tq][cols]
                Kr = _rotate_complex(Kh, np.arange(lens[b]), base, oracle.ROPE_INTERLEAVED)
                qr = _rotate_complex(q[b, tq, h], q_pos[b], base, oracle.ROPE_INTERLEAVED)
                o_ref, lse_ref = sdpa(qr, Kr, Vh, s)
                np.testing.assert_allclose(o[b, tq, h], o_ref, atol=1e-11)
                assert lse[b, tq, h] == pytest.approx(lse_ref, abs=1e-11)


@pytest.mark.parametrize("variant", VARIANTS)
def test_tiny_workload_against_brute_force_without_max_subtraction(variant):
    """The 64-token fp32 workload exactly as generated (fitted low-rank codec, all four
    loops): the oracle against a third expression written with Python loops and exact
    sums, exp of the raw logits with no max subtraction, normalised at the end."""
    w = S.WORKLOADS["tiny-fp32"]
    p = S.decode_inputs(w, 0, "cpu")
    to64 = lambda t: t.double().numpy()
    cK, cV = to64(p["k"][0]), to64(p["v"][0])
    WK, WV, mK, mV = (to64(p[k][0]) for k in ("W_up_k", "W_up_v", "mu_k", "mu_v"))
    q = to64(p["q"])
    n = int(p["lens"][0])
    s0 = int(p["starts"][0])
    o, lse = oracle.decode_layer(variant, q, cK, cV, p["starts"], p["lens"], WK, mK, WV, mV,
                                 0, 1.0, threads=1)
    for t in range(w.T):
        for h in range(w.H):
            Kh = [[math.fsum([cK[h, s0 + i, j] * WK[h, t, j, k] for j in range(w.r_k)]) + mK[h, t, k]
                   for k in range(w.d)] for i in range(n)]
            Vh = [[math.fsum([cV[h, s0 + i, j] * WV[h, t, j, k] for j in range(w.r_v)]) + mV[h, t, k]
                   for k in range(w.d)] for i in range(n)]
            e = [math.exp(math.fsum([q[0, t, h, k] * Kh[i][k] for k in range(w.d)])) for i in range(n)]
            Z = math.fsum(e)
            o_ref = [math.fsum([e[i] * Vh[i][k] for i in range(n)]) / Z for k in range(w.d)]
            np.testing.assert_allclose(o[0, t, h], o_ref, atol=1e-12, rtol=0)
            assert lse[0, t, h] == pytest.approx(math.log(Z), abs=1e-12)

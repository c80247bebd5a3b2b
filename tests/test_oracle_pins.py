"""Pins for the fp64 oracle, each tied to something other than the oracle.

Every check below is one of: a closed form the pages or the mathematics fix,
a special case that reduces to a known result, an invariant of the method,
or a value printed on the pages ("Looped Latent Attention", arXiv
2607.15456). Shapes are deliberately non-square and inputs non-symmetric so
that a transposed operand, a dropped mean term or a wrong stacking index
breaks at least one check.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_numbers.json")


def rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# textbook attention
# --------------------------------------------------------------------------

def test_attend_single_token_returns_its_value():
    r = rng(1)
    q, K, V = r.normal(size=5), r.normal(size=(1, 5)), r.normal(size=(1, 3))
    out, lse = oracle.attend(q, K, V, 0.7)
    np.testing.assert_allclose(out, V[0], rtol=0, atol=1e-15)
    assert lse == pytest.approx(0.7 * float(q @ K[0]), abs=1e-14)


def test_attend_two_tokens_is_a_sigmoid_mix():
    # softmax over two scores is (sigmoid(d), 1 - sigmoid(d)) with d = s0 - s1
    r = rng(2)
    q, K, V = r.normal(size=4), r.normal(size=(2, 4)), r.normal(size=(2, 6))
    scale = 0.5
    s0, s1 = scale * q @ K[0], scale * q @ K[1]
    w = 1.0 / (1.0 + math.exp(-(s0 - s1)))
    out, lse = oracle.attend(q, K, V, scale)
    np.testing.assert_allclose(out, w * V[0] + (1 - w) * V[1], atol=1e-14)
    assert lse == pytest.approx(max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))), abs=1e-13)


def test_attend_equal_keys_average_values():
    r = rng(3)
    q, V = r.normal(size=8), r.normal(size=(9, 5))
    K = np.tile(r.normal(size=8), (9, 1))
    out, lse = oracle.attend(q, K, V, 0.3)
    np.testing.assert_allclose(out, V.mean(axis=0), atol=1e-14)
    assert lse == pytest.approx(0.3 * q @ K[0] + math.log(9), abs=1e-13)


def test_attend_merge_identity_over_a_split_context():
    # Attention over a concatenation equals the lse-weighted mix of the two
    # halves: a property of softmax, not a restatement of the code.
    r = rng(4)
    q, K, V = r.normal(size=6), r.normal(size=(17, 6)), r.normal(size=(17, 3))
    o, l = oracle.attend(q, K, V, 0.9)
    o1, l1 = oracle.attend(q, K[:7], V[:7], 0.9)
    o2, l2 = oracle.attend(q, K[7:], V[7:], 0.9)
    m = max(l1, l2)
    w1, w2 = math.exp(l1 - m), math.exp(l2 - m)
    np.testing.assert_allclose(o, (w1 * o1 + w2 * o2) / (w1 + w2), atol=1e-13)
    assert l == pytest.approx(m + math.log(w1 + w2), abs=1e-12)


def test_attend_permutation_and_duplication():
    r = rng(5)
    q, K, V = r.normal(size=4), r.normal(size=(6, 4)), r.normal(size=(6, 2))
    o, l = oracle.attend(q, K, V, 1.1)
    perm = r.permutation(6)
    o_p, l_p = oracle.attend(q, K[perm], V[perm], 1.1)
    np.testing.assert_allclose(o, o_p, atol=1e-14)
    assert l == pytest.approx(l_p, abs=1e-13)
    # duplicating every token doubles each weight's mass: same output, lse + ln 2
    o_d, l_d = oracle.attend(q, np.vstack([K, K]), np.vstack([V, V]), 1.1)
    np.testing.assert_allclose(o, o_d, atol=1e-14)
    assert l_d == pytest.approx(l + math.log(2), abs=1e-13)


def test_attend_hard_limit_picks_the_argmax():
    r = rng(6)
    q, K, V = r.normal(size=5), r.normal(size=(8, 5)), r.normal(size=(8, 3))
    out, _ = oracle.attend(q, K, V, 1e4)
    np.testing.assert_allclose(out, V[np.argmax(K @ q)], atol=1e-9)


def test_attend_rejects_empty_context():
    with pytest.raises(ValueError):
        oracle.attend(np.zeros(2), np.zeros((0, 2)), np.zeros((0, 2)), 1.0)


# --------------------------------------------------------------------------
# per-head decode: explicit reconstruction (Eq. 3) then attention
# --------------------------------------------------------------------------

def _unit(seed, d=16, N=11, r_k=8, r_v=24, mu=True):
    r = rng(seed)
    return dict(q=r.normal(size=d), zk=r.normal(size=(N, r_k)), zv=r.normal(size=(N, r_v)),
                dk=r.normal(size=(d, r_k)), dv=r.normal(size=(d, r_v)),
                mu_k=r.normal(size=d) if mu else None, mu_v=r.normal(size=d) if mu else None)


def test_decode_single_token_is_its_reconstruction():
    u = _unit(10, N=1)
    out, lse = oracle.decode_unit(**u, scale=0.25)
    # Eq. 3 with a library matmul: vhat = W^V_up zv + mu_v
    np.testing.assert_allclose(out, u["dv"] @ u["zv"][0] + u["mu_v"], atol=1e-13)
    khat = u["dk"] @ u["zk"][0] + u["mu_k"]
    assert lse == pytest.approx(0.25 * u["q"] @ khat, abs=1e-13)


def test_decode_zero_query_averages_reconstructions():
    u = _unit(11)
    u["q"] = np.zeros_like(u["q"])
    out, lse = oracle.decode_unit(**u, scale=0.25)
    np.testing.assert_allclose(out, u["dv"] @ u["zv"].mean(axis=0) + u["mu_v"], atol=1e-13)
    assert lse == pytest.approx(math.log(u["zk"].shape[0]), abs=1e-13)


def test_decode_identity_codec_is_plain_attention():
    # T = 1, r = d_h, W_up = I, mu = 0: the latent is the key/value itself.
    r = rng(12)
    d, N = 8, 13
    q, Kr, Vr = r.normal(size=d), r.normal(size=(N, d)), r.normal(size=(N, d))
    out, lse = oracle.decode_unit(q, Kr, Vr, np.eye(d), np.eye(d), scale=0.4)
    o_ref, l_ref = oracle.attend(q, Kr, Vr, 0.4)
    np.testing.assert_allclose(out, o_ref, atol=1e-14)
    assert lse == pytest.approx(l_ref, abs=1e-13)


def test_decode_key_mean_shifts_only_lse_value_mean_shifts_output():
    u = _unit(13)
    base = dict(u, mu_k=None, mu_v=None)
    o0, l0 = oracle.decode_unit(**base, scale=0.3)
    o1, l1 = oracle.decode_unit(**dict(base, mu_k=u["mu_k"]), scale=0.3)
    np.testing.assert_allclose(o1, o0, atol=1e-13)           # softmax shift invariance
    assert l1 == pytest.approx(l0 + 0.3 * u["q"] @ u["mu_k"], abs=1e-12)
    o2, l2 = oracle.decode_unit(**dict(base, mu_v=u["mu_v"]), scale=0.3)
    np.testing.assert_allclose(o2, o0 + u["mu_v"], atol=1e-13)  # sum_j p_j = 1
    assert l2 == pytest.approx(l0, abs=1e-13)


def test_decode_absorbed_equals_explicit_by_brute_force():
    # §7: q^T (W_up c) = (W_up^T q)^T c and sum_i a_i W_up c_i = W_up sum_i a_i c_i.
    for seed in range(20):
        r = rng(100 + seed)
        d = int(r.choice([4, 16, 32]))
        N = int(r.integers(1, 65))
        r_k, r_v = int(r.choice([8, 16, 24])), int(r.choice([8, 16, 40]))
        u = _unit(200 + seed, d=d, N=N, r_k=r_k, r_v=r_v, mu=bool(seed % 2))
        o_e, l_e = oracle.decode_unit(**u, scale=1 / math.sqrt(d))
        o_a, l_a = oracle.decode_unit_absorbed(**u, scale=1 / math.sqrt(d))
        np.testing.assert_allclose(o_a, o_e, atol=1e-12)
        assert l_a == pytest.approx(l_e, abs=1e-12)


def test_decode_low_rank_codec_is_attention_over_projected_cache():
    # With an orthonormal W_down and its loop slices as decoders, the decoded
    # loop-t key is the loop-t block of the projection P (x - mu) + mu,
    # P = W W^T. Compare against attention over projected raw K/V built
    # with numpy linear algebra, not with the oracle's reconstruction.
    r = rng(14)
    T, d, N, rank = 3, 8, 10, 7
    Wk = np.linalg.qr(r.normal(size=(T * d, rank)))[0]
    Wv = np.linalg.qr(r.normal(size=(T * d, rank)))[0]
    xk, xv = r.normal(size=(N, T * d)), r.normal(size=(N, T * d))
    mk, mv = r.normal(size=T * d), r.normal(size=T * d)
    zk, zv = (xk - mk) @ Wk, (xv - mv) @ Wv
    Pk, Pv = Wk @ Wk.T, Wv @ Wv.T
    Kp, Vp = (xk - mk) @ Pk + mk, (xv - mv) @ Pv + mv
    q = r.normal(size=d)
    for t in range(T):
        sl = slice(t * d, (t + 1) * d)
        out, lse = oracle.decode_unit(q, zk, zv, Wk[sl], Wv[sl], mk[sl], mv[sl], scale=0.35)
        o_ref, l_ref = oracle.attend(q, Kp[:, sl], Vp[:, sl], 0.35)
        np.testing.assert_allclose(out, o_ref, atol=1e-12)
        assert lse == pytest.approx(l_ref, abs=1e-12)


def test_full_rank_svd_codec_reproduces_uncompressed_per_loop_attention():
    # Full rank r = T d_h: the SVD codec is an orthogonal change of basis, so
    # LLA decode of loop t equals textbook attention on the raw loop-t K/V.
    r = rng(15)
    T, d, N, n_cal = 4, 8, 12, 200
    cal_k = r.normal(size=(n_cal, T * d)) + r.normal(size=T * d)
    cal_v = r.normal(size=(n_cal, T * d)) * 2.0 - 1.0
    wk, upk, mk = oracle.svd_init(cal_k, T * d, T)
    wv, upv, mv = oracle.svd_init(cal_v, T * d, T)
    xk = r.normal(size=(T, N, 1, d))      # loop-major, one group
    xv = r.normal(size=(T, N, 1, d))
    zk = oracle.encode(xk, wk[None], mk[None])[0]
    zv = oracle.encode(xv, wv[None], mv[None])[0]
    q = r.normal(size=d)
    for t in range(T):
        sl = slice(t * d, (t + 1) * d)
        out, lse = oracle.decode_unit(q, zk, zv, upk[t], upv[t], mk[sl], mv[sl],
                                      scale=d ** -0.5)
        o_ref, l_ref = oracle.attend(q, xk[t, :, 0], xv[t, :, 0], d ** -0.5)
        np.testing.assert_allclose(out, o_ref, atol=1e-11)
        assert lse == pytest.approx(l_ref, abs=1e-11)


def test_batched_decode_matches_units_and_2d_shares_the_latent():
    r = rng(16)
    B, H, d, N, ncap, rk, rv = 2, 3, 8, 9, 12, 8, 16
    q = r.normal(size=(B, H, d))
    zk, zv = r.normal(size=(B, H, ncap, rk)), r.normal(size=(B, H, ncap, rv))
    dk, dv = r.normal(size=(H, d, rk)), r.normal(size=(H, d, rv))
    mk, mv = r.normal(size=(H, d)), r.normal(size=(H, d))
    out, lse = oracle.lla_decode(q, zk, zv, dk, dv, mk, mv, 0.3, N=N)
    for b in range(B):
        for h in range(H):
            o1, l1 = oracle.decode_unit(q[b, h], zk[b, h, :N], zv[b, h, :N], dk[h], dv[h],
                                        mk[h], mv[h], 0.3)
            np.testing.assert_allclose(out[b, h], o1, atol=0)
            assert lse[b, h] == l1
    # LLA-2D: every head reads the same per-token latent
    zk2, zv2 = r.normal(size=(B, ncap, rk)), r.normal(size=(B, ncap, rv))
    out2, _ = oracle.lla2d_decode(q, zk2, zv2, dk, dv, mk, mv, 0.3, N=N)
    zk_b = np.broadcast_to(zk2[:, None], (B, H, ncap, rk))
    zv_b = np.broadcast_to(zv2[:, None], (B, H, ncap, rv))
    out3, _ = oracle.lla_decode(q, zk_b, zv_b, dk, dv, mk, mv, 0.3, N=N)
    np.testing.assert_allclose(out2, out3, atol=0)
    sub, _ = oracle.lla2d_decode(q, zk2, zv2, dk, dv, mk, mv, 0.3, N=N, units=[(1, 2), (0, 1)])
    np.testing.assert_allclose(sub, np.stack([out2[1, 2], out2[0, 1]]), atol=0)


# --------------------------------------------------------------------------
# encode (Eq. 2) and stacking order (Eq. 1)
# --------------------------------------------------------------------------

def test_encode_stacking_order_is_loop_major():
    # A single unit entry at loop t, channel i selects row t*d + i of W_down.
    r = rng(20)
    T, N, G, d, rk = 3, 2, 2, 4, 5
    w = r.normal(size=(G, T * d, rk))
    for (t, n, g, i) in [(0, 0, 0, 0), (2, 1, 1, 3), (1, 0, 1, 2)]:
        x = np.zeros((T, N, G, d))
        x[t, n, g, i] = 1.0
        z = oracle.encode(x, w)
        expect = np.zeros((G, N, rk))
        expect[g, n] = w[g, t * d + i]
        np.testing.assert_allclose(z, expect, atol=0)


def test_encode_subtracts_the_mean_and_is_linear():
    r = rng(21)
    T, N, G, d, rk = 2, 5, 3, 4, 6
    w = r.normal(size=(G, T * d, rk))
    mu = r.normal(size=(G, T * d))
    x = r.normal(size=(T, N, G, d))
    # a token equal to its group's mean encodes to zero
    x_mu = np.transpose(mu.reshape(G, T, d), (1, 0, 2))[:, None]
    np.testing.assert_allclose(oracle.encode(x_mu, w, mu), 0.0, atol=1e-13)
    # (x - mu) W == x W - mu W
    z = oracle.encode(x, w, mu)
    z0 = oracle.encode(x, w)
    np.testing.assert_allclose(z, z0 - np.einsum("gk,gkr->gr", mu, w)[:, None], atol=1e-12)
    # linearity in x (without mean)
    x2 = r.normal(size=x.shape)
    np.testing.assert_allclose(oracle.encode(2 * x - x2, w), 2 * z0 - oracle.encode(x2, w), atol=1e-12)


def test_encode_decode_round_trip_is_a_projection():
    r = rng(22)
    T, N, d, rk = 4, 7, 6, 5
    cal = r.normal(size=(300, T * d)) @ r.normal(size=(T * d, T * d)) + 3.0
    w, up, mu = oracle.svd_init(cal, rk, T)
    x = r.normal(size=(T, N, 1, d))
    z = oracle.encode(x, w[None], mu[None])[0]
    xhat = oracle.reconstruct(z, up, mu)             # [N, T, d]
    # re-encoding the reconstruction gives the same latent (idempotent)
    z2 = oracle.encode(np.transpose(xhat, (1, 0, 2))[:, :, None], w[None], mu[None])[0]
    np.testing.assert_allclose(z2, z, atol=1e-11)
    # full rank: exact reconstruction
    wf, upf, muf = oracle.svd_init(cal, T * d, T)
    zf = oracle.encode(x, wf[None], muf[None])[0]
    np.testing.assert_allclose(oracle.reconstruct(zf, upf, muf),
                               np.transpose(x[:, :, 0], (1, 0, 2)), atol=1e-11)


# --------------------------------------------------------------------------
# SVD initialisation (§3 "Initialization and conversion")
# --------------------------------------------------------------------------

def test_svd_init_mean_orthonormality_and_eckart_young():
    r = rng(30)
    T, d, n, rk = 3, 5, 400, 4
    X = r.normal(size=(n, T * d)) @ np.diag(np.linspace(3, 0.2, T * d)) + np.arange(T * d)
    w, up, mu = oracle.svd_init(X, rk, T)
    np.testing.assert_allclose(mu, X.mean(axis=0), atol=1e-12)
    np.testing.assert_allclose(w.T @ w, np.eye(rk), atol=1e-12)
    np.testing.assert_allclose(up, w.reshape(T, d, rk), atol=0)
    Xc = X - mu
    resid = np.sum((Xc - Xc @ w @ w.T) ** 2)
    # Eckart-Young via the eigenvalues of the Gram matrix (a different routine)
    ev = np.sort(np.linalg.eigvalsh(Xc.T @ Xc))[::-1]
    assert resid == pytest.approx(ev[rk:].sum(), rel=1e-9)
    # no random rank-rk subspace does better
    for s in range(5):
        Qr = np.linalg.qr(rng(31 + s).normal(size=(T * d, rk)))[0]
        assert np.sum((Xc - Xc @ Qr @ Qr.T) ** 2) >= resid - 1e-9


def test_svd_init_recovers_planted_low_rank_data_exactly():
    r = rng(32)
    T, d, n, rk = 4, 4, 100, 3
    X = r.normal(size=(n, rk)) @ r.normal(size=(rk, T * d)) + r.normal(size=T * d)
    w, up, mu = oracle.svd_init(X, rk, T)
    x = np.transpose(X[:7].reshape(7, T, d), (1, 0, 2))[:, :, None]
    z = oracle.encode(x, w[None], mu[None])[0]
    np.testing.assert_allclose(oracle.reconstruct(z, up, mu).reshape(7, T * d), X[:7], atol=1e-10)


# --------------------------------------------------------------------------
# compression ratio and sizes printed on the pages (Eq. 4, §3, §7)
# --------------------------------------------------------------------------

def test_compression_ratio_matches_printed_points():
    g = json.load(open(GOLDEN))
    geo = g["ouro_geometry"]
    T, H, dh = geo["T"], geo["H"], geo["d_head"]
    assert 2 * T * H * dh == g["teacher_scalars_per_token_layer"]["value_at_ouro"]
    s = g["rank_split_4x"]
    assert oracle.compression_ratio(T, dh, s["r_k"], s["r_v"], H=H) == s["rho"]
    assert oracle.compression_ratio(T, dh, s["shared_r_k"], s["shared_r_v"]) == s["rho"]
    x21 = g["rho_21x"]
    assert round(oracle.compression_ratio(T, dh, x21["r_sum"] // 2, x21["r_sum"] // 2), 1) == x21["rho_printed"]
    # the build's workloads: 8x (tiny), 4x, 21.33x, 32x per head, 32x for LLA-2D
    assert oracle.compression_ratio(4, 16, 8, 8) == 8.0
    assert oracle.compression_ratio(4, 128, 128, 128) == 4.0
    assert oracle.compression_ratio(4, 128, 24, 24) == pytest.approx(512 / 24)
    assert oracle.compression_ratio(4, 128, 16, 16) == 32.0
    assert oracle.compression_ratio(4, 128, 256, 256, H=16, two_d=True) == 32.0
    # LLA-2D is a factor H below per-head LLA at the same (r_k, r_v)
    assert (oracle.compression_ratio(4, 128, 24, 24, H=16, two_d=True)
            == 16 * oracle.compression_ratio(4, 128, 24, 24, H=16))


def test_one_million_context_cache_size():
    g = json.load(open(GOLDEN))
    c = g["one_million_context_cache"]
    geo = g["ouro_geometry"]
    nbytes = c["tokens_kept"] * geo["D"] * geo["H"] * c["r_sum"] * c["bytes_per_scalar"]
    assert nbytes == c["printed_mib"] * 2 ** 20


def test_capacity_ratios_follow_the_scalar_reduction():
    # Measured batch capacity is not a closed form, but the printed points
    # must not exceed what the exact scalar reduction allows in the same
    # memory: batch ratio <= rho.
    g = json.load(open(GOLDEN))
    c = g["capacity_at_4k"]
    assert c["batch_4x"] / c["teacher_batch"] <= 4.0
    assert c["batch_21x"] / c["teacher_batch"] <= 512 / 24 * 1.13  # within one measured step
    # bytes of the build's 21.3x workload store (24 layers, batch 768, 4k)
    store = 24 * 768 * 4096 * 16 * 48 * 2
    assert store / 1e9 == pytest.approx(115.96, abs=0.01)


# ---------------------------------------------------------------------------
# paged / ragged store and sink + window eviction
# ---------------------------------------------------------------------------

def test_kept_positions_match_the_printed_eviction_budget():
    g = json.load(open(GOLDEN))["eviction_budget_gsm8k"]
    N = g["prompt_tokens_approx"]
    pos = oracle.kept_positions(N, g["sink"], g["window"])
    assert pos.size == g["budget"] == g["sink"] + g["window"]
    assert list(pos[:g["sink"]]) == list(range(g["sink"]))
    assert list(pos[g["sink"]:]) == list(range(N - g["window"], N))
    assert abs(1 - pos.size / N - g["evicted_fraction_approx"]) < 0.01
    # the budget caps the set; shorter sequences keep everything
    assert list(oracle.kept_positions(200, 4, 256)) == list(range(200))
    assert list(oracle.kept_positions(260, 4, 256)) == list(range(260))
    assert list(oracle.kept_positions(50, 0, 0)) == list(range(50))
    assert oracle.kept_positions(0, 4, 256).size == 0


def _paged_store(r, B, H, d, ps, lens, r_k=16, r_v=24, mu=True, spare=3):
    """Dense per-sequence stores scattered into a shuffled page pool."""
    maxb = max(1, max((n + ps - 1) // ps for n in lens))
    npages = B * maxb + spare
    order = r.permutation(npages)
    bt = np.full((B, maxb), -1, dtype=np.int64)
    zkp = r.standard_normal((npages, H, ps, r_k))
    zvp = r.standard_normal((npages, H, ps, r_v))
    dense_k = r.standard_normal((B, H, maxb * ps, r_k))
    dense_v = r.standard_normal((B, H, maxb * ps, r_v))
    k = 0
    for b in range(B):
        for blk in range((lens[b] + ps - 1) // ps):
            pg = order[k]; k += 1
            bt[b, blk] = pg
            zkp[pg] = dense_k[b, :, blk * ps:(blk + 1) * ps]
            zvp[pg] = dense_v[b, :, blk * ps:(blk + 1) * ps]
    q = r.standard_normal((B, H, d)) / np.sqrt(d)
    dk = r.standard_normal((H, d, r_k)) / np.sqrt(r_k)
    dv = r.standard_normal((H, d, r_v)) / np.sqrt(r_v)
    mk = r.standard_normal((H, d)) if mu else None
    mv = r.standard_normal((H, d)) if mu else None
    return dict(q=q, zkp=zkp, zvp=zvp, bt=bt, dense_k=dense_k, dense_v=dense_v, dk=dk, dv=dv,
                mk=mk, mv=mv)


def test_paged_equals_dense_decode_per_sequence_length():
    r = rng(41)
    lens = [1, 7, 8, 9, 23, 0, 16]
    B, H, d, ps = len(lens), 3, 8, 8
    s = _paged_store(r, B, H, d, ps, lens)
    out, lse = oracle.paged_decode(s["q"], s["zkp"], s["zvp"], s["bt"], lens, s["dk"], s["dv"],
                                   s["mk"], s["mv"])
    for b, n in enumerate(lens):
        if n == 0:
            continue
        ob, lb = oracle.lla_decode(s["q"][b:b + 1], s["dense_k"][b:b + 1], s["dense_v"][b:b + 1],
                                   s["dk"], s["dv"], s["mk"], s["mv"], N=n)
        np.testing.assert_allclose(out[b], ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], lb[0], rtol=0, atol=1e-12)


def test_paged_single_token_is_the_reconstruction_from_its_page():
    # one cached token: out is that token's reconstructed value, read from
    # head h of the page the block table names (§3 Eq. 3)
    r = rng(42)
    B, H, d, ps = 3, 4, 6, 5
    s = _paged_store(r, B, H, d, ps, [1, 1, 1])
    out, lse = oracle.paged_decode(s["q"], s["zkp"], s["zvp"], s["bt"], [1, 1, 1], s["dk"],
                                   s["dv"], s["mk"], s["mv"])
    for b in range(B):
        pg = s["bt"][b, 0]
        for h in range(H):
            vhat = s["dv"][h] @ s["zvp"][pg, h, 0] + s["mv"][h]
            khat = s["dk"][h] @ s["zkp"][pg, h, 0] + s["mk"][h]
            np.testing.assert_allclose(out[b, h], vhat, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], s["q"][b, h] @ khat / np.sqrt(d), atol=1e-12)


def test_paged_page_relabelling_and_unused_pages_do_not_matter():
    r = rng(43)
    lens = [13, 4, 30]
    B, H, d, ps = 3, 2, 8, 4
    s = _paged_store(r, B, H, d, ps, lens)
    out, lse = oracle.paged_decode(s["q"], s["zkp"], s["zvp"], s["bt"], lens, s["dk"], s["dv"])
    perm = r.permutation(s["zkp"].shape[0])
    inv = np.argsort(perm)
    bt2 = np.where(s["bt"] >= 0, inv[np.maximum(s["bt"], 0)], -1)
    zk2, zv2 = s["zkp"][perm].copy(), s["zvp"][perm].copy()
    used = set(bt2[bt2 >= 0].tolist())
    for pg in range(zk2.shape[0]):
        if pg not in used:
            zk2[pg] = np.nan
            zv2[pg] = np.nan
    # rows past each sequence's length inside its last page are never read
    for b, n in enumerate(lens):
        if n % ps:
            zk2[bt2[b, n // ps], :, n % ps:] = np.nan
            zv2[bt2[b, n // ps], :, n % ps:] = np.nan
    out2, lse2 = oracle.paged_decode(s["q"], zk2, zv2, bt2, lens, s["dk"], s["dv"])
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


def test_paged_eviction_attends_exactly_the_kept_positions():
    r = rng(44)
    lens = [40, 9, 26]
    sink, window = 3, 6
    B, H, d, ps = 3, 2, 8, 4
    s = _paged_store(r, B, H, d, ps, lens, mu=True)
    out, lse = oracle.paged_decode(s["q"], s["zkp"], s["zvp"], s["bt"], lens, s["dk"], s["dv"],
                                   s["mk"], s["mv"], sink=sink, window=window)
    for b, n in enumerate(lens):
        pos = oracle.kept_positions(n, sink, window)
        assert pos.size == min(n, sink + window)
        ob, lb = oracle.lla_decode(s["q"][b:b + 1], s["dense_k"][b:b + 1, :, pos],
                                   s["dense_v"][b:b + 1, :, pos], s["dk"], s["dv"], s["mk"],
                                   s["mv"])
        np.testing.assert_allclose(out[b], ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], lb[0], rtol=0, atol=1e-12)
    # evicted tokens may hold anything
    zk2, zv2 = s["zkp"].copy(), s["zvp"].copy()
    for b, n in enumerate(lens):
        kept = set(oracle.kept_positions(n, sink, window).tolist())
        for j in range(n):
            if j not in kept:
                zk2[s["bt"][b, j // ps], :, j % ps] = 1e3
                zv2[s["bt"][b, j // ps], :, j % ps] = -1e3
    out2, lse2 = oracle.paged_decode(s["q"], zk2, zv2, s["bt"], lens, s["dk"], s["dv"], s["mk"],
                                     s["mv"], sink=sink, window=window)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)


def test_paged_empty_sequence_has_no_attention_mass():
    r = rng(45)
    s = _paged_store(r, 2, 2, 4, 4, [0, 5])
    out, lse = oracle.paged_decode(s["q"], s["zkp"], s["zvp"], s["bt"], [0, 5], s["dk"], s["dv"],
                                   s["mk"], s["mv"])
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(out[1])) and np.all(np.isfinite(lse[1]))


# ---------------------------------------------------------------------------
# decoupled RoPE
# ---------------------------------------------------------------------------

def test_rope_is_a_rotation_that_sees_only_relative_position():
    r = rng(51)
    d = 16
    q, k = r.standard_normal(d), r.standard_normal(d)
    # position 0 is the identity; norms are kept
    np.testing.assert_allclose(oracle.rope_rotate(q, 0), q, atol=0)
    np.testing.assert_allclose(np.linalg.norm(oracle.rope_rotate(q, 37)), np.linalg.norm(q),
                               rtol=1e-13)
    # the score depends on p - j only
    s1 = oracle.rope_rotate(q, 100) @ oracle.rope_rotate(k, 40)
    s2 = oracle.rope_rotate(q, 1060) @ oracle.rope_rotate(k, 1000)
    s3 = oracle.rope_rotate(q, 60) @ k
    assert abs(s1 - s2) < 1e-10 and abs(s1 - s3) < 1e-10
    # pair 0 turns by exactly pos radians (theta^0 = 1); the last pair slowest
    x = np.zeros(d); x[0] = 1.0
    y = oracle.rope_rotate(x, 0.5)
    np.testing.assert_allclose(y[:2], [np.cos(0.5), np.sin(0.5)], atol=1e-15)
    x = np.zeros(d); x[d - 2] = 1.0
    y = oracle.rope_rotate(x, 3.0)
    a = 3.0 * 10000.0 ** (-(d - 2) / d)
    np.testing.assert_allclose(y[d - 2:], [np.cos(a), np.sin(a)], atol=1e-15)


def test_rope_unit_reduces_to_the_nope_unit_and_to_rotary_attention():
    r = rng(52)
    u = _unit(52)
    q, zk, zv, dk, dv, mk, mv = (u[k] for k in ("q", "zk", "zv", "dk", "dv", "mu_k", "mu_v"))
    N, d_r = zk.shape[0], 8
    k_rope = r.standard_normal((N, d_r))
    # zero rotary query: the NoPE latent unit
    o0, l0 = oracle.decode_unit_rope(q, np.zeros(d_r), zk, k_rope, zv, dk, dv, mk, mv)
    o1, l1 = oracle.decode_unit(q, zk, zv, dk, dv, mk, mv)
    np.testing.assert_allclose(o0, o1, atol=1e-12)
    assert abs(l0 - l1) < 1e-12
    # zero content query and key mean: plain attention over the rotary keys
    q_rope = r.standard_normal(d_r)
    o2, l2 = oracle.decode_unit_rope(np.zeros_like(q), q_rope, zk, k_rope, zv, dk, dv, None, mv)
    vhat = zv @ dv.T + mv
    o3, l3 = oracle.attend(q_rope, k_rope, vhat, 1.0 / np.sqrt(q.shape[0]))
    np.testing.assert_allclose(o2, o3, atol=1e-12)
    assert abs(l2 - l3) < 1e-12


def test_rope_unit_matches_absorbed_query_with_appended_rotary_part():
    # the §7 absorption applies to the content part only: q' = dk^T q,
    # scores q'.z_j + q.mu_k + q_rope.k_rope_j (brute force, tiny inputs)
    r = rng(53)
    u = _unit(53)
    q, zk, zv, dk, dv, mk, mv = (u[k] for k in ("q", "zk", "zv", "dk", "dv", "mu_k", "mu_v"))
    N, d_r = zk.shape[0], 6
    k_rope = r.standard_normal((N, d_r))
    q_rope = r.standard_normal(d_r)
    sc = 1.0 / np.sqrt(q.shape[0])
    o, l = oracle.decode_unit_rope(q, q_rope, zk, k_rope, zv, dk, dv, mk, mv)
    qa = np.concatenate([dk.T @ q, q_rope])
    s = sc * (np.concatenate([zk, k_rope], axis=1) @ qa + q @ mk)
    p = np.exp(s - s.max())
    ubar = (p / p.sum()) @ zv
    np.testing.assert_allclose(o, dv @ ubar + mv, atol=1e-12)
    assert abs(l - (s.max() + np.log(p.sum()))) < 1e-12


def test_paged2d_equals_dense_2d_decode_per_sequence_length():
    r = rng(61)
    lens = [1, 5, 8, 0, 13, 16]
    B, H, d, ps, rk, rv = len(lens), 3, 8, 4, 16, 24
    maxb = 4
    npages = B * maxb + 2
    order = r.permutation(npages)
    bt = np.full((B, maxb), -1)
    zkp = r.standard_normal((npages, ps, rk))
    zvp = r.standard_normal((npages, ps, rv))
    dense_k = r.standard_normal((B, maxb * ps, rk))
    dense_v = r.standard_normal((B, maxb * ps, rv))
    k = 0
    for b, n in enumerate(lens):
        for blk in range((n + ps - 1) // ps):
            pg = order[k]; k += 1
            bt[b, blk] = pg
            zkp[pg] = dense_k[b, blk * ps:(blk + 1) * ps]
            zvp[pg] = dense_v[b, blk * ps:(blk + 1) * ps]
    q = r.standard_normal((B, H, d))
    dk, dv = r.standard_normal((H, d, rk)), r.standard_normal((H, d, rv))
    mk, mv = r.standard_normal((H, d)), r.standard_normal((H, d))
    out, lse = oracle.paged2d_decode(q, zkp, zvp, bt, lens, dk, dv, mk, mv)
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        ob, lb = oracle.lla2d_decode(q[b:b + 1], dense_k[b:b + 1], dense_v[b:b + 1], dk, dv, mk,
                                     mv, N=n)
        np.testing.assert_allclose(out[b], ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], lb[0], rtol=0, atol=1e-12)
    # one token: every head's output is that token's reconstruction
    o1, _ = oracle.paged2d_decode(q[:1], zkp, zvp, bt[:1], [1], dk, dv, mk, mv)
    pg = bt[0, 0]
    for h in range(H):
        np.testing.assert_allclose(o1[0, h], dv[h] @ zvp[pg, 0] + mv[h], atol=1e-12)


def test_lla2d_rope_is_per_head_rope_with_the_row_shared_by_every_head():
    r = rng(71)
    B, H, d, N, rk, dr, rv = 2, 3, 8, 9, 8, 4, 12
    zk = r.standard_normal((B, N, rk + dr))
    zv = r.standard_normal((B, N, rv))
    q, qr = r.standard_normal((B, H, d)), r.standard_normal((B, H, dr))
    dk, dv = r.standard_normal((H, d, rk)), r.standard_normal((H, d, rv))
    mk, mv = r.standard_normal((H, d)), r.standard_normal((H, d))
    o2, l2 = oracle.lla2d_decode_rope(q, qr, zk, zv, dk, dv, mk, mv)
    zk_h = np.repeat(zk[:, None], H, axis=1)
    zv_h = np.repeat(zv[:, None], H, axis=1)
    o1, l1 = oracle.lla_decode_rope(q, qr, zk_h, zv_h, dk, dv, mk, mv)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(l2, l1, atol=1e-12)
    # and with a zero rotary query it is the plain LLA-2D decode
    o3, l3 = oracle.lla2d_decode_rope(q, np.zeros_like(qr), zk, zv, dk, dv, mk, mv)
    o4, l4 = oracle.lla2d_decode(q, zk[:, :, :rk], zv, dk, dv, mk, mv)
    np.testing.assert_allclose(o3, o4, atol=1e-12)
    np.testing.assert_allclose(l3, l4, atol=1e-12)


def _rope_batch(seed, B=3, H=4, d=8, n_cap=11, rk=8, dr=6, rv=12):
    """Per-head store with a DIFFERENT latent and rotary key for every
    (b, h): zk [B, H, n_cap, rk + dr], zv [B, H, n_cap, rv]."""
    r = rng(seed)
    return dict(q=r.normal(size=(B, H, d)), qr=r.normal(size=(B, H, dr)),
                zk=r.normal(size=(B, H, n_cap, rk + dr)), zv=r.normal(size=(B, H, n_cap, rv)),
                dk=r.normal(size=(H, d, rk)), dv=r.normal(size=(H, d, rv)),
                mk=r.normal(size=(H, d)), mv=r.normal(size=(H, d)), rk=rk, dr=dr)


def test_per_head_rope_reads_each_heads_own_row_and_units_pick_their_unit():
    # §7 "Per-head LLA versus LLA-2D at inference": each (b, h) unit is the
    # decoupled-RoPE unit on ITS OWN latent rows. Distinct rows per head, so
    # reading another head's (or batch row's) latents fails here.
    u = _rope_batch(301)
    q, qr, zk, zv, dk, dv, mk, mv = (u[k] for k in ("q", "qr", "zk", "zv", "dk", "dv", "mk", "mv"))
    rk = u["rk"]
    B, H = q.shape[:2]
    N = 9  # rows [N, n_cap) must be ignored
    out, lse = oracle.lla_decode_rope(q, qr, zk, zv, dk, dv, mk, mv, scale=0.3, N=N)
    for b in range(B):
        for h in range(H):
            o1, l1 = oracle.decode_unit_rope(q[b, h], qr[b, h], zk[b, h, :N, :rk],
                                             zk[b, h, :N, rk:], zv[b, h, :N], dk[h], dv[h],
                                             mk[h], mv[h], 0.3)
            np.testing.assert_allclose(out[b, h], o1, rtol=0, atol=1e-12)
            assert abs(lse[b, h] - l1) < 1e-12
    # a shuffled subset of units, with a repeat, returns one row per listed unit
    units = [(2, 3), (0, 1), (1, 0), (2, 0), (0, 1), (1, 3)]
    sub_o, sub_l = oracle.lla_decode_rope(q, qr, zk, zv, dk, dv, mk, mv, scale=0.3, N=N,
                                          units=units)
    assert sub_o.shape == (len(units), q.shape[2])
    for i, (b, h) in enumerate(units):
        np.testing.assert_allclose(sub_o[i], out[b, h], rtol=0, atol=1e-12)
        assert abs(sub_l[i] - lse[b, h]) < 1e-12


def test_per_head_rope_is_nope_decode_on_a_block_embedded_codec():
    # An independent route through the NoPE decode: append the rotary part to
    # the query, the identity on the rotary coordinates to W^K_up, zeros to
    # W^V_up and to the means. Then q'.(W' z' + mu') = q.(W z + mu) + q_rope.k_rope,
    # so lla_decode on the block-embedded codec gives the rotary scores, and
    # its output is [out | 0]. Distinct per-head rows, on a shuffled subset.
    u = _rope_batch(302, B=2, H=3, d=8, n_cap=10, rk=8, dr=4, rv=16)
    q, qr, zk, zv, dk, dv, mk, mv = (u[k] for k in ("q", "qr", "zk", "zv", "dk", "dv", "mk", "mv"))
    rk, dr = u["rk"], u["dr"]
    H, d = q.shape[1], q.shape[2]
    rv = zv.shape[-1]
    q_e = np.concatenate([q, qr], axis=-1)
    dk_e = np.zeros((H, d + dr, rk + dr))
    dk_e[:, :d, :rk] = dk
    dk_e[:, d:, rk:] = np.eye(dr)
    dv_e = np.zeros((H, d + dr, rv))
    dv_e[:, :d] = dv
    mk_e = np.concatenate([mk, np.zeros((H, dr))], axis=-1)
    mv_e = np.concatenate([mv, np.zeros((H, dr))], axis=-1)
    units = [(1, 2), (0, 0), (1, 0), (0, 2)]
    sc = 0.25
    o_r, l_r = oracle.lla_decode_rope(q, qr, zk, zv, dk, dv, mk, mv, scale=sc, N=7, units=units)
    o_e, l_e = oracle.lla_decode(q_e, zk, zv, dk_e, dv_e, mk_e, mv_e, sc, N=7, units=units)
    np.testing.assert_allclose(o_r, o_e[:, :d], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_e[:, d:], 0.0, atol=0)
    np.testing.assert_allclose(l_r, l_e, rtol=0, atol=1e-12)


def test_lla2d_rope_units_pick_their_unit_from_the_shared_row():
    r = rng(303)
    B, H, d, n_cap, rk, dr, rv = 3, 4, 8, 10, 8, 4, 12
    zk = r.normal(size=(B, n_cap, rk + dr))
    zv = r.normal(size=(B, n_cap, rv))
    q, qr = r.normal(size=(B, H, d)), r.normal(size=(B, H, dr))
    dk, dv = r.normal(size=(H, d, rk)), r.normal(size=(H, d, rv))
    mk, mv = r.normal(size=(H, d)), r.normal(size=(H, d))
    N = 8
    out, lse = oracle.lla2d_decode_rope(q, qr, zk, zv, dk, dv, mk, mv, scale=0.3, N=N)
    for b in range(B):
        for h in range(H):
            o1, l1 = oracle.decode_unit_rope(q[b, h], qr[b, h], zk[b, :N, :rk], zk[b, :N, rk:],
                                             zv[b, :N], dk[h], dv[h], mk[h], mv[h], 0.3)
            np.testing.assert_allclose(out[b, h], o1, rtol=0, atol=1e-12)
            assert abs(lse[b, h] - l1) < 1e-12
    units = [(2, 1), (0, 3), (2, 1), (1, 0)]
    sub_o, sub_l = oracle.lla2d_decode_rope(q, qr, zk, zv, dk, dv, mk, mv, scale=0.3, N=N,
                                            units=units)
    for i, (b, h) in enumerate(units):
        np.testing.assert_allclose(sub_o[i], out[b, h], rtol=0, atol=1e-12)
        assert abs(sub_l[i] - lse[b, h]) < 1e-12


def test_merge_of_context_parts_equals_attention_over_the_whole():
    # split the cached tokens into disjoint parts, attend each, merge
    r = rng(81)
    u = _unit(81, N=37)
    q, zk, zv, dk, dv, mk, mv = (u[k] for k in ("q", "zk", "zv", "dk", "dv", "mu_k", "mu_v"))
    full_o, full_l = oracle.decode_unit(q, zk, zv, dk, dv, mk, mv)
    cuts = [0, 5, 6, 20, 37]
    outs, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = oracle.decode_unit(q, zk[a:b], zv[a:b], dk, dv, mk, mv)
        outs.append(o)
        lses.append(l)
    # an empty part contributes nothing
    outs.append(np.full_like(full_o, 123.0))
    lses.append(-np.inf)
    o, l = oracle.merge_attn(np.stack(outs), np.array(lses))
    np.testing.assert_allclose(o, full_o, atol=1e-12)
    assert abs(l - full_l) < 1e-12
    # order of the parts does not matter; all-empty gives 0 / -inf
    o2, l2 = oracle.merge_attn(np.stack(outs[::-1]), np.array(lses[::-1]))
    np.testing.assert_allclose(o2, o, atol=1e-12)
    oe, le = oracle.merge_attn(np.zeros((3, 4)), np.full(3, -np.inf))
    assert np.all(oe == 0) and np.isneginf(le)


def test_paged2d_eviction_attends_exactly_the_kept_positions():
    r = rng(91)
    lens = [40, 9, 26, 0]
    sink, window = 3, 6
    B, H, d, ps, rk, rv = len(lens), 2, 8, 4, 8, 12
    maxb = 10
    npages = B * maxb
    bt = np.arange(npages).reshape(B, maxb)
    zkp = r.standard_normal((npages, ps, rk))
    zvp = r.standard_normal((npages, ps, rv))
    q = r.standard_normal((B, H, d))
    dk, dv = r.standard_normal((H, d, rk)), r.standard_normal((H, d, rv))
    out, lse = oracle.paged2d_decode(q, zkp, zvp, bt, lens, dk, dv, sink=sink, window=window)
    for b, n in enumerate(lens):
        pos = oracle.kept_positions(n, sink, window)
        if pos.size == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        zk = zkp[bt[b, pos // ps], pos % ps][None]
        zv = zvp[bt[b, pos // ps], pos % ps][None]
        ob, lb = oracle.lla2d_decode(q[b:b + 1], zk, zv, dk, dv)
        np.testing.assert_allclose(out[b], ob[0], atol=1e-12)
        np.testing.assert_allclose(lse[b], lb[0], atol=1e-12)
    # no eviction when window is 0
    o0, _ = oracle.paged2d_decode(q, zkp, zvp, bt, lens, dk, dv)
    o1, _ = oracle.paged2d_decode(q, zkp, zvp, bt, lens, dk, dv, sink=5, window=0)
    np.testing.assert_allclose(o0, o1, atol=0)


# --------------------------------------------------------------------------
# the latent write into a paged store (the write side of the paged layout)
# --------------------------------------------------------------------------

def _shuffled_table(r, lens, ps, extra_pages=3):
    need = [(n + ps - 1) // ps for n in lens]
    P = sum(need) + extra_pages
    order = r.permutation(P)
    bt = np.full((len(lens), max(need)), -1)
    k = 0
    for b, nb in enumerate(need):
        bt[b, :nb] = order[k:k + nb]
        k += nb
    return bt, P


def test_paged_write_then_paged_decode_equals_a_dense_prefill():
    # Appending each sequence's tokens one decode step at a time (a serving
    # loop: position = current length) into a shuffled page pool, then
    # decoding the pool, gives the same result as encoding every token at
    # once into a dense [B, H, n, r] store and decoding that. This ties the
    # write side's addresses to the read side's gather (itself pinned
    # against the dense decode above).
    r = rng(401)
    lens = [5, 1, 9, 4]
    B, T, H, d, rk, ps = len(lens), 2, 3, 4, 5, 3
    n_max = max(lens)
    bt, P = _shuffled_table(r, lens, ps)
    w = r.normal(size=(H, T * d, rk))
    mu = r.normal(size=(H, T * d))
    x = r.normal(size=(n_max, T, B, H, d))            # token j of every sequence
    pool = r.normal(size=(P, H, ps, rk))              # stale contents
    for j in range(n_max):
        live = [b for b in range(B) if j < lens[b]]
        z = oracle.encode(x[j][:, live], w, mu)       # one step's newest tokens
        pool, skipped = oracle.paged_write(pool, z, bt, positions=[j] * len(live),
                                           seq_idx=live)
        assert skipped == []
    dense = np.zeros((B, H, n_max, rk))
    for b in range(B):
        xb = np.transpose(x[:lens[b], :, b], (1, 0, 2, 3))   # [T, n_b, H, d]
        dense[b, :, :lens[b]] = oracle.encode(xb, w, mu)      # [H, n_b, rk]
    q = r.normal(size=(B, H, 6))
    dk, dv = r.normal(size=(H, 6, rk)), r.normal(size=(H, 6, rk))
    out_p, lse_p = oracle.paged_decode(q, pool, pool, bt, lens, dk, dv, scale=0.4)
    for b in range(B):
        o, l = oracle.lla_decode(q[b:b + 1], dense[b:b + 1], dense[b:b + 1], dk, dv, scale=0.4,
                                 N=lens[b])
        np.testing.assert_allclose(out_p[b], o[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse_p[b], l[0], rtol=0, atol=1e-12)


def test_paged_write_touches_exactly_the_addressed_rows():
    r = rng(402)
    G, N, rk, ps, r_row = 2, 6, 4, 4, 7                 # rows wider than the latent
    bt = np.array([[3, 0, 5], [1, 4, 2]])
    pool = r.normal(size=(7, G, ps, r_row))
    z = r.normal(size=(G, N, rk))
    seq = [0, 1, 1, 0, 1, 0]
    pos = [0, 5, 11, 9, 12, 6]                          # 12 is past the table: skipped
    new, skipped = oracle.paged_write(pool, z, bt, pos, seq_idx=seq)
    assert skipped == [4]
    expect = pool.copy()
    for n in (0, 1, 2, 3, 5):
        page, row = bt[seq[n], pos[n] // ps], pos[n] % ps
        expect[page, :, row, :rk] = z[:, n]
    np.testing.assert_array_equal(new, expect)          # the rotary tail is untouched too
    # bad sequence index and a page outside the pool are skipped as well
    bt2 = np.array([[3, 9]])
    new2, sk2 = oracle.paged_write(pool, z[:, :3], bt2, [1, 5, 0], seq_idx=[0, 0, 2])
    assert sk2 == [1, 2]
    expect2 = pool.copy()
    expect2[3, :, 1, :rk] = z[:, 0]
    np.testing.assert_array_equal(new2, expect2)


def test_paged_write_lla2d_rows_and_default_sequence_per_token():
    r = rng(403)
    N, rk, ps = 4, 6, 2
    bt = np.array([[2, 0], [5, 1], [3, 4], [6, 7]])
    pool = r.normal(size=(8, ps, rk))
    z = r.normal(size=(1, N, rk))
    pos = [3, 0, 2, 1]                                  # token n is sequence n's newest
    new, skipped = oracle.paged_write(pool, z, bt, pos)
    assert skipped == []
    expect = pool.copy()
    for n in range(N):
        expect[bt[n, pos[n] // ps], pos[n] % ps] = z[0, n]
    np.testing.assert_array_equal(new, expect)
    # reading the rows back through the LLA-2D paged decode with one token
    # gives each token's own reconstruction
    H, d = 3, 5
    dv = r.normal(size=(H, d, rk))
    q = r.normal(size=(N, H, d))
    bt1 = np.array([[bt[n, pos[n] // ps]] for n in range(N)])
    rows = [pos[n] % ps for n in range(N)]
    for n in range(N):
        one = new[bt1[n, 0], rows[n]][None, None]        # a 1-row page holding that row
        o, _ = oracle.paged2d_decode(q[n:n + 1], one, one, np.array([[0]]), [1],
                                     r.normal(size=(H, d, rk)), dv)
        np.testing.assert_allclose(o[0], (dv @ z[0, n]), atol=1e-12)

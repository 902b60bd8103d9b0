"""Pins for the float64 oracle: page numbers, closed forms, invariants, brute force.

Each test ties the oracle to something other than itself, so that a dropped
term, a wrong sign or index, or a transposed operand in ``oracle/`` fails one
of them.  CPU only.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))
KiB, MiB, GiB = 1 << 10, 1 << 20, 1 << 30


# --------------------------------------------------------------------------- bookkeeping

def ouro(r_k, r_v, mode=O.MODE_PER_HEAD):
    g = GOLDEN["ouro_1p4b"]
    return O.Cfg(g["T"], g["H"], g["d_head"], r_k, r_v, mode)


def test_worked_example_scalars_and_ratio():
    w = GOLDEN["ouro_1p4b"]["worked_example"]
    cfg = ouro(w["r_k"], w["r_v"])
    assert O.teacher_scalars_per_token_layer(cfg) == w["scalars_per_layer_teacher"]
    assert O.lla_scalars_per_token_layer(cfg) == w["scalars_per_layer_lla"]
    assert O.compression_ratio(cfg) == w["ratio"]


def test_table5_kib_per_token_full_model():
    g = GOLDEN["table5_kv_per_token_kib"]
    D = GOLDEN["ouro_1p4b"]["D"]
    base = ouro(96, 160)
    assert O.teacher_cache_bytes(base, 1, D) == g["teacher"] * KiB
    for key in ("lla_4x", "lla_21p3x"):
        s = g["ranks_sum"][key]
        cfg = ouro(s // 3, s - s // 3)
        assert O.cache_bytes(cfg, 1, D) == g[key] * KiB


def test_table5_one_million_context():
    g = GOLDEN["table5_1m_context_gib"]
    D = GOLDEN["ouro_1p4b"]["D"]
    assert O.teacher_cache_bytes(ouro(96, 160), g["tokens"], D) == g["teacher"] * GiB
    assert O.cache_bytes(ouro(96, 160), g["tokens"], D) == g["lla_4x"] * GiB
    assert O.cache_bytes(ouro(16, 32), g["tokens"], D) == g["lla_21p3x"] * GiB


def test_capacity_arithmetic_and_eviction():
    g = GOLDEN["table5_max_batch_4k"]
    D = GOLDEN["ouro_1p4b"]["D"]
    n = g["context"]
    teacher = O.teacher_cache_bytes(ouro(96, 160), n * g["teacher"], D)
    four = O.cache_bytes(ouro(96, 160), n * g["lla_4x"], D)
    big = O.cache_bytes(ouro(16, 32), n * g["lla_21p3x"], D)
    assert (teacher, four, big) == (96 * GiB, 96 * GiB, 108 * GiB)
    e = GOLDEN["eviction_budget"]
    assert O.cache_bytes(ouro(16, 32), e["tokens"], D) == e["mib"] * MiB


def test_ratio_labels_ouro_and_huginn():
    lab = GOLDEN["ouro_ratio_labels"]
    for printed, s in lab["labels"].items():
        cfg = ouro(s // 2, s - s // 2)
        r = O.compression_ratio(cfg)
        assert r == Fraction(lab["two_T_d"], s)
        # the printed label is the exact ratio rounded to the page's digits
        digits = len(printed.split(".")[1]) if "." in printed else 0
        assert round(float(r), digits) == pytest.approx(float(printed))
    hug = GOLDEN["huginn_table3"]
    for row in hug["rows"]:
        cfg = O.Cfg(hug["T"], 1, 96, row["r_k"], row["r_v"])
        assert O.compression_ratio(cfg) == row["ratio"]
    # d_head = 96 is the only width consistent with every Table 3 row
    for d in (64, 80, 112, 128):
        assert any(O.compression_ratio(O.Cfg(hug["T"], 1, d, x["r_k"], x["r_v"])) != x["ratio"]
                   for x in hug["rows"])


def test_workload_ratios_and_2d_fold():
    want = [Fraction(64, 3), Fraction(4), Fraction(64, 3), Fraction(256, 3), Fraction(32)]
    for name, r in zip(synth.WORKLOAD_ORDER, want):
        w = synth.WORKLOADS[name]
        assert O.compression_ratio(O.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode)) == r
    # LLA-2D at fixed ranks stores H times fewer scalars than per-head
    a = O.Cfg(4, 16, 128, 64, 128, O.MODE_PER_HEAD)
    b = O.Cfg(4, 16, 128, 64, 128, O.MODE_2D)
    assert O.lla_scalars_per_token_layer(a) == 16 * O.lla_scalars_per_token_layer(b)


# --------------------------------------------------------------------------- bf16

def test_bf16_round_matches_library_conversion():
    torch = pytest.importorskip("torch")
    g = synth.rng(7)
    x = np.concatenate([
        g.standard_normal(20000).astype(np.float32),
        (g.standard_normal(2000) * 1e-39).astype(np.float32),       # fp32 subnormals
        g.uniform(-3.39e38, 3.39e38, 2000).astype(np.float32),      # near overflow
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.4e38], np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even mantissa (1.0)
    assert O.bf16_round(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even)
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    # just above the halfway point rounds up
    assert O.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7


# --------------------------------------------------------------------------- RoPE

def test_rope_hand_values():
    # d = 2: theta_0 = 1, the pair rotates by pos radians
    x = np.array([0.3, -1.2])
    got = O.rope(x, 2, 10000.0)
    c, s = math.cos(2.0), math.sin(2.0)
    assert got == pytest.approx([0.3 * c + 1.2 * s, 0.3 * s - 1.2 * c], abs=1e-15)
    # d = 4, base 100: theta = [1, 0.1]; pairs are (0, 2) and (1, 3)
    x = np.array([1.0, 2.0, 3.0, 4.0])
    got = O.rope(x, 5, 100.0)
    a0, a1 = 5.0, 0.5
    want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
            1 * math.sin(a0) + 3 * math.cos(a0), 2 * math.sin(a1) + 4 * math.cos(a1)]
    assert got == pytest.approx(want, abs=1e-14)


def test_rope_complex_form_and_invariants():
    g = synth.rng(11)
    d, base = 64, 10000.0
    x = g.standard_normal((50, d))
    pos = g.integers(0, 40000, size=50)
    got = O.rope(x, pos, base)
    # independent form: pair (i, i+d/2) as a complex number times e^{i pos theta_i}
    theta = np.array([base ** (-(2 * i) / d) for i in range(d // 2)])
    z = (x[:, : d // 2] + 1j * x[:, d // 2:]) * np.exp(1j * pos[:, None] * theta[None])
    np.testing.assert_allclose(got, np.concatenate([z.real, z.imag], 1), atol=1e-11)
    np.testing.assert_allclose(np.linalg.norm(got, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_array_equal(O.rope(x, 0, base), x)
    # scores depend on the position difference only
    q, k = g.standard_normal(d), g.standard_normal(d)
    s1 = O.rope(q, 1000, base) @ O.rope(k, 400, base)
    s2 = O.rope(q, 30600, base) @ O.rope(k, 30000, base)
    assert s1 == pytest.approx(s2, rel=1e-10)


# --------------------------------------------------------------------------- codec

def test_full_rank_codec_is_exact_and_loop_specific():
    g = synth.rng(3)
    T, d = 4, 16
    W = synth.random_orthonormal(g, T * d, T * d)
    mu = g.standard_normal(T * d)
    W_up = O.loop_slices(W, T, d)
    x = g.standard_normal((10, T, d))
    c = O.encode(x.reshape(10, T * d), mu, W)
    for t in range(T):
        np.testing.assert_allclose(O.reconstruct(c, W_up[t], mu[t * d:(t + 1) * d]), x[:, t],
                                   atol=1e-12)
    # a different loop's slice gives a different state
    assert np.abs(O.reconstruct(c, W_up[1], mu[d:2 * d]) - x[:, 0]).max() > 0.1


def test_2d_codec_block_diagonal_equals_per_head():
    """LLA-2D with a head-block-diagonal codec reduces to per-head LLA, head by head."""
    g = synth.rng(5)
    T, H, d, rk, rv, n = 3, 2, 8, 4, 6, 7
    ph = O.Cfg(T, H, d, rk, rv, O.MODE_PER_HEAD)
    p2 = O.Cfg(T, H, d, rk * H, rv * H, O.MODE_2D)
    Wdk = np.stack([synth.random_orthonormal(g, T * d, rk) for _ in range(H)])
    Wdv = np.stack([synth.random_orthonormal(g, T * d, rv) for _ in range(H)])
    Wuk = g.standard_normal((H, T, d, rk))
    Wuv = g.standard_normal((H, T, d, rv))
    muk = g.standard_normal((H, T * d))
    muv = g.standard_normal((H, T * d))
    per = O.Codec(Wdk, Wdv, Wuk, Wuv, muk, muv)

    def fold_down(W, r):
        out = np.zeros((T * H * d, H * r))
        for h in range(H):
            for t in range(T):
                out[(t * H + h) * d:(t * H + h + 1) * d, h * r:(h + 1) * r] = W[h, t * d:(t + 1) * d]
        return out

    def fold_up(W, r):
        out = np.zeros((T, H, d, H * r))
        for h in range(H):
            out[:, h, :, h * r:(h + 1) * r] = W[h]
        return out

    def fold_mu(mu):
        return np.stack([mu[h].reshape(T, d) for h in range(H)], 1).reshape(-1)

    two = O.Codec(fold_down(Wdk, rk), fold_down(Wdv, rv), fold_up(Wuk, rk), fold_up(Wuv, rv),
                  fold_mu(muk), fold_mu(muv))
    xk = g.standard_normal((n, T, H, d))
    xv = g.standard_normal((n, T, H, d))
    ck, cv = O.encode_tokens(ph, per, xk, xv)
    ck2, cv2 = O.encode_tokens(p2, two, xk, xv)
    np.testing.assert_allclose(ck2, ck.reshape(n, -1), atol=1e-12)
    np.testing.assert_allclose(cv2, cv.reshape(n, -1), atol=1e-12)
    q, ks, vs = (g.standard_normal((1, H, d)) for _ in range(3))
    pos = np.arange(n)[None]
    for t in range(T):
        a = O.decode_attn_cache(ph, per, t, q, ks, vs, ck[None], cv[None], pos, [n], [n])
        b = O.decode_attn_cache(p2, two, t, q, ks, vs, ck2[None], cv2[None], pos, [n], [n])
        np.testing.assert_allclose(b, a, atol=1e-12)


def test_eckart_young_and_monotone_error():
    """Calibration error of the SVD codec equals the discarded spectrum, so falls with r."""
    g = synth.rng(9)
    T, H, d = 4, 1, 16
    model = synth.trajectory_model(g, T, H, d, R=5)
    X = synth.sample_trajectories(g, model, 400)[:, :, 0, :].reshape(400, T * d)
    Xh = synth.sample_trajectories(g, model, 400)[:, :, 0, :].reshape(400, T * d)
    cal, held = [], []
    for r in range(1, T * d + 1, 3):
        mu, W, sigma = O.svd_init(X, r)
        W_up = O.loop_slices(W, T, d)
        for data, acc in ((X, cal), (Xh, held)):
            c = O.encode(data, mu, W)
            rec = np.concatenate([O.reconstruct(c, W_up[t], mu[t * d:(t + 1) * d])
                                  for t in range(T)], 1)
            acc.append(((data - rec) ** 2).sum())
        assert cal[-1] == pytest.approx((sigma[r:] ** 2).sum(), rel=1e-9, abs=1e-9)
        assert np.allclose(W.T @ W, np.eye(r), atol=1e-12)
    assert all(a >= b - 1e-9 for a, b in zip(cal, cal[1:]))
    assert all(a >= b - 1e-9 for a, b in zip(held, held[1:]))
    # rank-5-plus-noise: nearly all energy is captured once r >= 5
    assert cal[2] < 1e-2 * cal[0]


def test_2d_svd_codec_full_rank_is_exact_and_slice_order_matters():
    """LLA-2D branch of svd_codec and loop_slices (close reading §二.4, §二.6; gist.science
    "Training und Initialisierung", "LLA-2D-Variante"): with r = T H d the SVD basis of
    the (t, h, i)-ordered calibration rows is a full orthonormal basis, so encoding and
    then rebuilding with the (t, h) slice returns x_{t,h} exactly.  Slicing the rows in
    (h, t) order instead (a transposed reshape) does not."""
    g = synth.rng(41)
    T, H, d = 2, 3, 4                             # width T H d = 24
    W = T * H * d
    cfg = O.Cfg(T, H, d, W, W, O.MODE_2D)
    model = synth.trajectory_model(g, T, H, d, R=5, shared=True)
    cal_k = synth.sample_trajectories(g, model, 400)
    cal_v = synth.sample_trajectories(g, model, 400)
    codec = O.svd_codec(cfg, cal_k, cal_v)
    assert codec.W_down_k.shape == (W, W) and codec.W_up_k.shape == (T, H, d, W)
    np.testing.assert_allclose(codec.W_down_k.T @ codec.W_down_k, np.eye(W), atol=1e-12)
    x = synth.sample_trajectories(g, model, 10)
    ck, cv = O.encode_tokens(cfg, codec, x, x)
    wrong_order = codec.W_down_k.reshape(H, T, d, W)
    worst_wrong = 0.0
    for t in range(T):
        for h in range(H):
            mu = O.mu_t(cfg, codec.mu_k, t, h)
            rec = O.reconstruct(ck, O.w_up_t(cfg, codec.W_up_k, t, h), mu)
            np.testing.assert_allclose(rec, x[:, t, h], atol=1e-12)
            np.testing.assert_allclose(O.reconstruct(cv, O.w_up_t(cfg, codec.W_up_v, t, h),
                                                     O.mu_t(cfg, codec.mu_v, t, h)),
                                       x[:, t, h], atol=1e-12)
            bad = O.reconstruct(ck, wrong_order[h, t], mu)
            worst_wrong = max(worst_wrong, np.abs(bad - x[:, t, h]).max())
    assert worst_wrong > 0.1


def test_2d_eckart_young_and_monotone_error():
    """LLA-2D codec by SVD: the calibration error summed over every (t, h) rebuild equals
    the discarded spectrum, so it falls monotonically with r (held-out error too, on the
    seeded low-rank-plus-noise trajectories shared across heads)."""
    g = synth.rng(43)
    T, H, d = 2, 2, 6
    W = T * H * d
    model = synth.trajectory_model(g, T, H, d, R=4, shared=True)
    X = synth.sample_trajectories(g, model, 300)
    Xh = synth.sample_trajectories(g, model, 300)
    cal, held = [], []
    for r in range(1, W + 1, 2):
        mu, Wd, sigma = O.svd_init(X.reshape(300, W), r)
        W_up = O.loop_slices(Wd, T, d, H)
        assert W_up.shape == (T, H, d, r)
        cfg = O.Cfg(T, H, d, r, r, O.MODE_2D)
        for data, acc in ((X, cal), (Xh, held)):
            c = O.encode(data.reshape(len(data), W), mu, Wd)
            err = 0.0
            for t in range(T):
                for h in range(H):
                    rec = O.reconstruct(c, W_up[t, h], O.mu_t(cfg, mu, t, h))
                    err += ((data[:, t, h] - rec) ** 2).sum()
            acc.append(err)
        assert cal[-1] == pytest.approx((sigma[r:] ** 2).sum(), rel=1e-9, abs=1e-9)
    assert all(a >= b - 1e-9 for a, b in zip(cal, cal[1:]))
    assert all(a >= b - 1e-9 for a, b in zip(held, held[1:]))
    assert cal[2] < 1e-2 * cal[0]      # rank 4 plus noise: captured once r >= 5


def test_2d_svd_codec_error_is_the_discarded_spectrum():
    """The whole LLA-2D codec path (svd_codec on [N, T, H, d] calibration tokens,
    encode_tokens, the (t, h) slices of W_up and mu) at ranks below full: the
    calibration error over every (t, h) rebuild equals the sum of the discarded
    squared singular values of the centred (t, h, i)-ordered calibration matrix, as
    numpy's SVD gives them.  A codec built in another concatenation order, or with a
    mis-sliced mean, misses it."""
    g = synth.rng(47)
    T, H, d = 2, 3, 4
    W = T * H * d
    model = synth.trajectory_model(g, T, H, d, R=6, shared=True)
    N = 300
    X = synth.sample_trajectories(g, model, N)
    flat = X.reshape(N, W)                               # (t, h, i) order, [CR] §二.6
    sigma = np.linalg.svd(flat - flat.mean(0), compute_uv=False)
    for r in (3, 6, 11):
        cfg = O.Cfg(T, H, d, r, r, O.MODE_2D)
        codec = O.svd_codec(cfg, X, X)
        ck, _ = O.encode_tokens(cfg, codec, X, X)
        err = 0.0
        for t in range(T):
            for h in range(H):
                rec = O.reconstruct(ck, O.w_up_t(cfg, codec.W_up_k, t, h),
                                    O.mu_t(cfg, codec.mu_k, t, h))
                err += ((X[:, t, h] - rec) ** 2).sum()
        assert err == pytest.approx((sigma[r:] ** 2).sum(), rel=1e-9, abs=1e-9)


# --------------------------------------------------------------------------- attention

def brute_force(q, K, V, pos, ks, vs, qpos, base):
    """Pure-Python decode attention: explicit rotations, dot products and softmax."""
    d = len(q)
    h = d // 2

    def rot(x, p):
        out = [0.0] * d
        for i in range(h):
            a = p * base ** (-2.0 * i / d)
            out[i] = x[i] * math.cos(a) - x[i + h] * math.sin(a)
            out[i + h] = x[i] * math.sin(a) + x[i + h] * math.cos(a)
        return out

    qr = rot(q, qpos)
    keys = [rot(k, p) for k, p in zip(K, pos)] + [rot(ks, qpos)]
    vals = list(V) + [vs]
    s = [sum(a * b for a, b in zip(qr, k)) / math.sqrt(d) for k in keys]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    z = sum(e)
    return [sum(e[j] * vals[j][i] for j in range(len(vals))) / z for i in range(d)]


@pytest.mark.parametrize("n", [0, 1, 2, 4])
def test_decode_attention_brute_force(n):
    g = synth.rng(20 + n)
    d, r, base = 4, 3, 100.0
    W_k, W_v = g.standard_normal((d, r)), g.standard_normal((d, r))
    mu_k, mu_v = g.standard_normal(d), g.standard_normal(d)
    ck, cv = g.standard_normal((n, r)), g.standard_normal((n, r))
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    pos = g.integers(0, 50, size=n)
    K = [[sum(ck[j, m] * W_k[i, m] for m in range(r)) + mu_k[i] for i in range(d)] for j in range(n)]
    V = [[sum(cv[j, m] * W_v[i, m] for m in range(r)) + mu_v[i] for i in range(d)] for j in range(n)]
    want = brute_force(list(q), K, V, list(pos), list(ks), list(vs), 60, base)
    for fn in (O.decode_attention, O.decode_attention_absorbed):
        got = fn(q, ks, vs, ck, cv, W_k, W_v, mu_k, mu_v, pos, 60, base)
        np.testing.assert_allclose(got, want, atol=1e-12)


def test_constant_keys_give_uniform_weights():
    g = synth.rng(31)
    d, n = 8, 5
    K = np.tile(g.standard_normal(d), (n, 1))
    V = g.standard_normal((n, d))
    vs = g.standard_normal(d)
    # same key at every position 0 (history and self): every score equal
    out, p, ps = O.attention_plain(g.standard_normal(d), K, V, np.zeros(n, int), K[0], vs, 0,
                                   10000.0)
    np.testing.assert_allclose(p, 1.0 / (n + 1), rtol=1e-14)
    np.testing.assert_allclose(out, (V.sum(0) + vs) / (n + 1), atol=1e-14)


def test_empty_history_returns_in_flight_value():
    g = synth.rng(32)
    d = 8
    vs = g.standard_normal(d)
    out = O.decode_attention(g.standard_normal(d), g.standard_normal(d), vs,
                             np.zeros((0, 3)), np.zeros((0, 3)), g.standard_normal((d, 3)),
                             g.standard_normal((d, 3)), np.zeros(d), np.zeros(d), np.zeros(0, int),
                             0, 10000.0)
    np.testing.assert_allclose(out, vs, atol=1e-15)


def test_v_absorption_identity():
    g = synth.rng(33)
    d, r, n = 32, 12, 50
    args = (g.standard_normal(d), g.standard_normal(d), g.standard_normal(d),
            g.standard_normal((n, 7)), g.standard_normal((n, r)), g.standard_normal((d, 7)),
            g.standard_normal((d, r)), g.standard_normal(d), g.standard_normal(d),
            g.permutation(200)[:n], 300, 10000.0)
    np.testing.assert_allclose(O.decode_attention_absorbed(*args), O.decode_attention(*args),
                               atol=1e-12)


def test_full_rank_lla_attention_equals_plain_attention():
    """r = T d with an orthonormal codec: LLA attention == attention over the per-loop cache."""
    g = synth.rng(34)
    T, H, d, n = 2, 2, 8, 9
    cfg = O.Cfg(T, H, d, T * d, T * d)
    Wk = np.stack([synth.random_orthonormal(g, T * d, T * d) for _ in range(H)])
    Wv = np.stack([synth.random_orthonormal(g, T * d, T * d) for _ in range(H)])
    muk, muv = g.standard_normal((H, T * d)), g.standard_normal((H, T * d))
    codec = O.Codec(Wk, Wv, np.stack([O.loop_slices(w, T, d) for w in Wk]),
                    np.stack([O.loop_slices(w, T, d) for w in Wv]), muk, muv)
    xk, xv = g.standard_normal((n, T, H, d)), g.standard_normal((n, T, H, d))
    ck, cv = O.encode_tokens(cfg, codec, xk, xv)
    q, ks, vs = (g.standard_normal((1, H, d)) for _ in range(3))
    pos = np.arange(n)[None]
    for t in range(T):
        got = O.decode_attn_cache(cfg, codec, t, q, ks, vs, ck[None], cv[None], pos, [n], [n])
        for h in range(H):
            want, _, _ = O.attention_plain(q[0, h], xk[:, t, h], xv[:, t, h], pos[0], ks[0, h],
                                           vs[0, h], n, 10000.0)
            np.testing.assert_allclose(got[0, h], want, atol=1e-12)


def test_svd_codec_on_low_rank_trajectories():
    """SVD codec of rank >= R reproduces rank-R-plus-noise trajectories to the noise level."""
    g = synth.rng(35)
    T, H, d, R = 4, 2, 16, 3
    mk = synth.trajectory_model(g, T, H, d, R)
    mv = synth.trajectory_model(g, T, H, d, R)
    cal_k, cal_v = synth.sample_trajectories(g, mk, 1024), synth.sample_trajectories(g, mv, 1024)
    cfg = O.Cfg(T, H, d, 8, 16)
    codec = O.svd_codec(cfg, cal_k, cal_v)
    xk, xv = synth.sample_trajectories(g, mk, 64), synth.sample_trajectories(g, mv, 64)
    ck, cv = O.encode_tokens(cfg, codec, xk, xv)
    for t in range(T):
        for h in range(H):
            rec = O.reconstruct(ck[:, h], O.w_up_t(cfg, codec.W_up_k, t, h),
                                O.mu_t(cfg, codec.mu_k, t, h))
            assert np.abs(rec - xk[:, t, h]).max() < 0.06   # noise sigma = 0.01 per entry

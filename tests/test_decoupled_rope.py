"""Decoupled RoPE attention (close reading §四.10, Appendix J, Tables 13-14): a
NoPE content path absorbed into the query plus an explicit rotary branch over the
first d_rope dims of each head.

CPU: the oracle pinned to the full-RoPE decode (d_rope = d), to a NoPE attention
written out by hand (d_rope = 0), to its own absorbed form, and to the
relative-position property of the rotary branch.
"""
from __future__ import annotations

import numpy as np

import oracle as O
import synth


def _head(g, d, r_k, r_v, n):
    c_k, c_v = g.standard_normal((n, r_k)), g.standard_normal((n, r_v))
    Wk, Wv = g.standard_normal((d, r_k)) / np.sqrt(r_k), g.standard_normal((d, r_v)) / np.sqrt(r_v)
    mk, mv = 0.1 * g.standard_normal(d), 0.1 * g.standard_normal(d)
    return c_k, c_v, Wk, Wv, mk, mv


def test_rotary_branch_over_every_dim_is_full_rope():
    g = synth.rng(21)
    d, r_k, r_v, n = 16, 6, 5, 30
    c_k, c_v, Wk, Wv, mk, mv = _head(g, d, r_k, r_v, n)
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    pos = g.permutation(300)[:n]
    got = O.decode_attention_decoupled(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 301, 500.0, d)
    want = O.decode_attention(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 301, 500.0)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_no_rotary_branch_is_plain_softmax_attention():
    """d_rope = 0: scores are scale * q . k of the rebuilt keys, written out here."""
    g = synth.rng(22)
    d, r_k, r_v, n = 8, 4, 3, 12
    c_k, c_v, Wk, Wv, mk, mv = _head(g, d, r_k, r_v, n)
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    K = np.array([[sum(c_k[j, k] * Wk[i, k] for k in range(r_k)) + mk[i] for i in range(d)]
                  for j in range(n)])
    V = np.array([[sum(c_v[j, k] * Wv[i, k] for k in range(r_v)) + mv[i] for i in range(d)]
                  for j in range(n)])
    s = [float(np.dot(q, K[j])) / np.sqrt(d) for j in range(n)] + [float(np.dot(q, ks)) / np.sqrt(d)]
    w = np.exp(np.array(s) - max(s))
    w /= w.sum()
    want = sum(w[j] * V[j] for j in range(n)) + w[-1] * vs
    pos = g.permutation(100)[:n]
    got = O.decode_attention_decoupled(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 77, 10000.0, 0)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_absorbed_content_path_equals_the_direct_form():
    g = synth.rng(23)
    d, r_k, r_v, n = 32, 7, 6, 25
    c_k, c_v, Wk, Wv, mk, mv = _head(g, d, r_k, r_v, n)
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    pos = g.permutation(400)[:n]
    for d_rope in (0, 8, 16, 32):
        a = O.decode_attention_decoupled(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 401, 1e4, d_rope)
        b = O.decode_attention_decoupled_absorbed(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 401,
                                                  1e4, d_rope)
        np.testing.assert_allclose(b, a, rtol=1e-11, atol=1e-12)


def test_rotary_branch_depends_on_relative_positions_only():
    g = synth.rng(24)
    d, r_k, r_v, n = 32, 6, 6, 20
    c_k, c_v, Wk, Wv, mk, mv = _head(g, d, r_k, r_v, n)
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    pos = g.permutation(50)[:n]
    ref = O.decode_attention_decoupled(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 60, 100.0, 16)
    for shift in (1000, 54321):
        got = O.decode_attention_decoupled(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos + shift,
                                           60 + shift, 100.0, 16)
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-9)
    moved = O.decode_attention_decoupled(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 61, 100.0, 16)
    assert not np.allclose(moved, ref)


def test_only_the_leading_dims_rotate_on_their_own_frequency_ladder():
    """rope_partial turns pair (i, i + d_rope/2) of the leading d_rope dims by
    pos * base^(-2i/d_rope) and leaves the rest alone."""
    g = synth.rng(25)
    d, d_rope, base, pos = 12, 4, 100.0, 7
    x = g.standard_normal(d)
    y = O.rope_partial(x, pos, base, d_rope)
    np.testing.assert_array_equal(y[d_rope:], x[d_rope:])
    for i in range(d_rope // 2):
        ang = pos * base ** (-2.0 * i / d_rope)
        a, b = x[i], x[i + d_rope // 2]
        np.testing.assert_allclose(y[i], a * np.cos(ang) - b * np.sin(ang), rtol=1e-14, atol=1e-14)
        np.testing.assert_allclose(y[i + d_rope // 2], a * np.sin(ang) + b * np.cos(ang),
                                   rtol=1e-14, atol=1e-14)

"""Full-memory fast path: the loop-t K/V rebuilt once into a full bf16 cache
(keys rotated at their positions) and decoded with ordinary attention
(close reading §四.9, Table 5 and the paragraph after it; §二.3 for RoPE).

CPU: the oracle's fast path pinned to the latent path, to closed forms and to
the relative-position property of RoPE.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
from cases import decode_case


def _head(g, d, r_k, r_v, n):
    c_k, c_v = g.standard_normal((n, r_k)), g.standard_normal((n, r_v))
    Wk, Wv = g.standard_normal((d, r_k)) / np.sqrt(r_k), g.standard_normal((d, r_v)) / np.sqrt(r_v)
    mk, mv = 0.1 * g.standard_normal(d), 0.1 * g.standard_normal(d)
    return c_k, c_v, Wk, Wv, mk, mv


# ----------------------------------------------------------------------------- oracle pins

def test_full_path_without_rounding_equals_the_latent_path():
    """Keeping rebuilt, rotated K/V and attending over them is the LLA decode itself
    (the fast path changes where the rebuild happens, not what is computed)."""
    g = synth.rng(11)
    d, r_k, r_v, n = 16, 6, 5, 37
    c_k, c_v, Wk, Wv, mk, mv = _head(g, d, r_k, r_v, n)
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    pos = g.permutation(500)[:n]                 # gaps and disorder, not slot order
    K, V = O.full_memory_kv(c_k, c_v, Wk, Wv, mk, mv, pos, 10000.0, round_bf16=False)
    got = O.decode_attention_full(q, ks, vs, K, V, 611, 10000.0)
    want = O.decode_attention(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, 611, 10000.0)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_full_path_empty_history_is_the_in_flight_value():
    g = synth.rng(12)
    d = 8
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    out = O.decode_attention_full(q, ks, vs, np.zeros((0, d)), np.zeros((0, d)), 5, 10000.0)
    np.testing.assert_array_equal(out, vs)


def test_full_path_one_token_closed_form():
    """At position 0 RoPE is the identity, so with one history row the weights are a
    logistic of the score difference."""
    g = synth.rng(13)
    d = 8
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    k1, v1 = g.standard_normal(d), g.standard_normal(d)
    sc = 0.37
    s1, s2 = sc * q @ k1, sc * q @ ks
    p1 = 1.0 / (1.0 + np.exp(s2 - s1))
    out = O.decode_attention_full(q, ks, vs, k1[None], v1[None], 0, 10000.0, scale=sc)
    np.testing.assert_allclose(out, p1 * v1 + (1 - p1) * vs, rtol=1e-13, atol=1e-13)


def test_full_path_depends_on_relative_positions_only():
    """Shifting every history position and the query position by the same amount
    leaves the output unchanged: the keys must be rotated by +angle at their own
    positions and the query at q_pos, and a sign or index slip breaks this."""
    g = synth.rng(14)
    d, r_k, r_v, n = 16, 4, 4, 20
    c_k, c_v, Wk, Wv, mk, mv = _head(g, d, r_k, r_v, n)
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    pos = g.permutation(60)[:n]
    outs = []
    for shift in (0, 1000, 12345):
        K, V = O.full_memory_kv(c_k, c_v, Wk, Wv, mk, mv, pos + shift, 100.0, round_bf16=False)
        outs.append(O.decode_attention_full(q, ks, vs, K, V, 70 + shift, 100.0))
    np.testing.assert_allclose(outs[1], outs[0], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(outs[2], outs[0], rtol=1e-9, atol=1e-9)
    # the query rotated at another position does change it
    K, V = O.full_memory_kv(c_k, c_v, Wk, Wv, mk, mv, pos, 100.0, round_bf16=False)
    assert not np.allclose(O.decode_attention_full(q, ks, vs, K, V, 71, 100.0), outs[0])


def test_full_memory_kv_at_position_zero_is_the_rebuild_and_rounds_once():
    g = synth.rng(15)
    d, r_k, r_v, n = 8, 3, 5, 9
    c_k, c_v, Wk, Wv, mk, mv = _head(g, d, r_k, r_v, n)
    K, V = O.full_memory_kv(c_k, c_v, Wk, Wv, mk, mv, np.zeros(n, int), 10000.0,
                            round_bf16=False)
    np.testing.assert_allclose(K, c_k @ Wk.T + mk, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(V, c_v @ Wv.T + mv, rtol=1e-14, atol=1e-14)
    Kb, Vb = O.full_memory_kv(c_k, c_v, Wk, Wv, mk, mv, np.zeros(n, int), 10000.0)
    np.testing.assert_array_equal(Kb, O.bf16_round(K))
    np.testing.assert_array_equal(Vb, O.bf16_round(V))
    np.testing.assert_array_equal(O.bf16_round(Kb), Kb)


def test_full_cache_layout_is_head_major_and_zero_past_the_context():
    cfg = O.Cfg(2, 3, 8, 4, 4)
    case = decode_case(cfg, 2, 10, seed=16, ctx_len=[10, 4], codec="random")
    K, V = O.full_cache(cfg, case.codec, 1, case.c_k, case.c_v, case.positions, case.ctx_len)
    assert K.shape == (2, 3, 10, 8)
    assert not K[1, :, 4:].any() and not V[1, :, 4:].any()
    k_row, v_row = O.full_memory_kv(case.c_k[1, :4, 2], case.c_v[1, :4, 2],
                                    O.w_up_t(cfg, case.codec.W_up_k, 1, 2),
                                    O.w_up_t(cfg, case.codec.W_up_v, 1, 2),
                                    O.mu_t(cfg, case.codec.mu_k, 1, 2),
                                    O.mu_t(cfg, case.codec.mu_v, 1, 2),
                                    case.positions[1, :4], cfg.rope_base)
    np.testing.assert_array_equal(K[1, 2, :4], k_row)
    np.testing.assert_array_equal(V[1, 2, :4], v_row)

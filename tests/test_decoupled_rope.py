"""Decoupled RoPE attention (close reading §四.10, Appendix J, Tables 13-14): a
NoPE content path absorbed into the query plus an explicit rotary branch over the
first d_rope dims of each head.

CPU: the oracle pinned to the full-RoPE decode (d_rope = d), to a NoPE attention
written out by hand (d_rope = 0), to its own absorbed form, and to the
relative-position property of the rotary branch; host checks of the ABI.
GPU: the tensor-core decode (per head and LLA-2D) with d_rope in {32, 64} against
the oracle (ragged and random-position cases, several splits and one split per
head), and the refusal of the CUDA-core path.
"""
from __future__ import annotations

import numpy as np
import pytest

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


# ----------------------------------------------------------------------------- C ABI, host

def test_decoupled_rope_host_checks():
    import ctypes

    import looped_transformer_decode_b200 as lla

    def cfg_rc(**kw):
        c = lla.Cfg(4, 16, 128, 96, 160, **kw)
        return lla.lib.lla_codec_packed_bytes(ctypes.byref(c.c()))
    assert cfg_rc(d_rope=64) > 0 and cfg_rc(d_rope=32) > 0 and cfg_rc(d_rope=128) > 0
    assert cfg_rc(d_rope=48) == 0                       # unsupported width
    c = lla.Cfg(4, 4, 32, 16, 16, d_rope=64)            # wider than the head
    assert lla.lib.lla_codec_packed_bytes(ctypes.byref(c.c())) == 0
    # the RoPE table holds the rotary branch's pairs only
    for dr, half in ((0, 64), (64, 32), (32, 16), (128, 64)):
        c = lla.Cfg(4, 16, 128, 96, 160, d_rope=dr)
        assert lla.lib.lla_rope_table_bytes(ctypes.byref(c.c()), 10) == 10 * half * 8
    # the full-memory path rotates whole heads
    p = ctypes.c_void_p(0x1000)
    c = lla.Cfg(4, 16, 128, 96, 160, d_rope=64).c()
    assert lla.lib.lla_full_decode_attn(ctypes.byref(c), p, 1, 2, 16, p, p, p, p, p, p, p, p, p,
                                        1 << 20, None) == lla.ERR_UNSUPPORTED


# ----------------------------------------------------------------------------- GPU

def _dev_cfg(cfg, d_rope):
    import looped_transformer_decode_b200 as lla
    return lla.Cfg(cfg.T, cfg.H, cfg.d, cfg.r_k, cfg.r_v, cfg.mode, cfg.rope_base, d_rope=d_rope)


def _run_decoupled(case, d_rope, t, ws=None):
    import torch

    import looped_transformer_decode_b200 as lla
    from gpu_util import bf16_tensor, f32_tensor, i32_tensor, pack
    lc = _dev_cfg(case.cfg, d_rope)
    mp = int(max(case.positions.max(initial=0), case.q_pos.max())) + 1
    rope = lla.rope_table(lc, mp)
    if ws is None:
        ws = lla.decode_workspace(lc, case.B, case.n_cap)
    out = lla.decode_attn(lc, pack(case), rope, t, i32_tensor(case.ctx_len), f32_tensor(case.q),
                          f32_tensor(case.k_self[t]), f32_tensor(case.v_self[t]),
                          i32_tensor(case.positions), i32_tensor(case.q_pos),
                          bf16_tensor(case.c_k), bf16_tensor(case.c_v), ws=ws)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), ws


DECOUPLED_CASES = [
    (O.Cfg(4, 2, 128, 96, 160), 64, [300, 129, 1], "random"),
    (O.Cfg(4, 4, 128, 16, 32), 32, [200, 64], "arange"),
    (O.Cfg(2, 2, 96, 32, 48), 64, [130, 7], "random"),
    (O.Cfg(2, 4, 64, 24, 40), 32, [100], "random"),
    (O.Cfg(2, 4, 128, 64, 128, O.MODE_2D), 64, [260, 100], "random"),   # LLA-2D
    (O.Cfg(2, 8, 64, 32, 48, O.MODE_2D), 32, [200, 1, 129], "arange"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("spec", DECOUPLED_CASES, ids=lambda s: f"d{s[0].d}r{s[1]}n{max(s[2])}")
def test_decoupled_decode_matches_oracle(spec):
    from cases import ATTN_TOL, decode_case, rel_err
    cfg, d_rope, ctx, pos_kind = spec
    ctx = np.asarray(ctx)
    case = decode_case(cfg, len(ctx), int(ctx.max()), seed=900 + d_rope + cfg.d, ctx_len=ctx,
                       positions=pos_kind, codec="random")
    for t in (0, cfg.T - 1):
        got, ws = _run_decoupled(case, d_rope, t)
        want = O.decode_attn_cache_decoupled(cfg, case.codec, t, case.q, case.k_self[t],
                                             case.v_self[t], case.c_k, case.c_v, case.positions,
                                             case.q_pos, case.ctx_len, d_rope)
        assert np.isfinite(got).all()
        assert rel_err(got, want).max() <= ATTN_TOL, (t, rel_err(got, want).max())
        # and the kernel follows the decoupled scores, not full RoPE (the two outputs
        # differ by ~1e-3 here; the kernel sits ten times closer to the decoupled one)
        full = O.decode_attn_cache(cfg, case.codec, t, case.q, case.k_self[t], case.v_self[t],
                                   case.c_k, case.c_v, case.positions, case.q_pos, case.ctx_len)
        assert 10 * rel_err(got, want).max() < rel_err(got, full).max()
        import looped_transformer_decode_b200 as lla
        assert lla.decode_status(ws) == 0


@pytest.mark.gpu
def test_decoupled_one_split_per_head_plan():
    """Enough heads for one split each: the combine runs inside the partial kernel."""
    from cases import ATTN_TOL, decode_case, rel_err

    import looped_transformer_decode_b200 as lla
    cfg = O.Cfg(4, 16, 128, 96, 160)
    ctx = np.array([260, 255, 129, 1, 0, 200, 256, 77] * 2)
    lc = _dev_cfg(cfg, 64)
    assert lla.decode_launches(lc, len(ctx), int(ctx.max())) == 2
    case = decode_case(cfg, len(ctx), int(ctx.max()), seed=950, ctx_len=ctx, positions="random",
                       codec="random")
    got, _ = _run_decoupled(case, 64, 1)
    want = O.decode_attn_cache_decoupled(cfg, case.codec, 1, case.q, case.k_self[1],
                                         case.v_self[1], case.c_k, case.c_v, case.positions,
                                         case.q_pos, case.ctx_len, 64)
    assert rel_err(got, want).max() <= ATTN_TOL


@pytest.mark.gpu
def test_decoupled_rope_outside_the_tensor_core_path_is_refused(monkeypatch):
    import torch

    import looped_transformer_decode_b200 as lla
    from cases import decode_case
    for cfg in (O.Cfg(2, 2, 64, 16, 16), O.Cfg(2, 4, 64, 16, 16, O.MODE_2D)):
        case = decode_case(cfg, 1, 40, seed=960, codec="random")
        monkeypatch.setenv("LLA_DECODE_PATH", "cuda_core")
        with pytest.raises(lla.LLAError):
            _run_decoupled(case, 32, 0)
    torch.cuda.synchronize()

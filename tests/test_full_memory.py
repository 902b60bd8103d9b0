"""Full-memory fast path: the loop-t K/V rebuilt once into a full bf16 cache
(keys rotated at their positions) and decoded with ordinary attention
(close reading §四.9, Table 5 and the paragraph after it; §二.3 for RoPE).

CPU: the oracle's fast path pinned to the latent path, to closed forms and to
the relative-position property of RoPE; host-side argument checks of the ABI.
GPU: lla_full_rebuild against the oracle's bf16 cache element by element, and
lla_full_decode_attn against the oracle on that cache (small ragged cases, both
launch plans, and sampled pairs of the 4x bench workload).
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

import oracle as O
import synth
from cases import ATTN_TOL, decode_case, f32, rel_err

import looped_transformer_decode_b200 as lla


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


# ----------------------------------------------------------------------------- C ABI, host

def test_full_path_host_checks():
    c = lla.Cfg(4, 16, 128, 96, 160).c()
    p = ctypes.c_void_p(0x1000)
    assert lla.lib.lla_full_kv_bytes(ctypes.byref(c), 8, 4097) == 8 * 16 * 4097 * 128 * 2
    assert lla.lib.lla_full_kv_bytes(ctypes.byref(c), -1, 4) == 0
    rb = lla.lib.lla_full_rebuild
    # nothing to do
    assert rb(ctypes.byref(c), None, None, 1, 0, 2, 16, None, None, None, None, 0, None, None,
              None, None) == lla.OK
    # t outside [0, T), NULL pointers, too many rows without a slot list
    assert rb(ctypes.byref(c), p, p, 1, 4, 2, 16, p, p, p, None, 4, p, p, None,
              None) == lla.ERR_INVALID
    assert rb(ctypes.byref(c), p, None, 1, 0, 2, 16, p, p, p, None, 4, p, p, None,
              None) == lla.ERR_INVALID
    assert rb(ctypes.byref(c), p, p, 1, 0, 2, 16, p, p, p, None, 33, p, p, None,
              None) == lla.ERR_INVALID
    fd = lla.lib.lla_full_decode_attn
    need = lla.lib.lla_full_decode_workspace_bytes(ctypes.byref(c), 2, 4096)
    assert need >= 256
    assert fd(ctypes.byref(c), p, 1, 0, 16, p, p, p, p, p, p, p, p, p, 0, None) == lla.OK
    assert fd(ctypes.byref(c), p, 1, 2, 4096, p, p, p, p, p, p, p, p, p, need - 1,
              None) == lla.ERR_TOO_SMALL
    assert fd(ctypes.byref(c), p, 1, 2, 4096, p, p, p, p, p, None, p, p, p, need,
              None) == lla.ERR_INVALID
    assert fd(ctypes.byref(c), p, 1, 4096, 40000, p, p, p, p, p, p, p, p, p, 1 << 40,
              None) == lla.ERR_UNSUPPORTED
    assert fd(ctypes.byref(c), p, 0, 2, 16, p, p, p, p, p, p, p, p, p, need,
              None) == lla.ERR_INVALID
    # one launch when every head fits one split, two when splits need the combine
    assert lla.full_decode_launches(lla.Cfg(4, 16, 128, 96, 160), 8, 4097) == 1
    assert lla.full_decode_launches(lla.Cfg(4, 16, 128, 96, 160), 1, 4096) == 2


# ----------------------------------------------------------------------------- GPU

def _device_inputs(case, t):
    from gpu_util import bf16_tensor, f32_tensor, i32_tensor, lib_cfg, pack
    mp = int(max(case.positions.max(initial=0), case.q_pos.max())) + 1
    lc = lib_cfg(case.cfg)
    return dict(lc=lc, packed=pack(case), rope=lla.rope_table(lc, mp),
                ctx_len=i32_tensor(case.ctx_len), q=f32_tensor(case.q),
                k_self=f32_tensor(case.k_self[t]), v_self=f32_tensor(case.v_self[t]),
                positions=i32_tensor(case.positions), q_pos=i32_tensor(case.q_pos),
                c_k=bf16_tensor(case.c_k), c_v=bf16_tensor(case.c_v))


def _assert_bf16_cache_close(got, want):
    """GPU rebuild (fp32 sums, fp32 RoPE factors, one bf16 rounding) against the
    oracle's (fp64, one bf16 rounding): equal except where the two pre-rounding
    values straddle a rounding boundary, which moves one element by one bf16 ulp
    (at most 2^-7 of its magnitude); fp32 accumulation adds ~1e-6 of the row scale."""
    row = np.abs(want).max(-1, keepdims=True)
    tol = 2.0 ** -7 * np.abs(want) + 1e-5 * row
    assert (np.abs(got - want) <= tol).all(), np.abs(got - want).max()
    assert np.mean(got != want) < 0.02


FULL_CASES = [
    (O.Cfg(4, 4, 128, 32, 48), [200, 65, 0], "random"),
    (O.Cfg(2, 2, 64, 16, 24), [150, 1], "random"),
    (O.Cfg(4, 4, 96, 32, 48), [130, 64], "arange"),
    (O.Cfg(2, 4, 32, 16, 16, O.MODE_2D), [100, 63, 2], "random"),
    (O.Cfg(4, 8, 128, 64, 64, O.MODE_2D), [257, 128], "arange"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("spec", FULL_CASES, ids=lambda s: f"m{s[0].mode}d{s[0].d}n{max(s[1])}")
def test_full_rebuild_then_decode_matches_oracle(spec):
    import torch
    cfg, ctx, pos_kind = spec
    ctx = np.asarray(ctx)
    n_cap = int(ctx.max()) + 3
    case = decode_case(cfg, len(ctx), n_cap, seed=500 + cfg.d, ctx_len=ctx, positions=pos_kind,
                       codec="random")
    for t in (0, cfg.T - 1):
        x = _device_inputs(case, t)
        kf, vf = lla.full_cache_alloc(x["lc"], case.B, n_cap)
        # rebuild every row of every sequence (rows past ctx_len too: the cache is full)
        lla.full_rebuild(x["lc"], x["packed"], x["rope"], t, x["positions"], x["c_k"], x["c_v"],
                         kf, vf)
        torch.cuda.synchronize()
        full_ctx = np.full(case.B, n_cap)
        K, V = O.full_cache(cfg, case.codec, t, case.c_k, case.c_v, case.positions, full_ctx)
        _assert_bf16_cache_close(kf.double().cpu().numpy(), K)
        _assert_bf16_cache_close(vf.double().cpu().numpy(), V)
        # decode over the GPU's cache: the oracle attends over that same bf16 cache
        ws = lla.full_decode_workspace(x["lc"], case.B, n_cap)
        out = lla.full_decode_attn(x["lc"], x["rope"], x["ctx_len"], x["q"], x["k_self"],
                                   x["v_self"], x["q_pos"], kf, vf, ws=ws)
        torch.cuda.synchronize()
        want = O.decode_attn_full_cache(cfg, case.q, case.k_self[t], case.v_self[t],
                                        kf.double().cpu().numpy(), vf.double().cpu().numpy(),
                                        case.q_pos, ctx)
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, want).max() <= ATTN_TOL, (t, rel_err(got, want).max())
        assert int(ws[4:8].view(torch.int32).item()) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,n_cap,launches", [(1, 2, 700, 2), (40, 4, 70, 1)])
def test_full_decode_both_launch_plans(B, H, n_cap, launches):
    """Several splits per head (partial kernel + combine) and one split per head (the
    merge finished inside the kernel), on an oracle-made bf16 cache with ragged lengths."""
    import torch
    from gpu_util import bf16_tensor, f32_tensor, i32_tensor, lib_cfg
    cfg = O.Cfg(2, H, 64, 16, 16)
    lc = lib_cfg(cfg)
    assert lla.full_decode_launches(lc, B, n_cap) == launches
    g = synth.rng(600 + B)
    ctx = g.integers(0, n_cap + 1, size=B)
    ctx[0] = n_cap
    K = O.bf16_round(g.standard_normal((B, H, n_cap, cfg.d)))
    V = O.bf16_round(g.standard_normal((B, H, n_cap, cfg.d)))
    q = f32(g.standard_normal((B, H, cfg.d)))
    ks, vs = f32(g.standard_normal((B, H, cfg.d))), f32(g.standard_normal((B, H, cfg.d)))
    q_pos = g.integers(0, 5000, size=B)
    rope = lla.rope_table(lc, 5000)
    out = lla.full_decode_attn(lc, rope, i32_tensor(ctx), f32_tensor(q), f32_tensor(ks),
                               f32_tensor(vs), i32_tensor(q_pos), bf16_tensor(K), bf16_tensor(V))
    torch.cuda.synchronize()
    want = O.decode_attn_full_cache(cfg, q, ks, vs, K, V, q_pos, ctx)
    assert rel_err(out.double().cpu().numpy(), want).max() <= ATTN_TOL


@pytest.mark.gpu
def test_full_rebuild_of_listed_slots_only():
    """The append flow: rebuild only the rows a decode step added; other rows keep
    what they held."""
    import torch
    cfg = O.Cfg(4, 2, 64, 16, 24)
    case = decode_case(cfg, 3, 40, seed=700, codec="random", positions="random")
    x = _device_inputs(case, 2)
    kf, vf = lla.full_cache_alloc(x["lc"], case.B, case.n_cap)
    kf.fill_(3.0)
    vf.fill_(3.0)
    rows = np.array([0 * 40 + 39, 1 * 40 + 0, 2 * 40 + 17], np.int64)
    slot = torch.from_numpy(rows).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lla.full_rebuild(x["lc"], x["packed"], x["rope"], 2, x["positions"], x["c_k"], x["c_v"], kf, vf,
                     slot=slot, status=status)
    torch.cuda.synchronize()
    K, V = O.full_cache(cfg, case.codec, 2, case.c_k, case.c_v, case.positions, np.full(3, 40))
    kg, vg = kf.double().cpu().numpy(), vf.double().cpu().numpy()
    touched = np.zeros((3, 40), bool)
    for r in rows:
        b, j = divmod(int(r), 40)
        touched[b, j] = True
        _assert_bf16_cache_close(kg[b, :, j], K[b, :, j])
        _assert_bf16_cache_close(vg[b, :, j], V[b, :, j])
    assert (kg.transpose(0, 2, 1, 3)[~touched] == 3.0).all()
    assert int(status.item()) == 0
    # a slot outside the cache is skipped and reported
    bad = torch.tensor([5, 3 * 40], dtype=torch.int64, device="cuda")
    lla.full_rebuild(x["lc"], x["packed"], x["rope"], 2, x["positions"], x["c_k"], x["c_v"], kf, vf,
                     slot=bad, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == lla.STATUS_SLOT_RANGE


@pytest.mark.gpu
def test_full_decode_empty_cache_and_status_bits():
    """n_cap = 0 gives the in-flight value; a query position outside the table and a
    ctx_len above n_cap are clamped and reported in the status word."""
    import torch
    from gpu_util import f32_tensor, i32_tensor, lib_cfg
    cfg = O.Cfg(2, 2, 32, 8, 8)
    lc = lib_cfg(cfg)
    g = synth.rng(800)
    q, ks, vs = (f32(g.standard_normal((2, 2, 32))) for _ in range(3))
    rope = lla.rope_table(lc, 16)
    empty = torch.empty((2, 2, 0, 32), dtype=torch.bfloat16, device="cuda")
    ws = lla.full_decode_workspace(lc, 2, 0)
    out = lla.full_decode_attn(lc, rope, i32_tensor([0, 0]), f32_tensor(q), f32_tensor(ks),
                               f32_tensor(vs), i32_tensor([3, 4]), empty, empty, ws=ws)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out.double().cpu().numpy(), vs, rtol=1e-6, atol=1e-6)
    assert int(ws[4:8].view(torch.int32).item()) == 0
    kf, vf = lla.full_cache_alloc(lc, 2, 8)
    ws2 = lla.full_decode_workspace(lc, 2, 8)
    out = lla.full_decode_attn(lc, rope, i32_tensor([9, 2]), f32_tensor(q), f32_tensor(ks),
                               f32_tensor(vs), i32_tensor([3, 99]), kf, vf, ws=ws2)
    torch.cuda.synchronize()
    bits = int(ws2[4:8].view(torch.int32).item())
    assert bits == lla.STATUS_POSITION_RANGE | lla.STATUS_CTX_RANGE
    assert np.isfinite(out.double().cpu().numpy()).all()


@pytest.mark.gpu
def test_full_path_bench_workload_sampled():
    """The per-head 4x bench workload (B 8, H 16, d 128, n 4096) through the full
    path as bench.py runs it: rebuild of the whole cache, then decode; sampled (b, h)
    pairs against the oracle's rebuild and attention."""
    import torch
    name = "perhead_4x_T4_H16_d128_r96_160_B8_n4096"
    w = synth.WORKLOADS[name]
    cfg = O.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode)
    from gpu_util import lib_cfg
    lc = lib_cfg(cfg)
    codec_np = synth.workload_codec(w)
    codec = O.Codec(*(codec_np[k].astype(np.float64) for k in
                      ("W_down_k", "W_down_v", "W_up_k", "W_up_v", "mu_k", "mu_v")))
    packed = lla.codec_pack(lc, *(torch.from_numpy(codec_np[k]).cuda() for k in
                                  ("W_down_k", "W_down_v", "W_up_k", "W_up_v", "mu_k", "mu_v")))
    x = synth.workload_tensors(w, "cuda")
    rope = lla.rope_table(lc, w.n + 1)
    t = w.loops[-1]
    kf, vf = lla.full_cache_alloc(lc, w.B, w.n)
    lla.full_rebuild(lc, packed, rope, t, x["positions"], x["c_k"], x["c_v"], kf, vf)
    out = lla.full_decode_attn(lc, rope, x["ctx_len"], x["q"], x["k_self"], x["v_self"],
                               x["q_pos"], kf, vf)
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    g = synth.rng(w.seed + 1)
    pairs = {(0, 0), (w.B - 1, w.H - 1)} | {(int(g.integers(w.B)), int(g.integers(w.H)))
                                           for _ in range(4)}
    qn, ksn, vsn = (x[k].double().cpu().numpy() for k in ("q", "k_self", "v_self"))
    for b, h in sorted(pairs):
        n = int(x["ctx_len"][b].item())
        ck = x["c_k"][b, :n, h].double().cpu().numpy()
        cv = x["c_v"][b, :n, h].double().cpu().numpy()
        pos = x["positions"][b, :n].cpu().numpy()
        Kr, Vr = O.full_memory_kv(ck, cv, O.w_up_t(cfg, codec.W_up_k, t, h),
                                  O.w_up_t(cfg, codec.W_up_v, t, h), O.mu_t(cfg, codec.mu_k, t, h),
                                  O.mu_t(cfg, codec.mu_v, t, h), pos, cfg.rope_base)
        _assert_bf16_cache_close(kf[b, h, :n].double().cpu().numpy(), Kr)
        want = O.decode_attention_full(qn[b, h], ksn[b, h], vsn[b, h],
                                       kf[b, h, :n].double().cpu().numpy(),
                                       vf[b, h, :n].double().cpu().numpy(),
                                       int(x["q_pos"][b].item()), cfg.rope_base)
        e = np.abs(got[b, h] - want).max() / np.abs(want).max()
        assert e <= ATTN_TOL, (b, h, e)

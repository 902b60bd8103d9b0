"""Eviction composed with the latent cache: sink + window retention
(close reading §四.10, Table 9: 4 sink tokens + a 256-token window; Appendix J:
a 1024-token budget).

CPU: the oracle's kept set against its definition, eviction as attention over
the kept set, the slot map of the C ABI, argument checks, and the Appendix J
bookkeeping.  GPU: the decode over an evicted cache (filled once, and grown by
decode-time appends through lla_evict_append + lla_encode) against the oracle.
"""
from __future__ import annotations

import ctypes
import dataclasses

import numpy as np
import pytest

import oracle as O
import synth
from cases import ATTN_TOL, decode_case, rel_err

import looped_transformer_decode_b200 as lla


# ----------------------------------------------------------------------------- oracle

@pytest.mark.parametrize("n,sink,window", [(0, 4, 256), (100, 4, 256), (260, 4, 256),
                                           (261, 4, 256), (4096, 4, 256), (700, 0, 64),
                                           (700, 10, 1), (3, 5, 2)])
def test_evict_keep_is_first_sink_plus_last_window(n, sink, window):
    keep = O.evict_keep(n, sink, window)
    want = sorted({j for j in range(n) if j < sink or j >= n - window})
    assert list(keep) == want
    assert len(keep) == min(n, sink + window)


def test_evicted_attention_is_attention_over_the_kept_tokens():
    """Eviction composes with LLA: the rebuilt-and-rotated keys of the kept tokens,
    attended with plain attention, give the evicted LLA output."""
    g = synth.rng(7)
    d, r_k, r_v, n, sink, window = 8, 5, 6, 40, 3, 9
    c_k, c_v = g.standard_normal((n, r_k)), g.standard_normal((n, r_v))
    Wk, Wv = g.standard_normal((d, r_k)), g.standard_normal((d, r_v))
    mk, mv = 0.1 * g.standard_normal(d), 0.1 * g.standard_normal(d)
    q, ks, vs = g.standard_normal(d), g.standard_normal(d), g.standard_normal(d)
    pos = np.arange(n)
    got = O.decode_attention_evicted(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, n, 10000.0,
                                     sink, window)
    keep = [j for j in range(n) if j < sink or j >= n - window]
    K = c_k[keep] @ Wk.T + mk
    V = c_v[keep] @ Wv.T + mv
    want = O.attention_plain(q, K, V, pos[keep], ks, vs, n, 10000.0)[0]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # a budget covering the history changes nothing
    full = O.decode_attention(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos, n, 10000.0)
    np.testing.assert_allclose(O.decode_attention_evicted(q, ks, vs, c_k, c_v, Wk, Wv, mk, mv, pos,
                                                          n, 10000.0, 30, 10), full, rtol=1e-12)
    assert not np.allclose(got, full)


def test_appendix_j_budget_bookkeeping():
    """1024 kept tokens of the 21.3x model (24 layers) take 36 KiB each: 36 MiB."""
    cfg = O.Cfg(4, 16, 128, 16, 32)
    assert O.cache_bytes(cfg, 1024, 24) == 36 * 2**20
    assert lla.cache_bytes(lla.Cfg(4, 16, 128, 16, 32), 1024, 24) == 36 * 2**20


# ----------------------------------------------------------------------------- C ABI, host

@pytest.mark.parametrize("sink,window", [(4, 256), (0, 64), (10, 1), (3, 7)])
def test_evict_slots_cover_the_budget_once(sink, window):
    budget = sink + window
    for n in (1, sink + 1, budget - 1, budget, budget + 1, 3 * budget + 5):
        keep = O.evict_keep(n, sink, window)
        slots = [lla.evict_slot(sink, window, int(j)) for j in keep]
        assert sorted(slots) == list(range(len(keep)))
    # a window position is reused exactly by the position one window later
    for p in range(sink, sink + 3 * window):
        assert lla.evict_slot(sink, window, p + window) == lla.evict_slot(sink, window, p)
        assert sink <= lla.evict_slot(sink, window, p) < budget
    for p in range(sink):
        assert lla.evict_slot(sink, window, p) == p


def test_evict_slot_rejects_bad_arguments():
    assert lla.evict_slot(-1, 4, 0) == -1
    assert lla.evict_slot(0, 0, 5) == -1
    assert lla.evict_slot(2, 4, -3) == -1


def test_evict_append_validates_on_the_host():
    f = lla.lib.lla_evict_append
    p = ctypes.c_void_p(0x1000)
    assert f(0, 16, 4, 8, None, None, None, None, None) == lla.OK           # nothing to do
    assert f(2, 16, 4, 16, p, p, p, p, None) == lla.ERR_INVALID             # budget > n_cap
    assert f(2, 16, -1, 8, p, p, p, p, None) == lla.ERR_INVALID
    assert f(2, 16, 4, 0, p, p, p, p, None) == lla.ERR_INVALID
    assert f(2, 16, 4, 8, None, p, p, p, None) == lla.ERR_INVALID
    assert f(2, 16, 4, 8, p, ctypes.c_void_p(0x1004), p, p, None) == lla.ERR_INVALID
    assert f(-1, 16, 4, 8, p, p, p, p, None) == lla.ERR_INVALID


# ----------------------------------------------------------------------------- GPU

def _expected_evicted(case, t, sink, window, n_hist):
    """Oracle: evicted LLA decode from the full-history latents of ``case``."""
    cfg, cd = case.cfg, case.codec
    out = np.zeros((case.B, cfg.H, cfg.d))
    for b in range(case.B):
        n = int(n_hist[b])
        for h in range(cfg.H):
            if cfg.mode == O.MODE_PER_HEAD:
                ck, cv = case.c_k[b, :n, h], case.c_v[b, :n, h]
            else:
                ck, cv = case.c_k[b, :n], case.c_v[b, :n]
            out[b, h] = O.decode_attention_evicted(
                case.q[b, h], case.k_self[t][b, h], case.v_self[t][b, h], ck, cv,
                O.w_up_t(cfg, cd.W_up_k, t, h), O.w_up_t(cfg, cd.W_up_v, t, h),
                O.mu_t(cfg, cd.mu_k, t, h), O.mu_t(cfg, cd.mu_v, t, h),
                case.positions[b, :n], int(case.q_pos[b]), cfg.rope_base, sink, window)
    return out


def _evicted_cache(case, sink, window, n_hist):
    """The cache a sink + window budget leaves: kept rows at their slots."""
    budget = sink + window
    B = case.B
    ck = np.zeros((B, budget) + case.c_k.shape[2:])
    cv = np.zeros((B, budget) + case.c_v.shape[2:])
    pos = np.zeros((B, budget), np.int64)
    ctx = np.zeros(B, np.int64)
    for b in range(B):
        keep = O.evict_keep(int(n_hist[b]), sink, window)
        for j in keep:
            s = lla.evict_slot(sink, window, int(j))
            ck[b, s], cv[b, s], pos[b, s] = case.c_k[b, j], case.c_v[b, j], case.positions[b, j]
        ctx[b] = len(keep)
    return dataclasses.replace(case, n_cap=budget, c_k=ck, c_v=cv, positions=pos, ctx_len=ctx)


EVICT_CASES = [
    (O.Cfg(4, 2, 64, 16, 24), 4, 256, [700, 150]),          # the pages' 260-token budget
    (O.Cfg(4, 2, 128, 96, 160), 4, 60, [400, 64, 65]),      # at and just past the budget
    (O.Cfg(2, 4, 64, 32, 48, O.MODE_2D), 0, 100, [300, 99]),  # LLA-2D, no sink
    (O.Cfg(4, 2, 64, 16, 32), 6, 1, [50, 7, 3]),            # one-token window, history < sink
]


@pytest.mark.gpu
@pytest.mark.parametrize("spec", EVICT_CASES, ids=lambda s: f"m{s[0].mode}d{s[0].d}s{s[1]}w{s[2]}")
def test_decode_over_evicted_cache_matches_oracle(spec):
    from gpu_util import DeviceCase
    cfg, sink, window, n_hist = spec
    n_hist = np.asarray(n_hist)
    case = decode_case(cfg, len(n_hist), int(n_hist.max()), seed=300 + window, ctx_len=n_hist)
    dev = DeviceCase(_evicted_cache(case, sink, window, n_hist),
                     rope_max_pos=int(n_hist.max()) + 1)
    for t in range(cfg.T):
        got = dev.decode(t)
        want = _expected_evicted(case, t, sink, window, n_hist)
        assert np.isfinite(got).all()
        assert rel_err(got, want).max() <= ATTN_TOL, t
    assert lla.decode_status(dev.ws) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [O.MODE_PER_HEAD, O.MODE_2D])
def test_append_under_eviction_matches_oracle(mode):
    """Decode-time appends: lla_evict_append picks each new token's slot, lla_encode
    writes its latents there, and the decode sees exactly the kept set."""
    import torch
    from gpu_util import DeviceCase, bf16_tensor, i32_tensor, lib_cfg
    cfg = O.Cfg(4, 2, 64, 16, 24) if mode == O.MODE_PER_HEAD else O.Cfg(2, 4, 64, 32, 48, mode)
    sink, window, steps = 3, 40, 50
    n0 = np.array([120, 20])                  # the second sequence crosses the budget mid-way
    B, n_tot = len(n0), int(n0.max()) + steps
    g = synth.rng(31)
    shared = mode == O.MODE_2D
    mk = synth.trajectory_model(g, cfg.T, cfg.H, cfg.d, 3, shared=shared)
    mv = synth.trajectory_model(g, cfg.T, cfg.H, cfg.d, 3, shared=shared)
    case = decode_case(cfg, B, n_tot, seed=41, ctx_len=n0 + steps)
    # history rows n0[b] .. n0[b] + steps - 1 are re-drawn as trajectories and encoded
    # on the GPU; the oracle's latents for them come from the oracle's encode of the same x
    xk = O.bf16_round(synth.sample_trajectories(g, mk, B * steps)).reshape(B, steps, cfg.T, cfg.H, cfg.d)
    xv = O.bf16_round(synth.sample_trajectories(g, mv, B * steps)).reshape(B, steps, cfg.T, cfg.H, cfg.d)
    ck_new, cv_new = O.encode_tokens(cfg, case.codec, xk.reshape(-1, cfg.T, cfg.H, cfg.d),
                                     xv.reshape(-1, cfg.T, cfg.H, cfg.d))
    ck_new = O.bf16_round(ck_new).reshape(B, steps, *ck_new.shape[1:])
    cv_new = O.bf16_round(cv_new).reshape(B, steps, *cv_new.shape[1:])
    for b in range(B):
        case.c_k[b, n0[b]:n0[b] + steps] = ck_new[b]
        case.c_v[b, n0[b]:n0[b] + steps] = cv_new[b]
        case.positions[b, :] = np.arange(n_tot)
    case.q_pos[:] = n0 + steps
    dev = DeviceCase(_evicted_cache(case, sink, window, n0), rope_max_pos=n_tot + 1)
    budget = sink + window
    for i in range(steps):
        pos = i32_tensor(n0 + i)
        slot = lla.evict_append(B, budget, sink, window, pos, dev.positions, dev.ctx_len)
        lla.encode(lib_cfg(cfg), dev.packed, bf16_tensor(xk[:, i]), bf16_tensor(xv[:, i]), slot,
                   dev.c_k, dev.c_v)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(dev.ctx_len.cpu().numpy(), np.minimum(n0 + steps, budget))
    for t in range(cfg.T):
        got = dev.decode(t)
        want = _expected_evicted(case, t, sink, window, n0 + steps)
        assert rel_err(got, want).max() <= ATTN_TOL, t

"""Seeded test cases: synthetic inputs plus the oracle's expected values.

Inputs come from ``synth`` (random draws) and, for small cases, the oracle's
encode (so the latents are realistic); expected values come only from
``oracle``.  Both sides receive identical bf16 latents and fp32 weights.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

import oracle as O
import synth


def f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


@dataclass
class DecodeCase:
    cfg: O.Cfg
    codec: O.Codec               # fp64 copies of fp32 weights
    B: int
    n_cap: int
    ctx_len: np.ndarray          # [B] int
    positions: np.ndarray        # [B, n_cap] int
    q_pos: np.ndarray            # [B] int
    q: np.ndarray                # [B, H, d] fp32 values
    k_self: dict = field(default_factory=dict)   # t -> [B, H, d]
    v_self: dict = field(default_factory=dict)
    c_k: np.ndarray = None       # bf16-valued float64, library layout
    c_v: np.ndarray = None


def random_codec(g, cfg: O.Cfg) -> O.Codec:
    """Independent random W_down, W_up and mu (no SVD structure)."""
    W = cfg.width
    L = cfg.H if cfg.mode == O.MODE_PER_HEAD else None
    lead = (cfg.H,) if L else ()
    up = (cfg.H, cfg.T) if L else (cfg.T, cfg.H)
    sc = 1.0 / np.sqrt(max(cfg.r_k, 1))
    return O.Codec(f32(g.standard_normal((*lead, W, cfg.r_k)) / np.sqrt(W)),
                   f32(g.standard_normal((*lead, W, cfg.r_v)) / np.sqrt(W)),
                   f32(g.standard_normal((*up, cfg.d, cfg.r_k)) * sc),
                   f32(g.standard_normal((*up, cfg.d, cfg.r_v)) / np.sqrt(cfg.r_v)),
                   f32(0.1 * g.standard_normal((*lead, W))),
                   f32(0.1 * g.standard_normal((*lead, W))))


def f32_codec(c: O.Codec) -> O.Codec:
    return O.Codec(*(f32(a) for a in (c.W_down_k, c.W_down_v, c.W_up_k, c.W_up_v, c.mu_k, c.mu_v)))


def decode_case(cfg: O.Cfg, B: int, n_cap: int, seed: int, ctx_len=None, codec="svd", R=3,
                q_scale=1.0, positions="arange", gamma=None) -> DecodeCase:
    g = synth.rng(seed)
    shared = cfg.mode == O.MODE_2D
    mk = synth.trajectory_model(g, cfg.T, cfg.H, cfg.d, R, shared=shared, gamma=gamma)
    mv = synth.trajectory_model(g, cfg.T, cfg.H, cfg.d, R, shared=shared, gamma=gamma)
    if codec == "svd":
        cal = max(256, min(1024, 4 * cfg.width))
        cd = f32_codec(O.svd_codec(cfg, synth.sample_trajectories(g, mk, cal),
                                   synth.sample_trajectories(g, mv, cal)))
    else:
        cd = random_codec(g, cfg)
    ctx = np.full(B, n_cap, dtype=np.int64) if ctx_len is None else np.asarray(ctx_len, np.int64)
    xk = synth.sample_trajectories(g, mk, B * n_cap)
    xv = synth.sample_trajectories(g, mv, B * n_cap)
    ck, cv = O.encode_tokens(cfg, cd, xk, xv)
    ck = O.bf16_round(ck).reshape(B, n_cap, *ck.shape[1:])
    cv = O.bf16_round(cv).reshape(B, n_cap, *cv.shape[1:])
    if positions == "arange":
        pos = np.tile(np.arange(n_cap), (B, 1))
        qpos = ctx.copy()
    else:
        pos = np.stack([g.permutation(4 * n_cap + 8)[:n_cap] for _ in range(B)])
        qpos = g.integers(0, 4 * n_cap + 8, size=B)
    case = DecodeCase(cfg, cd, B, n_cap, ctx, pos, qpos,
                      f32(q_scale * synth.queries(g, B, cfg.H, cfg.d)), c_k=ck, c_v=cv)
    new_k = synth.sample_trajectories(g, mk, B)   # [B, T, H, d]
    new_v = synth.sample_trajectories(g, mv, B)
    for t in range(cfg.T):
        case.k_self[t] = f32(new_k[:, t])
        case.v_self[t] = f32(new_v[:, t])
    return case


def expected(case: DecodeCase, t: int, pairs=None) -> np.ndarray:
    return O.decode_attn_cache(case.cfg, case.codec, t, case.q, case.k_self[t], case.v_self[t],
                               case.c_k, case.c_v, case.positions, case.q_pos, case.ctx_len,
                               pairs=pairs)


def rel_err(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    """Per (b, h): max |got - want| / max |want| over the d entries."""
    return np.abs(got - want).max(-1) / np.abs(want).max(-1)


ATTN_TOL = 2e-3     # max relative error of attention outputs per (b, h)
LATENT_TOL = 1e-2   # max |c_gpu - c_ref| relative to ||c_ref||_2 per latent

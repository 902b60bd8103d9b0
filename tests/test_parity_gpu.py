"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerances (written here, from the contract): attention outputs within 2e-3 max
relative error per (b, h); encoded latents within 1e-2 of the latent's L2 norm
(against the unrounded fp64 value); RoPE table within 1e-7 absolute; status
bits and bookkeeping exact.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
import synth
from cases import ATTN_TOL, LATENT_TOL, decode_case, expected, f32, rel_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import looped_transformer_decode_b200 as lla
    from gpu_util import DeviceCase, bf16_tensor, i32_tensor, lib_cfg, pack


# ----------------------------------------------------------------------------- RoPE table

@pytest.mark.parametrize("d", [32, 96, 128])
def test_rope_table_matches_fp64_angles(d):
    cfg = lla.Cfg(1, 1, d, 8, 8, rope_base=10000.0)
    max_pos = 40000
    tab = lla.rope_table(cfg, max_pos).cpu().numpy().astype(np.float64)
    ang = np.arange(max_pos)[:, None] * O.rope_inv_freq(d, 10000.0)[None]
    np.testing.assert_allclose(tab[..., 0], np.cos(ang), atol=1e-7, rtol=0)
    np.testing.assert_allclose(tab[..., 1], np.sin(ang), atol=1e-7, rtol=0)


# ----------------------------------------------------------------------------- encode

ENCODE_CFGS = [
    O.Cfg(4, 2, 64, 8, 16),                       # tiny per-head workload
    O.Cfg(4, 16, 128, 96, 160),                   # per-head 4x
    O.Cfg(4, 16, 128, 16, 32),                    # per-head 21.3x
    O.Cfg(32, 2, 96, 64, 128),                    # deep loop, two heads
    O.Cfg(2, 4, 64, 32, 48, O.MODE_2D),           # LLA-2D small
    O.Cfg(4, 16, 128, 64, 128, O.MODE_2D),        # LLA-2D workload width
    O.Cfg(3, 1, 96, 24, 40, O.MODE_2D),           # width 288: 32-wide K chunks, r not a multiple of 16
    O.Cfg(8, 3, 32, 256, 8),                      # largest latent, smallest head
]
# tensor_core picks 128- or 256-token CTAs by size; tensor_core_m256 forces 256.
ENCODE_PATHS = ["tensor_core", "tensor_core_m256", "cuda_core"]


@pytest.mark.parametrize("path", ENCODE_PATHS)
@pytest.mark.parametrize("n_tok", [37, 300])
@pytest.mark.parametrize("cfg", ENCODE_CFGS, ids=lambda c: f"T{c.T}H{c.H}d{c.d}r{c.r_k}_{c.r_v}m{c.mode}")
def test_encode_matches_oracle(cfg, n_tok, path, monkeypatch):
    """Both encode kernels against the oracle: one ragged 128-token tile, and three tiles
    (two 256-token CTAs, the second one partly past the end, when forced)."""
    monkeypatch.delenv("LLA_ENCODE_PATH", raising=False)
    monkeypatch.delenv("LLA_ENC_MSUB", raising=False)
    if path == "cuda_core":
        monkeypatch.setenv("LLA_ENCODE_PATH", "cuda_core")
    elif path == "tensor_core_m256":
        monkeypatch.setenv("LLA_ENC_MSUB", "2")
    case = decode_case(cfg, 1, 4, seed=50 + cfg.r_k, R=3)
    g = synth.rng(77)
    shared = cfg.mode == O.MODE_2D
    mk = synth.trajectory_model(g, cfg.T, cfg.H, cfg.d, 3, shared=shared)
    n_slots = n_tok + 13
    xk = O.bf16_round(synth.sample_trajectories(g, mk, n_tok))
    xv = O.bf16_round(synth.sample_trajectories(g, mk, n_tok))
    slot = g.permutation(n_slots)[:n_tok]
    packed = pack(case)
    L = cfg.H if cfg.mode == O.MODE_PER_HEAD else 1
    lead = (n_slots, cfg.H) if cfg.mode == O.MODE_PER_HEAD else (n_slots,)
    ck = torch.zeros((*lead, cfg.r_k), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros((*lead, cfg.r_v), dtype=torch.bfloat16, device="cuda")
    lla.encode(lib_cfg(cfg), packed, bf16_tensor(xk), bf16_tensor(xv),
               torch.from_numpy(slot.astype(np.int64)).cuda(), ck, cv)
    torch.cuda.synchronize()
    want_k, want_v = O.encode_tokens(cfg, case.codec, xk, xv)
    got_k = ck.float().cpu().numpy().astype(np.float64)[slot]
    got_v = cv.float().cpu().numpy().astype(np.float64)[slot]
    for got, want in ((got_k, want_k), (got_v, want_v)):
        got = got.reshape(n_tok, L, -1)
        want = want.reshape(n_tok, L, -1)
        err = np.abs(got - want).max(-1) / np.linalg.norm(want, axis=-1)
        assert err.max() <= LATENT_TOL, err.max()
    # rows that received no token stay untouched
    untouched = np.setdiff1d(np.arange(n_slots), slot)
    assert np.all(ck.float().cpu().numpy()[untouched] == 0)


def test_encode_deep_loop_full_width_sampled():
    """The deep-loop codec at its full width (T = 32, H = 8, d = 96: 3072 entries per
    head's latent) on the tensor-core encode, 4096 tokens in scattered slots, sampled
    rows of every head against the oracle."""
    w = synth.WORKLOADS["deeploop_32x_T32_H8_d96_r64_128_B16_n32768"]
    cfg = O.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode)
    cod = synth.workload_codec(w)
    codec = O.Codec(*(cod[k].astype(np.float64) for k in
                      ("W_down_k", "W_down_v", "W_up_k", "W_up_v", "mu_k", "mu_v")))
    packed = lla.codec_pack(lib_cfg(cfg), *(torch.from_numpy(cod[k]).cuda() for k in
                                            ("W_down_k", "W_down_v", "W_up_k", "W_up_v",
                                             "mu_k", "mu_v")))
    n_tok, n_slots = 4096, 5000
    g = synth.rng(4242)
    model = synth.trajectory_model(g, w.T, w.H, w.d, w.R, gamma=w.gamma)
    xk = O.bf16_round(synth.sample_trajectories(g, model, n_tok))
    xv = O.bf16_round(synth.sample_trajectories(g, model, n_tok))
    slot = g.permutation(n_slots)[:n_tok]
    ck = torch.zeros((n_slots, w.H, w.r_k), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros((n_slots, w.H, w.r_v), dtype=torch.bfloat16, device="cuda")
    lla.encode(lib_cfg(cfg), packed, bf16_tensor(xk), bf16_tensor(xv),
               torch.from_numpy(slot.astype(np.int64)).cuda(), ck, cv)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 127, 128, n_tok - 1], g.integers(0, n_tok, 60)]))
    want_k, want_v = O.encode_tokens(cfg, codec, xk[rows], xv[rows])
    got_k = ck.double().cpu().numpy()[slot[rows]]
    got_v = cv.double().cpu().numpy()[slot[rows]]
    for got, want in ((got_k, want_k), (got_v, want_v)):
        err = np.abs(got - want).max(-1) / np.linalg.norm(want, axis=-1)
        assert err.max() <= LATENT_TOL, err.max()


def test_encode_out_of_range_slot_sets_status_and_skips():
    cfg = O.Cfg(4, 2, 64, 8, 16)
    case = decode_case(cfg, 1, 4, seed=3)
    packed = pack(case)
    x = bf16_tensor(O.bf16_round(0.3 * synth.rng(1).standard_normal((3, 4, 2, 64))))
    ck = torch.zeros((5, 2, 8), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros((5, 2, 16), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    slot = torch.tensor([0, 5, -1], dtype=torch.int64, device="cuda")
    lla.encode(lib_cfg(cfg), packed, x, x, slot, ck, cv, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == lla.STATUS_SLOT_RANGE
    assert ck[0].abs().sum() > 0 and ck[1:].abs().sum() == 0


# ----------------------------------------------------------------------------- decode, small

SMALL = [
    # (cfg, B, n_cap, ctx_len, kwargs)
    (O.Cfg(4, 2, 64, 8, 16), 1, 128, None, {}),                                  # tiny workload
    (O.Cfg(4, 3, 64, 16, 24), 3, 300, [300, 129, 1], {}),                        # ragged tails
    (O.Cfg(4, 2, 128, 96, 160), 2, 520, [520, 385], {}),
    (O.Cfg(4, 2, 96, 64, 128), 2, 700, [700, 256], {"R": 8, "gamma": 0.85}),
    (O.Cfg(3, 2, 32, 8, 8), 2, 130, [130, 0], {}),                               # empty history
    (O.Cfg(4, 2, 64, 16, 32), 1, 2000, None, {}),                                # many splits
    (O.Cfg(4, 2, 64, 24, 40), 2, 200, None, {"codec": "random"}),                # no SVD structure
    (O.Cfg(4, 2, 64, 16, 32), 2, 200, None, {"q_scale": 25.0}),                  # sharp softmax
    (O.Cfg(4, 2, 64, 16, 32), 2, 260, None, {"positions": "random"}),            # arbitrary positions
    (O.Cfg(2, 4, 64, 32, 48, O.MODE_2D), 2, 200, [200, 77], {}),                 # LLA-2D
    (O.Cfg(4, 4, 128, 64, 128, O.MODE_2D), 1, 300, None, {"q_scale": 10.0}),
    # LLA-2D head groups of 2 (H = 6) and 1 (H = 3), r_v above 128 (two row blocks of
    # the transposed V sum), small d, ragged and empty contexts, arbitrary positions
    (O.Cfg(4, 6, 96, 48, 160, O.MODE_2D), 2, 260, [260, 131], {}),
    (O.Cfg(2, 3, 32, 16, 24, O.MODE_2D), 3, 140, [140, 1, 0], {}),
    (O.Cfg(4, 8, 64, 32, 64, O.MODE_2D), 2, 390, None, {"positions": "random", "q_scale": 20.0}),
    # phase-operand kernel (per head, r_k 16 or 32, r_v 32: four heads per item):
    # the 21.3x shape, two head groups with random positions and a sharp softmax,
    # ragged and empty contexts, r_k 32, d 64 with a random codec, one sequence long
    # enough for several context splits (combine pass); the r_v 64 case runs on the
    # per-head kernel
    (O.Cfg(4, 4, 128, 16, 32), 2, 600, [600, 257], {}),
    (O.Cfg(4, 8, 128, 16, 32), 2, 300, None, {"positions": "random", "q_scale": 20.0}),
    (O.Cfg(4, 4, 64, 32, 64), 3, 300, [300, 129, 1], {}),
    (O.Cfg(4, 4, 128, 32, 32), 2, 400, [400, 0], {"q_scale": 25.0}),
    (O.Cfg(4, 4, 64, 16, 32), 2, 260, None, {"codec": "random"}),
    (O.Cfg(4, 4, 128, 16, 32), 1, 2000, None, {}),
]


@pytest.mark.parametrize("spec", SMALL, ids=lambda s: f"T{s[0].T}H{s[0].H}d{s[0].d}r{s[0].r_k}_{s[0].r_v}m{s[0].mode}B{s[1]}n{s[2]}")
def test_decode_matches_oracle_small(spec):
    cfg, B, n_cap, ctx, kw = spec
    case = decode_case(cfg, B, n_cap, seed=100 + n_cap, ctx_len=ctx, **kw)
    dev = DeviceCase(case)
    for t in range(cfg.T):
        got = dev.decode(t)
        want = expected(case, t)
        err = rel_err(got, want)
        assert np.isfinite(got).all()
        assert err.max() <= ATTN_TOL, (t, err.max())
    assert lla.decode_status(dev.ws) == 0


# The CUDA-core decode kernel: the path for shapes the tensor-core plan refuses (here
# d 128 with r_k = r_v = 256, whose K and V rings do not fit in shared memory), and
# the LLA_DECODE_PATH=cuda_core variant of every small case.
CUDA_CORE_ONLY = [
    (O.Cfg(4, 2, 128, 256, 256), 2, 300, [300, 131], {}),
    (O.Cfg(2, 2, 128, 256, 256, O.MODE_2D), 1, 200, None, {"q_scale": 10.0}),
]


def test_tensor_core_plan_refuses_the_cuda_core_shapes():
    for cfg, B, n_cap, _, _ in CUDA_CORE_ONLY:
        # partial kernel + combine: the CUDA-core plan
        assert lla.decode_launches(lib_cfg(cfg), B, n_cap) == 2
        ws = lla.lib.lla_decode_workspace_bytes(ctypes.byref(lib_cfg(cfg).c()), B, n_cap)
        assert ws > 0


@pytest.mark.parametrize("spec", SMALL + CUDA_CORE_ONLY,
                         ids=lambda s: f"T{s[0].T}H{s[0].H}d{s[0].d}r{s[0].r_k}_{s[0].r_v}m{s[0].mode}B{s[1]}n{s[2]}")
def test_cuda_core_decode_matches_oracle(spec, monkeypatch):
    monkeypatch.setenv("LLA_DECODE_PATH", "cuda_core")
    cfg, B, n_cap, ctx, kw = spec
    case = decode_case(cfg, B, n_cap, seed=300 + n_cap, ctx_len=ctx, **kw)
    dev = DeviceCase(case)
    for t in (0, cfg.T - 1):
        got = dev.decode(t)
        err = rel_err(got, expected(case, t))
        assert np.isfinite(got).all()
        assert err.max() <= ATTN_TOL, (t, err.max())
    assert lla.decode_status(dev.ws) == 0


@pytest.mark.parametrize("spec", [s for s in SMALL if s[0].mode == O.MODE_PER_HEAD
                                  and s[0].r_k in (16, 32) and s[0].r_v == 32
                                  and s[0].H % 4 == 0 and s[0].d in (64, 128)],
                         ids=lambda s: f"T{s[0].T}H{s[0].H}d{s[0].d}r{s[0].r_k}_{s[0].r_v}B{s[1]}n{s[2]}")
def test_per_head_kernel_on_phase_operand_shapes(spec, monkeypatch):
    """LLA_TC_FORM=u runs the shapes of the phase-operand kernel on the per-head
    tensor-core kernel instead: both against the oracle."""
    monkeypatch.setenv("LLA_TC_FORM", "u")
    cfg, B, n_cap, ctx, kw = spec
    case = decode_case(cfg, B, n_cap, seed=100 + n_cap, ctx_len=ctx, **kw)
    dev = DeviceCase(case)
    for t in (0, cfg.T - 1):
        err = rel_err(dev.decode(t), expected(case, t))
        assert err.max() <= ATTN_TOL, (t, err.max())
    assert lla.decode_status(dev.ws) == 0


def _phase_table_case(cfg, seed):
    """One call whose sequences take phase tiles from the table, computed, or both:
    consecutive positions from 0; offset by 100 (every tile inside the table's
    tile-rounded cache length plus one tile, 768 rows); offset by 200 (the last tile
    runs past those rows); a gap of 5 inside tile 2 (that tile computed, the next
    ones consecutive again); arbitrary positions; a ragged and an empty context."""
    B, n_cap = 7, 600
    case = decode_case(cfg, B, n_cap, seed=seed, ctx_len=[600, 600, 600, 600, 600, 130, 0])
    pos = np.tile(np.arange(n_cap), (B, 1))
    pos[1] += 100
    pos[2] += 200
    pos[3, 300:] += 5
    pos[4] = synth.rng(seed + 1).permutation(4 * n_cap)[:n_cap]
    case.positions = pos
    case.q_pos = np.array([600, 700, 800, 605, 2400, 130, 0])
    return case


@pytest.mark.parametrize("cfg", [O.Cfg(4, 4, 128, 16, 32), O.Cfg(4, 8, 64, 32, 32)],
                         ids=lambda c: f"H{c.H}d{c.d}r{c.r_k}")
def test_phase_table_and_computed_tiles_match_oracle(cfg, monkeypatch):
    """The phase-operand kernel copies a tile's phase rows from the phase table when
    the tile's positions are consecutive inside it and computes them otherwise
    (LLA_TCF_TABLE=0: always); both against the oracle on the same call."""
    case = _phase_table_case(cfg, seed=900 + cfg.d)
    dev = DeviceCase(case)
    for mode in ("1", "0"):
        monkeypatch.setenv("LLA_TCF_TABLE", mode)
        for t in (0, cfg.T - 1):
            got = dev.decode(t)
            assert np.isfinite(got).all(), (mode, t)
            err = rel_err(got, expected(case, t))
            assert err.max() <= ATTN_TOL, (mode, t, err.max())
        assert lla.decode_status(dev.ws) == 0


NAN_TAIL = [
    (O.Cfg(4, 2, 128, 96, 160), 2, 300, [300, 190], "tensor_core"),     # per-head kernel
    (O.Cfg(4, 4, 128, 16, 32), 2, 300, [300, 190], "tensor_core"),      # phase-operand kernel
    (O.Cfg(2, 4, 64, 32, 48, O.MODE_2D), 2, 300, [300, 150], "tensor_core"),   # LLA-2D kernel
    (O.Cfg(4, 2, 64, 16, 32), 1, 2000, [1500], "tensor_core"),          # several splits
    (O.Cfg(4, 2, 128, 96, 160), 2, 300, [300, 190], "cuda_core"),
]


@pytest.mark.parametrize("spec", NAN_TAIL, ids=lambda s: f"T{s[0].T}H{s[0].H}d{s[0].d}r{s[0].r_k}_{s[0].r_v}m{s[0].mode}n{s[2]}_{s[4]}")
def test_cache_rows_past_the_context_are_never_used(spec, monkeypatch):
    """Cache rows at or past ctx_len[b] may hold anything (here NaN): the output is
    the oracle's over the first ctx_len rows.  The tensor-core kernels stream whole
    128-token tiles, so they zero those rows of the staged V tile before the V MMA
    (zero weights times NaN would be NaN), and mask their scores."""
    cfg, B, n_cap, ctx, path = spec
    if path == "cuda_core":
        monkeypatch.setenv("LLA_DECODE_PATH", "cuda_core")
    case = decode_case(cfg, B, n_cap, seed=700 + n_cap, ctx_len=ctx)
    dev = DeviceCase(case)
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16, device="cuda")
    for b, n in enumerate(case.ctx_len):
        dev.c_k[b, int(n):] = nan
        dev.c_v[b, int(n):] = nan
    for t in (0, cfg.T - 1):
        got = dev.decode(t)
        assert np.isfinite(got).all(), t
        err = rel_err(got, expected(case, t))
        assert err.max() <= ATTN_TOL, (t, err.max())
    assert lla.decode_status(dev.ws) == 0


def test_decode_status_bits_for_bad_device_inputs():
    cfg = O.Cfg(4, 2, 64, 16, 32)
    case = decode_case(cfg, 2, 200, seed=9)
    dev = DeviceCase(case, rope_max_pos=201)
    dev.decode(0)
    assert lla.decode_status(dev.ws) == 0
    bad = case.positions.copy()
    bad[0, 10] = 5000                         # outside the RoPE table
    dev.positions = i32_tensor(bad)
    out = dev.decode(0)
    assert np.isfinite(out).all()
    assert lla.decode_status(dev.ws) & lla.STATUS_POSITION_RANGE
    dev.positions = i32_tensor(case.positions)
    dev.ctx_len = i32_tensor([250, 200])      # above n_cap: clamped
    out = dev.decode(0)
    assert np.isfinite(out).all()
    assert lla.decode_status(dev.ws) == lla.STATUS_CTX_RANGE
    dev.ctx_len = i32_tensor(case.ctx_len)
    dev.decode(0)
    assert lla.decode_status(dev.ws) == 0


def test_decode_is_deterministic():
    cfg = O.Cfg(4, 2, 128, 96, 160)
    case = decode_case(cfg, 2, 700, seed=12)
    dev = DeviceCase(case)
    a, b = dev.decode(2), dev.decode(2)
    np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------------------- decode, full size

def _sample_pairs(B, H, k, seed):
    g = synth.rng(seed)
    pairs = {(B - 1, H - 1), (0, 0)}
    while len(pairs) < min(k, B * H):
        pairs.add((int(g.integers(B)), int(g.integers(H))))
    return sorted(pairs)


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER[1:])
def test_decode_full_size_sampled(name):
    """Full-size workloads in the bench's launch configuration, sampled (b, h) pairs."""
    w = synth.WORKLOADS[name]
    cfg = O.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode)
    lc = lib_cfg(cfg)
    codec_np = synth.workload_codec(w)
    codec = O.Codec(*(codec_np[k].astype(np.float64) for k in
                      ("W_down_k", "W_down_v", "W_up_k", "W_up_v", "mu_k", "mu_v")))
    packed = lla.codec_pack(lc, *(torch.from_numpy(codec_np[k]).cuda() for k in
                                  ("W_down_k", "W_down_v", "W_up_k", "W_up_v", "mu_k", "mu_v")))
    x = synth.workload_tensors(w, "cuda")
    rope = lla.rope_table(lc, w.n + 1)
    ws = lla.decode_workspace(lc, w.B, w.n)
    pairs = _sample_pairs(w.B, w.H, 48, w.seed)
    bs = sorted({b for b, _ in pairs})
    ck = x["c_k"][bs].float().cpu().numpy().astype(np.float64)
    cv = x["c_v"][bs].float().cpu().numpy().astype(np.float64)
    remap = {b: i for i, b in enumerate(bs)}
    for t in w.loops:
        out = lla.decode_attn(lc, packed, rope, t, x["ctx_len"], x["q"], x["k_self"], x["v_self"],
                              x["positions"], x["q_pos"], x["c_k"], x["c_v"], ws=ws)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        sub = [(remap[b], h) for b, h in pairs]
        sel = lambda a: a[bs]  # noqa: E731
        want = O.decode_attn_cache(cfg, codec, t, sel(x["q"].double().cpu().numpy()),
                                   sel(x["k_self"].double().cpu().numpy()),
                                   sel(x["v_self"].double().cpu().numpy()), ck, cv,
                                   sel(x["positions"].cpu().numpy()), sel(x["q_pos"].cpu().numpy()),
                                   sel(x["ctx_len"].cpu().numpy()), pairs=sub)
        for (b, h), (i, _) in zip(pairs, sub):
            e = np.abs(got[b, h] - want[i, h]).max() / np.abs(want[i, h]).max()
            assert e <= ATTN_TOL, (name, t, b, h, e)
    assert lla.decode_status(ws) == 0

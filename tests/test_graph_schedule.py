"""Decode-step schedule captured as a CUDA graph (the fused multi-layer schedule of
the decode step: every layer's decode attention at each loop, then the encode of
the finished tokens, replayed as one graph).

The library's calls enqueue work only on the caller's stream and never allocate
or synchronise, so a whole step can be captured once and replayed; replays with
new inputs written in place must equal eager calls.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from cases import decode_case


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [O.MODE_PER_HEAD, O.MODE_2D])
def test_captured_step_replays_equal_eager_calls(mode):
    import torch

    import looped_transformer_decode_b200 as lla
    from gpu_util import DeviceCase, bf16_tensor, f32_tensor
    cfg = O.Cfg(4, 2, 64, 16, 24) if mode == O.MODE_PER_HEAD else O.Cfg(2, 4, 64, 32, 48, mode)
    layers = []
    for layer in range(3):
        case = decode_case(cfg, 2, 300, seed=1000 + layer, ctx_len=[300, 170], codec="random")
        layers.append(DeviceCase(case, rope_max_pos=302))
    dev0 = layers[0]
    g = np.random.default_rng(5)
    B, H, d, T = 2, cfg.H, cfg.d, cfg.T
    q = [f32_tensor(g.standard_normal((B, H, d))) for _ in layers]
    ks = [f32_tensor(g.standard_normal((B, H, d))) for _ in layers]
    vs = [f32_tensor(g.standard_normal((B, H, d))) for _ in layers]
    outs = [[torch.empty((B, H, d), device="cuda") for _ in range(T)] for _ in layers]
    xk = bf16_tensor(O.bf16_round(g.standard_normal((B, T, H, d))))
    xv = bf16_tensor(O.bf16_round(g.standard_normal((B, T, H, d))))
    slot = torch.tensor([299, 300 + 169], dtype=torch.int64, device="cuda")

    def step():
        for t in range(T):
            for L, dev in enumerate(layers):
                lla.decode_attn(dev.cfg, dev.packed, dev0.rope, t, dev.ctx_len, q[L], ks[L], vs[L],
                                dev.positions, dev.q_pos, dev.c_k, dev.c_v, out=outs[L][t],
                                ws=dev.ws)
        for dev in layers:
            lla.encode(dev.cfg, dev.packed, xk, xv, slot, dev.c_k, dev.c_v)

    step()                                     # warm-up (kernel attributes, maps)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for rep in range(2):
        for L in range(len(layers)):           # new inputs, written in place
            q[L].copy_(f32_tensor(g.standard_normal((B, H, d))))
        graph.replay()
        torch.cuda.synchronize()
        got = [[o.clone() for o in outs[L]] for L in range(len(layers))]
        step()
        torch.cuda.synchronize()
        for L in range(len(layers)):
            for t in range(T):
                np.testing.assert_array_equal(got[L][t].cpu().numpy(), outs[L][t].cpu().numpy())
    for dev in layers:
        assert lla.decode_status(dev.ws) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [O.MODE_PER_HEAD, O.MODE_2D])
def test_captured_multilayer_steps_match_oracle(mode):
    """The decode-step schedule against the oracle: one captured graph holds every
    layer's decode at every loop and then the encode of the token that has just
    finished its loops (close reading §二.6, the inference flow: the in-flight token is
    attended exactly at each loop and written to the latent cache after its last).
    Two steps are replayed with new inputs written in place; each layer's output at
    each loop is compared with the oracle, and the second step attends over the
    rows the first step's encode appended (the oracle over its own encode of that
    token)."""
    import torch

    import looped_transformer_decode_b200 as lla
    from cases import ATTN_TOL, LATENT_TOL, expected, f32, rel_err
    from gpu_util import DeviceCase, bf16_tensor, f32_tensor, i32_tensor
    cfg = O.Cfg(4, 4, 128, 16, 32) if mode == O.MODE_PER_HEAD else O.Cfg(2, 4, 64, 32, 48, mode)
    B, n_cap, T, H, d = 2, 260, cfg.T, cfg.H, cfg.d
    ctx0 = np.array([250, 121])
    cases, devs = [], []
    for layer in range(3):
        case = decode_case(cfg, B, n_cap, seed=2000 + layer, ctx_len=ctx0.copy())
        cases.append(case)
        devs.append(DeviceCase(case, rope_max_pos=n_cap + 2))
    g = np.random.default_rng(11)
    shape = (B, H, d)
    # per (layer, loop) device inputs and outputs, written in place between replays
    q = [[f32_tensor(np.zeros(shape)) for _ in range(T)] for _ in devs]
    ks = [[f32_tensor(np.zeros(shape)) for _ in range(T)] for _ in devs]
    vs = [[f32_tensor(np.zeros(shape)) for _ in range(T)] for _ in devs]
    outs = [[torch.empty(shape, device="cuda") for _ in range(T)] for _ in devs]
    xk = [bf16_tensor(np.zeros((B, T, H, d))) for _ in devs]
    xv = [bf16_tensor(np.zeros((B, T, H, d))) for _ in devs]
    slot = torch.zeros(B, dtype=torch.int64, device="cuda")
    ctx = i32_tensor(ctx0)
    qpos = i32_tensor(ctx0)

    def step():
        for t in range(T):
            for L, dev in enumerate(devs):
                lla.decode_attn(dev.cfg, dev.packed, devs[0].rope, t, ctx, q[L][t], ks[L][t],
                                vs[L][t], dev.positions, qpos, dev.c_k, dev.c_v, out=outs[L][t],
                                ws=dev.ws)
        for L, dev in enumerate(devs):
            lla.encode(dev.cfg, dev.packed, xk[L], xv[L], slot, dev.c_k, dev.c_v)

    def new_inputs(n_hist):
        """In-flight token of this step (bf16-valued per-loop K/V, as the encode takes
        them) and queries; returns the host copies."""
        host = []
        for L in range(len(devs)):
            qq = [f32(g.standard_normal(shape) / np.sqrt(d)) for _ in range(T)]
            kk = O.bf16_round(0.3 * g.standard_normal((B, T, H, d)))
            vv = O.bf16_round(0.3 * g.standard_normal((B, T, H, d)))
            for t in range(T):
                q[L][t].copy_(f32_tensor(qq[t]))
                ks[L][t].copy_(f32_tensor(kk[:, t]))
                vs[L][t].copy_(f32_tensor(vv[:, t]))
            xk[L].copy_(bf16_tensor(kk))
            xv[L].copy_(bf16_tensor(vv))
            host.append((qq, kk, vv))
        slot.copy_(torch.from_numpy((np.arange(B) * n_cap + n_hist).astype(np.int64)))
        ctx.copy_(i32_tensor(n_hist))
        qpos.copy_(i32_tensor(n_hist))
        return host

    new_inputs(ctx0)
    step()                                     # warm-up (kernel attributes, tensor maps)
    torch.cuda.synchronize()
    for dev, case in zip(devs, cases):         # undo the warm-up's encode
        dev.c_k.copy_(bf16_tensor(case.c_k))
        dev.c_v.copy_(bf16_tensor(case.c_v))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    n_hist = ctx0.copy()
    for rep in range(2):
        host = new_inputs(n_hist)
        graph.replay()
        torch.cuda.synchronize()
        for L, (case, (qq, kk, vv)) in enumerate(zip(cases, host)):
            case.ctx_len = n_hist.copy()
            case.q_pos = n_hist.copy()
            for t in range(T):
                case.q = qq[t]
                case.k_self[t] = kk[:, t]
                case.v_self[t] = vv[:, t]
                err = rel_err(outs[L][t].double().cpu().numpy(), expected(case, t))
                assert err.max() <= ATTN_TOL, (rep, L, t, err.max())
            # the encode appended the finished token at row n_hist[b]: the oracle's own
            # encode of it goes into the oracle's cache, the GPU's is checked against it
            want_k, want_v = O.encode_tokens(cfg, case.codec, kk, vv)
            got_k = devs[L].c_k.double().cpu().numpy()[np.arange(B), n_hist]
            got_v = devs[L].c_v.double().cpu().numpy()[np.arange(B), n_hist]
            for got, want in ((got_k, want_k), (got_v, want_v)):
                got = got.reshape(B, -1, want.shape[-1])
                want = want.reshape(B, -1, want.shape[-1])
                err = np.abs(got - want).max(-1) / np.linalg.norm(want, axis=-1)
                assert err.max() <= LATENT_TOL, (rep, L, err.max())
            case.c_k[np.arange(B), n_hist] = O.bf16_round(want_k)
            case.c_v[np.arange(B), n_hist] = O.bf16_round(want_v)
        n_hist = n_hist + 1
    for dev in devs:
        assert lla.decode_status(dev.ws) == 0

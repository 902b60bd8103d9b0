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

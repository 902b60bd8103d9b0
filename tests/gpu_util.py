"""Move test cases to the device and run them through the library's C ABI."""
from __future__ import annotations

import numpy as np
import torch

import synth
import looped_transformer_decode_b200 as lla


def lib_cfg(cfg) -> lla.Cfg:
    return lla.Cfg(cfg.T, cfg.H, cfg.d, cfg.r_k, cfg.r_v, cfg.mode, cfg.rope_base)


def bf16_tensor(x64: np.ndarray) -> torch.Tensor:
    bits = synth.to_bf16_bits(x64)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def f32_tensor(x) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(x, np.float32))).cuda()


def i32_tensor(x) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(x, np.int32))).cuda()


def pack(case):
    c = case.codec
    return lla.codec_pack(lib_cfg(case.cfg), *(f32_tensor(a) for a in (
        c.W_down_k, c.W_down_v, c.W_up_k, c.W_up_v, c.mu_k, c.mu_v)))


class DeviceCase:
    def __init__(self, case, rope_max_pos=None):
        self.case = case
        self.cfg = lib_cfg(case.cfg)
        self.packed = pack(case)
        mp = rope_max_pos or int(max(case.positions.max(initial=0), case.q_pos.max())) + 1
        self.rope = lla.rope_table(self.cfg, mp)
        self.ctx_len = i32_tensor(case.ctx_len)
        self.q = f32_tensor(case.q)
        self.positions = i32_tensor(case.positions)
        self.q_pos = i32_tensor(case.q_pos)
        self.c_k = bf16_tensor(case.c_k)
        self.c_v = bf16_tensor(case.c_v)
        self.ws = lla.decode_workspace(self.cfg, case.B, case.n_cap)

    def decode(self, t: int) -> np.ndarray:
        out = lla.decode_attn(self.cfg, self.packed, self.rope, t, self.ctx_len, self.q,
                              f32_tensor(self.case.k_self[t]), f32_tensor(self.case.v_self[t]),
                              self.positions, self.q_pos, self.c_k, self.c_v, ws=self.ws)
        torch.cuda.synchronize()
        return out.double().cpu().numpy()

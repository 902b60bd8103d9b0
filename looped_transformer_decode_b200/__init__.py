"""Looped Latent Attention (LLA) decode on NVIDIA B200: thin torch binding of liblla.so.

Functions here only check tensor shapes/dtypes and pass pointers plus the current
CUDA stream to the C ABI in ``include/lla.h``; all computation runs in the
library's CUDA kernels.  Tensors must be contiguous CUDA tensors.
"""
from __future__ import annotations

import ctypes
from fractions import Fraction

import torch

from ._lib import (ERR_CUDA, ERR_INVALID, ERR_TOO_SMALL, ERR_UNSUPPORTED, LIB_PATH, MODE_2D,
                   MODE_PER_HEAD, OK, SIGNATURES, STATUS_CTX_RANGE, STATUS_POSITION_RANGE,
                   STATUS_SLOT_RANGE, Cfg, LLAError, check, last_error, lib)

__all__ = [
    "Cfg", "LLAError", "MODE_PER_HEAD", "MODE_2D", "ratio", "cache_bytes", "codec_pack",
    "rope_table", "encode", "decode_workspace", "decode_attn", "decode_status", "lib",
    "decode_launches", "STATUS_POSITION_RANGE", "STATUS_CTX_RANGE", "STATUS_SLOT_RANGE",
    "evict_slot", "evict_append", "full_kv_bytes", "full_cache_alloc", "full_rebuild",
    "full_decode_workspace", "full_decode_launches", "full_decode_attn",
]


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor, dtype: torch.dtype, name: str, shape=None) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def ratio(cfg: Cfg) -> Fraction:
    num, den = ctypes.c_int64(), ctypes.c_int64()
    check(lib.lla_ratio(ctypes.byref(cfg.c()), ctypes.byref(num), ctypes.byref(den)))
    return Fraction(num.value, den.value)


def cache_bytes(cfg: Cfg, tokens: int, layers: int, teacher: bool = False) -> int:
    out = ctypes.c_int64()
    check(lib.lla_cache_bytes(ctypes.byref(cfg.c()), tokens, layers, int(teacher),
                              ctypes.byref(out)))
    return out.value


def _wshapes(cfg: Cfg, r: int):
    T, H, d = cfg.T, cfg.H, cfg.d_head
    if cfg.mode == MODE_PER_HEAD:
        return (H, T * d, r), (H, T, d, r), (H, T * d)
    return (T * H * d, r), (T, H, d, r), (T * H * d,)


def codec_pack(cfg: Cfg, W_down_k, W_down_v, W_up_k, W_up_v, mu_k, mu_v, out=None):
    """Pack fp32 codec tensors (layouts in ``lla_codec_pack``) into a uint8 device buffer."""
    c = cfg.c()
    nbytes = lib.lla_codec_packed_bytes(ctypes.byref(c))
    if nbytes == 0:
        raise LLAError(ERR_UNSUPPORTED, last_error())
    dk, uk, mk = _wshapes(cfg, cfg.r_k)
    dv, uv, mv = _wshapes(cfg, cfg.r_v)
    args = [_ptr(W_down_k, torch.float32, "W_down_k", dk), _ptr(W_down_v, torch.float32, "W_down_v", dv),
            _ptr(W_up_k, torch.float32, "W_up_k", uk), _ptr(W_up_v, torch.float32, "W_up_v", uv),
            _ptr(mu_k, torch.float32, "mu_k", mk), _ptr(mu_v, torch.float32, "mu_v", mv)]
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=W_down_k.device)
    check(lib.lla_codec_pack(ctypes.byref(c), *args, _ptr(out, torch.uint8, "packed"),
                             out.numel(), _stream()))
    return out


def rope_table(cfg: Cfg, max_pos: int, device="cuda", out=None):
    c = cfg.c()
    if out is None:
        rd = cfg.d_rope or cfg.d_head                 # rotary dims
        out = torch.empty((max_pos, rd // 2, 2), dtype=torch.float32, device=device)
    check(lib.lla_rope_table(ctypes.byref(c), max_pos, _ptr(out, torch.float32, "table"),
                             out.numel() * 4, _stream()))
    return out


def _cache_shape(cfg: Cfg, rows_lead, r):
    return (*rows_lead, cfg.H, r) if cfg.mode == MODE_PER_HEAD else (*rows_lead, r)


def encode(cfg: Cfg, packed, x_k, x_v, slot, c_k, c_v, status=None):
    """Write latents of finished tokens into the caches (in place).

    x_[kv]: bf16 [n_tok, T, H, d]; slot: int64 [n_tok] row indices into the caches,
    which are bf16 with any leading shape whose rows flatten to n_slots.
    """
    c = cfg.c()
    n_tok = x_k.shape[0]
    xs = (n_tok, cfg.T, cfg.H, cfg.d_head)
    r_per_row_k = cfg.r_k * (cfg.H if cfg.mode == MODE_PER_HEAD else 1)
    n_slots = c_k.numel() // r_per_row_k
    if c_v.numel() // (cfg.r_v * (cfg.H if cfg.mode == MODE_PER_HEAD else 1)) != n_slots:
        raise ValueError("c_k and c_v hold different numbers of rows")
    st = _ptr(status, torch.int32, "status") if status is not None else None
    check(lib.lla_encode(ctypes.byref(c), _ptr(packed, torch.uint8, "packed"), n_tok,
                         _ptr(x_k, torch.bfloat16, "x_k", xs), _ptr(x_v, torch.bfloat16, "x_v", xs),
                         _ptr(slot, torch.int64, "slot", (n_tok,)), n_slots,
                         _ptr(c_k, torch.bfloat16, "c_k"), _ptr(c_v, torch.bfloat16, "c_v"), st,
                         _stream()))


def decode_workspace(cfg: Cfg, B: int, n_cap: int, device="cuda"):
    n = lib.lla_decode_workspace_bytes(ctypes.byref(cfg.c()), B, n_cap)
    if n == 0:
        raise LLAError(ERR_UNSUPPORTED, last_error())
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_launches(cfg: Cfg, B: int, n_cap: int) -> int:
    return lib.lla_decode_launches(ctypes.byref(cfg.c()), B, n_cap)


def decode_status(ws) -> int:
    """Status bits of the last completed decode call on this workspace (synchronises)."""
    return int(ws[4:8].view(torch.int32).item())


def decode_attn(cfg: Cfg, packed, rope, t: int, ctx_len, q, k_self, v_self, positions, q_pos,
                c_k, c_v, out=None, ws=None):
    """Decode attention at loop t over the latent cache; returns out fp32 [B, H, d]."""
    c = cfg.c()
    B, H, d = q.shape
    n_cap = positions.shape[1]
    if H != cfg.H or d != cfg.d_head:
        raise ValueError("q shape does not match cfg")
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = decode_workspace(cfg, B, n_cap, q.device)
    check(lib.lla_decode_attn(
        ctypes.byref(c), _ptr(packed, torch.uint8, "packed"), _ptr(rope, torch.float32, "rope"),
        rope.shape[0], t, B, n_cap, _ptr(ctx_len, torch.int32, "ctx_len", (B,)),
        _ptr(q, torch.float32, "q", (B, H, d)), _ptr(k_self, torch.float32, "k_self", (B, H, d)),
        _ptr(v_self, torch.float32, "v_self", (B, H, d)),
        _ptr(positions, torch.int32, "positions", (B, n_cap)), _ptr(q_pos, torch.int32, "q_pos", (B,)),
        _ptr(c_k, torch.bfloat16, "c_k", _cache_shape(cfg, (B, n_cap), cfg.r_k)),
        _ptr(c_v, torch.bfloat16, "c_v", _cache_shape(cfg, (B, n_cap), cfg.r_v)),
        _ptr(out, torch.float32, "out", (B, H, d)), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream()))
    return out


def evict_slot(sink: int, window: int, pos: int) -> int:
    """Slot (row within its sequence) of history position ``pos`` under sink + window eviction."""
    return int(lib.lla_evict_slot(sink, window, pos))


def evict_append(B: int, n_cap: int, sink: int, window: int, pos, positions, ctx_len, slot=None):
    """Slots for one new history token per sequence under sink + window eviction.

    ``pos`` int32 [B] device: history position of each new token.  Updates ``positions``
    [B, n_cap] and ``ctx_len`` [B] in place; returns the flat slots int64 [B] for encode.
    """
    if slot is None:
        slot = torch.empty((B,), dtype=torch.int64, device=pos.device)
    check(lib.lla_evict_append(B, n_cap, sink, window, _ptr(pos, torch.int32, "pos", (B,)),
                               _ptr(slot, torch.int64, "slot", (B,)),
                               _ptr(positions, torch.int32, "positions", (B, n_cap)),
                               _ptr(ctx_len, torch.int32, "ctx_len", (B,)), _stream()))
    return slot


# ---------------------------------------------------------------- full-memory fast path

def full_kv_bytes(cfg: Cfg, B: int, n_cap: int) -> int:
    """Bytes of one loop's full K (or V) cache, bf16 [B, H, n_cap, d]."""
    return int(lib.lla_full_kv_bytes(ctypes.byref(cfg.c()), B, n_cap))


def full_cache_alloc(cfg: Cfg, B: int, n_cap: int, device="cuda"):
    """Empty full K and V caches of one loop, bf16 [B, H, n_cap, d] each."""
    shape = (B, cfg.H, n_cap, cfg.d_head)
    return (torch.zeros(shape, dtype=torch.bfloat16, device=device),
            torch.zeros(shape, dtype=torch.bfloat16, device=device))


def full_rebuild(cfg: Cfg, packed, rope, t: int, positions, c_k, c_v, k_full, v_full,
                 slot=None, n_rows=None, status=None):
    """Rebuild rows of the loop-t full cache (in place) from the latent cache.

    ``slot`` int64 [n] lists rows b * n_cap + j; without it rows 0 .. n_rows-1 (default:
    every row) are rebuilt.
    """
    c = cfg.c()
    B, n_cap = positions.shape
    fs = (B, cfg.H, n_cap, cfg.d_head)
    if slot is not None:
        n_rows = slot.shape[0]
        sp = _ptr(slot, torch.int64, "slot", (n_rows,))
    else:
        n_rows = B * n_cap if n_rows is None else n_rows
        sp = None
    st = _ptr(status, torch.int32, "status") if status is not None else None
    check(lib.lla_full_rebuild(
        ctypes.byref(c), _ptr(packed, torch.uint8, "packed"), _ptr(rope, torch.float32, "rope"),
        rope.shape[0], t, B, n_cap, _ptr(positions, torch.int32, "positions", (B, n_cap)),
        _ptr(c_k, torch.bfloat16, "c_k", _cache_shape(cfg, (B, n_cap), cfg.r_k)),
        _ptr(c_v, torch.bfloat16, "c_v", _cache_shape(cfg, (B, n_cap), cfg.r_v)),
        sp, n_rows, _ptr(k_full, torch.bfloat16, "k_full", fs),
        _ptr(v_full, torch.bfloat16, "v_full", fs), st, _stream()))


def full_decode_workspace(cfg: Cfg, B: int, n_cap: int, device="cuda"):
    n = lib.lla_full_decode_workspace_bytes(ctypes.byref(cfg.c()), B, n_cap)
    if n == 0:
        raise LLAError(ERR_UNSUPPORTED, last_error())
    return torch.zeros(n, dtype=torch.uint8, device=device)


def full_decode_launches(cfg: Cfg, B: int, n_cap: int) -> int:
    return lib.lla_full_decode_launches(ctypes.byref(cfg.c()), B, n_cap)


def full_decode_attn(cfg: Cfg, rope, ctx_len, q, k_self, v_self, q_pos, k_full, v_full,
                     out=None, ws=None):
    """Ordinary decode attention over the full cache; returns out fp32 [B, H, d]."""
    c = cfg.c()
    B, H, d = q.shape
    n_cap = k_full.shape[2]
    if H != cfg.H or d != cfg.d_head:
        raise ValueError("q shape does not match cfg")
    fs = (B, H, n_cap, d)
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = full_decode_workspace(cfg, B, n_cap, q.device)
    check(lib.lla_full_decode_attn(
        ctypes.byref(c), _ptr(rope, torch.float32, "rope"), rope.shape[0], B, n_cap,
        _ptr(ctx_len, torch.int32, "ctx_len", (B,)), _ptr(q, torch.float32, "q", (B, H, d)),
        _ptr(k_self, torch.float32, "k_self", (B, H, d)),
        _ptr(v_self, torch.float32, "v_self", (B, H, d)), _ptr(q_pos, torch.int32, "q_pos", (B,)),
        _ptr(k_full, torch.bfloat16, "k_full", fs), _ptr(v_full, torch.bfloat16, "v_full", fs),
        _ptr(out, torch.float32, "out", (B, H, d)), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream()))
    return out

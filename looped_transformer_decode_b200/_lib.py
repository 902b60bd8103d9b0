"""ctypes binding of ``liblla.so`` (the C ABI declared in ``include/lla.h``).

Argument marshalling only: torch tensors become device pointers and the current
CUDA stream; every step of the computation runs in the library's kernels.
There is no fallback: a missing library raises at import time, and a non-zero
status raises ``LLAError`` with the library's message.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblla.so")

MODE_PER_HEAD = 0
MODE_2D = 1
STATUS_POSITION_RANGE = 1
STATUS_CTX_RANGE = 2
STATUS_SLOT_RANGE = 4

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_TOO_SMALL, ERR_CUDA = 0, -1, -2, -3, -4


class LLAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"lla error {code}: {msg}")
        self.code = code


class CCfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("d_head", ctypes.c_int32),
                ("r_k", ctypes.c_int32), ("r_v", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("rope_base", ctypes.c_float), ("sm_scale", ctypes.c_float),
                ("d_rope", ctypes.c_int32)]


@dataclass(frozen=True)
class Cfg:
    T: int
    H: int
    d_head: int
    r_k: int
    r_v: int
    mode: int = MODE_PER_HEAD
    rope_base: float = 10000.0
    sm_scale: float = 0.0
    d_rope: int = 0          # decoupled RoPE: rotary dims (0 = the whole head)

    def c(self) -> CCfg:
        return CCfg(self.T, self.H, self.d_head, self.r_k, self.r_v, self.mode, self.rope_base,
                    self.sm_scale, self.d_rope)


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -c \"import __graft_entry__ as g; "
                      "g.build()\"` (nvcc, sm_100a). There is no CPU fallback.")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_CFG = ctypes.POINTER(CCfg)
_I32, _I64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t

SIGNATURES = {
    "lla_last_error": (ctypes.c_char_p, []),
    "lla_version": (ctypes.c_char_p, []),
    "lla_ratio": (ctypes.c_int, [_CFG, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "lla_cache_bytes": (ctypes.c_int, [_CFG, _I64, _I64, ctypes.c_int, ctypes.POINTER(_I64)]),
    "lla_codec_packed_bytes": (_SZ, [_CFG]),
    "lla_codec_pack": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "lla_rope_table_bytes": (_SZ, [_CFG, _I32]),
    "lla_rope_table": (ctypes.c_int, [_CFG, _I32, _P, _SZ, _P]),
    "lla_encode": (ctypes.c_int, [_CFG, _P, _I64, _P, _P, _P, _I64, _P, _P, _P, _P]),
    "lla_decode_workspace_bytes": (_SZ, [_CFG, _I32, _I32]),
    "lla_decode_attn": (ctypes.c_int, [_CFG, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P,
                                       _P, _P, _P, _P, _P, _SZ, _P]),
    "lla_decode_launches": (ctypes.c_int, [_CFG, _I32, _I32]),
    "lla_decode_attn_noalloc": (ctypes.c_int, [_CFG, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P,
                                               _P, _P, _P, _P, _P, _P, _P, _P]),
    "lla_evict_slot": (_I64, [_I32, _I32, _I64]),
    "lla_evict_append": (ctypes.c_int, [_I32, _I32, _I32, _I32, _P, _P, _P, _P, _P]),
    "lla_full_kv_bytes": (_SZ, [_CFG, _I32, _I32]),
    "lla_full_rebuild": (ctypes.c_int, [_CFG, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P,
                                        _I64, _P, _P, _P, _P]),
    "lla_full_decode_workspace_bytes": (_SZ, [_CFG, _I32, _I32]),
    "lla_full_decode_launches": (ctypes.c_int, [_CFG, _I32, _I32]),
    "lla_full_decode_attn": (ctypes.c_int, [_CFG, _P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P,
                                            _P, _P, _P, _SZ, _P]),
}
for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def last_error() -> str:
    return lib.lla_last_error().decode()


def check(code: int) -> None:
    if code != OK:
        raise LLAError(code, last_error())

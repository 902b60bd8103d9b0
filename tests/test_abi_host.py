"""Host-side checks of the C ABI: the library loads, exports every declared symbol,
and its bookkeeping and argument validation behave as documented.  No GPU needed:
nothing here reaches a kernel launch."""
import ctypes
import os
import re

import pytest

import oracle as O
import synth

lla = pytest.importorskip("looped_transformer_decode_b200")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "lla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lla_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "lla_decode_attn" in names and "lla_encode" in names
    lib = ctypes.CDLL(lla.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
        assert n in lla.SIGNATURES, f"{n} has no binding"


def cfgs():
    for name in synth.WORKLOAD_ORDER:
        w = synth.WORKLOADS[name]
        yield O.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode), lla.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode)


def test_ratio_and_cache_bytes_match_oracle_exactly():
    for oc, lc in cfgs():
        assert lla.ratio(lc) == O.compression_ratio(oc)
        for tokens, layers in ((1, 1), (4096, 24), (1 << 20, 24), (768 * 4096, 24)):
            assert lla.cache_bytes(lc, tokens, layers) == O.cache_bytes(oc, tokens, layers)
            assert lla.cache_bytes(lc, tokens, layers, teacher=True) == \
                O.teacher_cache_bytes(oc, tokens, layers)


def test_cache_bytes_overflow_is_an_error():
    lc = lla.Cfg(4, 16, 128, 96, 160)
    with pytest.raises(lla.LLAError) as e:
        lla.cache_bytes(lc, 1 << 62, 24)
    assert e.value.code == lla.ERR_INVALID


@pytest.mark.parametrize("bad,code", [
    (dict(T=0), -2), (dict(T=65), -2), (dict(H=0), -2), (dict(d_head=80), -2),
    (dict(r_k=12), -2), (dict(r_v=264), -2), (dict(mode=3), -1), (dict(rope_base=1.0), -1),
    (dict(sm_scale=-1.0), -1)])
def test_bad_config_rejected(bad, code):
    base = dict(T=4, H=16, d_head=128, r_k=96, r_v=160)
    base.update(bad)
    with pytest.raises(lla.LLAError) as e:
        lla.ratio(lla.Cfg(**base))
    assert e.value.code == code
    assert lla.lib.lla_codec_packed_bytes(ctypes.byref(lla.Cfg(**base).c())) == 0


def _decode_args(cfg, t=0, B=2, n_cap=256, ws_bytes=None, null=None):
    fake = 0x10000  # aligned host address, never dereferenced: validation fails first
    ptr = {k: ctypes.c_void_p(fake) for k in
           ("packed", "rope", "ctx", "q", "ks", "vs", "pos", "qpos", "ck", "cv", "out", "ws")}
    if null:
        ptr[null] = None
    if ws_bytes is None:
        ws_bytes = lla.lib.lla_decode_workspace_bytes(ctypes.byref(cfg.c()), B, n_cap)
    return (ctypes.byref(cfg.c()), ptr["packed"], ptr["rope"], 4096, t, B, n_cap, ptr["ctx"],
            ptr["q"], ptr["ks"], ptr["vs"], ptr["pos"], ptr["qpos"], ptr["ck"], ptr["cv"],
            ptr["out"], ptr["ws"], ws_bytes, None)


def test_decode_argument_validation_before_launch():
    cfg = lla.Cfg(4, 16, 128, 96, 160)
    f = lla.lib.lla_decode_attn
    assert f(*_decode_args(cfg, t=4)) == lla.ERR_INVALID
    assert f(*_decode_args(cfg, t=-1)) == lla.ERR_INVALID
    for name in ("packed", "q", "ck", "ws", "out"):
        assert f(*_decode_args(cfg, null=name)) == lla.ERR_INVALID, name
    assert f(*_decode_args(cfg, ws_bytes=16)) == lla.ERR_TOO_SMALL
    assert "workspace" in lla.last_error()
    args = list(_decode_args(cfg))
    args[1] = ctypes.c_void_p(0x10004)   # misaligned packed pointer
    assert f(*args) == lla.ERR_INVALID
    # B == 0 is a no-op
    assert f(*_decode_args(cfg, B=0)) == lla.OK


def test_workspace_and_launch_accounting():
    cfg = lla.Cfg(4, 16, 128, 96, 160)
    ws = lla.lib.lla_decode_workspace_bytes(ctypes.byref(cfg.c()), 8, 4096)
    assert ws >= 256 + 8 * 16 * (2 + 160) * 4
    assert lla.decode_launches(cfg, 8, 4096) >= 2
    assert lla.decode_launches(cfg, 8, 0) == 1
    assert lla.decode_launches(cfg, 0, 4096) == 0


def test_encode_validation():
    cfg = lla.Cfg(4, 16, 128, 96, 160)
    f = lla.lib.lla_encode
    p = ctypes.c_void_p(0x10000)
    c = ctypes.byref(cfg.c())
    assert f(c, p, 0, p, p, p, 10, p, p, None, None) == lla.OK          # nothing to do
    assert f(c, None, 4, p, p, p, 10, p, p, None, None) == lla.ERR_INVALID
    assert f(c, p, -1, p, p, p, 10, p, p, None, None) == lla.ERR_INVALID
    assert f(c, p, 4, p, p, p, 10, p, p, ctypes.c_void_p(0x10002), None) == lla.ERR_INVALID


def test_packed_and_rope_sizes():
    cfg = lla.Cfg(4, 16, 128, 96, 160)
    n = lla.lib.lla_codec_packed_bytes(ctypes.byref(cfg.c()))
    # W_up and mu in fp32, W_down in bf16 twice (row major and as encode operand tiles,
    # rows padded to 16), bias in fp32; each section 256-byte aligned
    want = (4 * 16 * 128 * (96 + 160) * 4 + 2 * 4 * 16 * 128 * 4 + 2 * 16 * (96 + 160) * 512 * 2
            + 16 * (96 + 160) * 4)
    assert want <= n < want + 8 * 256
    assert lla.lib.lla_rope_table_bytes(ctypes.byref(cfg.c()), 4097) == 4097 * 64 * 8


def test_decode_plans_of_the_bench_workloads():
    """The split plan per workload (kernel launches per call): one split per head
    group with the combine fused in (prep + partial kernel) for every bench
    workload (the deep loop's 128 heads of 257 tiles included: a second split
    would add more item work than the 20 idle SMs give back); several splits plus
    the combine pass for a single sequence of 16 heads."""
    assert lla.decode_launches(lla.Cfg(4, 16, 128, 96, 160), 8, 4097) == 2
    assert lla.decode_launches(lla.Cfg(4, 16, 128, 16, 32), 256, 4097) == 2
    assert lla.decode_launches(lla.Cfg(4, 16, 128, 64, 128, lla.MODE_2D), 512, 4097) == 2
    assert lla.decode_launches(lla.Cfg(32, 8, 96, 64, 128), 16, 32769) == 2
    assert lla.decode_launches(lla.Cfg(4, 16, 128, 96, 160), 1, 4097) == 3


def test_forced_split_count_is_clamped(monkeypatch):
    """LLA_TC_SPLITS obeys the planner's bounds: at most 64 splits per head (the
    combine's limit) and at most one per 128-token tile.  The workspace holds the
    split partials [B][H][S][2 + r_v] fp32, so its size shows the S in use."""
    cfg = lla.Cfg(4, 2, 64, 16, 32)
    B, n_cap = 1, 32768                      # 256 tiles
    c = ctypes.byref(cfg.c())

    def partial_bytes(splits):
        monkeypatch.setenv("LLA_TC_SPLITS", str(splits))
        return lla.lib.lla_decode_workspace_bytes(c, B, n_cap)

    per_split = B * cfg.H * (2 + cfg.r_v) * 4
    at64 = partial_bytes(64)
    assert partial_bytes(100) == at64 == partial_bytes(1000)
    assert partial_bytes(32) < at64
    # 64 splits of four tiles each: exactly 64 partials per head (256-byte sections)
    base = partial_bytes(1)
    assert at64 - base >= 63 * per_split - 256
    assert at64 - base <= 63 * per_split + 256
    # a short history: never more splits than tiles
    monkeypatch.setenv("LLA_TC_SPLITS", "64")
    short = lla.lib.lla_decode_workspace_bytes(c, B, 300)    # 3 tiles
    monkeypatch.setenv("LLA_TC_SPLITS", "3")
    assert short == lla.lib.lla_decode_workspace_bytes(c, B, 300)


def test_phase_operand_kernel_workspace():
    """Per-head shapes with r_k in {16, 32} and r_v = 32 run on the phase-operand
    kernel, whose operand images are one [4 r_k + 16, d] bf16 image per (sequence,
    group of four heads), followed (1024-byte aligned) by the phase table, bf16 rows
    of d entries for positions below the tile-rounded cache length plus one tile,
    and one int32 table mark per (sequence, tile); LLA_TC_FORM=u keeps them on the
    per-head kernel, whose images are per (sequence, head)."""
    import os
    cfg = lla.Cfg(4, 16, 128, 16, 32)
    c = ctypes.byref(cfg.c())
    B, n = 256, 4097
    ws_f = lla.lib.lla_decode_workspace_bytes(c, B, n)
    os.environ["LLA_TC_FORM"] = "u"
    try:
        ws_u = lla.lib.lla_decode_workspace_bytes(c, B, n)
    finally:
        del os.environ["LLA_TC_FORM"]
    img_f = B * (16 // 4) * (4 * 16 + 16) * 128 * 2
    n_tiles = -(-n // 128)
    table = (n_tiles * 128 + 128) * 128 * 2
    marks = B * n_tiles * 4
    assert img_f % 1024 == 0
    img_u = B * 16 * (128 * 16 * 2 + 128 * 32)
    assert ws_u - ws_f == img_u - (img_f + table + marks)
    assert lla.decode_launches(cfg, B, n) == 2


def test_phase_table_switch_keeps_the_workspace_size(monkeypatch):
    """The phase table and tile marks are always reserved: LLA_TCF_TABLE only decides
    whether a call uses them, so a workspace sized once serves either setting."""
    cfg = lla.Cfg(4, 16, 128, 16, 32)
    c = ctypes.byref(cfg.c())
    for B, n in ((256, 4096), (3, 300), (1, 1)):
        monkeypatch.setenv("LLA_TCF_TABLE", "1")
        on = lla.lib.lla_decode_workspace_bytes(c, B, n)
        monkeypatch.setenv("LLA_TCF_TABLE", "0")
        assert lla.lib.lla_decode_workspace_bytes(c, B, n) == on

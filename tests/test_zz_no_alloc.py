"""lla_decode_attn_noalloc: decode attention for callers that cannot allocate.

Callers such as allocator-free runtime regions, plugins handed only their
input and output buffers, or servers that freeze memory after start-up cannot
provide a workspace.  The allocation-free entry point keeps its scratch in a
fixed array inside the library.  This file checks, through the C ABI, that it
returns what the workspace entry point returns on two calls in a row, and that
it rejects shapes whose scratch would exceed the array.  It is named so that
pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from cases import ATTN_TOL, decode_case, expected, rel_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import looped_transformer_decode_b200 as lla
    from gpu_util import DeviceCase, f32_tensor


def _noalloc(dev, t, out, status):
    c = dev.case
    ks, vs = f32_tensor(c.k_self[t]), f32_tensor(c.v_self[t])
    p = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
    rc = lla.lib.lla_decode_attn_noalloc(
        ctypes.byref(dev.cfg.c()), p(dev.packed), p(dev.rope), dev.rope.shape[0], t, c.B,
        c.n_cap, p(dev.ctx_len), p(dev.q), p(ks), p(vs), p(dev.positions), p(dev.q_pos),
        p(dev.c_k), p(dev.c_v), p(out), p(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == lla.OK, lla.last_error()
    torch.cuda.synchronize()
    return out.double().cpu().numpy()


def test_noalloc_matches_workspace_entry_point_twice():
    cfg = O.Cfg(4, 4, 128, 96, 160)
    case = decode_case(cfg, 2, 900, seed=4242, ctx_len=[900, 333])
    dev = DeviceCase(case)
    out = torch.empty((case.B, cfg.H, cfg.d), dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for t in (1, 3):                                   # two calls in a row
        want = dev.decode(t)                           # existing entry point, caller workspace
        got = _noalloc(dev, t, out, status)
        assert np.isfinite(got).all()
        assert rel_err(got, want).max() <= ATTN_TOL
        # and element by element against the float64 oracle
        assert rel_err(got, expected(case, t)).max() <= ATTN_TOL
        assert int(status.item()) == 0


def test_noalloc_reports_then_clears_device_status():
    """A device-side range problem reaches status_out, and the next valid call,
    which shares the same array, reports a clean status again."""
    cfg = O.Cfg(4, 2, 64, 16, 32)
    case = decode_case(cfg, 2, 300, seed=77)
    dev = DeviceCase(case, rope_max_pos=301)
    out = torch.empty((case.B, cfg.H, cfg.d), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    good_qpos = dev.q_pos
    bad = case.q_pos.copy()
    bad[1] = 5000                                      # outside the 301-entry RoPE table
    dev.q_pos = torch.from_numpy(bad.astype(np.int32)).cuda()
    got = _noalloc(dev, 0, out, status)
    assert np.isfinite(got).all()
    assert int(status.item()) & lla.STATUS_POSITION_RANGE
    dev.q_pos = good_qpos
    got = _noalloc(dev, 2, out, status)
    assert int(status.item()) == 0
    assert rel_err(got, dev.decode(2)).max() <= ATTN_TOL
    assert rel_err(got, expected(case, 2)).max() <= ATTN_TOL


def test_noalloc_rejected_call_enqueues_nothing():
    """Arguments that lla_decode_attn rejects are rejected before anything is
    enqueued, so status_out keeps the last call's word."""
    cfg = O.Cfg(4, 2, 64, 16, 32)
    case = decode_case(cfg, 1, 200, seed=78)
    dev = DeviceCase(case)
    out = torch.empty((case.B, cfg.H, cfg.d), dtype=torch.float32, device="cuda")
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    p = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
    ks = f32_tensor(case.k_self[0])
    rc = lla.lib.lla_decode_attn_noalloc(
        ctypes.byref(dev.cfg.c()), p(dev.packed), p(dev.rope), dev.rope.shape[0], cfg.T, case.B,
        case.n_cap, p(dev.ctx_len), p(dev.q), p(ks), p(ks), p(dev.positions), p(dev.q_pos),
        p(dev.c_k), p(dev.c_v), p(out), p(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))          # t == T: invalid
    assert rc == lla.ERR_INVALID
    torch.cuda.synchronize()
    assert int(status.item()) == 12345


def test_noalloc_rejects_shapes_beyond_its_scratch():
    cfg = lla.Cfg(4, 128, 128, 96, 256)
    B, n_cap = 4096, 8192
    assert lla.lib.lla_decode_workspace_bytes(ctypes.byref(cfg.c()), B, n_cap) > (8 << 20)
    fake = ctypes.c_void_p(0x10000)   # never dereferenced: the size check comes first
    rc = lla.lib.lla_decode_attn_noalloc(ctypes.byref(cfg.c()), fake, fake, 8192, 0, B, n_cap,
                                         fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                         None, None)
    assert rc == lla.ERR_TOO_SMALL
    assert "8388608" in lla.last_error()

"""bench.py's algorithmic byte counts against the per-call totals worked out from
the workload shapes (latents, positions, the loop-t up-projection and means, the
in-flight token's q / k_self / v_self and the output), and the roofline fields'
arithmetic."""
from __future__ import annotations

import bench
import synth


def _decode_bytes_by_hand(w):
    L = w.H if w.mode == synth.MODE_PER_HEAD else 1
    latents = w.B * w.n * L * (w.r_k + w.r_v) * 2
    positions = w.B * w.n * 4
    weights = w.H * w.d * (w.r_k + w.r_v) * 4 + 2 * w.H * w.d * 4
    token_io = 4 * w.B * w.H * w.d * 4
    return latents + positions + weights + token_io


def test_decode_bytes_per_call_of_every_workload():
    want_mb = {"perhead_4x_T4_H16_d128_r96_160_B8_n4096": 270.9,
               "perhead_21x_T4_H16_d128_r16_32_B256_n4096_L24": 1623.6,
               "lla2d_T4_H16_d128_r64_128_B512_n4096": 832.1,
               "deeploop_32x_T32_H8_d96_r64_128_B16_n32768": 1613.5}
    for name, mb in want_mb.items():
        w = synth.WORKLOADS[name]
        got = bench.decode_bytes(w, w.n)
        assert got == _decode_bytes_by_hand(w)
        assert round(got / 1e6, 1) == mb, (name, got)


def test_full_memory_bytes_are_the_bf16_rows_read():
    w = synth.WORKLOADS["perhead_4x_T4_H16_d128_r96_160_B8_n4096"]
    got = bench.full_decode_bytes(w, w.n)
    assert got == w.B * w.H * w.n * 2 * w.d * 2 + 4 * w.B * w.H * w.d * 4 + 2 * w.B * 4
    # the 4x codec stores across four loops what one loop's full cache holds
    assert abs(got - bench.decode_bytes(w, w.n)) / got < 0.01


def test_encode_bytes_count_inputs_weights_and_latents():
    w = synth.WORKLOADS["perhead_4x_T4_H16_d128_r96_160_B8_n4096"]
    n = 8
    x = n * w.T * w.H * w.d * 2 * 2
    wd = w.H * (w.r_k + w.r_v) * (w.T * w.d) * 2 + w.H * (w.r_k + w.r_v) * 4
    out = n * w.H * (w.r_k + w.r_v) * 2 + n * 8
    assert bench.encode_bytes(w, n) == x + wd + out

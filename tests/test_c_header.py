"""The boundary is a plain C ABI: a C99 program that includes ``include/lla.h``
compiles with gcc, links against the built library, and calls the host-side
entry points (no GPU needed for these)."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "looped_transformer_decode_b200")

C_SRC = r"""
#include <stdio.h>
#include "lla.h"

int main(void) {
  lla_cfg c = {4, 16, 128, 16, 32, LLA_MODE_PER_HEAD, 10000.0f, 0.0f, 0};
  int64_t num = 0, den = 0, bytes = 0;
  if (lla_ratio(&c, &num, &den) != LLA_OK) return 1;
  if (lla_cache_bytes(&c, 1024, 24, 0, &bytes) != LLA_OK) return 2;
  lla_cfg bad = c;
  bad.d_head = 100;
  if (lla_ratio(&bad, &num, &den) != LLA_ERR_UNSUPPORTED) return 3;
  printf("%lld/%lld %lld %d %s\n", (long long)num, (long long)den, (long long)bytes,
         lla_evict_slot(4, 256, 300) == 4 + (300 - 4) % 256, lla_version());
  return 0;
}
"""


def test_c99_program_uses_the_header_and_library(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    lib = os.path.join(LIB_DIR, "liblla.so")
    assert os.path.exists(lib), "build the library first"
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    cuda_lib = "/usr/local/cuda/lib64"
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           "-o", str(exe), "-L", LIB_DIR, "-llla", f"-Wl,-rpath,{LIB_DIR}"]
    if os.path.isdir(cuda_lib):
        cmd += ["-L", cuda_lib, f"-Wl,-rpath,{cuda_lib}", "-Wl,--allow-shlib-undefined"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    ratio, nbytes, evict_ok = r.stdout.split()[:3]
    assert ratio == "64/3"                       # 2 T d / (r_k + r_v) = 1024 / 48
    assert int(nbytes) == 36 * 2**20             # 36 KiB per token x 1024 tokens (24 layers)
    assert evict_ok == "1"

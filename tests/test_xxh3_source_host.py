"""The device hash source (csrc/lt_xxh3.cuh), compiled for the host with
g++, against the system libxxhash: every length from 0 to 1109 bytes and
larger inputs across several scramble blocks, with secrets of 136 to 320
bytes. The kernel k_xxh3_blocks runs this same function per block."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

from tests._pins import libxxhash
from weight_dequantization_b200 import _build

HARNESS = r"""
#include "lt_xxh3.cuh"
#include <dlfcn.h>
#include <stdio.h>
#include <initializer_list>
typedef uint64_t (*fn_t)(const void *, size_t, const void *, size_t);
static uint8_t buf[100003], sec[320];
int main() {
  void *h = dlopen("libxxhash.so.0", RTLD_NOW);
  if (!h) return 2;
  fn_t ref = (fn_t)dlsym(h, "XXH3_64bits_withSecret");
  uint64_t x = 88172645463325252ull;
  auto rnd = [&]() { x ^= x << 13; x ^= x >> 7; x ^= x << 17; return (uint8_t)x; };
  const size_t extra[] = {2047, 2048, 2049, 4096, 47000, 65536, 100003};
  int bad = 0, total = 0;
  for (int sl : {136, 192, 193, 256, 320}) {
    for (int i = 0; i < sl; ++i) sec[i] = rnd();
    for (size_t k = 0; k < 1110 + 7; ++k) {
      size_t len = k < 1110 ? k : extra[k - 1110];
      for (size_t i = 0; i < len; ++i) buf[i] = rnd();
      ++total;
      if (lt::xxh3::hash64(buf, len, sec, sl) != ref(buf, len, sec, sl)) ++bad;
    }
  }
  printf("%d %d\n", bad, total);
  return bad != 0;
}
"""


@pytest.mark.skipif(libxxhash() is None or shutil.which("g++") is None, reason="needs g++ and libxxhash")
def test_device_hash_source_matches_libxxhash(tmp_path):
    src = tmp_path / "harness.cpp"
    src.write_text(HARNESS)
    exe = tmp_path / "harness"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", _build.CSRC, str(src), "-o", str(exe), "-ldl"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, env=dict(os.environ))
    assert r.returncode == 0, r.stdout + r.stderr
    bad, total = map(int, r.stdout.split())
    assert bad == 0 and total == 5 * 1117

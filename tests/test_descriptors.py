"""The shared-memory descriptor words the MMA issuer adds offsets to equal
the full 64-bit descriptor for every shared address and K-step offset
(CPU only: the header's host-callable helpers compiled with nvcc for the
host). The issuer relies on (start >> 4) + (offset >> 4) never carrying
into the leading-byte-offset field."""

import os
import subprocess

import pytest

from packed_attention_qk_b200 import build as pqk_build

SRC = r'''
#include <cstdio>
#include "sm100_ptx.cuh"
using namespace pqk;
int main() {
  long bad = 0, n = 0;
  for (uint32_t base = 0; base < 233472; base += 1024)
    for (uint32_t off = 0; base + off < 233472 && off < 200 * 1024; off += 32)
      for (uint32_t lbo : {16u, 16384u})
        for (uint32_t sbo : {1024u}) {
          const uint64_t full = smem_desc_sw128(base + off, lbo, sbo);
          const uint32_t lo = smem_desc_lo(base, lbo) + (off >> 4);
          const uint64_t words = (uint64_t)lo | ((uint64_t)smem_desc_hi_sw128(sbo) << 32);
          bad += full != words;
          ++n;
        }
  printf("%ld %ld\n", n, bad);
  return bad != 0;
}
'''


def test_descriptor_words_equal_the_full_descriptor(tmp_path):
    if not os.path.exists(pqk_build.NVCC):
        pytest.skip("nvcc not available")
    src = tmp_path / "desc.cu"
    src.write_text(SRC)
    exe = tmp_path / "desc"
    subprocess.check_call([pqk_build.NVCC, "-std=c++17", "-I", pqk_build.CSRC, "-o", str(exe), str(src)],
                          stderr=subprocess.DEVNULL)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    n, bad = map(int, out.stdout.split())
    assert out.returncode == 0 and bad == 0 and n > 1_000_000

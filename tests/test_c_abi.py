"""The C ABI from C: include/kvq.h compiles as C11 with every warning an
error, a C program links against libkvq.so and makes the host-only calls
(no GPU needed), and its results equal the Python binding's."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mixed_precision_kv_kvq_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "kvq.h"

int main(void) {
  const int f4[1] = {4};
  const int fmix[3] = {4, 2, 2};
  printf("pool %zu\n", kvq_pool_bytes(1, 1, 2, 128, (size_t)1114112, f4));
  printf("pool_mix %zu\n", kvq_pool_bytes(3, 2, 4, 128, (size_t)200000000, fmix));
  printf("pool_bad_dim %zu\n", kvq_pool_bytes(1, 1, 2, 64, (size_t)1114112, f4));
  kvq_status s = kvq_alloc(NULL, 1, 1, 2, 128, (size_t)1114112, f4, NULL, 0);
  printf("alloc_null %d %d\n", (int)s, (int)(strlen(kvq_last_error()) > 0));
  /* 3 blocks, widths {2, 4}: block 1 is the most sensitive at 2 bits */
  const int bits[2] = {2, 4};
  const double sens[6] = {1.0, 0.5, 9.0, 0.1, 1.0, 0.9};
  int fb[3] = {0, 0, 0};
  double obj = -1.0;
  /* budget for widths (4, 4, 2) at 512 tokens, batch 1, 2 KV heads: 4 * 512 * (68 + 68 + 36) */
  s = kvq_allocate_bits(3, 2, bits, sens, 1, 2, 128, 512LL, (size_t)(4 * 512 * (68 + 68 + 36)), fb, &obj);
  printf("alloc_bits %d %d %d %d %.3f\n", (int)s, fb[0], fb[1], fb[2], obj);
  s = kvq_allocate_bits(3, 2, bits, sens, 1, 2, 128, 512LL, (size_t)100, fb, &obj);
  printf("alloc_bits_small %d\n", (int)s);
  kvq_free(NULL);
  return 0;
}
"""


@pytest.fixture(scope="module")
def kvq():
    from mixed_precision_kv_kvq_b200 import build

    build.build()
    import mixed_precision_kv_kvq_b200 as m

    m.load()
    return m


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_links_and_agrees(kvq, tmp_path):
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", PKG, "-lkvq", f"-Wl,-rpath,{PKG}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = {line.split()[0]: line.split()[1:] for line in out.strip().splitlines()}
    assert int(got["pool"][0]) == kvq.kvq_pool_bytes(1, 1, 2, 128, 1114112, [4]) > 0
    assert int(got["pool_mix"][0]) == kvq.kvq_pool_bytes(3, 2, 4, 128, 200000000, [4, 2, 2]) > 0
    assert int(got["pool_bad_dim"][0]) == 0
    assert got["alloc_null"] == ["1", "1"]  # KVQ_ERR_INVALID, with a message
    status, f0, f1, f2, obj = got["alloc_bits"]
    # the cheapest fitting choice: one block drops to 2 bits, the least sensitive one (block 2)
    assert (int(status), int(f0), int(f1), int(f2)) == (0, 4, 4, 2)
    assert abs(float(obj) - (0.5 + 0.1 + 1.0)) < 1e-9
    assert got["alloc_bits_small"] == ["2"]  # KVQ_ERR_BUDGET

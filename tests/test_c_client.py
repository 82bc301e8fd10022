"""The boundary from plain C: a C99 program that includes nothing of the library but
include/kvq.h, compiled by gcc with warnings as errors and linked against libkvq.so, calls the
host-only queries (sizes, tables, status strings; nothing that launches, so it passes no
pointer the library could hand to a kernel). What it prints is checked against the layout's
closed forms and the oracle's tables."""
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

from oracle import blockgtq as bg
from oracle import codebooks as cb
from packed_cache_attention_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STATUS = {m.group(1): int(m.group(2)) for m in
          re.finditer(r"\b(KVQ_\w+) = (\d+)", open(os.path.join(ROOT, "include", "kvq.h")).read())}

C_SOURCE = r"""
#include <stdio.h>
#include "kvq.h"

int main(void) {
  const kvq_cache_desc c = {1, 2, KVQ_HEAD_DIM, 131072, 3, 3};
  const kvq_cache_desc keys_only = {3, 5, KVQ_HEAD_DIM, 100, 3, 0};
  const kvq_cache_desc bad = {1, 2, 64, 100, 3, 3};
  uint16_t c16[8];
  float t32[7], delta = 0.0f, levels[16], mids[15];
  int i, st;

  printf("abi %d\n", kvq_abi_version());
  printf("status0 %s\n", kvq_status_string(KVQ_OK));
  printf("packed %zu\n", kvq_packed_bytes(&c));
  printf("keys_only %zu\n", kvq_packed_bytes(&keys_only));
  printf("bad %zu\n", kvq_packed_bytes(&bad));
  printf("header %zu %zu\n", kvq_packed_header_bytes(8), kvq_packed_header_bytes(9));
  printf("alloc %zu %zu\n", kvq_alloc_bytes(2), sizeof(kvq_head_alloc));
  printf("nf4 %zu\n", kvq_nf4_packed_bytes(8, 56, 8192, KVQ_HEAD_DIM));
  printf("decode_ws %d\n", kvq_decode_workspace_bytes(&c, 16) > 0);
  printf("calib_ws %zu\n", kvq_calibrate_workspace_bytes(16, 8, 2048));
  printf("statuses");
  for (i = 0; i <= KVQ_ERR_MISMATCH; ++i) printf(" %d", kvq_status_string(i)[0] != '\0');
  printf("\nstatus_out_of_range %s\n", kvq_status_string(KVQ_ERR_MISMATCH + 1));
  st = kvq_codebook(3, c16, t32, &delta);
  printf("codebook %d", st);
  for (i = 0; i < 8; ++i) printf(" %u", (unsigned)c16[i]);
  for (i = 0; i < 7; ++i) printf(" %.9g", t32[i]);
  printf(" %.9g\n", delta);
  st = kvq_nf4_table(levels, mids);
  printf("nf4_table %d", st);
  for (i = 0; i < 16; ++i) printf(" %.9g", levels[i]);
  for (i = 0; i < 15; ++i) printf(" %.9g", mids[i]);
  printf("\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(kvq.LIB_PATH):
        from packed_cache_attention_b200 import build
        build.build()
    d = tmp_path_factory.mktemp("c_client")
    src, exe = d / "client.c", d / "client"
    src.write_text(C_SOURCE)
    libdir = os.path.dirname(kvq.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lkvq", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True, text=True)
    run = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60)
    return {line.split()[0]: line.split()[1:] for line in run.stdout.splitlines() if line.strip()}


def test_c_program_sees_the_layout(c_output):
    out = c_output
    assert int(out["abi"][0]) >= 1
    assert out["status0"] == ["ok"]
    assert int(out["packed"][0]) == bg.packed_bytes(1, 2, 131072, 128, 3, 3) == 26_214_400 + 128
    assert int(out["keys_only"][0]) == bg.packed_bytes(3, 5, 100, 128, 3, 0)
    assert int(out["bad"][0]) == 0
    assert [int(x) for x in out["header"]] == [bg.header_bytes(8), bg.header_bytes(9)]
    n_alloc, rec = (int(x) for x in out["alloc"])
    assert rec == 2048 and n_alloc == 2 * rec
    assert int(out["nf4"][0]) == 2 * 8 * 28 * 8192 * 130
    assert out["decode_ws"] == ["1"]


def test_c_program_reads_the_oracles_tables(c_output):
    vals = c_output["codebook"]
    assert int(vals[0]) == STATUS["KVQ_OK"]
    c16, t32 = cb.stored_codebook(3)
    np.testing.assert_array_equal(np.array([int(x) for x in vals[1:9]], np.uint16), c16.view(np.uint16))
    np.testing.assert_array_equal(np.array(vals[9:16], dtype=np.float32), t32)
    assert np.float32(vals[16]) == cb.delta_table()[3]
    nf = c_output["nf4_table"]
    assert int(nf[0]) == STATUS["KVQ_OK"]
    np.testing.assert_array_equal(np.array(nf[1:17], dtype=np.float32), cb.nf4_values())
    np.testing.assert_array_equal(np.array(nf[17:32], dtype=np.float32), cb.nf4_midpoints())


def test_c_program_gets_status_strings_and_workspace_sizes(c_output):
    assert c_output["statuses"] == ["1"] * (STATUS["KVQ_ERR_MISMATCH"] + 1)
    assert " ".join(c_output["status_out_of_range"]) == "unknown status"
    # counters + energies + segment sums + chunk sums (fp64) at least
    assert int(c_output["calib_ws"][0]) >= 8 * (16 * 2048 // 64) * 64 * 8 + 8 * 64 * 8

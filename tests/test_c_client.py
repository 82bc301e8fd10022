"""The boundary from plain C: a C99 program that includes nothing of the library but
include/kvq.h, compiled by gcc with warnings as errors and linked against libkvq.so, calls the
host-only queries (sizes, tables, status strings; nothing that launches, so it passes no
pointer the library could hand to a kernel). What it prints is checked against the layout's
closed forms and the oracle's tables."""
import ctypes
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


# header struct -> the binding's ctypes mirror of it
STRUCTS = [("kvq_tensor4", kvq.Tensor4), ("kvq_calib_params", kvq.CalibParams), ("kvq_cache_desc", kvq.CacheDesc),
           ("kvq_head_alloc", kvq.HeadAlloc), ("kvq_packed_header", kvq.PackedHeader),
           ("kvq_decode_extra", kvq.DecodeExtra)]


def _layout_source():
    """A C program printing sizeof of every header struct and offsetof of every field the
    binding declares (a field the header lacks fails the compile)."""
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "kvq.h"', "int main(void) {"]
    for cname, cls in STRUCTS:
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["  return 0;", "}"]
    return "\n".join(lines) + "\n"


def _build_and_run(tmp, name, source, link):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src, exe = tmp / f"{name}.c", tmp / name
    src.write_text(source)
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe)]
    if link:
        libdir = os.path.dirname(kvq.LIB_PATH)
        cmd += ["-L", libdir, "-lkvq", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60).stdout


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    if not os.path.exists(kvq.LIB_PATH):
        from packed_cache_attention_b200 import build
        build.build()
    out = _build_and_run(tmp_path_factory.mktemp("c_client"), "client", C_SOURCE, link=True)
    return {line.split()[0]: line.split()[1:] for line in out.splitlines() if line.strip()}


def test_binding_structs_have_the_headers_layout(tmp_path):
    """Every ctypes mirror has the C compiler's size and field offsets for its struct."""
    out = _build_and_run(tmp_path, "layout", _layout_source(), link=False)
    got = {}
    for line in out.splitlines():
        cname, key, val = line.split()
        got[(cname, key)] = int(val)
    for cname, cls in STRUCTS:
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert got[(cname, field)] == getattr(cls, field).offset, (cname, field)


def _c_params(text, name):
    """Parameter types of `name` in the header, comments removed; [] for (void)."""
    m = re.search(r"\b" + name + r"\s*\(([^)]*)\)\s*;", text)
    params = " ".join(m.group(1).split())
    if params in ("", "void"):
        return []
    return [re.sub(r"\s*\b\w+$", "", p.strip()) if not p.strip().endswith("*") else p.strip()
            for p in params.split(",")]


def _ctypes_kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "pointer"
    if t is ctypes.c_size_t:
        return "size_t"
    if t is ctypes.c_int:
        return "int"
    raise AssertionError(t)


def _c_kind(t):
    if "*" in t:
        return "pointer"
    if t.endswith("size_t"):
        return "size_t"
    if t in ("int", "kvq_status") or t.endswith("int32_t"):
        return "int"
    raise AssertionError(t)


def test_binding_signatures_follow_the_header():
    """Every entry point the binding declares takes as many arguments as the header's
    prototype, each of the same kind (pointer, int or size_t), and returns the same kind."""
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "kvq.h")).read(), flags=re.S)
    for name, (args, res) in kvq._SIGNATURES.items():
        params = _c_params(text, name)
        assert len(params) == len(args), (name, params)
        for c, t in zip(params, args):
            assert _c_kind(c) == _ctypes_kind(t), (name, c, t)
        ret = re.search(r"([\w\s\*]+?)\b" + name + r"\s*\(", text).group(1).split()
        ret_t = " ".join(ret).replace("const ", "")
        assert _c_kind(ret_t) == _ctypes_kind(res), (name, ret_t, res)


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


def test_readme_c_example_compiles(tmp_path):
    """The C example in README.md compiles against the header as C99 with warnings as errors,
    and links against libkvq.so with no undefined symbol."""
    text = open(os.path.join(ROOT, "README.md")).read()
    block = re.search(r"```c\n(.*?)```", text, flags=re.S).group(1)
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "example.c"
    src.write_text(block)
    if not os.path.exists(kvq.LIB_PATH):
        from packed_cache_attention_b200 import build
        build.build()
    libdir = os.path.dirname(kvq.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fPIC", "-shared",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(tmp_path / "example.so"),
                    "-Wl,--no-undefined", "-L", libdir, "-lkvq"], check=True, capture_output=True, text=True)

"""The boundary is a plain C ABI: include/cg.h compiles as C99 and as C++11 on its
own, and a C program that includes it links against libcg.so and calls it without
any Python or torch in between (sizes, status strings and argument validation,
which need no GPU)."""
import os
import shutil
import subprocess

import pytest

from quantization_cg_encode_b200 import cg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")

C_PROGRAM = r"""
#include <stdio.h>
#include "cg.h"

int main(void) {
  /* Llama-3-8B-shaped cache: 32 layers, K and V, 1 x 8 KV heads, 4096 tokens, d = 128 */
  cg_kv_desc kv = {32, 1, 8, 4096, 128};
  cg_codec_desc codec = {16, 4, 16, 16, CG_QUANT_BLOCK_UNIFORM, 32, 32, 0};
  cg_sizes sz;
  cg_status st = cg_sizes_for(&kv, &codec, &sz);
  if (st != CG_OK) return 10;
  printf("version %d\n", (int)cg_version());
  printf("sizes %llu %llu\n", (unsigned long long)sz.code_bytes, (unsigned long long)sz.scale_count);
  printf("invalid %s\n", cg_status_string(CG_ERR_INVALID));
  /* a null cache pointer is rejected before anything is enqueued */
  st = cg_encode(&kv, &codec, 0, 0, 0, 4096, 0, 0, 0, 0, 0);
  printf("encode_null %d\n", (int)st);
  return 0;
}
"""


def _need(tool):
    if shutil.which(tool) is None:
        pytest.skip("%s not installed" % tool)


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-x", "c", "-std=c99", "-pedantic"]),
                                            ("g++", ["-x", "c++", "-std=c++11", "-pedantic"])])
def test_header_compiles_on_its_own(compiler, flags, tmp_path):
    _need(compiler)
    src = tmp_path / "only_header.c"
    src.write_text('#include "cg.h"\n')
    r = subprocess.run([compiler] + flags + ["-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I", INCLUDE, str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_program_links_and_calls_the_library(tmp_path):
    _need("gcc")
    lib = cg.LIB_PATH
    if not os.path.exists(lib):
        pytest.skip("libcg.so not built")
    src = tmp_path / "use_cg.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_cg"
    libdir = os.path.dirname(lib)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, str(src), "-o", str(exe),
                        "-L" + libdir, "-lcg", "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    out = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    n = 32 * 2 * 1 * 8 * 4096 * 128
    assert out["sizes"].split() == [str(n * 4 // 8), str(n // 256)]   # 4-bit codes; one range per 16 x 16 block
    assert int(out["version"]) == cg.lib().cg_version()
    assert out["invalid"] == cg.status_string(cg.CG_ERR_INVALID)
    assert int(out["encode_null"]) == cg.CG_ERR_INVALID

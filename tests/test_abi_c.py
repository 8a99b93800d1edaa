"""The C ABI from C: a plain C99 program (and the same file as C++) includes
include/coli_moe.h, links libcolimoe.so and runs the host-only calls.  CPU only:
nothing here reaches a kernel launch."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "int4_routed_expert_renorm_b200")

PROGRAM = r"""
#include <stdio.h>
#include "coli_moe.h"

int main(void) {
  coli_moe_dims d = {6144, 2048, 256, 8, 1, 32, 4};
  int f1 = -1, f64 = -1, f4096 = -1, f0 = -1;
  if (coli_moe_ffn_form(&d, 1, 0, &f1) != COLI_OK) return 10;
  if (coli_moe_ffn_form(&d, 64, 0, &f64) != COLI_OK) return 11;
  if (coli_moe_ffn_form(&d, 4096, 0, &f4096) != COLI_OK) return 12;
  if (coli_moe_ffn_form(&d, 0, COLI_PATH_DECODE | COLI_PATH_PREFILL, &f0) != COLI_OK) return 13;
  if (coli_moe_ffn_form(&d, 4, COLI_PATH_DECODE | COLI_PATH_PREFILL, &f0) != COLI_ERR_INVALID_ARG) return 14;
  /* argument checks answer before anything touches a device */
  if (coli_moe_layer(&d, NULL, NULL, 4, NULL, NULL, 0, NULL, NULL, NULL, NULL, NULL, 0, NULL) !=
      COLI_ERR_INVALID_ARG) return 15;
  if (coli_moe_route(NULL, NULL, 0, 16, 2, NULL, NULL, NULL) != COLI_OK) return 16;
  d.group = 16;
  if (coli_moe_workspace_bytes(&d, 4) != 0) return 17;
  d.group = 32;
  printf("%d %d %d %d %d %s %zu\n", coli_moe_version(), f1, f64, f4096, f0,
         coli_status_str(COLI_ERR_WORKSPACE), coli_moe_workspace_bytes(&d, 1) > 0 ? (size_t)1 : (size_t)0);
  return 0;
}
"""


@pytest.fixture(scope="module")
def built():
    from int4_routed_expert_renorm_b200.build import build
    build()
    return os.path.join(PKG, "libcolimoe.so")


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++17")])
def test_header_compiles_links_and_runs(built, tmp_path, compiler, std):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    ext = "c" if compiler == "gcc" else "cpp"
    src, exe = tmp_path / f"use_abi.{ext}", tmp_path / "use_abi"
    src.write_text(PROGRAM)
    cmd = [compiler, std, "-Wall", "-Wextra", "-Werror", "-pedantic", f"-I{os.path.join(ROOT, 'include')}",
           str(src), "-o", str(exe), f"-L{PKG}", "-lcolimoe", f"-Wl,-rpath,{PKG}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.split() == ["100", "1", "2", "3", "0", "workspace", "too", "small", "1"]

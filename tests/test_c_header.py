"""The boundary from plain C: include/fvattn.h compiles as strict C99 and C++17, and a C
program linked against libfvattn.so runs the entry points that need no GPU (geometry
queries, workspace sizes, status strings, host-side argument checks)."""
import os
import shutil
import subprocess

import pytest

import free_adaptive_block_b200 as fv
from free_adaptive_block_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INC = os.path.join(ROOT, "include")

C_PROGRAM = r"""
#include <stdio.h>
#include "fvattn.h"

int main(void) {
  /* Wan2.1-480p latent: 21 x 30 x 52 tokens, 1 x 8 x 16 blocks, 12 heads */
  fvattn_geom_t g = {1, 12, 21, 30, 52, 128, 1, 8, 16};
  fvattn_geom_t bad = g;
  int nB = 0, words = 0, s;
  size_t ws, rws;
  if (fvattn_num_blocks(&g, &nB, &words) != FVATTN_OK) return 1;
  ws = fvattn_attn_workspace_size(&g);
  rws = fvattn_route_workspace_size(&g);
  printf("nB=%d words=%d attn_ws=%zu route_ws=%zu\n", nB, words, ws, rws);
  for (s = FVATTN_OK; s <= FVATTN_ERR_DEVICE; ++s)
    printf("status %d %s\n", s, fvattn_status_string((fvattn_status_t)s));
  /* host-side argument checks, before any CUDA call */
  printf("null geometry %d\n", (int)fvattn_num_blocks(NULL, &nB, &words));
  bad.d = 96;
  printf("d=96 route %d\n", (int)fvattn_route(&bad, (const float*)0x1000, (const float*)0x2000,
                                               0.9f, 4, 0.088f, (uint32_t*)0x3000, (int32_t*)0x4000, NULL));
  printf("p<0 route %d\n", (int)fvattn_route(&g, (const float*)0x1000, (const float*)0x2000,
                                              -0.5f, 4, 0.088f, (uint32_t*)0x3000, (int32_t*)0x4000, NULL));
  printf("small route ws %d\n", (int)fvattn_route_ws(&g, (const float*)0x1000, (const float*)0x2000,
                                                     0.9f, 4, 0.088f, (uint32_t*)0x3000, (int32_t*)0x4000,
                                                     (void*)0x5000, rws - 16, NULL));
  printf("small attn ws %d\n", (int)fvattn_block_sparse_attn(&g, (const void*)0x1000, (const void*)0x2000,
                                                             (const void*)0x3000, (const uint32_t*)0x4000,
                                                             0.088f, (void*)0x5000, (float*)0x6000,
                                                             (void*)0x7000, ws - 256, NULL, NULL));
  /* the attention calls take the mask alone, no per-row counts */
  printf("small dense ws %d\n", (int)fvattn_dense_attn(&g, (const void*)0x1000, (const void*)0x2000,
                                                       (const void*)0x3000, 0.088f, (void*)0x5000,
                                                       (float*)0x6000, (void*)0x7000, ws - 256, NULL, NULL));
  return 0;
}
"""


@pytest.fixture(scope="module")
def libdir():
    return os.path.dirname(_build.build())


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_strict_c99_and_cxx17(tmp_path):
    src = tmp_path / "h.c"
    src.write_text('#include "fvattn.h"\n#include "fvattn_testing.h"\nint main(void) { return 0; }\n')
    subprocess.run(["gcc", "-std=c99", "-pedantic-errors", "-Wall", "-Wextra", "-Werror", "-I", INC,
                    "-fsyntax-only", str(src)], check=True)
    srcpp = tmp_path / "h.cpp"
    srcpp.write_text('#include "fvattn.h"\n#include "fvattn_testing.h"\nint main() { return 0; }\n')
    subprocess.run(["g++", "-std=c++17", "-pedantic-errors", "-Wall", "-Wextra", "-Werror", "-I", INC,
                    "-fsyntax-only", str(srcpp)], check=True)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_runs_host_entry_points(tmp_path, libdir):
    src = tmp_path / "prog.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "prog"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", INC, str(src), "-o", str(exe),
                    "-L", libdir, "-lfvattn", f"-Wl,-rpath,{libdir}"], check=True)
    # the library links against the CUDA runtime; no device is touched by these calls
    env = dict(os.environ)
    cuda_lib = "/usr/local/cuda/lib64"
    if os.path.isdir(cuda_lib):
        env["LD_LIBRARY_PATH"] = cuda_lib + os.pathsep + env.get("LD_LIBRARY_PATH", "")
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, env=env).stdout
    lines = out.splitlines()
    assert lines[0].startswith("nB=336 words=11 attn_ws=")
    assert lines[0].endswith(f" route_ws={256 + 12 * 336 * 11 * 32 * 4 + 4 * 12 * 336 * 128 * 4}")
    # the same static strings the binding reads through ctypes
    assert lines[1:8] == [f"status {i} {fv.fvattn_status_string(i)}" for i in range(7)]
    assert lines[8:] == [
        "null geometry 1",     # FVATTN_ERR_INVALID_ARG
        "d=96 route 2",        # FVATTN_ERR_UNSUPPORTED
        "p<0 route 1",         # FVATTN_ERR_INVALID_ARG
        "small route ws 3",    # FVATTN_ERR_WORKSPACE
        "small attn ws 3",     # FVATTN_ERR_WORKSPACE
        "small dense ws 3",    # FVATTN_ERR_WORKSPACE
    ]

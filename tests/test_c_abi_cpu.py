"""The boundary from plain C (no GPU work is launched).

A C99 program includes include/muon_b200.h, compiled with warnings as
errors and -pedantic, so the header is valid C with no C++ in it.  It links
against libmuon_b200.so and calls the host-only parts of the ABI: status
strings, workspace sizing, the kernel-kind table, and argument validation of
muon_step / adamw_step / muon_reduce_mean, which reject bad calls with a
status and a reason before any CUDA call.
"""
import os
import shutil
import subprocess

import pytest

from muon_polar_orthogonalized_b200.build import LIB_PATH, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "muon_b200.h"

static int failures = 0;
#define EXPECT(cond) do { if (!(cond)) { printf("FAIL line %d: %s\n", __LINE__, #cond); ++failures; } } while (0)

int main(void) {
  muon_group g[2];
  float* params[3];
  const void* grads[3];
  float* mom[3];
  float coeffs[15];
  size_t ws, ws_min;
  int i, kinds;
  adamw_group ag;
  int64_t numel = 16;

  EXPECT(strcmp(muon_status_string(MUON_OK), "") != 0);
  EXPECT(strcmp(muon_status_string(MUON_ERR_WORKSPACE), muon_status_string(MUON_OK)) != 0);

  g[0].rows = 256; g[0].cols = 1024; g[0].count = 2; g[0].first = 0;
  g[0].grad_dtype = MUON_BF16; g[0].lr_scale = 1.0f;
  g[1].rows = 1024; g[1].cols = 256; g[1].count = 1; g[1].first = 2;
  g[1].grad_dtype = MUON_F32; g[1].lr_scale = 1.0f;
  ws = muon_workspace_size(g, 2, MUON_NESTEROV | MUON_CAUTIOUS_WD);
  ws_min = muon_workspace_min_size(g, 2, MUON_NESTEROV | MUON_CAUTIOUS_WD);
  EXPECT(ws > 0);
  EXPECT(ws_min > 0 && ws_min <= ws);
  EXPECT(muon_workspace_size(g, 2, MUON_NESTEROV | MUON_ROW_EQUILIBRATE) >= ws);

  g[1].first = 1;   /* overlaps group 0's range: invalid */
  EXPECT(muon_workspace_size(g, 2, 0) == 0);
  g[1].first = 2;

  kinds = muon_kernel_kind_count();
  EXPECT(kinds > 0);
  for (i = 0; i < kinds; ++i) EXPECT(muon_kernel_kind_name(i) != NULL);

  for (i = 0; i < 3; ++i) { params[i] = (float*)0x100000; grads[i] = (const void*)0x200000; mom[i] = (float*)0x300000; }
  for (i = 0; i < 15; ++i) coeffs[i] = 1.0f;
  /* no workspace */
  EXPECT(muon_step(params, grads, mom, g, 2, 0.02f, 0.95f, 0.01f, 5, coeffs, MUON_NESTEROV,
                   NULL, ws, NULL) == MUON_ERR_WORKSPACE);
  EXPECT(strlen(muon_last_error()) > 0);
  /* ns_steps out of range */
  EXPECT(muon_step(params, grads, mom, g, 2, 0.02f, 0.95f, 0.01f, 17, coeffs, MUON_NESTEROV,
                   (void*)0x400000, ws, NULL) == MUON_ERR_INVALID_ARG);
  /* misaligned parameter pointer */
  params[1] = (float*)0x100004;
  EXPECT(muon_step(params, grads, mom, g, 2, 0.02f, 0.95f, 0.01f, 5, coeffs, MUON_NESTEROV,
                   (void*)0x400000, ws, NULL) == MUON_ERR_INVALID_ARG);
  params[1] = (float*)0x100000;
  /* workspace smaller than the minimum */
  EXPECT(muon_step(params, grads, mom, g, 2, 0.02f, 0.95f, 0.01f, 5, coeffs, MUON_NESTEROV,
                   (void*)0x400000, ws_min - 1, NULL) == MUON_ERR_WORKSPACE);

  ag.params = params; ag.grads = grads; ag.exp_avg = mom; ag.exp_avg_sq = mom;
  ag.numel = &numel; ag.count = 1; ag.grad_dtype = MUON_F32;
  ag.lr = 3e-4f; ag.beta1 = 0.9f; ag.beta2 = 0.95f; ag.eps = 1e-8f; ag.wd = 0.0f;
  EXPECT(adamw_step(&ag, 1, 0, NULL) == MUON_ERR_INVALID_ARG);   /* step must be >= 1 */

  EXPECT(muon_reduce_mean(NULL, NULL, 0, NULL, 0, MUON_F32, NULL) == MUON_ERR_INVALID_ARG);

  printf("%s\n", failures ? "failed" : "ok");
  return failures ? 1 : 0;
}
"""


@pytest.fixture(scope="module")
def lib_dir():
    build()
    return os.path.dirname(LIB_PATH)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_host_entry_points_work_from_c(tmp_path, lib_dir):
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", lib_dir, "-lmuon_b200", "-Wl,-rpath," + lib_dir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip().endswith("ok"), run.stdout + run.stderr

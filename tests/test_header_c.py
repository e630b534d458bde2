"""The C ABI from C: include/fva.h compiles as strict C99 with warnings as errors, and a C
program linked against libfva.so runs the host-only entry points (status strings, size
queries, the RLB planner, SASA budgets) without a GPU. Expected values come from the
shapes' arithmetic and from the oracles (oracle/rlb_oracle.py, oracle/sasa_oracle.py)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "adaptive_block_sparse_hilbert_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fva.h"

/* The calls of one layer, as the README shows them: compiled and linked here, never run
   (the pointers would be device memory). */
int example_layer(const void* q, const void* k, const void* v, void* o, void* qh, void* kh, void* vh, void* oh,
                  double* pooled_q, double* pooled_k, int32_t* perm, int32_t* inv, fva_mask mask, void* ws,
                  size_t ws_bytes, int32_t* status, fva_stream_t stream) {
  fva_shape s = {1, 40, 128, 21, 45, 80, 64, FVA_BF16};
  int rc = fva_hilbert_perm(&s, perm, inv, stream);
  if (rc == FVA_OK) rc = fva_reorder(&s, q, qh, pooled_q, perm, FVA_FWD, stream);
  if (rc == FVA_OK) rc = fva_reorder(&s, k, kh, pooled_k, perm, FVA_FWD, stream);
  if (rc == FVA_OK) rc = fva_reorder(&s, v, vh, NULL, perm, FVA_FWD_F16, stream);
  if (rc == FVA_OK)
    rc = fva_route(&s, NULL, NULL, pooled_q, pooled_k, 0.9, 4, FVA_ORDER_HEAD_LPT, &mask, ws, ws_bytes, status, stream);
  if (rc == FVA_OK) rc = fva_sparse_attn(&s, qh, kh, vh, FVA_F16, &mask, oh, 0.0f, status, stream);
  if (rc == FVA_OK) rc = fva_reorder(&s, oh, o, NULL, perm, FVA_INV, stream);
  return rc;
}

int main(void) {
  fva_shape s = {1, 40, 128, 21, 45, 80, 64, FVA_BF16}; /* 720p: 75,600 tokens, nB = 1182 */
  if (fva_num_tokens(&s) != 75600) return 1;
  if (fva_num_blocks(&s) != 1182) return 2;
  if (fva_num_tiles(&s) != 40 * 591) return 3;
  if (fva_mask_capacity(&s) != 40LL * 1182 * 1182) return 4;
  if (fva_tile_capacity(&s) != 40LL * 591 * 1182) return 5;
  if (fva_route_workspace_bytes(&s, 0) == 0 || fva_tiles_workspace_bytes(&s) == 0) return 6;
  if (strcmp(fva_status_string(FVA_OK), "ok") != 0) return 7;

  fva_shape bad = s;
  bad.block = 32;
  if (fva_num_tokens(&bad) != -1 || fva_route_workspace_bytes(&bad, 1) != 0) return 8;

  /* RLB: loads 10, 1, 1, 1 over 2 ranks (rank 0: 11, rank 1: 2). Moving head 0 would make
     rank 1 the new maximum (12 > 11), so the heaviest paying move is head 1. */
  {
    double load[4] = {10.0, 1.0, 1.0, 1.0};
    int32_t rank_of[4];
    fva_rlb_move moves[2];
    int n = -1;
    if (fva_rlb_plan(load, 4, 2, 0.0, 0.0, 1.10, 1, rank_of, moves, 2, &n) != FVA_OK) return 9;
    if (n != 1 || moves[0].head != 1 || moves[0].from_rank != 0 || moves[0].to_rank != 1) return 10;
    if (moves[0].gain_ms != 1.0) return 11;
    if (rank_of[0] != 0 || rank_of[1] != 1 || rank_of[2] != 1 || rank_of[3] != 1) return 12;
    /* room for fewer than min(n_heads, n_ranks * max_per_rank) = 2 moves is refused */
    if (fva_rlb_plan(load, 4, 2, 0.0, 0.0, 1.10, 1, rank_of, moves, 1, &n) != FVA_ERR_CAPACITY) return 13;
    if (fva_rlb_plan(load, 4, 2, 0.0, 0.0, 0.5, 1, rank_of, moves, 2, &n) != FVA_ERR_INVALID_ARG) return 14;
  }
  /* SASA budgets: critical load 10; slack 1 and 5 clear n2 = 7%; floor(0.8 * slack / 0.5) */
  {
    double rank_load[3] = {10.0, 9.0, 5.0};
    int64_t budget[3] = {-1, -1, -1};
    if (fva_sasa_budgets(rank_load, 3, 0.5, 0.8, 0.07, budget) != FVA_OK) return 15;
    if (budget[0] != 0 || budget[1] != 1 || budget[2] != 8) return 16;
  }
  printf("c abi ok\n");
  return 0;
}
"""


def test_header_is_strict_c99_and_host_entry_points_run_from_c(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = os.path.join(PKG, "libfva.so")
    assert os.path.exists(lib), "libfva.so not built"
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-Wpedantic", "-Werror", "-I", INCLUDE, str(src), "-o", str(exe),
           "-L", PKG, "-lfva", f"-Wl,-rpath,{PKG}"]
    out = subprocess.run(cmd, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert run.stdout.strip() == "c abi ok"


def test_header_compiles_as_cpp17():
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "abi.cpp")
        with open(src, "w") as f:
            f.write('#include "fva.h"\nint main() { fva_shape s{}; return fva_num_tokens(&s) == -1 ? 0 : 1; }\n')
        out = subprocess.run([cxx, "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, "-fsyntax-only", src],
                             capture_output=True, text=True)
        assert out.returncode == 0, out.stderr


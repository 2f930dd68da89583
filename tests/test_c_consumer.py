"""The boundary from plain C: compile a C99 program against include/segpaged.h,
link it to libsegpaged.so and call the host-only entry points (no GPU, no
Python types).  Its numbers must match what the ctypes binding reports."""
from __future__ import annotations

import shutil
import subprocess
from pathlib import Path

import pytest

from head_aware_paged_build_b200 import segpaged as S

ROOT = Path(__file__).resolve().parent.parent

PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include "segpaged.h"

int main(void) {
  /* two sequences, 4 q-heads over 2 kv-heads, decode at the last token */
  int32_t ctx[2] = {300, 1000}, q0[2] = {299, 999};
  sp_head_policy pol[4] = {{SP_GLOBAL, 0, 0}, {SP_LOCAL, 4, 128}, {SP_LOCAL, 0, 64}, {SP_GLOBAL, 0, 0}};
  sp_problem p = {0};
  p.batch = 2; p.num_q_heads = 4; p.num_kv_heads = 2; p.head_dim = 128; p.page_size = 64;
  p.dtype = SP_BF16; p.ctx_len = ctx; p.q_start = q0; p.policy = pol; p.target_ctas = 5;
  sp_plan* plan = NULL;
  if (segpaged_plan_create(&p, &plan) != SP_OK) { printf("create: %s\n", segpaged_last_error()); return 1; }
  sp_sizes z;
  if (segpaged_plan_sizes(plan, &z) != SP_OK) return 2;
  int32_t n = 0;
  if (segpaged_plan_decode_items(plan, NULL, 0, &n) != SP_OK) return 3;
  int32_t* rec = (int32_t*)malloc(sizeof(int32_t) * SP_DECODE_ITEM_WORDS * (size_t)(n > 0 ? n : 1));
  if (segpaged_plan_decode_items(plan, rec, n, &n) != SP_OK) return 4;
  printf("%lld %lld %lld %lld %d %d\n", (long long)z.num_pages, (long long)z.stored_token_heads,
         (long long)z.workspace_bytes, (long long)z.table_bytes, z.num_decode_ctas, n);
  for (int32_t i = 0; i < n; ++i) {
    for (int k = 0; k < SP_DECODE_ITEM_WORDS; ++k) printf("%d ", rec[i * SP_DECODE_ITEM_WORDS + k]);
    printf("\n");
  }
  /* an invalid problem is refused with a status, not a crash */
  sp_problem bad = p;
  bad.head_dim = 96;
  sp_plan* none = NULL;
  const sp_status st = segpaged_plan_create(&bad, &none);
  printf("%d %s\n", (int)st, segpaged_status_string(st));
  free(rec);
  segpaged_plan_destroy(plan);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_program_links_and_matches_the_binding(tmp_path):
    lib_dir = ROOT / "head_aware_paged_build_b200"
    S.load()  # builds nothing; asserts the library exists
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", f"-I{ROOT / 'include'}", str(src),
                    f"-L{lib_dir}", "-lsegpaged", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    head = [int(x) for x in out[0].split()]
    n_items = head[5]
    c_items = [[int(x) for x in line.split()] for line in out[1:1 + n_items]]
    status_line = out[1 + n_items].split(maxsplit=1)

    pol = [("global", 0, 0), ("local", 4, 128), ("local", 0, 64), ("global", 0, 0)]
    prob = S.make_problem(2, 4, 2, 128, 64, "bf16", [300, 1000], [299, 999], pol, target_ctas=5)
    plan = S.segpaged_plan_create(prob)
    try:
        z = S.segpaged_plan_sizes(plan)
        items = S.segpaged_plan_decode_items(plan)
    finally:
        S.segpaged_plan_destroy(plan)
    assert head[:5] == [z.num_pages, z.stored_token_heads, z.workspace_bytes, z.table_bytes, z.num_decode_ctas]
    assert c_items == [[it[f] for f in S.DECODE_ITEM_FIELDS] for it in items]
    assert int(status_line[0]) == S.SP_ERR_UNSUPPORTED and status_line[1]

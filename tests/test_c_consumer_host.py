"""The C ABI from a plain C program: include/wf.h compiles as strict C99, the program links
against libwf_b200.so, and the calls that answer on the host (errors, sizes, the split plan)
return what the header states.  No GPU: every call here returns before device work."""
import os
import shutil
import subprocess

import pytest

from block_causal_streaming_b200 import build as wf_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_causal_streaming_b200")

PROGRAM = r"""
#include <stdio.h>
#include <stddef.h>
#include "wf.h"

#define CHECK(cond) do { if (!(cond)) { printf("failed: %s\n", #cond); return 1; } } while (0)

int main(void) {
  /* one context chunk of 64 keys, query chunks of 64 and 72 rows */
  int32_t offsets[] = {0, 64, 128, 200};
  int32_t stages[] = {0, 200, 1000};
  wf_wavefront_t wf = {3, 1, offsets, stages, 8};
  wf_kv_pool_t no_k = {NULL, (void*)0x10000, 8, 64, 2, 128};
  wf_kv_pool_t d96 = {(void*)0x10000, (void*)0x10000, 8, 64, 2, 96};
  const int32_t* pt = (const int32_t*)0x10000;
  void* buf = (void*)0x10000;
  size_t s8[6];
  int32_t parts = 0, tail = 0;

  CHECK(wf_version() >= 100);
  CHECK(wf_strerror(WF_OK) != NULL && wf_strerror(WF_ERR_SHAPE) != NULL);
  CHECK(wf_attn_forward(buf, &no_k, pt, &wf, 0.1f, buf, NULL, NULL) == WF_ERR_INVALID_ARG);
  CHECK(wf_attn_forward(buf, &d96, pt, &wf, 0.1f, buf, NULL, NULL) == WF_ERR_SHAPE);
  CHECK(wf_kv_append(&no_k, 0, 0, buf, buf, pt, &wf, NULL) == WF_ERR_INVALID_ARG);

  /* split workspace: S x T_q x H fp32 rows of D values plus one lse each, 256-byte rounded */
  CHECK(wf_attn_workspace_size(&wf, 2, 128, 1) == 0);
  CHECK(wf_attn_workspace_size(&wf, 2, 128, 2) ==
        (size_t)((2 * 136 * 2 * 128 * 4 + 255) / 256 * 256 + (2 * 136 * 2 * 4 + 255) / 256 * 256));

  /* the INT8 tier's buffers: codes one byte per element, scales per 128 rows */
  CHECK(wf_qk_i8_sizes(&wf, 2, 128, s8) == WF_OK);
  CHECK(s8[0] == 136 * 2 * 128 && s8[1] == 2 * 2 * 4 && s8[2] == 200 * 2 * 128 &&
        s8[3] == 2 * 2 * 4 && s8[4] == 2 * 128 * 4 && s8[5] == 2 * 128 * 8);
  CHECK(wf_qk_i8_sizes(&wf, 2, 64, s8) == WF_ERR_SHAPE);

  /* an explicit split count is used as given; a 4-unit grid on 148 SMs is split */
  CHECK(wf_attn_split_plan(&wf, 2, 2, 148, &parts, &tail) == WF_OK && parts == 2 && tail == 0);
  CHECK(wf_attn_split_plan(&wf, 2, 0, 148, &parts, &tail) == WF_OK && parts >= 1);
  CHECK(wf_attn_split_plan(&wf, 2, -1, 148, &parts, &tail) == WF_ERR_INVALID_ARG);
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_links_and_gets_host_answers(tmp_path):
    wf_build.build()
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-L", PKG, "-lwf_b200",
                    f"-Wl,-rpath,{PKG}", "-o", str(exe)], check=True)
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")        # host answers only
    run = subprocess.run([str(exe)], capture_output=True, text=True, env=env, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.strip().endswith("ok")

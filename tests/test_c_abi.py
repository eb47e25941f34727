"""bd.h is a C header and libbd.so a C library: a plain C99 program compiles
against the header with every warning an error, links the library, and calls
the entry points that need no GPU (version, status strings, host-side
validation, sizes of an empty call). On a GPU machine the same program runs the
same host-only calls."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_diffusion_lm_bd_b200")

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "bd.h"

static int check(const char *what, bd_status got, bd_status want) {
  if (got != want) {
    printf("%s: got %s, want %s\n", what, bd_status_string(got), bd_status_string(want));
    return 1;
  }
  return 0;
}

int main(void) {
  int bad = 0;
  char buf[64];
  float logits[4], conf[1];
  int32_t tok[1], draft[1], n_accept[1];
  uint8_t mask[1], commit[1];
  if (bd_version() < 100) bad |= 1;
  if (strcmp(bd_status_string(BD_ERR_TIMEOUT), "BD_ERR_TIMEOUT") != 0) bad |= 1;
  /* host-side validation: nothing is launched */
  bad |= check("attn d=96", bd_attn_step(buf, buf, buf, 1, buf, buf, (const int32_t *)buf,
                                         (const int64_t *)buf, 1, 16, 8, 2, 96, 0.f,
                                         BD_DTYPE_BF16, (float *)buf, NULL, buf, 1 << 20, NULL),
               BD_ERR_UNSUPPORTED);
  bad |= check("attn_ex flags", bd_attn_step_ex(buf, buf, buf, 1, buf, buf, (const int32_t *)buf,
                                                (const int64_t *)buf, 1, 16, 8, 2, 64, 0.f,
                                                BD_DTYPE_BF16, (float *)buf, NULL, buf, 1 << 20,
                                                4, NULL),
               BD_ERR_INVALID_ARG);
  bad |= check("unmask rows<0", bd_unmask(logits, mask, 0.9f, tok, conf, commit, NULL, -1, 4, 0, 0,
                                          buf, sizeof buf, NULL),
               BD_ERR_INVALID_ARG);
  bad |= check("unmask empty", bd_unmask(logits, mask, 0.9f, tok, conf, commit, NULL, 0, 4, 0, 0,
                                         buf, sizeof buf, NULL),
               BD_OK);
  bad |= check("append d=96", bd_kv_append(buf, buf, 1, buf, buf, (int32_t *)buf,
                                           (const int64_t *)buf, (const int64_t *)buf, NULL, 1, 1,
                                           1, 96, BD_DTYPE_F32, NULL),
               BD_ERR_UNSUPPORTED);
  bad |= check("lmhead D=96", bd_lmhead_unmask(buf, buf, mask, 0.9f, tok, conf, commit, NULL, 1, 8,
                                               96, 0, 0, buf, 1 << 20, NULL),
               BD_ERR_UNSUPPORTED);
  bad |= check("mamba P=48", bd_mamba_block_scan(logits, logits, logits, logits, logits, logits,
                                                 logits, logits, logits, logits, logits, logits, 1,
                                                 4, 2, 48, 32, 1, NULL),
               BD_ERR_UNSUPPORTED);
  bad |= check("verify S=0", bd_spec_verify(logits, draft, tok, conf, commit, n_accept, 1, 4, 0,
                                             buf, sizeof buf, NULL),
               BD_ERR_INVALID_ARG);
  printf(bad ? "FAIL\n" : "OK\n");
  return bad;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_header_is_c99_and_the_library_links(tmp_path):
    from block_diffusion_lm_bd_b200 import build

    build.build()
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
          str(src), "-L", PKG, "-lbd", f"-Wl,-rpath,{PKG}", "-o", str(exe)]
    r = subprocess.run(cc, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr

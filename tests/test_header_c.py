"""The C ABI is plain C: a C99 program that includes include/deltalog.h
compiles warning-free, links against libdeltalog.so and gets DL_ERR_ARG back
from every entry point given a NULL handle (no device is touched)."""
import os
import shutil
import subprocess

import pytest

from recurrent_state_update_deltalog_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "deltalog.h"

#define EXPECT(call, want)                                                    \
  do {                                                                        \
    int rc_ = (call);                                                         \
    if (rc_ != (want)) {                                                      \
      printf("FAIL %s -> %d (want %d): %s\n", #call, rc_, (int)(want),        \
             dl_last_error());                                                \
      return 1;                                                               \
    }                                                                         \
  } while (0)

int main(void) {
  dl_t h = NULL;
  float f = 0.f;
  int i = 0;
  const void* p = &f;
  EXPECT(dl_create(NULL, 1, 1, 64, 64, 8, DL_GDN, DL_BF16), DL_ERR_ARG);
  EXPECT(dl_create(&h, 1, 1, 64, 64, -1, DL_GDN, DL_BF16), DL_ERR_UNSUPPORTED);
  EXPECT(dl_suggest_m(DL_GDN, 128, 128, DL_BF16, &i), DL_OK);
  if (i < 2 || i > DL_MAX_M) { printf("FAIL suggest_m %d\n", i); return 1; }
  EXPECT(dl_merge_interval(h, &i), DL_ERR_ARG);
  EXPECT(dl_load_state(h, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_set_bonus(h, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_step(h, p, p, p, &f, &f, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_step_indexed(h, &i, 1, p, p, p, &f, &f, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_prefill(h, NULL, 1, &i, 1LL, DL_PREFILL_ZERO_STATE, p, p, p, &f, &f, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_step_host(h, p, p, p, &f, &f, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_eager_step(h, p, p, p, &f, &f, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_eager_step_indexed(h, &i, 1, p, p, p, &f, &f, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_merge(h, NULL), DL_ERR_ARG);
  EXPECT(dl_read_state(h, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_set_option(h, DL_OPT_PDL, 1), DL_ERR_ARG);
  EXPECT(dl_last_step_kernel(h, &i), DL_ERR_ARG);
  EXPECT(dl_log_len(h, &i), DL_ERR_ARG);
  EXPECT(dl_slot_load(h, 0, NULL, NULL), DL_ERR_ARG);
  EXPECT(dl_slot_merge(h, 0, NULL), DL_ERR_ARG);
  EXPECT(dl_slot_read(h, 0, &f, NULL), DL_ERR_ARG);
  EXPECT(dl_check_device(h, NULL), DL_ERR_ARG);
  EXPECT(dl_destroy(NULL), DL_OK);
  if (!dl_strerror(DL_ERR_STATE)[0]) return 1;
  printf("ok %s\n", dl_strerror(DL_OK));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_abi_rejects_null_handles(tmp_path):
    build()
    src = tmp_path / "abi.c"
    exe = tmp_path / "abi"
    src.write_text(PROGRAM)
    libdir = os.path.dirname(LIB)
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
          str(src), "-o", str(exe), "-L", libdir, "-ldeltalog", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cc, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr

"""The C ABI from C: include/h3.h compiles as C99 and libh3.so links and runs.

A small C program (no GPU needed) includes the header, links the library and
exercises the calls that validate arguments on the host: version, status
strings, workspace sizing, and the rejection of bad segment tables and rope
configurations before any launch.
"""
import os
import shutil
import subprocess

import pytest

from packed_mm_rope_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "h3.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAILED: %s (line %d)\n", #cond, __LINE__); return 1; } } while (0)

int main(void) {
  CHECK(h3_version() == 101);
  CHECK(strcmp(h3_status_str(H3_OK), "ok") == 0);
  CHECK(strcmp(h3_status_str(12345), "unknown status") == 0);
  CHECK(h3_host_workspace_bytes(100, 2) == 4 * 51200 + 1280 + 512);
  CHECK(h3_host_workspace_bytes(0, 2) == 0);

  h3_segment text;
  memset(&text, 0, sizeof(text));
  text.kind = H3_SEG_TEXT;
  text.count = 4;
  text.t_step_num = 1;
  text.t_den = 1;
  /* the row count must match the table; a zero denominator is rejected */
  CHECK(h3_build_coords(&text, 1, NULL, 5, (float*)0x1000, NULL) == H3_ERR_INVALID_ARG);
  text.t_den = 0;
  CHECK(h3_build_coords(&text, 1, NULL, 4, (float*)0x1000, NULL) == H3_ERR_INVALID_ARG);
  /* an empty problem is a no-op */
  text.t_den = 1;
  text.count = 0;
  CHECK(h3_build_coords(&text, 1, NULL, 0, NULL, NULL) == H3_OK);

  h3_rope_cfg cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.theta = 10000.0;
  cfg.head_dim = 128;
  cfg.sec_t = 32;
  cfg.sec_h = 48;
  cfg.sec_w = 48;
  CHECK(h3_mmrope_qk(NULL, NULL, NULL, NULL, NULL, 0, 1, 128, &cfg, NULL) == H3_OK);
  cfg.freq_rule = 2;
  CHECK(h3_mmrope_qk(NULL, NULL, NULL, NULL, NULL, 0, 1, 128, &cfg, NULL) == H3_ERR_INVALID_ARG);
  cfg.freq_rule = 1;
  cfg.sec_w = 46;
  CHECK(h3_mmrope_qk(NULL, NULL, NULL, NULL, NULL, 0, 1, 128, &cfg, NULL) == H3_ERR_INVALID_ARG);

  /* attention: head_dim other than 128 is unsupported, zero heads invalid */
  CHECK(h3_packed_attention((void*)0x10000, (void*)0x10000, (void*)0x10000, (void*)0x10000, NULL, NULL, NULL,
                            1, 10, 1, 64, 128, 0.f, NULL) == H3_ERR_UNSUPPORTED);
  CHECK(h3_packed_attention((void*)0x10000, (void*)0x10000, (void*)0x10000, (void*)0x10000, NULL, NULL, NULL,
                            1, 10, 0, 128, 128, 0.f, NULL) == H3_ERR_INVALID_ARG);
  printf("ok\n");
  return 0;
}
"""


def test_header_compiles_as_c99_and_links():
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    if not os.path.exists(_lib.LIB_PATH):
        pytest.skip("libh3.so not built")
    import tempfile
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "use_h3.c")
        exe = os.path.join(tmp, "use_h3")
        with open(src, "w") as f:
            f.write(C_PROGRAM)
        r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                            os.path.join(ROOT, "include"), src, "-o", exe, "-L", lib_dir, "-lh3",
                            "-Wl,-rpath," + lib_dir], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr

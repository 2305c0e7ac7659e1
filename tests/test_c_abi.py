"""include/gdit.h is a plain C ABI: a C99 program that includes it compiles
warning-free with gcc, links against libgdit.so and calls the entry points
that need no GPU (CPU only)."""

import ctypes
import os
import shutil
import subprocess

import pytest

from flow_matching_dit_b200.build import HEADER, LIB, build

PROGRAM = r"""
#include <stddef.h>
#include <stdio.h>
#include <string.h>
#include "gdit.h"

#define FIELD(T, f) printf(#T "." #f " %d\n", (int)offsetof(T, f))

int main(void) {
  gdit_config cfg;
  gdit_handle* h = (gdit_handle*)1;
  int rc;
  if (strncmp(gdit_version(), "gdit", 4) != 0) return 1;
  if (strcmp(gdit_strerror(GDIT_EINVAL), "invalid argument") != 0) return 2;
  memset(&cfg, 0, sizeof cfg);
  cfg.num_layers = 3;                                   /* odd: rejected on the host */
  rc = gdit_create(&cfg, NULL, 0, &h);
  if (rc != GDIT_EINVAL || h != NULL) return 3;
  if (strstr(gdit_last_error(NULL), "num_layers") == NULL) return 4;
  if (gdit_get_action(NULL, NULL, GDIT_BF16, NULL, NULL, NULL, NULL, 4, NULL, 1, 1, NULL) != GDIT_EINVAL) return 5;
  if (gdit_sync_status(NULL) != GDIT_EINVAL) return 6;
  gdit_destroy(NULL);
  printf("sizeof.gdit_config %d\n", (int)sizeof(gdit_config));
  printf("sizeof.gdit_tensor %d\n", (int)sizeof(gdit_tensor));
  printf("sizeof.gdit_kernel_stat %d\n", (int)sizeof(gdit_kernel_stat));
  FIELD(gdit_config, num_layers); FIELD(gdit_config, max_batch); FIELD(gdit_config, num_timestep_buckets);
  FIELD(gdit_config, ln_eps); FIELD(gdit_config, flags); FIELD(gdit_config, device);
  FIELD(gdit_config, attend_text_every_n_blocks);
  FIELD(gdit_tensor, name); FIELD(gdit_tensor, dtype); FIELD(gdit_tensor, ndim); FIELD(gdit_tensor, shape);
  FIELD(gdit_tensor, host_ptr);
  FIELD(gdit_kernel_stat, name); FIELD(gdit_kernel_stat, launches); FIELD(gdit_kernel_stat, total_ms);
  FIELD(gdit_kernel_stat, flops); FIELD(gdit_kernel_stat, bytes);
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_is_plain_c_and_the_library_links():
    build()
    work = os.path.join(os.path.dirname(LIB), os.pardir, "_build", "c_abi_test")
    os.makedirs(work, exist_ok=True)
    src = os.path.join(work, "abi.c")
    with open(src, "w") as f:
        f.write(PROGRAM)
    exe = os.path.join(work, "abi")
    inc = os.path.dirname(HEADER)
    libdir = os.path.dirname(LIB)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", inc, src, "-o", exe,
           "-L", libdir, "-l:libgdit.so", "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    lines = r.stdout.split()
    assert lines[-1] == "ok"
    c_layout = dict(zip(lines[:-1:2], map(int, lines[1:-1:2])))
    # the ctypes declarations of the binding must match the C compiler's layout
    from flow_matching_dit_b200 import _lib
    for name in ("gdit_config", "gdit_tensor", "gdit_kernel_stat"):
        T = getattr(_lib, name)
        assert ctypes.sizeof(T) == c_layout["sizeof." + name], name
        for key, off in c_layout.items():
            if key.startswith(name + "."):
                assert getattr(T, key.split(".")[1]).offset == off, key

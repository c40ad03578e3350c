"""The C ABI is C: a C99 program that includes include/ws.h, takes the address of
every function the header declares and calls the host-only ones compiles with
-Wall -Werror, links against libws.so and runs without a GPU."""
import os
import shutil
import subprocess

import pytest

from kv_cache_serving_ws_b200 import native as ws

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_include():
    for d in ("/usr/local/cuda/include", os.path.join(os.environ.get("CUDA_HOME", ""), "include")):
        if d and os.path.exists(os.path.join(d, "cuda_runtime_api.h")):
            return d
    return None


@pytest.mark.skipif(shutil.which("gcc") is None or _cuda_include() is None, reason="needs gcc and the CUDA headers")
def test_header_is_c99_and_links(tmp_path):
    ws.lib()                                               # builds must exist: no fallback
    names = ws.header_symbols()
    src = ['#include <stdio.h>', '#include <string.h>', '#include "ws.h"', "", "int main(void) {",
           "  const void* fns[] = {"]
    src += [f"    (const void*)&{n}," for n in names]
    src += ["  };",
            f"  if (sizeof(fns) / sizeof(fns[0]) != {len(names)}) return 2;",
            "  for (unsigned i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i) if (!fns[i]) return 3;",
            "  ws_cache_config cfg;",
            "  memset(&cfg, 0, sizeof cfg);",
            "  ws_cache_t* h = NULL;",
            "  if (ws_cache_create(&h, NULL, NULL) != WS_ERR_ARG) return 4;",      # rejected before any CUDA call
            "  if (ws_plan_visible(&cfg, NULL, NULL, 0, 0, NULL, NULL, 0, NULL) != WS_ERR_ARG) return 5;",
            '  printf("%s|%s\\n", ws_status_string(WS_OK), ws_status_string(WS_ERR_EVICTED));',
            "  return 0;", "}"]
    c = tmp_path / "abi.c"
    c.write_text("\n".join(src) + "\n")
    exe = tmp_path / "abi"
    lib_dir = os.path.join(ROOT, "kv_cache_serving_ws_b200")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I",
           _cuda_include(), str(c), "-o", str(exe), "-L", lib_dir, "-lws", f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.strip() == f"{ws.status_string(0)}|{ws.status_string(ws.WS_ERR_EVICTED)}"

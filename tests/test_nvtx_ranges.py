"""Every scoring and selection entry point of the C ABI opens an NVTX range
named after itself (balanced push / pop), so that a timeline tool can
attribute the kernels to the call.  Checked on the CPU: a small NVTX injection
library, built here, records the ranges of calls that the host rejects before
any device work."""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

# an NVTX v3 injection library: InitializeInjectionNvtx2 receives the export
# table and points the core module's RangePushA / RangePop slots at loggers
INJECTION_C = r"""
#include <stdio.h>
#include <stdlib.h>
#include <nvtx3/nvToolsExt.h>

static FILE* g_log;

static int log_push(const char* name) {
  if (g_log) { fprintf(g_log, "push %s\n", name); fflush(g_log); }
  return 0;
}

static int log_pop(void) {
  if (g_log) { fprintf(g_log, "pop\n"); fflush(g_log); }
  return 0;
}

int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks* cb =
      (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size)) return 0;
  if (size <= NVTX_CBID_CORE_RangePop) return 0;
  g_log = fopen(getenv("DROPKV_NVTX_LOG"), "w");
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)log_push;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)log_pop;
  return 1;
}
"""

# calls the host rejects (null shape, B = 0, no status pointer): no device work
CALLS = r"""
import ctypes, sys
sys.path.insert(0, sys.argv[1])
import kv_cache_eviction_scores_b200 as dk
L = dk.lib()
shape = dk.Shape(1, 4, 2, 64, 8, 2, 1, 1)
fake = ctypes.c_void_p(0x100000)
res = [
    L.dropkv_scores(None, fake, fake, fake, None, fake, fake, 1 << 20, None),
    L.dropkv_scores_async(ctypes.byref(shape), fake, fake, fake, None, fake, fake, 1 << 20,
                          None, None),
    L.dropkv_scores_ex(None, fake, fake, fake, None, fake, fake, 1 << 20, None, None, None),
    L.dropkv_scores_select(None, fake, fake, fake, None, None, fake, fake, 1, fake, 1, fake,
                           1 << 20, None, None, None),
    L.dropkv_select(0, 1, 64, fake, None, None, fake, 1, fake, 1, fake, 1 << 20, None),
    L.dropkv_select_ex(0, 1, 64, fake, None, None, fake, 1, fake, 1, fake, 1 << 20, None, None),
    L.dropkv_select_noalloc(0, 1, 64, fake, None, None, fake, 1, fake, 1, None),
]
assert all(r == dk.ERR_ARG for r in res), res
print("ok")
"""

ENTRY_POINTS = ["dropkv_scores", "dropkv_scores_async", "dropkv_scores_ex", "dropkv_scores_select",
                "dropkv_select", "dropkv_select_ex", "dropkv_select_noalloc"]


def test_entry_points_open_named_nvtx_ranges(tmp_path):
    if shutil.which("gcc") is None or not os.path.exists(
            os.path.join(CUDA_INC, "nvtx3", "nvToolsExt.h")):
        pytest.skip("needs gcc and the NVTX3 headers")
    src = tmp_path / "inject.c"
    src.write_text(INJECTION_C)
    so = tmp_path / "libinject.so"
    subprocess.run(["gcc", "-shared", "-fPIC", "-O1", "-I", CUDA_INC, str(src), "-o", str(so)],
                   check=True)
    log = tmp_path / "ranges.log"
    env = dict(os.environ, NVTX_INJECTION64_PATH=str(so), DROPKV_NVTX_LOG=str(log))
    out = subprocess.run([sys.executable, "-c", CALLS, ROOT], env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0 and "ok" in out.stdout, out.stderr[-2000:]
    lines = log.read_text().splitlines()
    pushes = [ln.split(" ", 1)[1] for ln in lines if ln.startswith("push ")]
    assert pushes == ENTRY_POINTS
    # each call's range is closed before the next opens
    assert lines == [x for name in ENTRY_POINTS for x in (f"push {name}", "pop")]

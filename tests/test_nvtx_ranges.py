"""Each C-ABI call opens one NVTX range named after itself and closes it on every
return path.  A profiler can therefore attribute kernels to calls, or capture one
call's kernels only.

NVTX v3 hands its calls to a tool library named by NVTX_INJECTION64_PATH.  This test
builds a minimal tool of that kind with gcc, from the callback interface NVTX v3
publishes: it appends every range push and pop to a log.  A child process loads
libduo.so with that tool and makes each call.  Launches are skipped by the dry-run
launch control, and the buffer is a fake address, so no GPU is needed.
"""
import os
import shutil
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

TOOL_C = r"""
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

/* the NVTX v3 injection interface: export table 1 (callbacks) hands out the function
   table of a module; module 1 (core) slot 9 is RangePushA, slot 11 RangePop */
typedef void (*fn_t)(void);
typedef fn_t **table_t;
typedef struct {
  size_t struct_size;
  int (*get_module_function_table)(int module, table_t *table, unsigned int *size);
} callbacks_t;
typedef const void *(*get_export_table_t)(uint32_t id);

static FILE *log_file;

static int range_push_a(const char *name) {
  fprintf(log_file, "push %s\n", name ? name : "");
  fflush(log_file);
  return 0;
}
static int range_pop(void) {
  fprintf(log_file, "pop\n");
  fflush(log_file);
  return 0;
}

int InitializeInjectionNvtx2(get_export_table_t get) {
  const callbacks_t *cb = (const callbacks_t *)get(1);
  table_t table = 0;
  unsigned int size = 0;
  if (!cb || !cb->get_module_function_table(1, &table, &size) || size < 11) return 0;
  log_file = fopen(getenv("DUO_TEST_NVTX_LOG"), "a");
  if (!log_file) return 0;
  *table[9] = (fn_t)range_push_a;
  *table[11] = (fn_t)range_pop;
  return 1;
}
"""

CHILD = textwrap.dedent("""
    import ctypes
    import numpy as np
    from head_split_kv_duo_b200 import duo

    FAKE = 1 << 40
    assert duo.duo_debug_launch_controls(1, -1) == duo.DUO_OK  # launches skipped
    mask = np.array([[1, 0, 1, 0]], dtype=np.uint8)
    opts = duo._opts(batch=1, q_heads=8)
    need = duo.duo_cache_bytes(1, 4, 128, mask, 4, 16, 1000, opts)
    st, h = duo.duo_cache_create(1, 4, 128, mask, 4, 16, 1000, opts, FAKE, need)
    assert st == duo.DUO_OK
    assert duo.duo_append_kv(h, 0, FAKE, FAKE, 10) == duo.DUO_OK
    assert duo.duo_prefill_chunk(h, 0, FAKE, FAKE, FAKE, 5, FAKE, None) == duo.DUO_OK
    assert duo.duo_decode_attention(h, 0, FAKE, FAKE, None) == duo.DUO_OK
    assert duo.duo_append_decode(h, 0, FAKE, FAKE, FAKE, FAKE, None) == duo.DUO_OK
    assert duo.duo_get_device_status(h) == duo.DUO_OK
    assert duo.duo_decode_attention(h, 5, FAKE, FAKE, None) == duo.DUO_ERR_INVALID  # an early return
    f = duo.lib().duo_decode_attention_static_scratch
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert f(None, 0, None, None, None, None) == duo.DUO_ERR_INVALID
    duo.duo_cache_destroy(h)
    pneed = duo.duo_pool_bytes(1, 4, 128, mask, 4, 16, 2, 1000, 8, opts)
    st, P = duo.duo_pool_create(1, 4, 128, mask, 4, 16, 2, 1000, 8, opts, FAKE, pneed)
    assert st == duo.DUO_OK
    st, s = duo.duo_pool_open(P)
    assert st == duo.DUO_OK
    assert duo.duo_pool_append_kv(P, 0, s, FAKE, FAKE, 3) == duo.DUO_OK
    assert duo.duo_pool_decode_step(P, 0, 1, [s], FAKE, FAKE, FAKE, FAKE, None) == duo.DUO_OK
    assert duo.duo_pool_device_status(P) == duo.DUO_OK
    duo.duo_pool_destroy(P)
    assert duo.duo_gated_attention(FAKE, FAKE, FAKE, 1, 100, 4, 2, 64, duo.DUO_FP32, FAKE, 2, 8, 0.0, FAKE) == duo.DUO_OK
    print("calls done")
""")

CALLS = ["duo_cache_create", "duo_append_kv", "duo_prefill_chunk", "duo_decode_attention", "duo_append_decode",
         "duo_get_device_status", "duo_decode_attention_static_scratch", "duo_pool_create", "duo_pool_open",
         "duo_pool_append_kv", "duo_pool_decode_step", "duo_pool_device_status", "duo_gated_attention"]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc builds the NVTX tool library")
def test_every_call_has_one_balanced_nvtx_range(tmp_path):
    src = tmp_path / "tool.c"
    src.write_text(TOOL_C)
    lib = tmp_path / "libtool.so"
    subprocess.run(["gcc", "-shared", "-fPIC", "-O1", "-o", str(lib), str(src)], check=True)
    log = tmp_path / "nvtx.log"
    log.write_text("")
    env = dict(os.environ, NVTX_INJECTION64_PATH=str(lib), DUO_TEST_NVTX_LOG=str(log), PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "calls done" in r.stdout, r.stderr[-2000:]
    # replay the log: every push of a duo_ range is closed by a pop, innermost first
    stack, seen = [], []
    for line in log.read_text().splitlines():
        if line.startswith("push "):
            stack.append(line[5:])
            if line[5:].startswith("duo_"):
                seen.append(line[5:])
        else:
            assert line == "pop" and stack, line
            stack.pop()
    assert not [n for n in stack if n.startswith("duo_")], stack
    for name in CALLS:
        assert name in seen, (name, seen)
    # one range per top-level call: the two decode_attention calls, and nothing named twice otherwise
    assert seen.count("duo_decode_attention") >= 2
    assert seen.count("duo_cache_create") == 1 and seen.count("duo_pool_decode_step") == 1

"""Host-side caching rules of the launchers (csrc/device_cache.h), built with
g++ against fake device calls: one shared-memory opt-in per (device, context,
kernel) and a new one for more bytes, an SM count per device, device-array
addresses looked up again after a context change (cudaDeviceReset), and the
table limits.  No GPU is needed."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "block_sparse_attention_logits_b200", "csrc")

PROGRAM = r"""
#include <cassert>
#include <cstdio>
#include "device_cache.h"

static int g_dev = 0;                 // current device
static int g_ctx_id[4] = {1, 2, 3, 4};  // current context of each device (0: none yet)
static int g_set_calls = 0, g_sm_calls = 0, g_sym_calls = 0;
static size_t g_last_bytes = 0;
static int g_sym_gen = 0;             // addresses move when a context is rebuilt

static int get_device(int* d) { *d = g_dev; return 0; }
static void* current_ctx() {
  return g_ctx_id[g_dev] ? reinterpret_cast<void*>(static_cast<size_t>(0x1000 * g_ctx_id[g_dev])) : nullptr;
}
static int set_smem(const void*, size_t b) {
  ++g_set_calls; g_last_bytes = b;
  if (!g_ctx_id[g_dev]) g_ctx_id[g_dev] = 9 + g_dev;  // the call makes a primary context current
  return 0;
}
static int sm_count(int d, int* n) { ++g_sm_calls; *n = 100 + d; return 0; }
static int symbol_address(const void*, void** a) {
  ++g_sym_calls;
  *a = reinterpret_cast<void*>(static_cast<size_t>(0x100000 * (1 + g_dev) + 0x10 * g_ctx_id[g_dev] + g_sym_gen));
  return 0;
}

int main() {
  const bsa::DeviceOps ops = {get_device, current_ctx, set_smem, sm_count, symbol_address, 101, 999};
  static bsa::DeviceCache<4, 2, 2> c;
  int k1 = 0, k2 = 0, k3 = 0, s1 = 0, s2 = 0, s3 = 0;

  // opt-in: once per (device, context, kernel); again for more bytes, not for fewer
  assert(c.smem_opt_in(ops, &k1, 100000) == 0 && g_set_calls == 1);
  assert(c.smem_opt_in(ops, &k1, 100000) == 0 && g_set_calls == 1);
  assert(c.smem_opt_in(ops, &k1, 60000) == 0 && g_set_calls == 1);
  assert(c.smem_opt_in(ops, &k1, 200000) == 0 && g_set_calls == 2 && g_last_bytes == 200000);
  assert(c.smem_opt_in(ops, &k2, 100000) == 0 && g_set_calls == 3);
  g_dev = 1;                                           // a second device: its own entries
  assert(c.smem_opt_in(ops, &k1, 60000) == 0 && g_set_calls == 4 && g_last_bytes == 60000);
  assert(c.smem_opt_in(ops, &k1, 60000) == 0 && g_set_calls == 4);
  g_dev = 0;
  assert(c.smem_opt_in(ops, &k1, 200000) == 0 && g_set_calls == 4);  // device 0 kept its entry
  g_ctx_id[0] = 5;                                     // device 0 reset: a new context
  assert(c.smem_opt_in(ops, &k1, 60000) == 0 && g_set_calls == 5 && g_last_bytes == 60000);
  assert(c.smem_opt_in(ops, &k1, 100000) == 0 && g_set_calls == 6);  // the new context holds 60000 only
  assert(c.smem_opt_in(ops, &k3, 100000) == 999);      // a third kernel: the table holds two per device
  g_dev = 2; g_ctx_id[2] = 0;                          // no context yet: set, then remember the new one
  assert(c.smem_opt_in(ops, &k1, 100000) == 0 && g_set_calls == 7);
  assert(c.smem_opt_in(ops, &k1, 100000) == 0 && g_set_calls == 7);
  g_dev = 7;
  assert(c.smem_opt_in(ops, &k1, 100000) == 101);      // ordinal outside the table

  // SM count: read once per device
  int n = 0;
  g_dev = 0; assert(c.sm_count(ops, &n) == 0 && n == 100 && g_sm_calls == 1);
  assert(c.sm_count(ops, &n) == 0 && n == 100 && g_sm_calls == 1);
  g_dev = 1; assert(c.sm_count(ops, &n) == 0 && n == 101 && g_sm_calls == 2);

  // device-array addresses: per device, looked up again after a context change
  void* a = nullptr; void* b = nullptr;
  g_dev = 0; assert(c.symbol_address(ops, &s1, &a) == 0 && g_sym_calls == 1);
  assert(c.symbol_address(ops, &s1, &b) == 0 && b == a && g_sym_calls == 1);
  g_dev = 1; assert(c.symbol_address(ops, &s1, &b) == 0 && b != a && g_sym_calls == 2);
  g_dev = 0; g_ctx_id[0] = 6; g_sym_gen = 8;          // reset: the array moved
  assert(c.symbol_address(ops, &s1, &b) == 0 && b != a && g_sym_calls == 3);
  assert(c.symbol_address(ops, &s2, &b) == 0 && g_sym_calls == 4);
  assert(c.symbol_address(ops, &s3, &b) == 999);       // two symbols per table
  std::printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_device_cache_rules(tmp_path):
    src = tmp_path / "t.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "t"
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", f"-I{CSRC}", str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"

"""CPU checks of the C ABI: the library loads, exports every entry point include/s3r.h
declares, and rejects bad arguments on the host (nothing is launched without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "s3r.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^S3R_API\s+[\w\s\*]+?\b(s3r_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_hot_path():
    syms = declared_symbols()
    for name in ("s3r_select_kv", "s3r_sparse_draft_attn", "s3r_verify_attn", "s3r_spec_sample",
                 "s3r_draft_sample", "s3r_commit", "s3r_workspace_size", "s3r_get_error"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    import sparse_dense_kv_b200 as s3r
    raw = ctypes.CDLL(s3r.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(raw, n)]
    assert not missing, missing


def test_status_strings_and_counter():
    import sparse_dense_kv_b200 as s3r
    for code, name in s3r.STATUS_NAMES.items():
        assert s3r.s3r_status_string(code)
    assert s3r.s3r_status_string(99) == "unknown status"
    assert s3r.s3r_launch_count() >= 0


def _cache(**kw):
    import sparse_dense_kv_b200 as s3r
    d = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16, num_pages=1000,
             k_pool=0x100000, v_pool=0x200000)
    d.update(kw)
    return s3r.KVCacheDesc(**d)


def test_workspace_size_is_host_only_and_monotone():
    import sparse_dense_kv_b200 as s3r
    c = _cache()
    a = s3r.s3r_workspace_size(c, 32, 1540, 6, 151936, 1232)
    b = s3r.s3r_workspace_size(c, 64, 1540, 6, 151936, 1232)
    assert 0 < a < b
    assert s3r.s3r_workspace_size(c, 32, 1540, 8, 151936, 1232) >= a
    with pytest.raises(s3r.S3RError):
        s3r.s3r_workspace_size(_cache(head_dim=96), 32, 1540, 6, 151936, 1232)


def test_host_validation_rejects_before_launch():
    import sparse_dense_kv_b200 as s3r
    L = s3r.lib
    null = ctypes.c_void_p(0)
    # NULL descriptors
    assert L.s3r_verify_attn(None, None, 6, null, null, null, null, null, null, null, 0, null) == 1
    b = s3r.BatchDesc(1, 1, None, 0x1000, 0x2000, 10)
    # unsupported head_dim / page size / group / k
    for bad in (_cache(head_dim=96), _cache(page_size=32), _cache(num_q_heads=72, num_kv_heads=8)):
        assert L.s3r_verify_attn(ctypes.byref(bad), ctypes.byref(b), 6, 0x10, 0x10, 0x10, 0x10,
                                 0x10, None, 0x100, 1 << 20, null) == 2
    c = _cache()
    assert L.s3r_verify_attn(ctypes.byref(c), ctypes.byref(b), 9, 0x10, 0x10, 0x10, 0x10, 0x10,
                             None, 0x100, 1 << 20, null) == 2
    # misaligned q
    assert L.s3r_verify_attn(ctypes.byref(c), ctypes.byref(b), 6, 0x18, 0x10, 0x10, 0x10, 0x10,
                             None, 0x100, 1 << 20, null) == 1
    # workspace too small / misaligned
    assert L.s3r_verify_attn(ctypes.byref(c), ctypes.byref(b), 6, 0x10, 0x10, 0x10, 0x10, 0x10,
                             None, 0x100, 16, null) == 4
    assert L.s3r_verify_attn(ctypes.byref(c), ctypes.byref(b), 6, 0x10, 0x10, 0x10, 0x10, 0x10,
                             None, 0x180, 1 << 30, null) == 4
    # selection: budget and window
    assert L.s3r_select_kv(ctypes.byref(c), ctypes.byref(b), 0x10, 0x10, 6, 0, 64, 0x10, 100,
                           0x10, 0x100, 1 << 30, null) == 1
    assert L.s3r_select_kv(ctypes.byref(c), ctypes.byref(b), 0x10, 0x10, 6, 500, 6, 0x10, 100,
                           0x10, 0x100, 1 << 30, null) == 1
    # sampling: vocabulary and k
    assert L.s3r_spec_sample(ctypes.byref(b), 9, 0x10, 0x10, 0x10, 64, 1, 0x10, 0x10, None, None,
                             0x100, 1 << 30, null) == 2
    assert L.s3r_draft_sample(ctypes.byref(b), 0x10, 6, 0x10, 0, 1, 0x10, None, None, 0x100, 1 << 30,
                              null) == 2
    # a misaligned margins output
    assert L.s3r_spec_sample(ctypes.byref(b), 6, 0x10, 0x10, 0x10, 64, 1, 0x10, 0x10, 0x11, None,
                             0x100, 1 << 30, null) == 1
    assert L.s3r_draft_sample(ctypes.byref(b), 0x10, 6, 0x10, 64, 1, 0x10, 0x11, None, 0x100, 1 << 30,
                              null) == 1
    # a misaligned normaliser array (8-byte records)
    assert L.s3r_spec_sample(ctypes.byref(b), 6, 0x10, 0x10, 0x10, 64, 1, 0x10, 0x10, None, 0x14,
                             0x100, 1 << 30, null) == 1
    assert L.s3r_draft_sample(ctypes.byref(b), 0x10, 6, 0x10, 64, 1, 0x10, None, 0x14, 0x100, 1 << 30,
                              null) == 1
    # position scores: misaligned output, a stride that is not a multiple of 4, k_prev
    assert L.s3r_position_scores(ctypes.byref(c), ctypes.byref(b), 0x10, 0x10, 6, 0x18, 1024,
                                 0x100, 1 << 20, null) == 1
    assert L.s3r_position_scores(ctypes.byref(c), ctypes.byref(b), 0x10, 0x10, 6, 0x10, 1022,
                                 0x100, 1 << 20, null) == 1
    assert L.s3r_position_scores(ctypes.byref(c), ctypes.byref(b), 0x10, 0x10, 9, 0x10, 1024,
                                 0x100, 1 << 20, null) == 2
    # the verify's wait bound
    assert L.s3r_set_wait_limit(-1) == 1
    assert L.s3r_set_wait_limit(0) == 0
    # an empty batch is a no-op that succeeds
    e = s3r.BatchDesc(0, 0, None, None, None, 0)
    assert L.s3r_commit(ctypes.byref(e), 6, 0x10, 0x10, None, null) == 0


def test_noalloc_draft_sample_validates_on_the_host():
    """The static-scratch draft sampler checks its size limits before touching the device."""
    import sparse_dense_kv_b200 as s3r
    L = s3r.lib
    null = ctypes.c_void_p(0)
    big = s3r.BatchDesc(1, 2049, None, 0x1000, None, 0)
    assert L.s3r_draft_sample_noalloc(ctypes.byref(big), 0x10, 6, 0x10, 1000, 1, 0x10, 0x10,
                                      null) == 2
    assert b"static scratch" in L.s3r_last_error_message()
    b = s3r.BatchDesc(1, 8, None, 0x1000, None, 0)
    assert L.s3r_draft_sample_noalloc(ctypes.byref(b), 0x10, 6, 0x10, 262145, 1, 0x10, 0x10,
                                      null) == 2
    # the caller's error word is required
    assert L.s3r_draft_sample_noalloc(ctypes.byref(b), 0x10, 6, 0x10, 1000, 1, 0x10, None,
                                      null) == 1
    assert L.s3r_draft_sample_noalloc(ctypes.byref(b), 0x10, 9, 0x10, 1000, 1, 0x10, 0x10,
                                      null) == 2


C_PROGRAM = r"""
#include <stdio.h>
#include "s3r.h"
int main(void) {
  double a[2] = {9.0, 8.0}, d[2] = {10.0, 10.0};
  int32_t k = 0;
  int st = s3r_choose_horizon(a, d, 2, 1.0, 100.0, 0.5, 1.0, &k);
  s3r_sched_config cfg = {50, 0, 0, 4, 1, 64, 0.85, 0.97, 1.0, 10.0, 0.0, 0.001, 0.1, 0.5, 0.5, 1000};
  int32_t prompt[1] = {16}, resp[1] = {32};
  uint8_t tau[64];
  for (int i = 0; i < 64; ++i) tau[i] = 4;
  s3r_sched_result res;
  int st2 = s3r_sched_simulate(&cfg, 1, prompt, resp, tau, 64, NULL, 0, &res, NULL, 0);
  size_t ws = s3r_workspace_size(NULL, 1, 1, 6, 64, 64);
  printf("%d %d %d %lld %lld %zu\n", st, k, st2, (long long)res.tokens, (long long)res.done, ws);
  return 0;
}
"""


def test_header_is_plain_c_and_host_calls_run_from_c(tmp_path):
    """The boundary as a C user sees it: the header compiles as strict C99, a C program
    links the library and runs its host-only calls (no GPU needed)."""
    import shutil
    import subprocess
    import sparse_dense_kv_b200 as s3r
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(s3r.LIB_PATH)
    res = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                          os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-ls3r",
                          f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    st, k, st2, tokens, done, ws = out.stdout.split()
    assert (st, k, st2, tokens, done) == ("0", "2", "0", "32", "1")
    assert ws == "0"   # a NULL cache descriptor is rejected (size 0)

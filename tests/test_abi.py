"""C ABI checks that need no GPU: the library loads, exports every declared
symbol, rejects bad arguments before launching anything, and its host-side
partition order matches the oracle bit for bit."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import block_sparse_attention_16_b200 as lbsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lbsa.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lbsa_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = lbsa.load_library()
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert lbsa.lbsa_version() == 101


def _desc(**kw):
    d = dict(B=1, H=2, N_valid=256, d=64, dtype=1, reserved=0, stride_b=2 * 256 * 64, stride_h=256 * 64, stride_n=64)
    d.update(kw)
    return lbsa._Desc(**d)


FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: validation fails first


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), lbsa.LBSA_ERR_UNSUPPORTED),
    (dict(N_valid=0), lbsa.LBSA_ERR_INVALID_ARG),
    (dict(dtype=7), lbsa.LBSA_ERR_INVALID_ARG),
    (dict(stride_n=60), lbsa.LBSA_ERR_INVALID_ARG),
    (dict(stride_n=65), lbsa.LBSA_ERR_INVALID_ARG),
])
def test_score_rejects_bad_desc(kw, code):
    lib = lbsa.load_library()
    d = _desc(**kw)
    rc = lib.lbsa_score(FAKE, FAKE, ctypes.byref(d), 64, 0, FAKE, None, None)
    assert rc == code
    assert lbsa.lbsa_last_error()


def test_score_rejects_bad_block_mode_and_pointers():
    lib = lbsa.load_library()
    d = _desc()
    assert lib.lbsa_score(FAKE, FAKE, ctypes.byref(d), 96, 0, FAKE, None, None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert lib.lbsa_score(FAKE, FAKE, ctypes.byref(d), 64, 9, FAKE, None, None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_score(None, FAKE, ctypes.byref(d), 64, 0, FAKE, None, None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_score(ctypes.c_void_p(0x10004), FAKE, ctypes.byref(d), 64, 0, FAKE, None, None) == \
        lbsa.LBSA_ERR_INVALID_ARG
    # lse is only defined for the exact mode
    assert lib.lbsa_score(FAKE, FAKE, ctypes.byref(d), 64, 1, FAKE, FAKE, None) == lbsa.LBSA_ERR_INVALID_ARG


@pytest.mark.parametrize("p", [0.0, -0.5, 1.5, float("nan")])
def test_select_rejects_bad_p(p):
    lib = lbsa.load_library()
    h = ctypes.c_void_p()
    assert lib.lbsa_select(FAKE, 1, 1, 4, 64, p, 0, ctypes.byref(h), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert not h.value


def test_select_rejects_bad_scope_block_and_size():
    lib = lbsa.load_library()
    h = ctypes.c_void_p()
    assert lib.lbsa_select(FAKE, 1, 1, 4, 64, 0.9, 5, ctypes.byref(h), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_select(FAKE, 1, 1, 4, 32, 0.9, 0, ctypes.byref(h), None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert lib.lbsa_select(FAKE, 1, 1, 4097, 64, 0.9, 0, ctypes.byref(h), None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert lib.lbsa_select(FAKE, 1, 1, 0, 64, 0.9, 0, ctypes.byref(h), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_select(FAKE, 1, 1, 4, 64, 0.9, 0, None, None) == lbsa.LBSA_ERR_INVALID_ARG


def test_attend_rejects_null_blockset_and_permute_aliasing():
    lib = lbsa.load_library()
    d = _desc()
    assert lib.lbsa_attend(FAKE, FAKE, FAKE, ctypes.byref(d), None, FAKE, None, None) == lbsa.LBSA_ERR_INVALID_ARG
    xs = (ctypes.c_void_p * 1)(0x10000)
    assert lib.lbsa_permute(xs, xs, 1, FAKE, ctypes.byref(d), 0, None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_permute(xs, xs, 4, FAKE, ctypes.byref(d), 0, None) == lbsa.LBSA_ERR_INVALID_ARG


def test_free_null_is_noop_and_info_rejects_null():
    lib = lbsa.load_library()
    lib.lbsa_free(None)
    assert lib.lbsa_blockset_info(None, None, None, None, None, None) == lbsa.LBSA_ERR_INVALID_ARG


@pytest.mark.parametrize("grid", [(4, 8, 8), (21, 30, 52), (5, 7, 9), (33, 45, 80)])
def test_host_partition_perm_matches_oracle(grid):
    T, H, W = grid
    assert np.array_equal(lbsa.lbsa_partition_perm(T, H, W, "raster").numpy(), oracle.perm_raster(T, H, W))
    assert np.array_equal(lbsa.lbsa_partition_perm(T, H, W, "1d").numpy(), oracle.perm_1d_temporal(T, H, W))
    assert np.array_equal(lbsa.lbsa_partition_perm(T, H, W, "2d", frame_tile=(8, 8)).numpy(),
                          oracle.perm_2d_frame_tiles(T, H, W, 8, 8))
    assert np.array_equal(lbsa.lbsa_partition_perm(T, H, W, "3d", tile=(4, 4, 4)).numpy(),
                          oracle.perm_3d_tiles(T, H, W, 4, 4, 4))
    assert np.array_equal(lbsa.lbsa_partition_perm(T, H, W, "3d", tile=(3, 5, 2)).numpy(),
                          oracle.perm_3d_tiles(T, H, W, 3, 5, 2))


def test_partition_perm_rejects_bad_args():
    lib = lbsa.load_library()
    buf = (ctypes.c_int32 * 8)()
    assert lib.lbsa_partition_perm(0, 2, 2, 0, 1, 1, 1, buf, 0, None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_partition_perm(2, 2, 2, 9, 1, 1, 1, buf, 0, None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_partition_perm(2, 2, 2, 3, 0, 1, 1, buf, 0, None) == lbsa.LBSA_ERR_INVALID_ARG


def test_select_tokens_rejects_bad_block_p_and_size():
    lib = lbsa.load_library()
    buf = np.zeros(4096, dtype=np.float32)                  # host memory: rejected before any launch
    h = ctypes.c_void_p()
    p = ctypes.c_void_p(buf.ctypes.data)
    assert lib.lbsa_select_tokens(p, 1, 1, 256, 128, 0.25, ctypes.byref(h), None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert lib.lbsa_select_tokens(p, 1, 1, 256, 64, 0.0, ctypes.byref(h), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_select_tokens(p, 1, 1, 256, 64, 1.5, ctypes.byref(h), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_select_tokens(p, 1, 1, 64 * 4097, 64, 0.25, ctypes.byref(h), None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert lib.lbsa_select_tokens(p, 0, 1, 256, 64, 0.25, ctypes.byref(h), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_select_tokens(p, 1, 1, 256, 64, 0.25, None, None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_select_tokens(None, 1, 1, 256, 64, 0.25, ctypes.byref(h), None) == lbsa.LBSA_ERR_INVALID_ARG


def test_select_routed_rejects_bad_args():
    lib = lbsa.load_library()
    buf = np.zeros(4096, dtype=np.float32)                  # host memory: rejected before any launch
    h = ctypes.c_void_p()
    p = ctypes.c_void_p(buf.ctypes.data)
    ok = dict(B=1, H=4, nB=8, block=64, p=0.9, thr=0.5, group=2)

    def call(**kw):
        a = {**ok, **kw}
        return lib.lbsa_select_routed(a.get("ptr", p), a["B"], a["H"], a["nB"], a["block"], a["p"], a["thr"],
                                      a["group"], None, None, a.get("out", ctypes.byref(h)), None)

    assert call(block=32) == lbsa.LBSA_ERR_UNSUPPORTED
    assert call(p=0.0) == lbsa.LBSA_ERR_INVALID_ARG
    assert call(p=1.5) == lbsa.LBSA_ERR_INVALID_ARG
    assert call(p=float("nan")) == lbsa.LBSA_ERR_INVALID_ARG
    assert call(thr=float("nan")) == lbsa.LBSA_ERR_INVALID_ARG
    assert call(group=0) == lbsa.LBSA_ERR_INVALID_ARG
    assert call(B=0) == lbsa.LBSA_ERR_INVALID_ARG
    assert call(B=20, H=4000) == lbsa.LBSA_ERR_UNSUPPORTED                # B*H > 65535
    assert call(nB=4097, group=1) == lbsa.LBSA_ERR_UNSUPPORTED             # past the wide row kernel
    assert call(H=4097) == lbsa.LBSA_ERR_UNSUPPORTED
    assert call(H=64, nB=1024, group=64) == lbsa.LBSA_ERR_UNSUPPORTED   # a 64-head pool of 1024 blocks: 256 KiB
    assert call(out=None) == lbsa.LBSA_ERR_INVALID_ARG
    assert call(ptr=None) == lbsa.LBSA_ERR_INVALID_ARG
    assert "200 KiB" in (call(H=64, nB=1024, group=64) and lbsa.lbsa_last_error())


def test_blockset_rows_beyond_int_range_are_rejected():
    lib = lbsa.load_library()
    buf = np.zeros(64, dtype=np.float32)                    # host memory: rejected before any launch
    h = ctypes.c_void_p()
    p = ctypes.c_void_p(buf.ctypes.data)
    assert lib.lbsa_select(p, 65535, 65535, 1, 64, 0.5, 0, ctypes.byref(h), None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert "2^31" in lbsa.lbsa_last_error()


def test_call_log_reports_calls_and_errors():
    """LBSA_LOG=1: the rejected calls of a fresh process each leave a call line and an error line on stderr."""
    import subprocess
    import sys
    code = (
        "import ctypes, numpy as np\n"
        "import block_sparse_attention_16_b200 as lbsa\n"
        "lib = lbsa.load_library()\n"
        "buf = np.zeros(64, dtype=np.float32)\n"
        "h = ctypes.c_void_p()\n"
        "rc = lib.lbsa_select(ctypes.c_void_p(buf.ctypes.data), 1, 1, 8, 64, 1.5, 0, ctypes.byref(h), None)\n"
        "rc2 = lib.lbsa_select_tokens(ctypes.c_void_p(buf.ctypes.data), 1, 1, 256, 128, 0.25, ctypes.byref(h), None)\n"
        "print(rc, rc2)\n")
    env = dict(os.environ, LBSA_LOG="1")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == [str(lbsa.LBSA_ERR_INVALID_ARG), str(lbsa.LBSA_ERR_UNSUPPORTED)]
    lines = [l for l in r.stderr.splitlines() if l.startswith("[lbsa]")]
    assert any("lbsa_select B=1 H=1 nB=8 block=64 p=1.5" in l for l in lines), lines
    assert any(l.startswith("[lbsa] error 1:") and "p = 1.5" in l for l in lines), lines
    assert any("lbsa_select_tokens" in l for l in lines) and any(l.startswith("[lbsa] error 2:") for l in lines), lines
    quiet = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           env=dict(os.environ, LBSA_LOG="0"),
                           cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), timeout=120)
    assert "[lbsa]" not in quiet.stderr


def test_noalloc_head_selection_bounds():
    """The allocation-free head selection takes the same nB bound as lbsa_select's
    head scope and rejects B*H past its static scratch without overflowing the
    head count it reports."""
    lib = lbsa.load_library()
    buf = np.zeros(64, dtype=np.int32)
    p = ctypes.c_void_p(buf.ctypes.data)                    # host memory: rejected before any launch
    assert lib.lbsa_select_head_noalloc(p, 1, 1, 4097, 0.25, p, p, p, None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert "4096" in lbsa.lbsa_last_error()
    assert lib.lbsa_select_head_noalloc(p, 65535, 65535, 1, 0.25, p, p, p, None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert "B*H=4294836225 heads" in lbsa.lbsa_last_error()


def test_bitmask_calls_reject_bad_args():
    lib = lbsa.load_library()
    out = ctypes.c_void_p()
    assert lib.lbsa_blockset_export_bitmask(None, FAKE, None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_blockset_from_bitmask(None, 1, 1, 4, 64, ctypes.byref(out), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_blockset_from_bitmask(FAKE, 1, 1, 4097, 64, ctypes.byref(out), None) == lbsa.LBSA_ERR_INVALID_ARG
    assert lib.lbsa_blockset_from_bitmask(FAKE, 1, 1, 4, 96, ctypes.byref(out), None) == lbsa.LBSA_ERR_UNSUPPORTED
    assert lib.lbsa_blockset_from_bitmask(FAKE, 1, 1, 4, 64, None, None) == lbsa.LBSA_ERR_INVALID_ARG


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "lbsa.h"

int main(void) {
  lbsa_blockset* bs = (lbsa_blockset*)0;
  lbsa_qkv_desc desc;
  int rc;
  memset(&desc, 0, sizeof desc);
  printf("version %d\n", lbsa_version());
  rc = lbsa_select((const float*)0, 1, 1, 4, 64, 0.5, LBSA_SCOPE_ROW, &bs, (void*)0);
  printf("select %d %s\n", rc, lbsa_last_error());
  rc = lbsa_blockset_from_bitmask((const uint32_t*)0, 1, 1, 4, 64, &bs, (void*)0);
  printf("from_bitmask %d %s\n", rc, lbsa_last_error());
  rc = lbsa_attend((const void*)0, (const void*)0, (const void*)0, &desc, bs, (void*)0, (float*)0, (void*)0);
  printf("attend %d\n", rc);
  return bs != (lbsa_blockset*)0;
}
"""


def test_header_compiles_as_c99_and_links(tmp_path):
    # the boundary is a plain C ABI: a C99 program built with gcc against the
    # header and the shared library calls it without any Python in between
    # (argument errors only: they return before any device work)
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    lib_dir = os.path.dirname(lbsa.load_library()._name)
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", lib_dir, "-llbsa", "-Wl,-rpath," + lib_dir],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = r.stdout.splitlines()
    assert lines[0] == "version 101"
    assert lines[1].startswith("select 1 ") and "NULL" in lines[1]
    assert lines[2].startswith("from_bitmask 1 ")
    assert lines[3] == "attend 1"

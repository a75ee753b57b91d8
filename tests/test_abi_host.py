"""The C ABI on the host (no GPU): libress.so loads, exports every function that
include/ress.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from block_sparse_global_b200 import build as B
from block_sparse_global_b200 import ress as R

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ress.h")
INVALID, UNSUPPORTED, OK = 1, 2, 0
FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    B.build()
    return R.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ress_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path(lib):
    names = declared_functions()
    for needed in ("ress_pool_blocks", "ress_block_scores", "ress_drift_scores",
                   "ress_select_blocks", "ress_block_sparse_attn"):
        assert needed in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libress.so does not export {name}"


def test_version_and_status_strings(lib):
    assert R.ress_abi_version() == 5
    assert R.ress_status_string(0) == "RESS_OK"
    assert R.ress_status_string(5) == "RESS_ERR_DEVICE_TIMEOUT"
    assert R.ress_status_string(99) == "RESS_ERR_UNKNOWN"


def _pool(lib, shape, ptrs):
    return lib.ress_pool_blocks(shape, *ptrs, None)


def test_shape_validation(lib):
    ptrs = [FAKE] * 6
    assert _pool(lib, None, ptrs) == INVALID
    assert _pool(lib, ctypes.byref(R.make_shape(1, 4, 1024, head_dim=128)), ptrs) == UNSUPPORTED
    assert _pool(lib, ctypes.byref(R.make_shape(1, 4, 1024, block=64)), ptrs) == UNSUPPORTED
    assert _pool(lib, ctypes.byref(R.make_shape(1, 129, 1024)), ptrs) == UNSUPPORTED
    assert _pool(lib, ctypes.byref(R.make_shape(1, 4, 4096 * 128 + 1)), ptrs) == UNSUPPORTED
    assert _pool(lib, ctypes.byref(R.make_shape(-1, 4, 1024)), ptrs) == INVALID
    assert _pool(lib, ctypes.byref(R.make_shape(1, 0, 1024)), ptrs) == INVALID
    # key blocks: 0 (= the query block), 128 or 64 tokens; at most 4096 key blocks
    for kb in (32, 96, 256, -64, 1):
        assert _pool(lib, ctypes.byref(R.make_shape(1, 4, 1024, key_block=kb)), ptrs) == UNSUPPORTED
    assert _pool(lib, ctypes.byref(R.make_shape(1, 4, 4096 * 64 + 1, key_block=64)),
                 ptrs) == UNSUPPORTED


def test_key_block_grid_sizes():
    assert R.grid(1024) == (8, 8) and R.grid(1024, 128) == (8, 8)
    assert R.grid(1024, 64) == (8, 16)
    assert R.grid(4122, 64) == (33, 65)     # 3 VGGT views: ragged last blocks of 26 tokens
    assert R.grid(1, 64) == (1, 1) and R.grid(0, 64) == (0, 0)


def test_empty_problem_is_ok_without_launch(lib):
    for shape in (R.make_shape(0, 4, 1024), R.make_shape(2, 4, 0)):
        assert _pool(lib, ctypes.byref(shape), [None] * 6) == OK
        assert lib.ress_block_sparse_attn(ctypes.byref(shape), *([None] * 6), 0.125, None, None,
                                          None, None) == OK


def test_pointer_validation(lib):
    shape = ctypes.byref(R.make_shape(1, 4, 1024))
    assert _pool(lib, shape, [FAKE, FAKE, None, FAKE, FAKE, FAKE]) == INVALID
    assert _pool(lib, shape, [FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE]) == INVALID  # misaligned
    assert lib.ress_block_scores(shape, FAKE, FAKE, FAKE, 0.0, FAKE, FAKE, None) == INVALID
    assert lib.ress_block_scores(shape, FAKE, FAKE, FAKE, float("nan"), FAKE, FAKE, None) == INVALID
    ws = lib.ress_drift_workspace_bytes(shape)
    assert ws >= 4 * 8 * 66
    assert lib.ress_drift_scores(shape, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 1, None) == INVALID
    assert lib.ress_attn_schedule(shape, FAKE, None, None) == INVALID
    assert lib.ress_block_sparse_attn(shape, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, 0.125, FAKE,
                                      None, None, None) == INVALID
    assert lib.ress_head_gram(shape, 0, FAKE, FAKE, None) == INVALID


def test_select_parameter_validation(lib):
    shape = ctypes.byref(R.make_shape(1, 2, 1024))   # nb = 8
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None]

    def call(method, budgets, rounds=2, rho=0.5, eps=1e-4):
        p, keep = R.select_params(method, budgets, rounds=rounds, rho=rho, eps=eps)
        return lib.ress_select_blocks(shape, ctypes.byref(p), *args)

    assert call(1, [4, 9]) == INVALID             # budget > nb
    # with 64-token key blocks the same sequence has 16 key blocks: budgets count those
    shape64 = ctypes.byref(R.make_shape(1, 2, 1024, key_block=64))
    p, keep = R.select_params(1, [4, 17], rounds=2)
    assert lib.ress_select_blocks(shape64, ctypes.byref(p), *args) == INVALID
    assert call(1, [4, -1]) == INVALID
    assert call(7, [4, 4]) == INVALID             # unknown method
    assert call(1, [4, 4], rounds=65) == INVALID
    assert call(1, [4, 4], rho=0.0) == INVALID
    assert call(1, [4, 4], eps=0.0) == INVALID
    p, keep = R.select_params(1, [4, 4], rounds=2)
    assert lib.ress_select_blocks(shape, ctypes.byref(p), FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  None, None, None) == INVALID          # drift needs s
    assert lib.ress_select_blocks(shape, None, *args) == INVALID
    # the sign flip is a drift-selection control; its value must be one of the three
    p, keep = R.select_params(0, [4, 4], objective=1)
    assert lib.ress_select_blocks(shape, ctypes.byref(p), *args) == INVALID
    p, keep = R.select_params(1, [4, 4], rounds=2, objective=3)
    assert lib.ress_select_blocks(shape, ctypes.byref(p), *args) == INVALID
    # the realized-drift output needs the pooled values, vbar and M, and a valid eps
    for bad in (0.0, -0.5, 1.5, float("nan")):   # the CDF threshold lies in (0, 1]
        p, keep = R.select_params(3, [4, 4], top_p=bad)
        assert lib.ress_select_blocks(shape, ctypes.byref(p), *args) == INVALID
    p, keep = R.select_params(0, [4, 4])
    p.drift = FAKE   # an aligned address that validation rejects before any use
    assert lib.ress_select_blocks(shape, ctypes.byref(p), FAKE, None, None, None, None, FAKE, FAKE,
                                  None, None, None) == INVALID
    p, keep = R.select_params(0, [4, 4], eps=0.0)
    p.drift = FAKE
    assert lib.ress_select_blocks(shape, ctypes.byref(p), *args) == INVALID


def test_token_gather_validation(lib):
    shape = ctypes.byref(R.make_shape(1, 2, 10 * 140))   # 10 views of 140 tokens
    ok = [FAKE, FAKE + 4096, None]
    assert lib.ress_token_gather(shape, 0, 5, 0, *ok) == INVALID      # no views
    assert lib.ress_token_gather(shape, 3, 5, 0, *ok) == INVALID      # 3 does not divide N
    assert lib.ress_token_gather(shape, 10, 141, 0, *ok) == INVALID   # more specials than tokens
    assert lib.ress_token_gather(shape, 10, -1, 0, *ok) == INVALID
    assert lib.ress_token_gather(shape, 10, 5, 2, *ok) == INVALID     # inverse is 0 or 1
    assert lib.ress_token_gather(shape, 10, 5, 0, FAKE, FAKE, None) == INVALID   # in place
    assert lib.ress_token_gather(shape, 10, 5, 0, FAKE + 8, FAKE + 4096, None) == INVALID
    assert lib.ress_token_gather(ctypes.byref(R.make_shape(0, 2, 1400)), 10, 5, 0, None, None,
                                 None) == OK


def test_fused_scores_select_validation(lib):
    shape = ctypes.byref(R.make_shape(1, 2, 1024))
    args = [FAKE, FAKE, FAKE, 0.125, None, None, FAKE, FAKE, None, None, None]
    p, keep = R.select_params(1, [4, 4])
    assert lib.ress_scores_select(shape, ctypes.byref(p), *args) == UNSUPPORTED   # drift
    p, keep = R.select_params(0, [4, 4], objective=1)
    assert lib.ress_scores_select(shape, ctypes.byref(p), *args) == INVALID
    p, keep = R.select_params(0, [4, 9])
    assert lib.ress_scores_select(shape, ctypes.byref(p), *args) == INVALID       # budget > nb
    p, keep = R.select_params(2, [4, 4])
    assert lib.ress_scores_select(shape, ctypes.byref(p), None, *args[1:]) == INVALID
    # v_bar requested without the pooled values
    assert lib.ress_scores_select(shape, ctypes.byref(p), FAKE, FAKE, None, 0.125, None, FAKE,
                                  FAKE, FAKE, None, None, None) == INVALID
    assert lib.ress_scores_select(shape, ctypes.byref(p), FAKE, FAKE, FAKE, 0.0, None, None,
                                  FAKE, FAKE, None, None, None) == INVALID    # scale
    assert lib.ress_scores_select(ctypes.byref(R.make_shape(0, 2, 1024)), ctypes.byref(p),
                                  *([None] * 3), 0.125, *([None] * 7)) == OK


def test_python_binding_raises(lib):
    with pytest.raises(R.RessError) as e:
        R.ress_attn_schedule(R.make_shape(1, 4, 1024, head_dim=32), None, None)
    assert e.value.status == UNSUPPORTED


def test_forced_timeout_diagnostic_validation(lib):
    """The diagnostic entry point validates like the attention call, and needs a dev_err
    word and a positive, bounded wait limit (checked on the host, nothing launched)."""
    shape = ctypes.byref(R.make_shape(1, 2, 1024))
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.125), FAKE]
    i64 = ctypes.c_int64
    assert lib.ress_debug_attn_forced_timeout(shape, *args, None, i64(1000), None) == INVALID
    assert lib.ress_debug_attn_forced_timeout(shape, *args, FAKE + 2, i64(1000), None) == INVALID
    assert lib.ress_debug_attn_forced_timeout(shape, *args, FAKE, i64(0), None) == INVALID
    assert lib.ress_debug_attn_forced_timeout(shape, *args, FAKE, i64(-5), None) == INVALID
    assert lib.ress_debug_attn_forced_timeout(shape, *args, FAKE, i64((1 << 32) + 1), None) == INVALID
    bad = [FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.0), FAKE]
    assert lib.ress_debug_attn_forced_timeout(shape, *bad, FAKE, i64(1000), None) == INVALID
    assert lib.ress_debug_attn_forced_timeout(None, *args, FAKE, i64(1000), None) == INVALID


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """include/ress.h compiles as strict C99 (no C++ or CUDA headers needed) and a C
    program links against libress.so and gets host-validation results from it."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(R.LIB_PATH)
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "ress.h"
int main(void) {
  ress_shape s = {1, 2, 1024, 64, 128, 0};
  ress_shape bad = {1, 2, 1024, 32, 128, 0};
  float *fake = (float *)(unsigned long)0x7F0000000000ul;
  if (ress_abi_version() != 5) return 2;
  if (ress_pool_blocks(&s, 0, 0, 0, 0, 0, 0, 0) != RESS_ERR_INVALID_ARG) return 3;
  if (ress_pool_blocks(&bad, fake, fake, fake, fake, fake, fake, 0) != RESS_ERR_UNSUPPORTED) return 4;
  printf("%s\n", ress_status_string(RESS_ERR_DEVICE_TIMEOUT));
  return 0;
}
''')
    exe = tmp_path / "abi"
    cc = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(root, "include"), str(src), "-L", libdir, "-lress",
                         f"-Wl,-rpath,{libdir}", "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert "TIMEOUT" in run.stdout


def test_fused_drift_select_validation(lib):
    """ress_drift_select rejects bad arguments on the host, before any launch."""
    shape = ctypes.byref(R.make_shape(1, 2, 1024))   # nq = nk = 8
    ws = lib.ress_drift_select_workspace_bytes(shape)
    assert ws >= 2 * 8 * 4 and ws % 256 == 0
    assert lib.ress_drift_select_workspace_bytes(None) == 0

    def call(method=1, budgets=(4, 4), rounds=2, rho=0.5, eps=1e-4, scale=0.125, qp=FAKE,
             wsb=None, work=FAKE, P=None, objective=0):
        p, keep = R.select_params(method, list(budgets), rounds=rounds, rho=rho, eps=eps,
                                  objective=objective)
        return lib.ress_drift_select(shape, ctypes.byref(p), qp, FAKE, FAKE, FAKE, scale, P, None,
                                     None, FAKE, FAKE, None, None, work,
                                     ws if wsb is None else wsb, None)

    assert call(method=0) == INVALID               # drift selection only
    assert call(budgets=(4, 9)) == INVALID         # budget > nk
    assert call(rounds=65) == INVALID
    assert call(rho=0.0) == INVALID
    assert call(eps=0.0) == INVALID
    assert call(scale=0.0) == INVALID
    assert call(scale=float("nan")) == INVALID
    assert call(objective=3) == INVALID
    assert call(qp=None) == INVALID
    assert call(qp=FAKE + 4) == INVALID            # misaligned
    assert call(work=None) == INVALID
    assert call(wsb=ws - 1) == INVALID             # workspace too small
    assert call(P=FAKE + 8) == INVALID             # misaligned optional output
    # an empty problem is fine without any pointer
    empty = ctypes.byref(R.make_shape(0, 2, 1024))
    p, keep = R.select_params(1, [4, 4], rounds=2)
    assert lib.ress_drift_select(empty, ctypes.byref(p), *([None] * 4), 0.125, *([None] * 8), 0,
                                 None) == OK

"""The C-ABI library loads without a GPU, exports every symbol the header
declares, and rejects bad arguments on the host before launching anything.
CPU only: no call here reaches a kernel launch."""

import ctypes
import os
import re

import pytest

from block_sparse_attention_ba_b200 import api
from block_sparse_attention_ba_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ba_att.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return api.load_library()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ba_att_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = header_functions()
    for n in ("ba_att_stats", "ba_att_select", "ba_att_sparse_fwd", "ba_att_merge_lse", "ba_att_split_lists",
              "ba_att_num_blocks", "ba_att_keep_count", "ba_att_get_device_error", "ba_att_status_string",
              "ba_att_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert set(header_functions()) == set(api._SIGS)


def test_version_and_status_strings(lib):
    assert lib.ba_att_version().decode().endswith("sm_100a")
    for code, name in api.STATUS_NAMES.items():
        assert lib.ba_att_status_string(code).decode() == name


def shape(**kw):
    base = dict(B=1, Hq=4, Hkv=2, N=1000, N_alloc=1024, d=128, block=128, dtype=api.DTYPE_BF16, sm_scale=0.0)
    base.update(kw)
    return api.CShape(**base)


def test_num_blocks_and_keep_count(lib):
    s = shape()
    assert lib.ba_att_num_blocks(ctypes.byref(s)) == 8
    assert lib.ba_att_keep_count(ctypes.byref(s), ctypes.c_double(0.5)) == 4
    assert lib.ba_att_keep_count(ctypes.byref(s), ctypes.c_double(1.0)) == 8
    assert lib.ba_att_keep_count(ctypes.byref(s), ctypes.c_double(1e-4)) == 1
    assert lib.ba_att_keep_count(ctypes.byref(s), ctypes.c_double(0.0)) == -1
    assert lib.ba_att_keep_count(ctypes.byref(s), ctypes.c_double(1.5)) == -1
    for n, keep, k in ((256, 0.5, 128), (256, 0.25, 64), (1024, 0.5, 512), (16, 0.5, 8)):
        s = shape(N=n * 128, N_alloc=n * 128)
        assert lib.ba_att_keep_count(ctypes.byref(s), ctypes.c_double(keep)) == k


P = ctypes.c_void_p(0x10000)       # aligned, never dereferenced: every call below fails validation
MIS = ctypes.c_void_p(0x10008)


@pytest.mark.parametrize("bad,status", [
    (dict(d=96), 2), (dict(block=100), 2), (dict(block=512), 2), (dict(block_k=100), 2), (dict(block_k=512), 2), (dict(Hq=3, Hkv=2), 1), (dict(N=0), 1),
    (dict(N_alloc=10), 1), (dict(dtype=7), 1), (dict(B=0), 1), (dict(sm_scale=float("nan")), 1),
])
def test_bad_shapes_rejected(lib, bad, status):
    s = shape(**bad)
    assert lib.ba_att_stats(ctypes.byref(s), P, P, P, P, P, P, None) == status
    assert lib.ba_att_sparse_fwd(ctypes.byref(s), P, P, P, P, P, 4, P, 1, P, None) == status
    assert lib.ba_att_select(ctypes.byref(s), ctypes.c_double(0.5), P, P, P, P, P, P, 8, None, None) == status
    assert lib.ba_att_num_blocks(ctypes.byref(s)) == -1


def test_null_and_misaligned_pointers(lib):
    s = shape()
    assert lib.ba_att_stats(None, P, P, P, P, P, P, None) == 1
    assert lib.ba_att_stats(ctypes.byref(s), None, P, P, P, P, P, None) == 1
    assert lib.ba_att_stats(ctypes.byref(s), MIS, P, P, P, P, P, None) == 3
    assert lib.ba_att_sparse_fwd(ctypes.byref(s), P, P, P, P, P, 4, None, 1, P, None) == 1
    assert lib.ba_att_sparse_fwd(ctypes.byref(s), P, P, MIS, P, P, 4, P, 1, P, None) == 3
    assert lib.ba_att_select(ctypes.byref(s), ctypes.c_double(0.5), P, P, P, P, P, MIS, 8, P, None) == 3
    assert lib.ba_att_select(ctypes.byref(s), ctypes.c_double(0.5), P, P, P, P, P, P, 8, None, None) == 1
    assert lib.ba_att_merge_lse(10, 128, 1, 1, P, P, None, P, P, P, None) == 1
    assert lib.ba_att_merge_lse(10, 128, 1, 1, MIS, P, P, P, P, P, None) == 3


def test_selection_arguments(lib):
    s = shape()
    # keep outside (0, 1]
    assert lib.ba_att_select(ctypes.byref(s), ctypes.c_double(0.0), P, P, P, P, P, P, 8, None, None) == 1
    assert lib.ba_att_select(ctypes.byref(s), ctypes.c_double(1.01), P, P, P, P, P, P, 8, None, None) == 1
    # kmax below the kept count (keep 0.5 of 8 blocks = 4)
    assert lib.ba_att_select(ctypes.byref(s), ctypes.c_double(0.5), P, P, P, P, P, P, 3, None, None) == 1
    # too many blocks for the in-shared-memory selector
    big = shape(N=4097 * 16, N_alloc=4097 * 16, block=16)
    assert lib.ba_att_select(ctypes.byref(big), ctypes.c_double(0.5), P, P, P, P, P, P, 4097, P, None) == 2
    # split point outside [0, nb]
    assert lib.ba_att_split_lists(ctypes.byref(s), 9, P, P, 8, P, P, P, P, None) == 1
    assert lib.ba_att_split_lists(ctypes.byref(s), -1, P, P, 8, P, P, P, P, None) == 1
    assert lib.ba_att_sparse_fwd(ctypes.byref(s), P, P, P, P, P, 0, P, 1, P, None) == 1


def test_merge_and_selftest_arguments(lib):
    assert lib.ba_att_merge_lse(10, 96, 1, 1, P, P, P, P, P, P, None) == 2
    assert lib.ba_att_merge_lse(10, 128, 5, 5, P, P, P, P, P, P, None) == 1
    assert lib.ba_att_merge_lse(-1, 128, 1, 1, P, P, P, P, P, P, None) == 1
    assert lib.ba_att_merge_lse(0, 128, 1, 1, P, P, P, P, P, P, None) == 0     # nothing to do
    # bf16 partials cannot widen to an fp32 output; unknown dtypes are rejected
    assert lib.ba_att_merge_lse(10, 128, 1, 0, P, P, P, P, P, P, None) == 2
    assert lib.ba_att_merge_lse(10, 128, 0, 3, P, P, P, P, P, P, None) == 1
    # sparse_fwd output dtype must be the input dtype or fp32
    s = shape()
    assert lib.ba_att_sparse_fwd(ctypes.byref(s), P, P, P, P, P, 4, P, 2, P, None) == 1
    assert lib.ba_att_selftest_bounded_wait(0, None) == 1
    assert lib.ba_att_selftest_bounded_wait(3_000_000, None) == 1


def test_forward_host_arguments(lib):
    s = shape(N=4096, N_alloc=4096, Hq=8, Hkv=4)
    ws = lib.ba_att_forward_host_workspace(ctypes.byref(s), ctypes.c_double(0.5), 10, 0)
    assert ws > 0
    # no split and smaller chunks need less (auto: every KV head in one chunk here, 64 tiles each);
    # bad keep, split past the end, bad shape -> -1
    assert lib.ba_att_forward_host_workspace(ctypes.byref(s), ctypes.c_double(0.5), -1, 0) < ws
    assert lib.ba_att_forward_host_workspace(ctypes.byref(s), ctypes.c_double(0.5), 10, 4) == ws
    assert lib.ba_att_forward_host_workspace(ctypes.byref(s), ctypes.c_double(0.5), 10, 1) < ws
    assert lib.ba_att_forward_host_workspace(ctypes.byref(s), ctypes.c_double(0.0), 10, 0) == -1
    assert lib.ba_att_forward_host_workspace(ctypes.byref(s), ctypes.c_double(0.5), 33, 0) == -1
    assert lib.ba_att_forward_host_workspace(ctypes.byref(shape(d=96)), ctypes.c_double(0.5), -1, 0) == -1
    W = ctypes.c_void_p(0x100000)                      # 256-byte aligned, never dereferenced
    call = lambda *a: lib.ba_att_forward_host(ctypes.byref(s), ctypes.c_double(0.5), 10, 0, *a, None)
    assert call(None, P, P, P, P, W, ws) == 1
    assert call(P, P, P, P, None, W, ws) == 1
    assert call(P, P, P, P, P, None, ws) == 1
    assert call(P, P, P, P, P, W, ws - 1) == 1                             # workspace too small
    assert call(P, P, P, P, P, ctypes.c_void_p(0x100010), ws) == 3         # workspace not 256-byte aligned
    assert lib.ba_att_forward_host(ctypes.byref(shape(d=96)), ctypes.c_double(0.5), -1, 0, P, P, P, P, P, W, ws,
                                   None) == 2


def test_sparse_fwd_merge_arguments(lib):
    s = shape()
    # the earlier partial is required and must be aligned like every other buffer
    assert lib.ba_att_sparse_fwd_merge(ctypes.byref(s), P, P, P, P, P, 4, None, P, P, 1, P, None) == 1
    assert lib.ba_att_sparse_fwd_merge(ctypes.byref(s), P, P, P, P, P, 4, P, None, P, 1, P, None) == 1
    assert lib.ba_att_sparse_fwd_merge(ctypes.byref(s), P, P, P, P, P, 4, MIS, P, P, 1, P, None) == 3
    assert lib.ba_att_sparse_fwd_merge(ctypes.byref(shape(d=96)), P, P, P, P, P, 4, P, P, P, 1, P, None) == 2


def test_sparse_fwd_rows_arguments(lib):
    s = shape()
    call = lambda sh, rows, stride, op, lp, *rest: lib.ba_att_sparse_fwd_rows(
        ctypes.byref(sh), rows, stride, P, P, P, P, P, 4, op, lp, *rest)
    assert call(s, 0, 64, None, None, P, 1, P, None) == 1             # no query rows
    assert call(s, 65, 64, None, None, P, 1, P, None) == 1            # stride below the row count
    assert call(s, 64, 64, P, None, P, 1, P, None) == 1               # the cached partial comes in pairs
    assert call(s, 64, 64, None, P, P, 1, P, None) == 1
    assert call(s, 64, 64, None, None, None, 1, P, None) == 1         # no output
    assert call(s, 64, 64, None, None, MIS, 1, P, None) == 3
    assert call(s, 64, 64, MIS, P, P, 1, P, None) == 3
    assert call(shape(d=96), 64, 64, None, None, P, 1, P, None) == 2
    assert lib.ba_att_sparse_fwd_rows(None, 64, 64, P, P, P, P, P, 4, None, None, P, 1, P, None) == 1


def test_complement_lists_arguments(lib):
    s = shape()                                          # nb = 8
    assert lib.ba_att_complement_lists(ctypes.byref(s), P, P, 4, P, P, 7, None) == 1       # stride below nb
    assert lib.ba_att_complement_lists(ctypes.byref(s), None, P, 4, P, P, 8, None) == 1
    assert lib.ba_att_complement_lists(ctypes.byref(s), P, P, 0, P, P, 8, None) == 1
    assert lib.ba_att_complement_lists(ctypes.byref(s), P, P, 4, MIS, P, 8, None) == 3
    big = shape(N=4097 * 16, N_alloc=4097 * 16, block=16)
    assert lib.ba_att_complement_lists(ctypes.byref(big), P, P, 4, P, P, 4097, None) == 2


def test_select_variant_arguments(lib):
    s = shape()
    args = (P, P, P, P, P, P, 8, P, None)
    assert lib.ba_att_select_ex(ctypes.byref(s), ctypes.c_double(0.5), ctypes.c_uint32(0x10), *args) == 1
    # by-mass lists need room for every block, and do not combine with the forced diagonal
    assert lib.ba_att_select_ex(ctypes.byref(s), ctypes.c_double(0.5), ctypes.c_uint32(api.SELECT_BY_MASS),
                                P, P, P, P, P, P, 7, P, None) == 1
    assert lib.ba_att_select_ex(ctypes.byref(s), ctypes.c_double(0.5),
                                ctypes.c_uint32(api.SELECT_BY_MASS | api.SELECT_FORCE_DIAGONAL), *args) == 2
    big = shape(N=1025 * 16, N_alloc=1025 * 16, block=16)
    bigargs = (P, P, P, P, P, P, 1025, P, None)
    for flag in (api.SELECT_FORCE_DIAGONAL, api.SELECT_SHARED_GQA, api.SELECT_BY_MASS):
        assert lib.ba_att_select_ex(ctypes.byref(big), ctypes.c_double(0.5), ctypes.c_uint32(flag), *bigargs) == 2
    # the plain variant-free flag set of ba_att_select still reaches the same checks
    assert lib.ba_att_select_ex(ctypes.byref(s), ctypes.c_double(0.5), ctypes.c_uint32(0), P, P, P, P, P, P, 3,
                                P, None) == 1


def test_selector_workspace_and_arguments(lib):
    s = shape()
    nb = lib.ba_att_num_blocks(ctypes.byref(s))
    up = lambda x: (x + 255) // 256 * 256
    feats = 6 * s.B * (s.Hq + s.Hkv) * nb * s.d * 2          # score features, hi and lo
    scores = 4 * s.B * s.Hq * nb * nb                          # room for the map when none is passed
    assert lib.ba_att_selector_workspace(ctypes.byref(s)) == up(feats) + up(scores)
    assert lib.ba_att_selector_workspace(ctypes.byref(shape(d=96))) == -1
    call = lambda sh, keep, *ptrs, kmax=8: lib.ba_att_selector(ctypes.byref(sh), ctypes.c_double(keep), *ptrs[:9],
                                                               ptrs[9], kmax, None)
    ptrs = [P] * 10
    for i in range(10):                        # every pointer but block_scores (index 7) is required
        bad = list(ptrs)
        if i != 7:
            bad[i] = None
            assert call(s, 0.5, *bad) == 1
        bad[i] = MIS
        assert call(s, 0.5, *bad) == 3
    assert call(s, 0.0, *ptrs) == 1            # keep outside (0, 1]
    assert call(s, 0.5, *ptrs, kmax=3) == 1    # kmax below the keep count
    big = shape(N=4097 * 16, N_alloc=4097 * 16, block=16)
    assert call(big, 0.5, *ptrs, kmax=4097) == 2


def test_key_block_geometry(lib):
    s = shape(N=1000, block=128, block_k=64)
    assert lib.ba_att_num_blocks(ctypes.byref(s)) == 8
    assert lib.ba_att_num_key_blocks(ctypes.byref(s)) == 16
    assert lib.ba_att_keep_count(ctypes.byref(s), ctypes.c_double(0.5)) == 8       # a fraction of the key blocks
    assert lib.ba_att_num_key_blocks(ctypes.byref(shape())) == lib.ba_att_num_blocks(ctypes.byref(shape()))
    # the forced diagonal pairs query block i with key block i: equal sizes only
    assert lib.ba_att_select_ex(ctypes.byref(s), ctypes.c_double(0.5), ctypes.c_uint32(api.SELECT_FORCE_DIAGONAL),
                                P, P, P, P, P, P, 8, P, None) == 2


def test_topk_arguments(lib):
    assert lib.ba_att_topk(None, 4, 16, 8, P, P, 8, None) == 1
    assert lib.ba_att_topk(MIS, 4, 16, 8, P, P, 8, None) == 3
    assert lib.ba_att_topk(P, 0, 16, 8, P, P, 8, None) == 1
    assert lib.ba_att_topk(P, 4, 16, 0, P, P, 8, None) == 1
    assert lib.ba_att_topk(P, 4, 16, 8, P, P, 7, None) == 1
    assert lib.ba_att_topk(P, 4, 4097, 8, P, P, 8, None) == 2


C_CALLER = r"""
#include <stdio.h>
#include "ba_att.h"
/* a plain C caller of the boundary: shape geometry and host-side checks only */
int main(void) {
  ba_att_shape s = {0};
  s.B = 1; s.Hq = 4; s.Hkv = 2; s.N = 1000; s.N_alloc = 1024; s.d = 128; s.block = 128;
  s.dtype = BA_DTYPE_BF16; s.sm_scale = 0.f; s.block_k = 0;
  if (ba_att_num_blocks(&s) != 8 || ba_att_keep_count(&s, 0.5) != 4) return 1;
  s.block_k = 64;
  if (ba_att_num_key_blocks(&s) != 16) return 2;
  if (ba_att_stats(&s, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != BA_ERR_INVALID_ARG) return 3;
  printf("%s\n", ba_att_status_string(BA_OK));
  return 0;
}
"""


def test_header_is_plain_c_and_links(lib):
    # the boundary compiles as strict C99 (no C++ in the header) and a C
    # program links against the library and calls it
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    out = os.path.join(ROOT, "tests", "_build")
    os.makedirs(out, exist_ok=True)
    src, exe = os.path.join(out, "c_caller.c"), os.path.join(out, "c_caller")
    with open(src, "w") as f:
        f.write(C_CALLER)
    so = os.path.abspath(api.library_path())
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-o", exe, src, so, "-Wl,-rpath," + os.path.dirname(so)], check=True)
    res = subprocess.run([exe], capture_output=True, text=True)
    assert res.returncode == 0, res.returncode
    assert res.stdout.strip() == "BA_OK"

"""ba_att_forward_host_noalloc: the host-buffer forward on the library's static
device scratch (no workspace argument, nothing allocated per call).

CPU tests check the header constant and the argument checks (none of them
reaches a CUDA call); GPU tests check that the results equal the
device-resident calls bit for bit and the oracle at the parity bar, that calls
on two streams sharing the scratch stay correct, and that a shape whose
workspace cannot fit is refused."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from block_sparse_attention_ba_b200 import api
from block_sparse_attention_ba_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
P = ctypes.c_void_p(0x10000)


@pytest.fixture(scope="module")
def lib():
    build()
    return api.load_library()


def shape(**kw):
    base = dict(B=1, Hq=8, Hkv=4, N=4096, N_alloc=4096, d=128, block=128, dtype=api.DTYPE_BF16, sm_scale=0.0)
    base.update(kw)
    return api.CShape(**base)


def test_static_scratch_size_matches_header():
    text = open(os.path.join(ROOT, "include", "ba_att.h")).read()
    m = re.search(r"#define BA_ATT_STATIC_SCRATCH_BYTES \((\d+)ull << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == api.STATIC_SCRATCH_BYTES


def test_noalloc_arguments(lib):
    s = shape()
    call = lambda sh, keep, *ptrs: lib.ba_att_forward_host_noalloc(ctypes.byref(sh), ctypes.c_double(keep), 10,
                                                                   *ptrs, None)
    assert call(s, 0.5, None, P, P, P, P) == 1
    assert call(s, 0.5, P, P, P, P, None) == 1
    assert call(s, 0.0, P, P, P, P, P) == 1                                   # keep outside (0, 1]
    assert call(shape(d=96), 0.5, P, P, P, P, P) == 2
    # 32 query heads on one KV head at 128K with a split: one chunk needs more than the scratch
    big = shape(Hq=32, Hkv=1, N=131072, N_alloc=131072)
    need = lib.ba_att_forward_host_workspace(ctypes.byref(big), ctypes.c_double(0.5), 10, 1)
    assert need > api.STATIC_SCRATCH_BYTES
    assert call(big, 0.5, P, P, P, P, P) == 2


def _inputs(name, **over):
    from block_sparse_attention_ba_b200.workloads import make_inputs
    Q, K, V, meta = make_inputs(name, **over)
    return Q, K, V, meta["workload"], meta


def _pinned(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return (t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float32)).pin_memory()


@pytest.mark.gpu
@pytest.mark.parametrize("name,over,split", [
    ("extreme_128k", dict(N=4096 - 50, N_alloc=4096, Hq=8, Hkv=4), True),
    ("tiny_fp32", dict(N=1000, N_alloc=1024), False),
])
def test_noalloc_matches_workspace_path_and_oracle(name, over, split):
    import oracle as O
    from gpu_util import TOL, max_abs, rel_l2
    Q, K, V, w, meta = _inputs(name, **over)
    Qh, Kh, Vh = (_pinned(x, w.dtype) for x in (Q, K, V))
    split_block = meta.get("split_block", w.nb // 2) if split else -1
    On, Ln = api.forward_host_noalloc(Qh, Kh, Vh, w.N, w.block, 0.5, split_block=split_block)
    Ow, Lw = api.forward_host(Qh, Kh, Vh, w.N, w.block, 0.5, split_block=split_block)
    torch.cuda.synchronize()
    n = w.N
    assert torch.equal(On[:, :, :n], Ow[:, :, :n]) and torch.equal(Ln[:, :, :n], Lw[:, :, :n])
    # against the oracle on the GPU's own selection
    Qd, Kd = (torch.from_numpy(np.ascontiguousarray(x)).to(Qh.dtype).cuda() for x in (Q, K))
    sh = api.Shape.of(Qd, Kd, w.N, w.block)
    idx, cnt = api.select(api.stats(Qd, Kd, sh), sh, 0.5)
    Oref, Lref = O.masked_attention(Q, K, V, idx.cpu().numpy(), cnt.cpu().numpy(), w.N, w.block, w.d ** -0.5)
    tol = TOL[w.dtype]
    got = On[:, :, :n].float().numpy()
    assert max_abs(got, Oref[:, :, :n]) <= tol["max_abs"] and rel_l2(got, Oref[:, :, :n]) <= tol["rel_l2"]
    assert max_abs(Ln[:, :, :n].numpy(), Lref[:, :, :n]) <= tol["lse_abs"]


@pytest.mark.gpu
def test_noalloc_calls_on_two_streams_share_the_scratch():
    # two different inputs, issued back to back on two streams: the second
    # call waits for the first on the shared scratch, so both come out right
    Qa, Ka, Va, w, _ = _inputs("dlm_16k", N=2048, Hq=4, Hkv=2)
    Qb, Kb, Vb, _, _ = _inputs("dlm_16k", N=2048, Hq=4, Hkv=2, seed=11)
    ha = [_pinned(x, w.dtype) for x in (Qa, Ka, Va)]
    hb = [_pinned(x, w.dtype) for x in (Qb, Kb, Vb)]
    ref_a = api.forward_host(*ha, w.N, w.block, 0.5)
    ref_b = api.forward_host(*hb, w.N, w.block, 0.5)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        got_a = api.forward_host_noalloc(*ha, w.N, w.block, 0.5)
    with torch.cuda.stream(s2):
        got_b = api.forward_host_noalloc(*hb, w.N, w.block, 0.5)
    torch.cuda.synchronize()
    for got, ref in ((got_a, ref_a), (got_b, ref_b)):
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    st, word = api.get_device_error()
    assert st == 0, f"device error word {word:#x}"

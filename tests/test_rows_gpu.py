"""ba_att_sparse_fwd_rows through the C ABI: attention for one range of query
rows (the current block of a block-diffusion step), merged with a cached
partial of those rows over the keys outside the block.

FlashBlock ("Core claim", "What carries the argument", Eq. 5 and Eq. 9):
caching the block-external attention and recomputing only the block-internal
part, then merging in log space, equals attention over every key. The tests
check that identity against the oracle's textbook dense attention, and that
the range call equals the whole-sequence call on the same rows bit for bit."""

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_ba_b200 import api
from block_sparse_attention_ba_b200.workloads import make_inputs
from gpu_util import TOL, max_abs, rel_l2, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.load_library()
    yield
    st, word = api.get_device_error()
    assert st == 0, f"device error word {word:#x}"


# (generator, overrides, prefix rows r0, current-block rows R): N = r0 + R tokens so far
CASES = [
    ("dlm_16k", dict(Hq=4, Hkv=2), 1024, 200),                        # tcgen05, ragged second tile (72 rows)
    ("dlm_16k", dict(Hq=4, Hkv=2, block_k=64), 512, 128),             # tcgen05, 64-row key blocks
    ("dlm_16k", dict(Hq=4, Hkv=2, d=64), 768, 256 + 40),              # tcgen05 d = 64, three tiles
    ("dlm_16k", dict(Hq=2, Hkv=1, block=256), 1024, 256 + 100),       # 256-row query blocks (two tiles each)
    ("dlm_16k", dict(Hq=2, Hkv=1), 0, 300),                           # no prefix: the cache is empty
    ("tiny_fp32", dict(Hq=2, Hkv=2), 256, 100),                       # fp32 on the CUDA cores, block 64
    ("dlm_16k", dict(Hq=2, Hkv=1, d=64, block=64), 320, 64 + 30),     # tcgen05, 64-row query blocks
    ("dlm_16k", dict(Hq=2, Hkv=1, block=32), 320, 64 + 30),           # bf16 block 32 (CUDA cores)
]


def _case(name, over, r0, R):
    N = r0 + R
    Q, K, V, meta = make_inputs(name, N=N, N_alloc=N + 24, **over)
    return Q, K, V, meta["workload"]


@pytest.mark.parametrize("name,over,r0,R", CASES)
def test_rows_cached_external_plus_internal_is_dense(name, over, r0, R):
    Q, K, V, w = _case(name, over, r0, R)
    s = w.d ** -0.5
    rows = np.arange(r0, r0 + R)
    q_stride = R + 8                                   # a compact range buffer with spare rows
    Qr = np.zeros((w.B, w.Hq, q_stride, w.d), np.float32)
    Qr[:, :, :R] = Q[:, :, rows]
    # the cached block-external partial: the oracle's attention of these rows over keys [0, r0)
    Oc = np.zeros((w.B, w.Hq, q_stride, w.d), np.float32)
    Lc = np.full((w.B, w.Hq, q_stride), -np.inf, np.float32)
    if r0 > 0:
        Oe, Le = O.dense_attention(Q, K, V, r0, s, rows=rows)
        Oc[:, :, :R], Lc[:, :, :R] = Oe, Le
    # block-internal lists: the key blocks of [r0, N)
    internal = np.arange(r0 // w.kb, -(-w.N // w.kb), dtype=np.int32)
    nqr = -(-R // w.block)
    idx = np.tile(internal, (w.B, w.Hq, nqr, 1))
    cnt = np.full((w.B, w.Hq, nqr), internal.size, np.int32)

    Kd, Vd = to_dev(K, w.dtype), to_dev(V, w.dtype)
    shape = api.Shape(w.B, w.Hq, w.Hkv, w.N, w.N_alloc, w.d, w.block,
                      api.DTYPE_BF16 if w.dtype == "bf16" else api.DTYPE_F32, 0.0, w.block_k)
    Qd = to_dev(Qr, w.dtype)
    Ocd = torch.from_numpy(Oc).cuda()
    Lcd = torch.from_numpy(Lc).cuda()
    Og = torch.full_like(Qd, 7.0)
    Lg = torch.full((w.B, w.Hq, q_stride), 7.0, device="cuda")
    api.sparse_fwd_rows(Qd, Kd, Vd, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), shape,
                        q_rows=R, O_prev=Ocd, L_prev=Lcd, out=(Og, Lg))
    torch.cuda.synchronize()
    Od, Ld = O.dense_attention(Q, K, V, w.N, s, rows=rows)
    got, gl = Og.float().cpu().numpy(), Lg.cpu().numpy()
    tol = TOL[w.dtype]
    assert max_abs(got[:, :, :R], Od) <= tol["max_abs"], max_abs(got[:, :, :R], Od)
    assert rel_l2(got[:, :, :R], Od) <= tol["rel_l2"], rel_l2(got[:, :, :R], Od)
    assert max_abs(gl[:, :, :R], Ld) <= tol["lse_abs"], max_abs(gl[:, :, :R], Ld)
    assert (got[:, :, R:] == 7.0).all() and (gl[:, :, R:] == 7.0).all()     # rows past the range untouched
    # and against the oracle's own range routine (the same split, merged in float64)
    Orr, Lrr = O.block_rows_attention(Qr, K, V, idx, cnt, R, w.N, w.block, s, O_prev=Oc, L_prev=Lc, b_k=w.kb)
    assert max_abs(got[:, :, :R], Orr[:, :, :R]) <= tol["max_abs"]
    assert max_abs(gl[:, :, :R], Lrr[:, :, :R]) <= tol["lse_abs"]


@pytest.mark.parametrize("name,over,i0,nqr_take", [
    ("dlm_16k", dict(N=2048 - 50, N_alloc=2048, Hq=4, Hkv=2), 5, 11),        # tcgen05, to the ragged end
    ("dlm_16k", dict(N=2048, Hq=4, Hkv=2), 3, 2),                             # tcgen05, interior range
    ("dlm_16k", dict(N=2048, Hq=2, Hkv=1, block=256), 2, 3),                  # 256-row blocks
    ("tiny_fp32", dict(N=1000, N_alloc=1024), 4, 12),                         # CUDA cores, to the ragged end
])
@pytest.mark.parametrize("merge", [False, True])
def test_rows_equal_whole_sequence_call_bit_for_bit(name, over, i0, nqr_take, merge):
    # the range call on rows of the full tensors (slices of Q, O and LSE, at
    # the full row stride) gives the same bits as the whole-sequence call on
    # those rows, and leaves every other row alone
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    Qd, Kd, Vd = to_dev(Q, w.dtype), to_dev(K, w.dtype), to_dev(V, w.dtype)
    shape = api.Shape.of(Qd, Kd, w.N, w.block)
    idx, cnt = api.select(api.stats(Qd, Kd, shape), shape, 0.5)
    r0 = i0 * w.block
    R = min(w.N, (i0 + nqr_take) * w.block) - r0
    nqr = -(-R // w.block)
    sl = slice(r0, r0 + R)
    li, lc = idx[:, :, i0:i0 + nqr].contiguous(), cnt[:, :, i0:i0 + nqr].contiguous()
    if merge:
        g = torch.Generator(device="cuda").manual_seed(3)
        Op = torch.randn(Qd.shape, device="cuda", generator=g)
        Lp = torch.randn((w.B, w.Hq, w.N_alloc), device="cuda", generator=g) + 5.0
        Of, Lf = api.sparse_fwd_merge(Qd, Kd, Vd, idx, cnt, shape, Op, Lp)
    else:
        Op = Lp = None
        Of, Lf = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, shape)
    Ox = torch.full_like(Of, 3.0)
    Lx = torch.full_like(Lf, 3.0)
    api.sparse_fwd_rows(Qd[:, :, sl], Kd, Vd, li, lc, shape, O_prev=None if Op is None else Op[:, :, sl],
                        L_prev=None if Lp is None else Lp[:, :, sl], out=(Ox[:, :, sl], Lx[:, :, sl]))
    torch.cuda.synchronize()
    assert torch.equal(Ox[:, :, sl], Of[:, :, sl]) and torch.equal(Lx[:, :, sl], Lf[:, :, sl])
    assert (Ox[:, :, :r0] == 3.0).all() and (Ox[:, :, r0 + R:] == 3.0).all()
    assert (Lx[:, :, :r0] == 3.0).all() and (Lx[:, :, r0 + R:] == 3.0).all()

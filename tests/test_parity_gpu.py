"""GPU path vs the CPU oracle, element by element, through the C ABI.

Small cases span several tiles and a ragged tail and are compared in full;
the full-size workloads are compared on sampled query blocks (attention) and
in full (statistics, scores, masks). Block masks must match bit-exactly
except for blocks within the near-tie band of the selection threshold, which
are counted and reported."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_ba_b200 import api
from block_sparse_attention_ba_b200.workloads import WORKLOADS, make_inputs
from gpu_util import NEAR_TIE_REL, TOL, mask_of, max_abs, rel_l2, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.load_library()
    yield
    st, word = api.get_device_error()
    assert st == 0, f"device error word {word:#x}"


def run_gpu(Q, K, V, w, keep, kmax=None, with_scores=True):
    Qd, Kd, Vd = to_dev(Q, w.dtype), to_dev(K, w.dtype), to_dev(V, w.dtype)
    shape = api.Shape.of(Qd, Kd, w.N, w.block, block_k=w.block_k)
    st = api.stats(Qd, Kd, shape)
    idx, cnt, sc = api.select(st, shape, keep, kmax=kmax, with_scores=True)
    Od, Ld = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, shape)
    torch.cuda.synchronize()
    return dict(shape=shape, Qd=Qd, Kd=Kd, Vd=Vd, stats=[t.cpu().numpy() for t in st], idx=idx.cpu().numpy(),
                cnt=cnt.cpu().numpy(), scores=sc.cpu().numpy(), O=Od.float().cpu().numpy(), L=Ld.cpu().numpy(),
                idx_d=idx, cnt_d=cnt)


def check_stats(r, Q, K, w):
    qm, qv, _ = O.block_stats(Q, w.N, w.block)
    km, kv, kc = O.block_stats(K, w.N, w.kb)            # key blocks (asymmetric shapes: w.kb rows)
    for got, ref, name in zip(r["stats"], (qm, qv, km, kv), ("q_mean", "q_var", "k_mean", "k_var")):
        err = np.abs(got - ref)
        assert np.all(err <= 1e-5 * np.abs(ref) + 2e-6 * (1 + np.abs(ref).max())), (name, err.max())
    return qm, qv, km, kv, kc


def check_selection(r, stats_ref, w, keep):
    qm, qv, km, kv, kc = stats_ref
    s = w.d ** -0.5
    S = O.corrected_scores(qm, qv, km, kv, kc, s)
    k = O.keep_count(keep, w.nk)
    err = np.abs(r["scores"] - S)
    assert np.all(err <= 1e-5 * np.abs(S) + 5e-5), err.max()
    idx_ref, cnt_ref = O.select_topk(S, k)
    assert (r["cnt"] == k).all()
    got = mask_of(r["idx"], r["cnt"], w.nk)
    ref = mask_of(idx_ref, cnt_ref, w.nk)
    near = O.near_tie_mask(S, k, NEAR_TIE_REL)
    mism = (got != ref) & ~near
    assert not mism.any(), f"{int(mism.sum())} mask mismatches outside the near-tie band"
    # lists ascending, -1 padded
    idx = r["idx"]
    kmax = idx.shape[-1]
    for pos in np.ndindex(r["cnt"].shape):
        row = idx[pos]
        assert (np.diff(row[:k]) > 0).all() and (row[k:kmax] == -1).all()
    return int(((got != ref) & near).sum()), int(near.sum())


def check_attention(r, Q, K, V, w, blocks):
    s = w.d ** -0.5
    Oref, Lref = O.masked_attention(Q, K, V, r["idx"], r["cnt"], w.N, w.block, s, query_blocks=blocks,
                                    b_k=w.kb)
    tol = TOL[w.dtype]
    rows = []
    for (bb, h, i) in blocks:
        lo, hi = i * w.block, min(w.N, (i + 1) * w.block)
        rows.append((bb, h, slice(lo, hi)))
    got = np.concatenate([r["O"][bb, h, sl] for bb, h, sl in rows])
    ref = np.concatenate([Oref[bb, h, sl] for bb, h, sl in rows])
    gl = np.concatenate([r["L"][bb, h, sl] for bb, h, sl in rows])
    rl = np.concatenate([Lref[bb, h, sl] for bb, h, sl in rows])
    assert max_abs(got, ref) <= tol["max_abs"], max_abs(got, ref)
    assert rel_l2(got, ref) <= tol["rel_l2"], rel_l2(got, ref)
    assert max_abs(gl, rl) <= tol["lse_abs"], max_abs(gl, rl)


def all_blocks(w):
    return [(bb, h, i) for bb in range(w.B) for h in range(w.Hq) for i in range(w.nb)]


def sample_blocks(w, per_head=2, seed=0):
    rng = np.random.default_rng(seed)
    out = []
    for bb in range(w.B):
        for h in range(w.Hq):
            for i in rng.choice(w.nb, size=min(per_head, w.nb), replace=False):
                out.append((bb, h, int(i)))
            out.append((bb, h, w.nb - 1))                 # always include the (possibly ragged) last block
    return sorted(set(out))


# ------------------------------------------------------------------ small cases

SMALL = [
    ("tiny_fp32", {}, 0.5),                                           # the fp32 configuration, in full
    ("tiny_fp32", dict(N=1000, N_alloc=1024), 0.25),                  # ragged tail, padding rows
    ("dlm_16k", dict(N=2048, Hq=8, Hkv=2), 0.5),                      # tcgen05 path, GQA, 16 blocks
    ("dlm_16k", dict(N=1920 + 77, N_alloc=2048, Hq=4, Hkv=2), 0.5),   # tcgen05 path, ragged last block
    ("sweep_32k", dict(N=4096, Hq=4, Hkv=1), 0.25),                   # needle generator, 32 blocks
    ("video_32k", dict(N=600, N_alloc=640, Hq=2, Hkv=2, grid=(3, 10, 20)), 0.5),
    ("dlm_16k", dict(N=1024, Hq=2, Hkv=1, d=64, block=64), 0.5),      # tcgen05, 64-row query blocks, d = 64
    ("dlm_16k", dict(N=1600 - 23, N_alloc=1600, Hq=4, Hkv=2, block=64), 0.5),   # tcgen05, 64-row blocks, ragged
    ("tiny_fp32", dict(N=768, d=128, block=32), 0.3),                 # fp32 d=128, block 32
    ("tiny_fp32", dict(N=9600 - 7, N_alloc=9600, block=16, Hq=2, Hkv=1), 0.5),   # 600 blocks: 5x5 score tiles
    ("dlm_16k", dict(N=64 * 128, Hq=2, Hkv=1), 0.5),                 # 512 blocks: 16 keys per lane in the top-k
    ("dlm_16k", dict(N=300 * 128 - 5, Hq=2, Hkv=2), 0.3),             # 300 blocks: ragged score tiles
    ("dlm_16k", dict(N=2048 - 17, N_alloc=2048, Hq=4, Hkv=2, d=64), 0.5),   # tcgen05 path with d = 64, ragged
    ("sweep_32k", dict(N=4096, Hq=4, Hkv=1, d=64), 0.25),            # d = 64, needle generator
    ("dlm_16k", dict(N=4096, Hq=4, Hkv=2, block=256), 0.5),          # tcgen05 path, 256-row blocks
    ("dlm_16k", dict(N=3 * 256 + 200, N_alloc=1024, Hq=2, Hkv=1, block=256), 0.5),   # 256-row blocks, ragged
    ("dlm_16k", dict(N=2048 - 40, N_alloc=2048, Hq=4, Hkv=2, d=64, block=256), 0.5),  # 256-row blocks, d = 64
    ("dlm_16k", dict(N=2 * 256 + 60, N_alloc=640, Hq=2, Hkv=1, block=256), 0.5),   # CTA pair: rank 1 of the last block holds no row
    ("dlm_16k", dict(N=3072 - 50, N_alloc=3072, B=2, Hq=8, Hkv=2, block=256), 0.3),   # CTA pair: B = 2, 4 heads per KV head
    ("dlm_16k", dict(N=4096 - 70, N_alloc=4096, Hq=2, Hkv=1, block=256, block_k=256), 0.5),   # CTA pair, 256 x 256
    # asymmetric blocks: query blocks of `block` rows, key blocks of `block_k` rows
    ("dlm_16k", dict(N=2048 - 30, N_alloc=2048, Hq=4, Hkv=2, block_k=64), 0.5),      # tcgen05, 128 x 64
    ("dlm_16k", dict(N=2048, Hq=4, Hkv=2, block=256, block_k=128), 0.5),             # tcgen05, 256 x 128
    ("dlm_16k", dict(N=3000, N_alloc=3072, Hq=2, Hkv=1, block=128, block_k=256), 0.3),  # tcgen05, 128 x 256
    ("dlm_16k", dict(N=1500, N_alloc=1536, Hq=2, Hkv=1, d=64, block=128, block_k=64), 0.5),  # tcgen05, d 64
    ("dlm_16k", dict(N=1024 - 9, N_alloc=1024, Hq=2, Hkv=1, block=64, block_k=128), 0.5),   # tcgen05, 64 x 128
    ("dlm_16k", dict(N=1024, Hq=2, Hkv=1, block=32), 0.5),                         # CUDA cores, bf16 block 32
    ("tiny_fp32", dict(block=32, block_k=64), 0.5),                                  # fp32, 32 x 64
]


@pytest.mark.parametrize("name,over,keep", SMALL)
def test_small_full_parity(name, over, keep):
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    r = run_gpu(Q, K, V, w, keep)
    st = check_stats(r, Q, K, w)
    check_selection(r, st, w, keep)
    check_attention(r, Q, K, V, w, all_blocks(w))
    # padding rows are never written: fill and re-run
    if w.N_alloc > w.N:
        Od = torch.full_like(r["Qd"], 7.0)
        Ld = torch.full((w.B, w.Hq, w.N_alloc), 7.0, device="cuda")
        api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], r["idx_d"], r["cnt_d"], r["shape"], out=(Od, Ld))
        assert (Od[:, :, w.N:] == 7.0).all() and (Ld[:, :, w.N:] == 7.0).all()


@pytest.mark.parametrize("block_k", [128, 256])
@pytest.mark.parametrize("merge", [False, True])
def test_cta_pair_equals_two_single_tiles(block_k, merge):
    # A 256-row query block on the CTA pair computes, per 128-row half, what
    # the one-CTA kernel computes for a 128-row block holding the same list:
    # the same key halves in the same order, the same MMA k-steps. The two
    # are compared bit for bit (the pair against the kernel the oracle pins).
    Q, K, V, meta = make_inputs("dlm_16k", N=1536 - 70, N_alloc=1536, Hq=4, Hkv=2)
    w = meta["workload"]
    Qd, Kd, Vd = to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16")
    s256 = api.Shape.of(Qd, Kd, w.N, 256, block_k=block_k)
    s128 = api.Shape.of(Qd, Kd, w.N, 128, block_k=block_k)
    idx, cnt = api.select(api.stats(Qd, Kd, s256), s256, 0.5)
    idx[0, 1, 2] = torch.arange(idx.shape[-1], device="cuda", dtype=torch.int32)    # consecutive blocks
    cnt[0, 2, 1] = 0                                                   # one empty list
    idx128 = idx.repeat_interleave(2, dim=2)[:, :, : s128.nb].contiguous()
    cnt128 = cnt.repeat_interleave(2, dim=2)[:, :, : s128.nb].contiguous()
    if merge:
        g = torch.Generator(device="cuda").manual_seed(5)
        Op = torch.randn(Qd.shape, device="cuda", generator=g)
        Lp = torch.randn((w.B, w.Hq, w.N_alloc), device="cuda", generator=g)
        O2, L2 = api.sparse_fwd_merge(Qd, Kd, Vd, idx, cnt, s256, Op, Lp)
        O1, L1 = api.sparse_fwd_merge(Qd, Kd, Vd, idx128, cnt128, s128, Op, Lp)
    else:
        O2, L2 = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, s256)
        O1, L1 = api.sparse_fwd(Qd, Kd, Vd, idx128, cnt128, s128)
    torch.cuda.synchronize()
    n = w.N
    assert torch.equal(O2[:, :, :n], O1[:, :, :n]) and torch.equal(L2[:, :, :n], L1[:, :, :n])
    Oref, Lref = O.masked_attention(Q, K, V, idx.cpu().numpy(), cnt.cpu().numpy(), n, 256, w.d ** -0.5, b_k=block_k)
    if not merge:
        assert max_abs(O2[:, :, :n].float().cpu().numpy(), Oref[:, :, :n]) <= TOL["bf16"]["max_abs"]
        got_l = L2[:, :, :n].cpu().numpy()
        fin = np.isfinite(Lref[:, :, :n])
        assert (np.isneginf(got_l) == ~fin).all()
        assert np.abs(got_l[fin] - Lref[:, :, :n][fin]).max() <= TOL["bf16"]["lse_abs"]


@pytest.mark.parametrize("name,over", [("tiny_fp32", {}), ("dlm_16k", dict(N=1536, Hq=4, Hkv=2)),
                                       ("dlm_16k", dict(N=1536 - 9, N_alloc=1536, Hq=4, Hkv=2, d=64)),
                                       ("dlm_16k", dict(N=1536, Hq=4, Hkv=2, block=256)),
                                       ("dlm_16k", dict(N=1536, Hq=4, Hkv=2, block=256, block_k=64)),
                                       ("dlm_16k", dict(N=1536 - 5, N_alloc=1536, Hq=4, Hkv=2, block=64)),
                                       ("video_32k", dict(N=600, N_alloc=640, Hq=2, Hkv=2, grid=(3, 10, 20)))])
def test_keep_all_equals_dense(name, over):
    # check (1): keep = 1.0 selects every block and equals dense attention
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    r = run_gpu(Q, K, V, w, 1.0)
    assert (r["cnt"] == w.nk).all()
    Od, Ld = O.dense_attention(Q, K, V, w.N, w.d ** -0.5)
    tol = TOL[w.dtype]
    assert max_abs(r["O"][:, :, : w.N], Od) <= tol["max_abs"]
    assert rel_l2(r["O"][:, :, : w.N], Od) <= tol["rel_l2"]
    assert max_abs(r["L"][:, :, : w.N], Ld) <= tol["lse_abs"]


def test_split_and_merge_equals_union():
    # check (2) on the GPU: split kept lists at a block boundary, attend each
    # span, merge in log space; equals single-pass attention over the union
    Q, K, V, meta = make_inputs("extreme_128k", N=4096, Hq=4, Hkv=2)
    w = meta["workload"]
    r = run_gpu(Q, K, V, w, 0.5)
    shape = r["shape"]
    for split in (0, meta["split_block"], w.nb // 2, w.nb):
        lo_i, lo_c, hi_i, hi_c = api.split_lists(r["idx_d"], r["cnt_d"], shape, split)
        ref = O.split_lists(r["idx"], r["cnt"], split)
        for got, exp in zip((lo_i, lo_c, hi_i, hi_c), ref):
            np.testing.assert_array_equal(got.cpu().numpy(), exp)
        # partials in fp32, merged output rounded once to bf16
        O1, L1 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], lo_i, lo_c, shape, out_dtype=torch.float32)
        O2, L2 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], hi_i, hi_c, shape, out_dtype=torch.float32)
        Om, Lm = api.merge_lse(O1, L1, O2, L2, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        Om = Om.float().cpu().numpy()
        Lm = Lm.cpu().numpy()
        tol = TOL[w.dtype]
        Oref, Lref = O.masked_attention(Q, K, V, r["idx"], r["cnt"], w.N, w.block, w.d ** -0.5)
        assert max_abs(Om, Oref) <= tol["max_abs"], max_abs(Om, Oref)
        assert rel_l2(Om, Oref) <= tol["rel_l2"]
        assert max_abs(Lm, Lref) <= tol["lse_abs"]
        # against the single pass: both sit within the bar of the oracle, and
        # their bf16 P roundings differ, so they agree within twice the bar
        assert max_abs(Om, r["O"]) <= 2 * tol["max_abs"] and rel_l2(Om, r["O"]) <= 2 * tol["rel_l2"]
        assert max_abs(Lm, r["L"]) <= 2 * tol["lse_abs"]


@pytest.mark.parametrize("flags", [api.SELECT_NO_VAR_PRODUCT, api.SELECT_FORCE_DIAGONAL, api.SELECT_SHARED_GQA,
                                   api.SELECT_NO_VAR_PRODUCT | api.SELECT_FORCE_DIAGONAL | api.SELECT_SHARED_GQA])
@pytest.mark.parametrize("name,over,keep", [
    ("dlm_16k", dict(N=2048 - 40, N_alloc=2048, Hq=8, Hkv=2), 0.25),       # 16 blocks, 4 heads per group
    ("tiny_fp32", dict(N=1000, N_alloc=1024, Hq=4, Hkv=2), 0.5),            # d = 64
    ("dlm_16k", dict(N=300 * 128 - 5, Hq=2, Hkv=1), 0.3),                   # 300 blocks, 16 keys per lane
])
def test_selection_variants(name, over, keep, flags):
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    Qd, Kd = to_dev(Q, w.dtype), to_dev(K, w.dtype)
    shape = api.Shape.of(Qd, Kd, w.N, w.block)
    st = api.stats(Qd, Kd, shape)
    idx, cnt, sc = api.select(st, shape, keep, with_scores=True, flags=flags)
    torch.cuda.synchronize()
    qm, qv, _ = O.block_stats(Q, w.N, w.block)
    km, kv, kc = O.block_stats(K, w.N, w.block)
    S = O.corrected_scores(qm, qv, km, kv, kc, w.d ** -0.5, var_product=not (flags & api.SELECT_NO_VAR_PRODUCT))
    err = np.abs(sc.cpu().numpy() - S)
    assert np.all(err <= 1e-5 * np.abs(S) + 5e-5), err.max()
    R = O.selection_scores(S, w.Hkv, force_diagonal=bool(flags & api.SELECT_FORCE_DIAGONAL),
                           shared_gqa=bool(flags & api.SELECT_SHARED_GQA))
    k = O.keep_count(keep, w.nb)
    idx_ref, cnt_ref = O.select_topk(R, k)
    got = mask_of(idx.cpu().numpy(), cnt.cpu().numpy(), w.nb)
    ref = mask_of(idx_ref, cnt_ref, w.nb)
    near = O.near_tie_mask(R, k, NEAR_TIE_REL)
    assert not ((got != ref) & ~near).any()
    if flags & api.SELECT_FORCE_DIAGONAL:
        assert got[..., np.arange(w.nb), np.arange(w.nb)].all()
    if flags & api.SELECT_SHARED_GQA:
        G = w.Hq // w.Hkv
        g_idx = idx.cpu().numpy().reshape(w.B, w.Hkv, G, w.nb, -1)
        assert (g_idx == g_idx[:, :, :1]).all()


@pytest.mark.parametrize("tau", [0.3, 0.7, 0.95])
@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("name,over", [
    ("dlm_16k", dict(N=2048 - 40, N_alloc=2048, Hq=8, Hkv=2)),     # 16 blocks
    ("video_32k", dict(N=600, N_alloc=640, Hq=2, Hkv=2, grid=(3, 10, 20))),
    ("dlm_16k", dict(N=300 * 128 - 5, Hq=2, Hkv=1)),               # 300 blocks
])
def test_selection_by_mass(name, over, tau, shared):
    # the shortest top-ranked prefix reaching the softmax share tau; the GPU
    # sums in fp32, so where its cut differs from the oracle's the oracle's
    # shares must put that cut within 1e-4 of tau, and the kept set must be
    # the top m of the ranking outside near-ties
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    Qd, Kd = to_dev(Q, w.dtype), to_dev(K, w.dtype)
    shape = api.Shape.of(Qd, Kd, w.N, w.block)
    flags = api.SELECT_BY_MASS | (api.SELECT_SHARED_GQA if shared else 0)
    idx, cnt = api.select(api.stats(Qd, Kd, shape), shape, tau, flags=flags)
    torch.cuda.synchronize()
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    qm, qv, _ = O.block_stats(Q, w.N, w.block)
    km, kv, kc = O.block_stats(K, w.N, w.block)
    R = O.selection_scores(O.corrected_scores(qm, qv, km, kv, kc, w.d ** -0.5), w.Hkv, shared_gqa=shared)
    idx_ref, cnt_ref = O.select_by_mass(R, tau)
    band = 1e-4
    moved = 0
    for pos in np.ndindex(cnt.shape):
        m = int(cnt[pos])
        assert 1 <= m <= w.nb and (idx[pos][m:] == -1).all() and (np.diff(idx[pos][:m]) > 0).all()
        if m == cnt_ref[pos] and (idx[pos][:m] == idx_ref[pos][:m]).all():
            continue
        moved += 1
        row = R[pos]
        order = np.argsort(-row, kind="stable")
        e = np.exp(row - row.max())
        share = np.cumsum(e[order]) / e.sum()
        assert share[m - 1] >= tau - band and (m == 1 or share[m - 2] < tau + band), (pos, m, cnt_ref[pos])
        got = np.zeros(w.nb, bool)
        got[idx[pos][:m]] = True
        top = np.zeros(w.nb, bool)
        top[order[:m]] = True
        near = O.near_tie_mask(row[None], m, NEAR_TIE_REL)[0]
        assert not ((got != top) & ~near).any()
    assert moved <= max(2, cnt.size // 50), moved


def test_complement_lists_long_rows_and_odd_entries():
    # 2000 blocks (63 bitmap words, two rounds of 32), random kept sets of
    # every size, duplicate and out-of-range entries (ignored and flagged)
    B, H, nb, kmax = 1, 3, 2000, 64
    N = nb * 16
    rng = np.random.default_rng(9)
    idx = np.full((B, H, nb, kmax), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nb), dtype=np.int32)
    for pos in np.ndindex(cnt.shape):
        c = int(rng.integers(0, kmax + 1))
        idx[pos][:c] = np.sort(rng.choice(nb, size=c, replace=False))
        cnt[pos] = c
    idx[0, 0, 0, :3] = [5, 5, 7]                         # a duplicate
    cnt[0, 0, 0] = 3
    shape = api.Shape(B, H, H, N, N, 64, 16, api.DTYPE_F32)
    c_idx, c_cnt = api.complement_lists(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), shape)
    torch.cuda.synchronize()
    ref_idx, ref_cnt = O.complement_lists(idx, cnt, nb)
    np.testing.assert_array_equal(c_cnt.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(c_idx.cpu().numpy(), ref_idx)
    idx[0, 1, 0, 0] = nb + 3                              # out of range: ignored, flagged
    cnt[0, 1, 0] = max(int(cnt[0, 1, 0]), 1)
    c_idx, c_cnt = api.complement_lists(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), shape)
    st, word = api.get_device_error()
    assert st == 5 and word & 0x1                          # BA_ERR_DEVICE, BA_DEVERR_BAD_INDEX
    ref_idx, ref_cnt = O.complement_lists(idx, cnt, nb)
    np.testing.assert_array_equal(c_idx.cpu().numpy(), ref_idx)


@pytest.mark.parametrize("name,over,keep", [
    ("dlm_16k", dict(N=2048 - 30, N_alloc=2048, Hq=4, Hkv=2), 0.25),    # tensor-core path, ragged tail
    ("tiny_fp32", dict(N=1000, N_alloc=1024), 0.5),                      # CUDA-core path, fp32
    ("tiny_fp32", dict(N=4800 - 7, N_alloc=4800, block=16, Hq=2, Hkv=1), 0.3),   # 300 blocks, 10 bitmap words
])
def test_complement_lists_and_cached_residual_is_dense(name, over, keep):
    # the complement lists equal the oracle's exactly; attention over the kept
    # blocks merged with attention over the rest is dense attention
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    r = run_gpu(Q, K, V, w, keep)
    shape = r["shape"]
    c_idx, c_cnt = api.complement_lists(r["idx_d"], r["cnt_d"], shape)
    ref_idx, ref_cnt = O.complement_lists(r["idx"], r["cnt"], w.nb)
    np.testing.assert_array_equal(c_cnt.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(c_idx.cpu().numpy(), ref_idx)
    O1, L1 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], r["idx_d"], r["cnt_d"], shape, out_dtype=torch.float32)
    Of, Lf = api.sparse_fwd_merge(r["Qd"], r["Kd"], r["Vd"], c_idx, c_cnt, shape, O1, L1)
    torch.cuda.synchronize()
    Od, Ld = O.dense_attention(Q, K, V, w.N, w.d ** -0.5)
    tol = TOL[w.dtype]
    got = Of[:, :, :w.N].float().cpu().numpy()
    assert max_abs(got, Od) <= tol["max_abs"] and rel_l2(got, Od) <= tol["rel_l2"]
    assert max_abs(Lf[:, :, :w.N].cpu().numpy(), Ld) <= tol["lse_abs"]
    # keep = 1: nothing is left out
    idx_all, cnt_all = api.select(api.stats(r["Qd"], r["Kd"], shape), shape, 1.0)
    c_idx, c_cnt = api.complement_lists(idx_all, cnt_all, shape)
    torch.cuda.synchronize()
    assert int(c_cnt.max()) == 0 and bool((c_idx == -1).all())


@pytest.mark.parametrize("name,over", [
    ("extreme_128k", dict(N=4096 - 50, N_alloc=4096, Hq=4, Hkv=2)),      # tensor-core path, ragged tail
    ("tiny_fp32", dict(N=1000, N_alloc=1024)),                             # CUDA-core path, fp32
    ("dlm_16k", dict(N=1024, Hq=2, Hkv=1, d=64, block=64)),                # tensor-core path, 64-row blocks
    ("dlm_16k", dict(N=1024 - 3, N_alloc=1024, Hq=2, Hkv=1, block=32)),    # CUDA-core path, bf16 inputs
    ("dlm_16k", dict(N=2048 - 40, N_alloc=2048, Hq=4, Hkv=2, d=64)),       # tensor-core path, d = 64
])
def test_fused_merge_equals_separate_merge(name, over):
    # attention over span B merged in the epilogue with the partial over span A
    # equals the separate partial + ba_att_merge_lse bit for bit, and the
    # oracle's attention over the union at the parity bar
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    r = run_gpu(Q, K, V, w, 0.5)
    shape = r["shape"]
    split = w.nb // 2
    lo_i, lo_c, hi_i, hi_c = api.split_lists(r["idx_d"], r["cnt_d"], shape, split)
    O1, L1 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], lo_i, lo_c, shape, out_dtype=torch.float32)
    O2, L2 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], hi_i, hi_c, shape, out_dtype=torch.float32)
    for odt in {r["Qd"].dtype, torch.float32}:
        Om, Lm = api.merge_lse(O1, L1, O2, L2, out_dtype=odt)
        Of, Lf = api.sparse_fwd_merge(r["Qd"], r["Kd"], r["Vd"], hi_i, hi_c, shape, O1, L1, out_dtype=odt)
        torch.cuda.synchronize()
        n = w.N
        assert torch.equal(Of[:, :, :n], Om[:, :, :n]) and torch.equal(Lf[:, :, :n], Lm[:, :, :n])
    # in place into the fp32 partial
    O1c, L1c = O1.clone(), L1.clone()
    api.sparse_fwd_merge(r["Qd"], r["Kd"], r["Vd"], hi_i, hi_c, shape, O1c, L1c, out=(O1c, L1c))
    Om, Lm = api.merge_lse(O1, L1, O2, L2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(O1c[:, :, :w.N], Om[:, :, :w.N]) and torch.equal(L1c[:, :, :w.N], Lm[:, :, :w.N])
    tol = TOL[w.dtype]
    Oref, Lref = O.masked_attention(Q, K, V, r["idx"], r["cnt"], w.N, w.block, w.d ** -0.5)
    got = Of[:, :, :w.N].float().cpu().numpy()
    assert max_abs(got, Oref[:, :, :w.N]) <= tol["max_abs"] and rel_l2(got, Oref[:, :, :w.N]) <= tol["rel_l2"]
    assert max_abs(Lf[:, :, :w.N].cpu().numpy(), Lref[:, :, :w.N]) <= tol["lse_abs"]


@pytest.mark.parametrize("name,over,split,chunk", [
    ("extreme_128k", dict(N=4096 - 50, N_alloc=4096, Hq=8, Hkv=4), True, 0),    # split + merge, 4 chunks of 1
    ("extreme_128k", dict(N=4096, Hq=8, Hkv=4), False, 3),                      # chunks of 3 + 1 KV heads
    ("dlm_16k", dict(N=2048, Hq=4, Hkv=2, B=2), True, 2),                       # one chunk per batch entry
    ("tiny_fp32", dict(N=1000, N_alloc=1024), False, 1),                        # fp32, CUDA-core attention
    ("dlm_16k", dict(N=3000, N_alloc=3072, Hq=4, Hkv=2, block_k=64), True, 1),   # asymmetric 128 x 64, split
    ("dlm_16k", dict(N=2048 - 20, N_alloc=2048, Hq=4, Hkv=2, block=256), False, 0),  # 256-row blocks
    ("dlm_16k", dict(N=2048, Hq=12, Hkv=4), False, 1),        # 3 query heads per KV head, 4 chunks
    ("dlm_16k", dict(N=1024, B=2, Hq=4, Hkv=2), True, 1),     # chunks across batch entries, split
])
def test_forward_host_pipeline(name, over, split, chunk):
    # host buffers in and out, chunked and pipelined: bit-identical to the
    # device-resident calls on the same heads, and at the parity bar
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    keep = 0.5
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Qh, Kh, Vh = (torch.from_numpy(np.ascontiguousarray(x)).to(tdt).pin_memory() for x in (Q, K, V))
    split_block = meta.get("split_block", w.nk // 2) if split else -1
    Oh = torch.full(Qh.shape, 7.0, dtype=tdt).pin_memory()              # padding rows must stay untouched
    Lh = torch.full(Qh.shape[:3], 7.0, dtype=torch.float32).pin_memory()
    api.forward_host(Qh, Kh, Vh, w.N, w.block, keep, split_block=split_block, kv_heads_per_chunk=chunk, out=(Oh, Lh),
                     block_k=w.block_k)
    torch.cuda.synchronize()
    # the same steps on device-resident buffers
    r = run_gpu(Q, K, V, w, keep)
    if split:
        lo_i, lo_c, hi_i, hi_c = api.split_lists(r["idx_d"], r["cnt_d"], r["shape"], split_block)
        O1, L1 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], lo_i, lo_c, r["shape"], out_dtype=torch.float32)
        O2, L2 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], hi_i, hi_c, r["shape"], out_dtype=torch.float32)
        Od, Ld = api.merge_lse(O1, L1, O2, L2, out_dtype=tdt)
    else:
        Od, Ld = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], r["idx_d"], r["cnt_d"], r["shape"])
    torch.cuda.synchronize()
    n = w.N
    assert torch.equal(Oh[:, :, :n], Od[:, :, :n].cpu()), "host pipeline differs from the device-resident calls"
    assert torch.equal(Lh[:, :, :n], Ld[:, :, :n].cpu())
    assert (Oh[:, :, n:] == 7.0).all() and (Lh[:, :, n:] == 7.0).all()
    tol = TOL[w.dtype]
    Oref, Lref = O.masked_attention(Q, K, V, r["idx"], r["cnt"], w.N, w.block, w.d ** -0.5, b_k=w.kb)
    got = Oh[:, :, :n].float().numpy()
    assert max_abs(got, Oref[:, :, :n]) <= tol["max_abs"] and rel_l2(got, Oref[:, :, :n]) <= tol["rel_l2"]
    assert max_abs(Lh[:, :, :n].numpy(), Lref[:, :, :n]) <= tol["lse_abs"]


@pytest.mark.parametrize("dtype,out,d", [("bf16", "bf16", 128), ("f32", "f32", 64), ("bf16", "bf16", 64),
                                         ("f32", "f32", 128), ("f32", "bf16", 128), ("f32", "bf16", 64)])
def test_merge_parity_and_edges(dtype, out, d):
    rng = np.random.default_rng(3)
    rows = 1000
    O1 = rng.standard_normal((rows, d)).astype(np.float32)
    O2 = rng.standard_normal((rows, d)).astype(np.float32)
    L1 = (rng.standard_normal(rows) * 5).astype(np.float32)
    L2 = (rng.standard_normal(rows) * 5).astype(np.float32)
    L1[:10] = -np.inf
    L2[5:15] = -np.inf                    # rows 5..9 empty on both sides
    L1[20] = 80.0
    L2[20] = -80.0
    O1d, O2d = to_dev(O1, dtype), to_dev(O2, dtype)
    L1d, L2d = torch.from_numpy(L1).cuda(), torch.from_numpy(L2).cuda()
    out_dt = torch.bfloat16 if out == "bf16" else torch.float32
    Om, Lm = api.merge_lse(O1d, L1d, O2d, L2d, out_dtype=out_dt)
    Oref, Lref = O.merge_lse(O1d.float().cpu().numpy(), L1, O2d.float().cpu().numpy(), L2)
    err = np.abs(Om.float().cpu().numpy() - Oref)
    if out == "bf16":        # one round-to-nearest-even to bf16: half an ulp, 2^-9 relative
        assert np.all(err <= 2.0 ** -8 * np.abs(Oref) + 1e-6), err.max()
    else:
        assert np.all(err <= 1e-6 * np.abs(Oref) + 1e-6), err.max()
    Lg = Lm.cpu().numpy()
    assert np.isneginf(Lg[5:10]).all() and (Om[5:10].float() == 0).all()
    fin = np.isfinite(Lref)
    assert np.all(np.abs(Lg[fin] - Lref[fin]) <= 1e-6 * np.abs(Lref[fin]) + 1e-5)
    if dtype == out:
        # in place: the output aliases the first input
        api.merge_lse(O1d, L1d, O2d, L2d, out=(O1d, L1d))
        torch.cuda.synchronize()
        assert torch.equal(O1d, Om) and torch.equal(L1d, Lm)


@pytest.mark.parametrize("block", [128, 256])
def test_empty_lists_and_single_block_lists(block):
    Q, K, V, meta = make_inputs("dlm_16k", N=1024, Hq=2, Hkv=1, block=block)
    w = meta["workload"]
    Qd, Kd, Vd = to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16")
    shape = api.Shape.of(Qd, Kd, w.N, w.block)
    nb = w.nb
    idx = torch.full((1, 2, nb, 4), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, 2, nb), dtype=torch.int32, device="cuda")
    idx[0, 0, :, 0] = torch.arange(nb, dtype=torch.int32)         # head 0: the diagonal block only
    cnt[0, 0] = 1
    Od, Ld = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, shape)
    torch.cuda.synchronize()
    assert (Od[0, 1] == 0).all() and torch.isneginf(Ld[0, 1]).all()
    Oref, Lref = O.masked_attention(Q, K, V, idx.cpu().numpy(), cnt.cpu().numpy(), w.N, w.block, w.d ** -0.5,
                                    query_blocks=[(0, 0, i) for i in range(nb)])
    assert max_abs(Od[0, 0].float().cpu().numpy(), Oref[0, 0]) <= TOL["bf16"]["max_abs"]
    assert max_abs(Ld[0, 0].cpu().numpy(), Lref[0, 0]) <= TOL["bf16"]["lse_abs"]


def test_post_downsample_mass_via_single_block_lists():
    # check (4) through the GPU: per-block LSEs from single-block lists give
    # the exact post-downsample map, matched against the oracle's brute force
    Q, K, V, meta = make_inputs("tiny_fp32", N=512)
    w = meta["workload"]
    Qd, Kd, Vd = to_dev(Q, "f32"), to_dev(K, "f32"), to_dev(V, "f32")
    shape = api.Shape.of(Qd, Kd, w.N, w.block)
    nb = w.nb
    L_single = np.empty((w.Hq, nb, w.N))
    for j in range(nb):
        idx = torch.full((1, w.Hq, nb, 1), j, dtype=torch.int32, device="cuda")
        cnt = torch.ones((1, w.Hq, nb), dtype=torch.int32, device="cuda")
        _, L = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, shape)
        L_single[:, j] = L[0].cpu().numpy()
    idx = torch.arange(nb, dtype=torch.int32, device="cuda").expand(1, w.Hq, nb, nb).contiguous()
    cnt = torch.full((1, w.Hq, nb), nb, dtype=torch.int32, device="cuda")
    _, Lf = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, shape)
    A = O.post_downsample_map(Q, K, w.N, w.block, w.d ** -0.5)
    for h in range(w.Hq):
        A_gpu = O.block_mass_via_lse(L_single[h], Lf[0, h].cpu().numpy(), O.block_counts(w.N, w.block))
        assert max_abs(A_gpu, A[0, h]) <= 1e-4


def test_device_checks_flag_bad_lists_without_trapping():
    Q, K, V, meta = make_inputs("dlm_16k", N=1024, Hq=2, Hkv=1)
    w = meta["workload"]
    for dtype, d, block in (("bf16", 128, 128), ("bf16", 128, 256), ("f32", 128, 64)):
        Qd, Kd, Vd = to_dev(Q, dtype), to_dev(K, dtype), to_dev(V, dtype)
        shape = api.Shape.of(Qd, Kd, w.N, block)
        nb = shape.nb
        idx = torch.tensor([[0, 1, 2, 3]], dtype=torch.int32, device="cuda").repeat(2 * nb, 1).reshape(1, 2, nb, 4)
        cnt = torch.full((1, 2, nb), 4, dtype=torch.int32, device="cuda")
        ref_O, ref_L = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, shape)
        bad = idx.clone()
        bad[0, 0, 0, 3] = nb + 5                     # out of range: skipped, flagged
        Ob, Lb = api.sparse_fwd(Qd, Kd, Vd, bad, cnt, shape)
        st, word = api.get_device_error()
        assert st == 5 and word & 0x1, (st, word)
        three = idx.clone()
        three[0, 0, 0, 3] = -1
        O3, L3 = api.sparse_fwd(Qd, Kd, Vd, three[..., :3].contiguous(), torch.full_like(cnt, 3), shape)
        api.get_device_error()
        assert torch.allclose(Ob[0, 0, :block].float(), O3[0, 0, :block].float(), atol=1e-6)
        # count above kmax: clamped and flagged
        api.sparse_fwd(Qd, Kd, Vd, idx, torch.full_like(cnt, 9), shape)
        st, word = api.get_device_error()
        assert st == 5 and word & 0x2
        # not ascending
        desc = idx.flip(-1).contiguous()
        api.sparse_fwd(Qd, Kd, Vd, desc, cnt, shape)
        st, word = api.get_device_error()
        assert st == 5 and word & 0x4
        # the context stays usable
        O4, L4 = api.sparse_fwd(Qd, Kd, Vd, idx, cnt, shape)
        assert torch.equal(O4, ref_O)
        assert api.get_device_error() == (0, 0)


def test_bounded_wait_gives_up_and_context_survives():
    api.selftest_bounded_wait(20_000)                 # 20 ms on a barrier nobody arrives on
    st, word = api.get_device_error()
    assert st == 6 and word & 0x8
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0
    assert api.get_device_error() == (0, 0)


FUZZ = [("bf16", 128), ("bf16", 128), ("bf16", 128), ("bf16", 64), ("f32", 64), ("f32", 128), ("bf16", 128),
        ("f32", 64)]


@pytest.mark.parametrize("seed", range(len(FUZZ)))
def test_fuzz_small_shapes(seed):
    rng = np.random.default_rng(100 + seed)
    dtype, d = FUZZ[seed]
    # bf16 with d = 128 takes the tensor-core path only at block 128
    block = 128 if (dtype == "bf16" and d == 128 and seed != 6) else int(rng.choice([32, 64, 128]))
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.integers(1, 4))
    N = int(rng.integers(block + 1, 9 * block))
    N_alloc = N + int(rng.integers(0, 40))
    B = int(rng.integers(1, 3))
    keep = float(rng.uniform(0.05, 1.0))
    Q = rng.standard_normal((B, Hq, N_alloc, d)).astype(np.float32)
    K = rng.standard_normal((B, Hkv, N_alloc, d)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, N_alloc, d)).astype(np.float32)
    from block_sparse_attention_ba_b200.workloads import Workload, round_to
    Q, K, V = (round_to(x, dtype) for x in (Q, K, V))
    w = Workload("fuzz", B, Hq, Hkv, N, N_alloc, d, block, dtype, (keep,), seed, "iid_planted")
    r = run_gpu(Q, K, V, w, keep, kmax=O.keep_count(keep, w.nb) + 3)
    st = check_stats(r, Q, K, w)
    check_selection(r, st, w, keep)
    check_attention(r, Q, K, V, w, all_blocks(w))


@pytest.mark.parametrize("seed", range(5))
def test_fuzz_cta_pair(seed):
    # 256-row query blocks at d = 128 (the CTA pair) on random shapes: ragged
    # tails (a pair whose second CTA holds no row included), GQA ratios, key
    # blocks of 64, 128 or 256 rows, keep ratios from sparse to dense
    rng = np.random.default_rng(500 + seed)
    block_k = int(rng.choice([64, 128, 256]))
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.integers(1, 4))
    N = int(rng.integers(257, 9 * 256))
    if seed == 0:
        N = 2 * 256 + 40                          # the last pair's second CTA is past the end
    N_alloc = N + int(rng.integers(0, 40))
    B = int(rng.integers(1, 3))
    keep = float(rng.uniform(0.05, 1.0))
    Q = rng.standard_normal((B, Hq, N_alloc, 128)).astype(np.float32)
    K = rng.standard_normal((B, Hkv, N_alloc, 128)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, N_alloc, 128)).astype(np.float32)
    from block_sparse_attention_ba_b200.workloads import Workload, round_to
    Q, K, V = (round_to(x, "bf16") for x in (Q, K, V))
    w = Workload("fuzz", B, Hq, Hkv, N, N_alloc, 128, 256, "bf16", (keep,), seed, "iid_planted", block_k=block_k)
    r = run_gpu(Q, K, V, w, keep, kmax=O.keep_count(keep, w.nk) + 2)
    st = check_stats(r, Q, K, w)
    check_selection(r, st, w, keep)
    check_attention(r, Q, K, V, w, all_blocks(w))


# ------------------------------------------------------------- full-size cases

@pytest.mark.parametrize("name", ["dlm_16k", "sweep_32k", "video_32k", "extreme_128k"])
def test_full_size_workloads(name):
    Q, K, V, meta = make_inputs(name)
    w = meta["workload"]
    for keep in w.keeps:
        r = run_gpu(Q, K, V, w, keep)
        st = check_stats(r, Q, K, w)
        flipped, near = check_selection(r, st, w, keep)
        print(f"{name} keep={keep}: near-tie blocks {near}, of which decided differently {flipped}")
        check_attention(r, Q, K, V, w, sample_blocks(w, per_head=1 if w.N > 65536 else 2))
        if w.split:
            shape = r["shape"]
            lo_i, lo_c, hi_i, hi_c = api.split_lists(r["idx_d"], r["cnt_d"], shape, meta["split_block"])
            O1, L1 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], lo_i, lo_c, shape, out_dtype=torch.float32)
            O2, L2 = api.sparse_fwd(r["Qd"], r["Kd"], r["Vd"], hi_i, hi_c, shape, out_dtype=torch.float32)
            Om, Lm = api.merge_lse(O1, L1, O2, L2, out_dtype=torch.bfloat16)
            torch.cuda.synchronize()
            Om = Om.float().cpu().numpy()
            assert max_abs(Om, r["O"]) <= TOL["bf16"]["max_abs"] and rel_l2(Om, r["O"]) <= TOL["bf16"]["rel_l2"]
            assert max_abs(Lm.cpu().numpy(), r["L"]) <= TOL["bf16"]["lse_abs"]
            # the merged output against the oracle on the sampled query blocks
            r2 = dict(r, O=Om, L=Lm.cpu().numpy())
            check_attention(r2, Q, K, V, w, sample_blocks(w, per_head=1, seed=1))
        del r
        torch.cuda.empty_cache()


@pytest.mark.parametrize("name,over", [
    ("tiny_fp32", dict(N=16384 - 5, N_alloc=16384, Hq=8, Hkv=8, block=16)),       # fp32, d 64: 16384 blocks
    ("dlm_16k", dict(N=16384, Hq=16, Hkv=4, d=64, block=16, block_k=32)),        # bf16, asymmetric: 18432 blocks
])
def test_stats_many_blocks(name, over):
    # enough blocks for the warp-per-block statistics kernel: statistics and
    # selection against the oracle
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    Qd, Kd = to_dev(Q, w.dtype), to_dev(K, w.dtype)
    shape = api.Shape.of(Qd, Kd, w.N, w.block, block_k=w.block_k)
    assert w.B * (w.Hq * w.nb + w.Hkv * w.nk) >= 16384
    st = api.stats(Qd, Kd, shape)
    idx, cnt, sc = api.select(st, shape, 0.5, with_scores=True)
    torch.cuda.synchronize()
    r = dict(stats=[t.cpu().numpy() for t in st], scores=sc.cpu().numpy(), idx=idx.cpu().numpy(), cnt=cnt.cpu().numpy())
    stats_ref = check_stats(r, Q, K, w)
    check_selection(r, stats_ref, w, 0.5)

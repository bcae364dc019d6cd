"""ba_att_selector: the selector stage in one call (statistics, scores, top-k),
with the augmented score features written once by the statistics pass and read
by a TMA-fed score GEMM. It must reproduce ba_att_stats followed by
ba_att_select bit for bit: statistics, score map and kept lists. That sequence
is itself held to the oracle by test_parity_gpu.py; here one case is also
checked against the oracle directly."""

import numpy as np
import pytest
import torch

from block_sparse_attention_ba_b200 import api
from block_sparse_attention_ba_b200.workloads import make_inputs

CASES = [
    ("tiny_fp32", {}, 0.5),                                            # fp32, d 64, block 64: 16 blocks in one tile
    ("tiny_fp32", dict(N=1000, N_alloc=1024), 0.25),                   # ragged tail
    ("tiny_fp32", dict(N=768, d=128, block=32), 0.3),                  # fp32 d 128, block 32
    ("dlm_16k", dict(N=2048, Hq=8, Hkv=2), 0.5),                       # bf16, GQA, 16 blocks
    ("dlm_16k", dict(N=1920 + 77, N_alloc=2048, Hq=4, Hkv=2), 0.5),    # ragged last block
    ("dlm_16k", dict(N=300 * 128 - 5, Hq=2, Hkv=2), 0.3),              # 300 blocks: 3 x 3 tiles, partial
    ("dlm_16k", dict(N=2048 - 17, N_alloc=2048, Hq=4, Hkv=2, d=64), 0.5),   # d 64
    ("dlm_16k", dict(N=1024, Hq=2, Hkv=1, d=64, block=64), 0.5),       # bf16 block 64
    ("dlm_16k", dict(N=1024, B=2, Hq=4, Hkv=2), 0.5),                  # two batches
    ("dlm_16k", dict(N=2048 - 40, N_alloc=2048, Hq=4, Hkv=2, d=64, block=256), 0.5),   # 256-row blocks, d 64
    ("dlm_16k", dict(N=2048 - 30, N_alloc=2048, Hq=4, Hkv=2, block_k=64), 0.5),      # asymmetric: 16 x 32 blocks
    ("dlm_16k", dict(N=3000, N_alloc=3072, Hq=2, Hkv=1, d=64, block_k=256), 0.3),    # asymmetric: 24 x 12 blocks
    ("tiny_fp32", dict(N=2048, d=128, block=128), 0.5),                # fp32 64 KB blocks, streamed in chunks
    ("dlm_16k", dict(N=4096 - 100, N_alloc=4096, Hq=4, Hkv=2, block=256), 0.5),   # bf16 d 128, 64 KB blocks
    # long key ranges: 4 to 6 key tiles per query tile, ragged last tile
    ("dlm_16k", dict(N=32768 - 100, N_alloc=32768, Hq=2, Hkv=1, block_k=64), 0.5),   # 256 x 511 blocks
    ("dlm_16k", dict(N=32768, B=2, Hq=4, Hkv=2, d=64, block_k=64), 0.3),            # d 64, two batches
    ("dlm_16k", dict(N=16384 * 3 - 7, N_alloc=16384 * 3, Hq=3, Hkv=1, block=64), 0.5),   # 768 x 768 blocks
]


def _run_both(name, over, keep):
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Qd, Kd = (torch.from_numpy(np.ascontiguousarray(x)).to(dt).cuda() for x in (Q, K))
    shape = api.Shape.of(Qd, Kd, w.N, w.block, block_k=w.block_k)
    st_ref = api.stats(Qd, Kd, shape)
    idx_ref, cnt_ref, sc_ref = api.select(st_ref, shape, keep, with_scores=True)
    # poison the outputs so that every written element is checked
    k = api.keep_count(shape, keep)
    out = (tuple(torch.full_like(t, float("nan")) for t in st_ref), torch.full_like(idx_ref, 7),
           torch.full_like(cnt_ref, 7), torch.full_like(sc_ref, float("nan")))
    ws = torch.full((api.selector_workspace_bytes(shape),), 0xFF, device="cuda", dtype=torch.uint8)
    st, idx, cnt, sc = api.selector(Qd, Kd, shape, keep, kmax=k, out=out, workspace=ws)
    torch.cuda.synchronize()
    status, word = api.get_device_error()
    assert status == 0, f"device error word {word:#x}"
    return (st_ref, idx_ref, cnt_ref, sc_ref), (st, idx, cnt, sc), (Q, K, w)


@pytest.mark.gpu
@pytest.mark.parametrize("name,over,keep", CASES)
def test_selector_equals_stats_then_select(name, over, keep):
    ref, got, _ = _run_both(name, over, keep)
    for a, b in zip(ref[0], got[0]):
        assert torch.equal(a, b)
    assert torch.equal(ref[3], got[3])
    assert torch.equal(ref[2], got[2])
    assert torch.equal(ref[1], got[1])


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["sweep_32k", "extreme_128k"])
def test_selector_full_size(name):
    keep = 0.5
    ref, got, _ = _run_both(name, {}, keep)
    for a, b in zip(ref[0], got[0]):
        assert torch.equal(a, b)
    assert torch.equal(ref[3], got[3])
    assert torch.equal(ref[2], got[2]) and torch.equal(ref[1], got[1])


@pytest.mark.gpu
def test_selector_against_oracle():
    from test_parity_gpu import check_selection, check_stats
    keep = 0.5
    _, (st, idx, cnt, sc), (Q, K, w) = _run_both("dlm_16k", dict(N=300 * 128 - 5, Hq=2, Hkv=2), keep)
    r = {"stats": [t.cpu().numpy() for t in st], "scores": sc.cpu().numpy(), "idx": idx.cpu().numpy(),
         "cnt": cnt.cpu().numpy()}
    stats_ref = check_stats(r, Q, K, w)
    check_selection(r, stats_ref, w, keep)


@pytest.mark.gpu
@pytest.mark.parametrize("name,over", [("dlm_16k", dict(N=2048 - 40, N_alloc=2048, Hq=8, Hkv=2)),
                                       ("dlm_16k", dict(N=300 * 128 - 5, Hq=2, Hkv=2)),
                                       ("dlm_16k", dict(N=1024, B=2, Hq=4, Hkv=2, d=64))])
def test_selector_without_score_map_and_reused_workspace(name, over):
    # block_scores NULL: the map stays in the workspace and the lists are the
    # same; a second call on the same (now used) workspace gives them again
    keep = 0.5
    (st_ref, idx_ref, cnt_ref, _), _, _ = _run_both(name, over, keep)
    Q, K, V, meta = make_inputs(name, **over)
    w = meta["workload"]
    Qd, Kd = (torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda() for x in (Q, K))
    shape = api.Shape.of(Qd, Kd, w.N, w.block)
    ws = torch.full((api.selector_workspace_bytes(shape),), 0x5A, device="cuda", dtype=torch.uint8)
    for _ in range(2):
        st, idx, cnt, sc = api.selector(Qd, Kd, shape, keep, workspace=ws, with_scores=False)
        torch.cuda.synchronize()
        assert sc is None
        assert torch.equal(idx, idx_ref) and torch.equal(cnt, cnt_ref)
        for a, b in zip(st, st_ref):
            assert torch.equal(a, b)
    status, word = api.get_device_error()
    assert status == 0, f"device error word {word:#x}"

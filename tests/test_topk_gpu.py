"""ba_att_topk (the norm sorting step on a given score map) against the
oracle's select_topk, element for element: the kept columns are exact integer
work, so every list must match, ties, signed zeros, infinities and NaN
included (equal scores go to the lower column, NaN ranks last)."""

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_ba_b200 import api

pytestmark = pytest.mark.gpu


def _maps(nk, rows, seed):
    rng = np.random.default_rng(seed)
    out = {
        "normal": rng.standard_normal((rows, nk)).astype(np.float32),
        "few_values": rng.integers(0, 5, (rows, nk)).astype(np.float32),          # many exact ties
        "narrow_band": (1.0 + 1e-6 * rng.integers(0, 3, (rows, nk))).astype(np.float32),
        "constant": np.full((rows, nk), 0.25, dtype=np.float32),
    }
    wild = rng.standard_normal((rows, nk)).astype(np.float32)
    picks = rng.random((rows, nk))
    wild[picks < 0.05] = 0.0
    wild[(picks >= 0.05) & (picks < 0.10)] = -0.0
    wild[(picks >= 0.10) & (picks < 0.12)] = np.inf
    wild[(picks >= 0.12) & (picks < 0.15)] = -np.inf
    wild[(picks >= 0.15) & (picks < 0.17)] = np.nan
    wild[(picks >= 0.17) & (picks < 0.20)] = 3e38
    wild[(picks >= 0.20) & (picks < 0.23)] = 1e-38
    out["wild"] = wild
    # a long upper tail over a tight band, the shape of real block scores
    tail = (rng.standard_normal((rows, nk)) * 1e-3).astype(np.float32)
    tail[rng.random((rows, nk)) < 0.05] += 5.0
    out["band_and_tail"] = tail
    return out


@pytest.mark.parametrize("nk", [16, 64, 100, 255, 256, 257, 300, 512, 700, 1000, 1024, 1500, 4096])
def test_topk_matches_oracle(nk):
    rows = 300 if nk <= 1024 else 40
    for name, S in _maps(nk, rows, nk).items():
        Sd = torch.from_numpy(S).cuda()
        for k in sorted({1, max(1, nk // 4), max(1, nk // 2), max(1, nk - 1), nk, nk + 3}):
            kmax = max(k, nk // 2) + 2
            idx, cnt = api.topk(Sd, k, kmax=kmax)
            torch.cuda.synchronize()
            ref_idx, ref_cnt = O.select_topk(S, k, kmax=kmax)
            got_idx, got_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
            assert np.array_equal(got_cnt, ref_cnt), (name, k)
            bad = np.nonzero((got_idx != ref_idx).any(axis=1))[0]
            assert bad.size == 0, (name, k, int(bad[0]), got_idx[bad[0]][:16], ref_idx[bad[0]][:16])
    st, word = api.get_device_error()
    assert st == 0, f"device error word {word:#x}"

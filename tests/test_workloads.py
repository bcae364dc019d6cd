"""The seeded input generators follow the stated recipe: deterministic draws,
bf16 rounding to nearest even, the planted x3 key blocks, the needle's
added dot product, the video field's smoothness and zero padding, and the
split point's range. These inputs feed both the GPU path and the oracle."""

import numpy as np
import pytest
import torch

from block_sparse_attention_ba_b200.workloads import WORKLOADS, make_inputs, round_to


def test_draws_are_deterministic():
    a = make_inputs("dlm_16k", N=1024, Hq=4, Hkv=2)
    b = make_inputs("dlm_16k", N=1024, Hq=4, Hkv=2)
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(x, y)
    assert a[3] == b[3]


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(100000).astype(np.float32) * np.float32(37.0)
    # exact ties: a bf16 value plus half an ulp of its last kept bit
    base = round_to(x[:1000], "bf16").view(np.uint32)
    ties = (base | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, np.array([0.0, -0.0, 1.0, -2.5], dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(round_to(x, "bf16").view(np.uint32), ref.view(np.uint32))
    assert round_to(x, "f32") is x or np.array_equal(round_to(x, "f32"), x)


def test_inputs_are_exactly_representable_in_their_dtype():
    Q, K, V, _ = make_inputs("dlm_16k", N=512, Hq=2, Hkv=1)
    for x in (Q, K, V):
        assert np.array_equal(round_to(x, "bf16"), x)


def test_planted_key_blocks_are_scaled_by_three():
    w = WORKLOADS["dlm_16k"].with_(N=4096, N_alloc=4096, Hq=4, Hkv=2)
    Q, K, V, meta = make_inputs(w)
    planted = np.array(meta["planted_blocks"])
    assert planted.shape == (1, 2, max(1, round(0.05 * w.nb)))
    for g in range(w.Hkv):
        blocks = K[0, g].reshape(w.nb, w.block, w.d)
        # the shared direction adds 0.25 to E|k|^2 / d; x3 scales everything by 9
        msq = (blocks.astype(np.float64) ** 2).mean(axis=(1, 2))
        hot = np.zeros(w.nb, dtype=bool)
        hot[planted[0, g]] = True
        ratio = msq[hot].mean() / msq[~hot].mean()
        assert 8.5 < ratio < 9.5
        assert msq[~hot].max() < 2.0 and msq[hot].min() > 7.0


def test_needle_adds_four_standard_deviations_to_its_dot_products():
    w = WORKLOADS["sweep_32k"].with_(N=4096, N_alloc=4096, Hq=2, Hkv=1)
    Q, K, V, meta = make_inputs(w)
    s0, s1 = meta["needle_span"]
    rows = np.array(meta["needle_rows"])
    assert s1 - s0 == 512 and len(rows) == 8
    q = Q[0, 0].astype(np.float64)
    k = K[0, 0].astype(np.float64)
    span = np.arange(s0, s1)
    others = np.setdiff1d(np.arange(w.N), np.concatenate([span, rows]))
    rng = np.random.default_rng(0)
    far_keys = rng.choice(np.setdiff1d(np.arange(w.N), span), size=512, replace=False)
    needle = (q[rows] @ k[span].T).mean()
    base = (q[rows] @ k[far_keys].T).mean()
    # a^2 = 4 sqrt(d), plus what the planted x3 blocks inside the span add
    lift = needle - base
    assert 0.8 * 4 * np.sqrt(w.d) < lift < 3.5 * 4 * np.sqrt(w.d)
    # queries outside the needle rows see no such lift
    plain = (q[others[:64]] @ k[span].T).mean() - (q[others[:64]] @ k[far_keys].T).mean()
    assert abs(plain) < 0.5 * 4 * np.sqrt(w.d)


def test_video_field_is_smooth_along_tokens_and_padding_is_zero():
    w = WORKLOADS["video_32k"].with_(grid=(3, 6, 40), N=720, N_alloc=768, Hq=2, Hkv=2)
    Q, K, V, meta = make_inputs(w)
    assert meta["grid"] == [3, 6, 40]
    for x in (Q, K, V):
        assert not x[:, :, w.N:].any()
        t = x[0, 0, :w.N].astype(np.float64)
        # neighbours along w (t-major flattening) share the smoothed field;
        # unit noise of equal variance bounds the correlation near 1/2
        a, b = t[:-1].reshape(-1), t[1:].reshape(-1)
        c = np.corrcoef(a, b)[0, 1]
        assert 0.3 < c < 0.6
        assert 1.5 < t.var() < 2.5          # unit-variance field + unit noise


def test_split_point_is_an_interior_key_block():
    w = WORKLOADS["extreme_128k"].with_(N=8192, N_alloc=8192, Hq=2, Hkv=1)
    _, _, _, meta = make_inputs(w)
    assert 1 <= meta["split_block"] <= w.nk - 1

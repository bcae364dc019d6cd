"""Seeded synthetic inputs for the BA-Att hot path.

This module only draws random tensors with the shapes and structure of the
long-context language and video workloads the BA-Att paper evaluates on
(bidirectional diffusion-LM attention at 16K-128K tokens with grouped KV
heads; video-DiT attention over a flattened latent grid). It holds none of the
method's arithmetic, and it serves the GPU library, the CPU oracle, the tests
and the benchmark alike. No public benchmark item is reproduced: every tensor
is drawn from NumPy's PCG64 generator.

Each workload returns float32 NumPy arrays Q [B,Hq,N_alloc,d], K and V
[B,Hkv,N_alloc,d] rounded once to the compute dtype (bf16 via round-to-nearest
-even), so the GPU and the oracle see identical values.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    N_alloc: int
    d: int
    block: int
    dtype: str              # "f32" or "bf16"
    keeps: tuple
    seed: int
    kind: str               # "iid_planted" | "shared_dir" | "video_field"
    needle: bool = False
    split: bool = False
    grid: tuple | None = None   # (t, h, w) for video_field
    block_k: int = 0            # key block size when it differs from block (0: equal)

    @property
    def nb(self) -> int:
        """Query blocks."""
        return -(-self.N // self.block)

    @property
    def kb(self) -> int:
        return self.block_k if self.block_k > 0 else self.block

    @property
    def nk(self) -> int:
        """Key blocks."""
        return -(-self.N // self.kb)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads. Sizes follow the paper's settings: a tiny fp32 case,
# diffusion-LM long context (16K, 32K keep sweep, 128K with a partial merge)
# and a video-DiT latent grid (21 x 30 x 52 tokens, padded to 32768).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 2, 2, 1024, 1024, 64, 64, "f32", (0.5,), 0, "iid_planted"),
    "dlm_16k": Workload("dlm_16k", 1, 32, 8, 16384, 16384, 128, 128, "bf16", (0.5,), 1, "shared_dir"),
    "sweep_32k": Workload("sweep_32k", 1, 32, 8, 32768, 32768, 128, 128, "bf16", (1.0, 0.5, 0.25), 2,
                          "shared_dir", needle=True),
    "video_32k": Workload("video_32k", 1, 12, 12, 32760, 32768, 128, 128, "bf16", (0.5,), 3,
                          "video_field", grid=(21, 30, 52)),
    "extreme_128k": Workload("extreme_128k", 1, 32, 8, 131072, 131072, 128, 128, "bf16", (0.5,), 4,
                             "shared_dir", split=True),
}


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the storage dtype, returned as float32."""
    if dtype == "f32":
        return x.astype(np.float32, copy=False)
    if dtype == "bf16":
        u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
        # round to nearest even on the upper 16 bits (finite inputs)
        r = ((u >> 16) & 1) + np.uint32(0x7FFF)
        return ((u + r) & np.uint32(0xFFFF0000)).view(np.float32)
    raise ValueError(dtype)


def _normal(rng, shape):
    return rng.standard_normal(shape, dtype=np.float32)


def _gen_iid_planted(w: Workload):
    rng = np.random.default_rng(w.seed)
    Q = _normal(rng, (w.B, w.Hq, w.N_alloc, w.d))
    K = _normal(rng, (w.B, w.Hkv, w.N_alloc, w.d))
    V = _normal(rng, (w.B, w.Hkv, w.N_alloc, w.d))
    planted = np.sort(rng.choice(w.nb, size=2, replace=False))
    for j in planted:
        K[:, :, j * w.block:(j + 1) * w.block] *= 3.0
    return Q, K, V, {"planted_blocks": planted.tolist()}


def _gen_shared_dir(w: Workload):
    """Q,K = N(0,1) + 0.5 u_g (u_g a unit direction per KV head, shared by
    the query heads of its group); 5% of key blocks per KV head scaled by 3;
    V ~ N(0,1). Optionally a 512-token needle span of keys aligned with 8
    query rows (added dot product 4 standard deviations of q.k)."""
    rng = np.random.default_rng(w.seed)
    meta_rng = np.random.default_rng([w.seed, 1])
    group = w.Hq // w.Hkv
    u = _normal(rng, (w.B, w.Hkv, w.d))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    Q = _normal(rng, (w.B, w.Hq, w.N_alloc, w.d))
    Q += 0.5 * np.repeat(u, group, axis=1)[:, :, None, :]
    K = _normal(rng, (w.B, w.Hkv, w.N_alloc, w.d))
    K += 0.5 * u[:, :, None, :]
    V = _normal(rng, (w.B, w.Hkv, w.N_alloc, w.d))
    n_planted = max(1, int(round(0.05 * w.nb)))
    planted = np.zeros((w.B, w.Hkv, n_planted), dtype=np.int64)
    for bb in range(w.B):
        for g in range(w.Hkv):
            blocks = np.sort(meta_rng.choice(w.nb, size=n_planted, replace=False))
            planted[bb, g] = blocks
            for j in blocks:
                K[bb, g, j * w.block:min(w.N, (j + 1) * w.block)] *= 3.0
    meta = {"planted_blocks": planted.tolist()}
    if w.needle:
        span = min(512, w.N)
        start = int(meta_rng.integers(0, w.N - span + 1))
        rows = np.sort(meta_rng.choice(w.N, size=min(8, w.N), replace=False))
        wv = _normal(meta_rng, (w.d,))
        wv /= np.linalg.norm(wv)
        a = 2.0 * w.d ** 0.25          # a^2 = 4 sqrt(d): four standard deviations of q.k
        K[:, :, start:start + span] += a * wv
        Q[:, :, rows] += a * wv
        meta.update(needle_span=[start, start + span], needle_rows=rows.tolist())
    if w.split:
        meta["split_block"] = int(meta_rng.integers(1, w.nk))
    if w.N_alloc > w.N:
        Q[:, :, w.N:] = 0
        K[:, :, w.N:] = 0
        V[:, :, w.N:] = 0
    return Q, K, V, meta


def _smooth_axis(x: np.ndarray, axis: int, sigma: float) -> np.ndarray:
    """Separable Gaussian smoothing along one axis (zero padding at the edges)."""
    radius = int(math.ceil(4 * sigma))
    t = np.arange(-radius, radius + 1, dtype=np.float32)
    kern = np.exp(-0.5 * (t / sigma) ** 2)
    kern /= kern.sum()
    x = np.moveaxis(x, axis, -1)
    n = x.shape[-1]
    pad = np.zeros(x.shape[:-1] + (n + 2 * radius,), dtype=np.float32)
    pad[..., radius:radius + n] = x
    out = np.zeros_like(x)
    for o, c in enumerate(kern):
        out += c * pad[..., o:o + n]
    return np.moveaxis(out, -1, axis)


def _video_field(rng, heads: int, d: int, grid, sigma: float = 3.0):
    T, Hh, Ww = grid
    f = _normal(rng, (heads, d, T, Hh, Ww))
    for ax in (2, 3, 4):
        f = _smooth_axis(f, ax, sigma)
    f /= f.reshape(heads, d, -1).std(axis=-1)[:, :, None, None, None] + 1e-12
    f += _normal(rng, f.shape)
    # flatten t-major (t, h, w) -> token, then [heads, tokens, d]
    return np.ascontiguousarray(f.reshape(heads, d, T * Hh * Ww).transpose(0, 2, 1))


def _gen_video_field(w: Workload):
    rng = np.random.default_rng(w.seed)
    n_tok = int(np.prod(w.grid))
    assert n_tok == w.N and w.B == 1
    out = []
    for H in (w.Hq, w.Hkv, w.Hkv):
        X = np.zeros((1, H, w.N_alloc, w.d), dtype=np.float32)
        X[0, :, :n_tok] = _video_field(rng, H, w.d, w.grid)
        out.append(X)
    return out[0], out[1], out[2], {"grid": list(w.grid)}


def make_inputs_device(w: Workload | str, device, **overrides):
    """The same recipe drawn on a CUDA device with torch's generator, for
    timing runs at full size: (Q, K, V, meta) as bf16 (or fp32) device
    tensors. The structure (shared direction per KV head, planted x3 key
    blocks, needle, smoothed video field, zero padding rows, split point)
    matches make_inputs; the values differ, since the generator does. Parity
    tests use make_inputs, whose arrays the oracle also reads."""
    import torch
    import torch.nn.functional as F

    if isinstance(w, str):
        w = WORKLOADS[w]
    if overrides:
        if "N" in overrides and "N_alloc" not in overrides:
            overrides["N_alloc"] = overrides["N"]
        w = w.with_(**overrides)
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(1_000_003 * w.seed + 17)
    meta_rng = np.random.default_rng([w.seed, 1])
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    meta = {}
    if w.kind == "video_field":
        T, Hh, Ww = w.grid
        sigma = 3.0
        radius = int(math.ceil(4 * sigma))
        t = torch.arange(-radius, radius + 1, device=dev, dtype=torch.float32)
        kern = torch.exp(-0.5 * (t / sigma) ** 2)
        kern = (kern / kern.sum()).view(1, 1, -1)
        out = []
        for H in (w.Hq, w.Hkv, w.Hkv):
            f = randn(H * w.d, T, Hh, Ww)
            for ax in (1, 2, 3):                   # separable smoothing along t, h, w
                x = f.movedim(ax, -1)
                shp = x.shape
                x = F.conv1d(x.reshape(-1, 1, shp[-1]), kern, padding=radius).reshape(shp)
                f = x.movedim(-1, ax)
            f = f / (f.reshape(H * w.d, -1).std(dim=-1).view(-1, 1, 1, 1) + 1e-12)
            f = f + randn(*f.shape)
            X = torch.zeros((1, H, w.N_alloc, w.d), device=dev, dtype=tdt)
            X[0, :, :T * Hh * Ww] = f.reshape(H, w.d, -1).transpose(1, 2).to(tdt)
            out.append(X)
        Q, K, V = out
        meta["grid"] = list(w.grid)
    else:
        Q = randn(w.B, w.Hq, w.N_alloc, w.d)
        K = randn(w.B, w.Hkv, w.N_alloc, w.d)
        V = randn(w.B, w.Hkv, w.N_alloc, w.d)
        if w.kind == "shared_dir":
            group = w.Hq // w.Hkv
            u = randn(w.B, w.Hkv, w.d)
            u = u / u.norm(dim=-1, keepdim=True)
            Q += 0.5 * u.repeat_interleave(group, dim=1)[:, :, None, :]
            K += 0.5 * u[:, :, None, :]
            n_planted = max(1, int(round(0.05 * w.nb)))
        else:
            n_planted = 2
        for bb in range(w.B):
            for gg in range(w.Hkv if w.kind == "shared_dir" else 1):
                for j in np.sort(meta_rng.choice(w.nb, size=n_planted, replace=False)):
                    rows = slice(j * w.block, min(w.N, (j + 1) * w.block))
                    if w.kind == "shared_dir":
                        K[bb, gg, rows] *= 3.0
                    else:
                        K[:, :, rows] *= 3.0
        if w.needle:
            span = min(512, w.N)
            start = int(meta_rng.integers(0, w.N - span + 1))
            rows = np.sort(meta_rng.choice(w.N, size=min(8, w.N), replace=False))
            wv = randn(w.d)
            wv = wv / wv.norm()
            a = 2.0 * w.d ** 0.25
            K[:, :, start:start + span] += a * wv
            Q[:, :, torch.as_tensor(rows, device=dev)] += a * wv
            meta.update(needle_span=[start, start + span], needle_rows=rows.tolist())
        if w.N_alloc > w.N:
            Q[:, :, w.N:] = 0
            K[:, :, w.N:] = 0
            V[:, :, w.N:] = 0
        Q, K, V = Q.to(tdt), K.to(tdt), V.to(tdt)
    if w.split:
        meta["split_block"] = int(meta_rng.integers(1, w.nk))
    meta["workload"] = w
    return Q, K, V, meta


def make_inputs(w: Workload | str, **overrides):
    """Draw (Q, K, V, meta) for a workload; float32 arrays rounded to w.dtype.

    overrides (e.g. N=..., N_alloc=..., Hq=..., grid=...) build a smaller case
    of the same generator for fast tests.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if overrides:
        if "N" in overrides and "N_alloc" not in overrides:
            overrides["N_alloc"] = overrides["N"]
        w = w.with_(**overrides)
    gen = {"iid_planted": _gen_iid_planted, "shared_dir": _gen_shared_dir,
           "video_field": _gen_video_field}[w.kind]
    Q, K, V, meta = gen(w)
    if w.split and "split_block" not in meta:      # generators without their own split point
        meta["split_block"] = int(np.random.default_rng([w.seed, 2]).integers(1, w.nk))
    meta["workload"] = w
    return round_to(Q, w.dtype), round_to(K, w.dtype), round_to(V, w.dtype), meta

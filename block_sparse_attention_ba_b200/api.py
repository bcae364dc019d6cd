"""Thin ctypes binding over libbaatt.so (declared in include/ba_att.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels. PyTorch supplies device memory and the current stream; outputs
not passed in are allocated with ``torch.empty`` on the inputs' device. A
missing library, a CPU tensor, or a non-OK status raises.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))

BA_OK = 0
BA_ERR_INVALID_ARG = 1
STATUS_NAMES = {0: "BA_OK", 1: "BA_ERR_INVALID_ARG", 2: "BA_ERR_UNSUPPORTED", 3: "BA_ERR_MISALIGNED",
                4: "BA_ERR_CUDA", 5: "BA_ERR_DEVICE", 6: "BA_ERR_TIMEOUT"}
DTYPE_F32, DTYPE_BF16 = 0, 1
SELECT_NO_VAR_PRODUCT, SELECT_FORCE_DIAGONAL, SELECT_SHARED_GQA, SELECT_BY_MASS = 0x1, 0x2, 0x4, 0x8   # select_ex flags

# Entry points declared in include/ba_att.h: name -> (restype, argtypes)
_P = ctypes.c_void_p
_I32 = ctypes.c_int32


class CShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("N", ctypes.c_int32),
                ("N_alloc", ctypes.c_int32), ("d", ctypes.c_int32), ("block", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("sm_scale", ctypes.c_float), ("block_k", ctypes.c_int32)]


_SIGS = {
    "ba_att_version": (ctypes.c_char_p, []),
    "ba_att_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ba_att_num_blocks": (_I32, [ctypes.POINTER(CShape)]),
    "ba_att_num_key_blocks": (_I32, [ctypes.POINTER(CShape)]),
    "ba_att_keep_count": (_I32, [ctypes.POINTER(CShape), ctypes.c_double]),
    "ba_att_stats": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P, _P]),
    "ba_att_select": (ctypes.c_int, [ctypes.POINTER(CShape), ctypes.c_double, _P, _P, _P, _P, _P, _P, _I32, _P, _P]),
    "ba_att_select_ex": (ctypes.c_int, [ctypes.POINTER(CShape), ctypes.c_double, ctypes.c_uint32, _P, _P, _P, _P, _P,
                                         _P, _I32, _P, _P]),
    "ba_att_topk": (ctypes.c_int, [_P, ctypes.c_int64, _I32, _I32, _P, _P, _I32, _P]),
    "ba_att_selector_workspace": (ctypes.c_int64, [ctypes.POINTER(CShape)]),
    "ba_att_selector": (ctypes.c_int, [ctypes.POINTER(CShape), ctypes.c_double, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                        _P, _I32, _P]),
    "ba_att_split_lists": (ctypes.c_int, [ctypes.POINTER(CShape), _I32, _P, _P, _I32, _P, _P, _P, _P, _P]),
    "ba_att_complement_lists": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _I32, _P, _P, _I32, _P]),
    "ba_att_sparse_fwd": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _I32, _P, _I32, _P, _P]),
    "ba_att_merge_lse": (ctypes.c_int, [ctypes.c_int64, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P]),
    "ba_att_sparse_fwd_rows": (ctypes.c_int, [ctypes.POINTER(CShape), _I32, _I32, _P, _P, _P, _P, _P, _I32, _P, _P,
                                               _P, _I32, _P, _P]),
    "ba_att_sparse_fwd_merge": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _I32, _P, _P, _P, _I32, _P,
                                                _P]),
    "ba_att_get_device_error": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "ba_att_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint32, _P]),
    "ba_att_forward_host_workspace": (ctypes.c_int64, [ctypes.POINTER(CShape), ctypes.c_double, _I32, _I32]),
    "ba_att_forward_host": (ctypes.c_int, [ctypes.POINTER(CShape), ctypes.c_double, _I32, _I32, _P, _P, _P, _P, _P,
                                            _P, ctypes.c_int64, _P]),
    "ba_att_forward_host_noalloc": (ctypes.c_int, [ctypes.POINTER(CShape), ctypes.c_double, _I32, _P, _P, _P, _P,
                                                    _P, _P]),
}
STATIC_SCRATCH_BYTES = 512 << 20      # BA_ATT_STATIC_SCRATCH_BYTES

_lib = None
_lock = threading.Lock()


class BaAttError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


def library_path() -> str:
    return os.environ.get("BA_ATT_LIB", os.path.join(_HERE, "libbaatt.so"))


def load_library():
    """Load libbaatt.so (once). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing: build it with `python -m block_sparse_attention_ba_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _check(fn: str, status: int):
    if status != BA_OK:
        raise BaAttError(fn, status)


@dataclass(frozen=True)
class Shape:
    B: int
    Hq: int
    Hkv: int
    N: int
    N_alloc: int
    d: int
    block: int
    dtype: int
    sm_scale: float = 0.0
    block_k: int = 0          # key block size when it differs from block (0: equal)

    @property
    def nb(self) -> int:
        """Query blocks, ceil(N / block)."""
        return -(-self.N // self.block)

    @property
    def kb(self) -> int:
        """Key block size."""
        return self.block_k if self.block_k > 0 else self.block

    @property
    def nk(self) -> int:
        """Key blocks, ceil(N / key block size)."""
        return -(-self.N // self.kb)

    @property
    def scale(self) -> float:
        return self.sm_scale if self.sm_scale > 0 else 1.0 / math.sqrt(self.d)

    def c(self) -> CShape:
        return CShape(self.B, self.Hq, self.Hkv, self.N, self.N_alloc, self.d, self.block, self.dtype,
                      float(self.sm_scale), self.block_k)

    @staticmethod
    def of(Q: torch.Tensor, K: torch.Tensor, N: int | None = None, block: int = 128,
           sm_scale: float = 0.0, block_k: int = 0) -> "Shape":
        B, Hq, N_alloc, d = Q.shape
        dt = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(Q.dtype)
        if dt is None:
            raise TypeError(f"unsupported dtype {Q.dtype}")
        return Shape(B, Hq, K.shape[1], N_alloc if N is None else N, N_alloc, d, block, dt, sm_scale, block_k)


def _stream(t: torch.Tensor | None = None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _dev(t: torch.Tensor, name: str) -> ctypes.c_void_p:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def num_blocks(shape: Shape) -> int:
    return int(load_library().ba_att_num_blocks(ctypes.byref(shape.c())))


def keep_count(shape: Shape, keep: float) -> int:
    return int(load_library().ba_att_keep_count(ctypes.byref(shape.c()), ctypes.c_double(keep)))


def stats(Q: torch.Tensor, K: torch.Tensor, shape: Shape, out=None):
    """Per-block mean / population variance of Q and K (fp32)."""
    lib = load_library()
    dev = Q.device
    if out is None:
        out = (torch.empty((shape.B, shape.Hq, shape.nb, shape.d), device=dev, dtype=torch.float32),
               torch.empty((shape.B, shape.Hq, shape.nb, shape.d), device=dev, dtype=torch.float32),
               torch.empty((shape.B, shape.Hkv, shape.nk, shape.d), device=dev, dtype=torch.float32),
               torch.empty((shape.B, shape.Hkv, shape.nk, shape.d), device=dev, dtype=torch.float32))
    qm, qv, km, kv = out
    _check("ba_att_stats", lib.ba_att_stats(ctypes.byref(shape.c()), _dev(Q, "Q"), _dev(K, "K"), _dev(qm, "q_mean"),
                                            _dev(qv, "q_var"), _dev(km, "k_mean"), _dev(kv, "k_var"), _stream(Q)))
    return out


def select(stats_out, shape: Shape, keep: float, kmax: int | None = None, with_scores: bool = False, out=None,
           flags: int = 0):
    """Corrected block scores + top-k -> (idx, cnt), or (idx, cnt, scores) with with_scores.

    The score map [B, Hq, nq, nk] fp32 is always written; out = (idx, cnt, scores) may pass
    a preallocated one. flags: SELECT_* variants (ba_att_select_ex)."""
    lib = load_library()
    qm, qv, km, kv = stats_out
    k = keep_count(shape, keep)
    if k < 1:
        raise BaAttError("ba_att_keep_count", 1)
    if kmax is None:                     # by-mass counts vary per row, up to nk
        kmax = shape.nk if flags & SELECT_BY_MASS else k
    dev = qm.device
    if out is None:
        idx = torch.empty((shape.B, shape.Hq, shape.nb, kmax), device=dev, dtype=torch.int32)
        cnt = torch.empty((shape.B, shape.Hq, shape.nb), device=dev, dtype=torch.int32)
        sc = None
    else:
        idx, cnt, sc = out
    if sc is None:       # the score map is always written (the selection reads it back)
        sc = torch.empty((shape.B, shape.Hq, shape.nb, shape.nk), device=dev, dtype=torch.float32)
    _check("ba_att_select_ex", lib.ba_att_select_ex(
        ctypes.byref(shape.c()), ctypes.c_double(keep), ctypes.c_uint32(flags), _dev(qm, "q_mean"),
        _dev(qv, "q_var"), _dev(km, "k_mean"), _dev(kv, "k_var"), _dev(idx, "kv_idx"), _dev(cnt, "kv_cnt"),
        idx.shape[-1], _dev(sc, "block_scores"), _stream(qm)))
    return (idx, cnt, sc) if with_scores else (idx, cnt)


def topk(scores: torch.Tensor, k: int, kmax: int | None = None, out=None):
    """Norm sorting of a given fp32 score map [..., nk] (ba_att_topk) -> (idx [..., kmax], cnt [...])."""
    lib = load_library()
    if scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be a contiguous float32 tensor")
    nk = scores.shape[-1]
    rows = scores.numel() // nk
    kmax = k if kmax is None else kmax
    if out is None:
        idx = torch.empty(scores.shape[:-1] + (kmax,), device=scores.device, dtype=torch.int32)
        cnt = torch.empty(scores.shape[:-1], device=scores.device, dtype=torch.int32)
    else:
        idx, cnt = out
    _check("ba_att_topk", lib.ba_att_topk(_dev(scores, "block_scores"), rows, nk, k, _dev(idx, "kv_idx"),
                                          _dev(cnt, "kv_cnt"), idx.shape[-1], _stream(scores)))
    return idx, cnt


def selector_workspace_bytes(shape: Shape) -> int:
    """Device workspace bytes of ba_att_selector for this shape."""
    n = int(load_library().ba_att_selector_workspace(ctypes.byref(shape.c())))
    if n < 0:
        raise BaAttError("ba_att_selector_workspace", 1)
    return n


def selector(Q: torch.Tensor, K: torch.Tensor, shape: Shape, keep: float, kmax: int | None = None, out=None,
             workspace: torch.Tensor | None = None, with_scores: bool = True):
    """The whole selector in one call (ba_att_selector): stats, scores and top-k.

    Returns (stats, idx, cnt, scores) with stats = (q_mean, q_var, k_mean, k_var); out may
    pass the same tuple preallocated (its scores may be None), workspace a uint8 device
    tensor of at least selector_workspace_bytes(shape). With with_scores=False (or a None
    scores entry in out) no score map is returned (scores is None): the map stays in the
    workspace."""
    lib = load_library()
    k = keep_count(shape, keep)
    if k < 1:
        raise BaAttError("ba_att_keep_count", 1)
    kmax = k if kmax is None else kmax
    dev = Q.device
    if out is None:
        st = (torch.empty((shape.B, shape.Hq, shape.nb, shape.d), device=dev, dtype=torch.float32),
              torch.empty((shape.B, shape.Hq, shape.nb, shape.d), device=dev, dtype=torch.float32),
              torch.empty((shape.B, shape.Hkv, shape.nk, shape.d), device=dev, dtype=torch.float32),
              torch.empty((shape.B, shape.Hkv, shape.nk, shape.d), device=dev, dtype=torch.float32))
        idx = torch.empty((shape.B, shape.Hq, shape.nb, kmax), device=dev, dtype=torch.int32)
        cnt = torch.empty((shape.B, shape.Hq, shape.nb), device=dev, dtype=torch.int32)
        sc = (torch.empty((shape.B, shape.Hq, shape.nb, shape.nk), device=dev, dtype=torch.float32)
              if with_scores else None)
    else:
        st, idx, cnt, sc = out
    if workspace is None:
        workspace = torch.empty(selector_workspace_bytes(shape), device=dev, dtype=torch.uint8)
    qm, qv, km, kv = st
    _check("ba_att_selector", lib.ba_att_selector(
        ctypes.byref(shape.c()), ctypes.c_double(keep), _dev(Q, "Q"), _dev(K, "K"), _dev(qm, "q_mean"),
        _dev(qv, "q_var"), _dev(km, "k_mean"), _dev(kv, "k_var"), _dev(workspace, "workspace"),
        ctypes.c_void_p(0) if sc is None else _dev(sc, "block_scores"), _dev(idx, "kv_idx"), _dev(cnt, "kv_cnt"),
        idx.shape[-1], _stream(Q)))
    return st, idx, cnt, sc


def split_lists(idx: torch.Tensor, cnt: torch.Tensor, shape: Shape, split_block: int, out=None):
    """Partition kept lists at a key-block boundary -> (lo_idx, lo_cnt, hi_idx, hi_cnt)."""
    lib = load_library()
    if out is None:
        out = (torch.empty_like(idx), torch.empty_like(cnt), torch.empty_like(idx), torch.empty_like(cnt))
    lo_i, lo_c, hi_i, hi_c = out
    _check("ba_att_split_lists", lib.ba_att_split_lists(
        ctypes.byref(shape.c()), int(split_block), _dev(idx, "kv_idx"), _dev(cnt, "kv_cnt"), idx.shape[-1],
        _dev(lo_i, "lo_idx"), _dev(lo_c, "lo_cnt"), _dev(hi_i, "hi_idx"), _dev(hi_c, "hi_cnt"), _stream(idx)))
    return out


_TORCH_DT = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}


def complement_lists(idx, cnt, shape: Shape, out=None):
    """The key blocks each kept-block list leaves out -> (c_idx [.., nb], c_cnt)."""
    lib = load_library()
    if out is None:
        out = (torch.empty(idx.shape[:-1] + (shape.nk,), device=idx.device, dtype=torch.int32), torch.empty_like(cnt))
    c_idx, c_cnt = out
    _check("ba_att_complement_lists", lib.ba_att_complement_lists(
        ctypes.byref(shape.c()), _dev(idx, "kv_idx"), _dev(cnt, "kv_cnt"), idx.shape[-1], _dev(c_idx, "c_idx"),
        _dev(c_cnt, "c_cnt"), c_idx.shape[-1], _stream(idx)))
    return out


def sparse_fwd(Q, K, V, idx, cnt, shape: Shape, out=None, out_dtype=None):
    """Block-sparse attention over the kept blocks -> (O, LSE).

    out_dtype=torch.float32 keeps O in fp32 (for partials merged later)."""
    lib = load_library()
    if out is None:
        odt = Q.dtype if out_dtype is None else out_dtype
        out = (torch.empty(Q.shape, device=Q.device, dtype=odt),
               torch.empty((shape.B, shape.Hq, shape.N_alloc), device=Q.device, dtype=torch.float32))
    O, LSE = out
    _check("ba_att_sparse_fwd", lib.ba_att_sparse_fwd(
        ctypes.byref(shape.c()), _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(idx, "kv_idx"), _dev(cnt, "kv_cnt"),
        idx.shape[-1], _dev(O, "O"), _TORCH_DT[O.dtype], _dev(LSE, "LSE"), _stream(Q)))
    return out


def sparse_fwd_merge(Q, K, V, idx, cnt, shape: Shape, O_prev, L_prev, out=None, out_dtype=None):
    """Block-sparse attention over the kept blocks, merged in the epilogue with
    an earlier fp32 partial (O_prev, L_prev) over a disjoint key set -> (O, LSE).
    out may be (O_prev, L_prev) for an in-place fp32 merge."""
    lib = load_library()
    if O_prev.dtype != torch.float32 or L_prev.dtype != torch.float32:
        raise TypeError("O_prev and L_prev must be float32")
    if out is None:
        odt = Q.dtype if out_dtype is None else out_dtype
        out = (torch.empty(Q.shape, device=Q.device, dtype=odt),
               torch.empty((shape.B, shape.Hq, shape.N_alloc), device=Q.device, dtype=torch.float32))
    O, LSE = out
    _check("ba_att_sparse_fwd_merge", lib.ba_att_sparse_fwd_merge(
        ctypes.byref(shape.c()), _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(idx, "kv_idx"), _dev(cnt, "kv_cnt"),
        idx.shape[-1], _dev(O_prev, "O_prev"), _dev(L_prev, "L_prev"), _dev(O, "O"), _TORCH_DT[O.dtype],
        _dev(LSE, "LSE"), _stream(Q)))
    return out


def _rows_view(t: torch.Tensor, name: str, q_rows: int, d: int | None) -> int:
    """Row stride of a [B, H, rows, d] (or [B, H, rows]) CUDA tensor that is
    either contiguous or a slice of rows of a contiguous one (heads at a fixed
    stride of whole rows); the call reads and writes through its data pointer."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    inner = 1 if d is None else d
    st = t.stride()
    if (d is not None and st[3] != 1) or st[2] != inner or st[1] % inner != 0:
        raise ValueError(f"{name} must be contiguous or a slice of rows of a contiguous tensor")
    stride = st[1] // inner
    if stride < q_rows or st[0] != t.shape[1] * st[1]:
        raise ValueError(f"{name} must be contiguous or a slice of rows of a contiguous tensor")
    return stride


def sparse_fwd_rows(Qr, K, V, idx, cnt, shape: Shape, q_rows: int | None = None, O_prev=None, L_prev=None,
                    out=None, out_dtype=None):
    """Attention for one range of query rows only (ba_att_sparse_fwd_rows) -> (O, LSE).

    Qr [B, Hq, R, d] holds the range's rows: a contiguous tensor, or a slice of
    rows of a full one (e.g. Q[:, :, r0:r0 + R], r0 a multiple of 8), whose head
    stride becomes the call's row stride; q_rows defaults to R. K, V and `shape`
    describe the keys. idx/cnt list key blocks per query block of the range
    ([B, Hq, ceil(q_rows / block), kmax]). With (O_prev, L_prev), fp32, laid out
    like Qr, the result is merged with that cached partial in the epilogue; out
    (laid out like Qr, e.g. slices of full O/LSE tensors) may be (O_prev, L_prev)
    for an in-place fp32 merge."""
    lib = load_library()
    B, Hq, R, d = Qr.shape
    q_rows = R if q_rows is None else q_rows
    q_stride = _rows_view(Qr, "Q", q_rows, d)
    if (O_prev is None) != (L_prev is None):
        raise ValueError("pass both O_prev and L_prev, or neither")
    if O_prev is not None:
        if O_prev.dtype != torch.float32 or L_prev.dtype != torch.float32:
            raise TypeError("O_prev and L_prev must be float32")
        if _rows_view(O_prev, "O_prev", q_rows, d) != q_stride or _rows_view(L_prev, "L_prev", q_rows, None) != q_stride:
            raise ValueError("O_prev and L_prev must have Q's row stride")
    if out is None:
        odt = Qr.dtype if out_dtype is None else out_dtype
        full = (torch.empty((B, Hq, q_stride, d), device=Qr.device, dtype=odt),
                torch.empty((B, Hq, q_stride), device=Qr.device, dtype=torch.float32))
        out = (full[0][:, :, :R], full[1][:, :, :R])
    O, LSE = out
    if _rows_view(O, "O", q_rows, d) != q_stride or _rows_view(LSE, "LSE", q_rows, None) != q_stride:
        raise ValueError("O and LSE must have Q's row stride")
    null = ctypes.c_void_p(0)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    _check("ba_att_sparse_fwd_rows", lib.ba_att_sparse_fwd_rows(
        ctypes.byref(shape.c()), int(q_rows), int(q_stride), ptr(Qr), _dev(K, "K"), _dev(V, "V"),
        _dev(idx, "kv_idx"), _dev(cnt, "kv_cnt"), idx.shape[-1],
        null if O_prev is None else ptr(O_prev), null if L_prev is None else ptr(L_prev),
        ptr(O), _TORCH_DT[O.dtype], ptr(LSE), _stream(Qr)))
    return out


def merge_lse(O1, L1, O2, L2, out=None, out_dtype=None):
    """Log-space merge of two partial attentions -> (O, L).

    out may alias (O1, L1) when the dtypes agree; out_dtype=torch.bfloat16
    rounds fp32 partials once into a bf16 output."""
    lib = load_library()
    d = O1.shape[-1]
    rows = O1.numel() // d
    if out is None:
        out = (torch.empty(O1.shape, device=O1.device, dtype=O1.dtype if out_dtype is None else out_dtype),
               torch.empty_like(L1))
    O, L = out
    _check("ba_att_merge_lse", lib.ba_att_merge_lse(
        rows, d, _TORCH_DT[O1.dtype], _TORCH_DT[O.dtype], _dev(O1, "O1"), _dev(L1, "L1"), _dev(O2, "O2"),
        _dev(L2, "L2"), _dev(O, "O"), _dev(L, "L"), _stream(O1)))
    return out


def forward(Q, K, V, N: int, block: int, keep: float, sm_scale: float = 0.0, block_k: int = 0):
    """Full BA-Att forward: stats -> select -> sparse attention. Returns (O, LSE, idx, cnt)."""
    shape = Shape.of(Q, K, N, block, sm_scale, block_k)
    st = stats(Q, K, shape)
    idx, cnt = select(st, shape, keep)
    O, LSE = sparse_fwd(Q, K, V, idx, cnt, shape)
    return O, LSE, idx, cnt


def forward_host_workspace_bytes(shape: Shape, keep: float, split_block: int = -1, kv_heads_per_chunk: int = 0) -> int:
    """Device workspace bytes ba_att_forward_host needs (raises on arguments it would reject)."""
    n = load_library().ba_att_forward_host_workspace(ctypes.byref(shape.c()), float(keep), int(split_block),
                                                     int(kv_heads_per_chunk))
    if n < 0:
        raise BaAttError("ba_att_forward_host_workspace", BA_ERR_INVALID_ARG)
    return int(n)


def _host(t: torch.Tensor, name: str) -> ctypes.c_void_p:
    if t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host (CPU) tensor")
    return ctypes.c_void_p(t.data_ptr())


def forward_host(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, N: int, block: int, keep: float,
                 split_block: int = -1, kv_heads_per_chunk: int = 0, sm_scale: float = 0.0,
                 workspace: torch.Tensor | None = None, out=None, device=None, block_k: int = 0):
    """Whole forward from host tensors to host tensors (ba_att_forward_host):
    copies in, stats, select, sparse attention (split + merge when
    split_block >= 0), copies out, pipelined per chunk of KV heads. Q, K, V,
    and the outputs should be pinned for the copies to overlap compute.
    Asynchronous on the current stream; synchronise before reading (O, LSE)."""
    shape = Shape.of(Q, K, N, block, sm_scale, block_k)
    dev = torch.device("cuda") if device is None else torch.device(device)
    need = forward_host_workspace_bytes(shape, keep, split_block, kv_heads_per_chunk)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if not workspace.is_cuda or workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace must be a CUDA tensor of at least {need} bytes")
    if out is None:
        O = torch.empty(Q.shape, dtype=Q.dtype).pin_memory()
        LSE = torch.empty(Q.shape[:3], dtype=torch.float32).pin_memory()
    else:
        O, LSE = out
    lib = load_library()
    _check("ba_att_forward_host",
           lib.ba_att_forward_host(ctypes.byref(shape.c()), float(keep), int(split_block), int(kv_heads_per_chunk),
                                   _host(Q, "Q"), _host(K, "K"), _host(V, "V"), _host(O, "O"), _host(LSE, "LSE"),
                                   ctypes.c_void_p(workspace.data_ptr()), int(workspace.numel() * workspace.element_size()),
                                   ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))
    return O, LSE


def forward_host_noalloc(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, N: int, block: int, keep: float,
                         split_block: int = -1, sm_scale: float = 0.0, out=None, device=None, block_k: int = 0):
    """forward_host on the library's static device scratch (ba_att_forward_host_noalloc):
    no workspace argument, nothing allocated on the device by this call."""
    shape = Shape.of(Q, K, N, block, sm_scale, block_k)
    dev = torch.device("cuda") if device is None else torch.device(device)
    if out is None:
        O = torch.empty(Q.shape, dtype=Q.dtype).pin_memory()
        LSE = torch.empty(Q.shape[:3], dtype=torch.float32).pin_memory()
    else:
        O, LSE = out
    lib = load_library()
    _check("ba_att_forward_host_noalloc",
           lib.ba_att_forward_host_noalloc(ctypes.byref(shape.c()), float(keep), int(split_block), _host(Q, "Q"),
                                           _host(K, "K"), _host(V, "V"), _host(O, "O"), _host(LSE, "LSE"),
                                           ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))
    return O, LSE


def get_device_error(device=None):
    """Synchronise the current stream, read and clear the device error word -> (status, word)."""
    lib = load_library()
    word = ctypes.c_uint32(0)
    dev = torch.device("cuda") if device is None else torch.device(device)
    st = lib.ba_att_get_device_error(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream),
                                     ctypes.byref(word))
    return int(st), int(word.value)


def selftest_bounded_wait(timeout_us: int):
    lib = load_library()
    _check("ba_att_selftest_bounded_wait", lib.ba_att_selftest_bounded_wait(int(timeout_us), _stream()))

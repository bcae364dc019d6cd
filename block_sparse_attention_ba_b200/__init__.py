"""BA-Att for B200: block-wise pre-downsample selector + block-sparse attention.

The compute lives in a C-ABI shared library of hand-written sm_100a CUDA
kernels (``libbaatt.so``, declared in ``include/ba_att.h``). This package is
the thin Python binding over it: argument marshalling and stream plumbing
only. The library is loaded on first use; a missing library raises.
"""

from .api import (  # noqa: F401
    BaAttError,
    Shape,
    library_path,
    load_library,
    num_blocks,
    keep_count,
    stats,
    select,
    split_lists,
    sparse_fwd,
    merge_lse,
    forward,
    get_device_error,
)

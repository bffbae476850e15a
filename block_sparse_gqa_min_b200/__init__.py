"""Group-shared block-sparse GQA decode attention for NVIDIA B200 (sm_100a).

The compute path is libsba.so (CUDA kernels behind the C ABI in include/sba.h);
`sba` is its thin ctypes binding and `workloads` the seeded synthetic inputs.
The library is built in-tree on first use (nvcc, sm_100a) and every call goes
through it; there is no CPU fallback.
"""
from . import sba, workloads  # noqa: F401
from .sba import (  # noqa: F401
    Cache,
    SbaError,
    alloc_step,
    decode_step,
    sba_append_kv,
    sba_budget_from_sparsity,
    sba_combine,
    sba_default_num_splits,
    sba_num_selected,
    sba_score_select,
    sba_sparse_decode,
    sba_status_string,
    sba_update_descriptors,
    sba_workspace_size,
    select_params,
)

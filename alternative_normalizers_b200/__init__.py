"""B200-native fused attention with selectable row normalizers.

``O = N(scale * Q K^T + mask) V`` with N one of softmax, softmax1, sparsemax
and 1.5-entmax (and its backward), computed by the CUDA kernels of
``libnattn.so`` (sm_100a).
The Python layer only allocates with PyTorch and marshals arguments; build the
library with ``python -m alternative_normalizers_b200.build``.
"""

from .binding import (  # noqa: F401
    NattnArgs,
    NattnBwdArgs,
    NattnError,
    attention,
    attention_backward,
    build_args,
    build_bwd_args,
    lib,
    nattn_bwd,
    nattn_bwd_workspace_size,
    nattn_fwd,
    nattn_fwd_ex,
    nattn_get_device_status,
    nattn_selftest_wait_timeout,
    nattn_strerror,
    nattn_version,
    nattn_workspace_size,
    paged_attention,
    varlen_attention,
)
from .workloads import NORMALIZER_IDS, WORKLOADS, Workload  # noqa: F401

__version__ = "0.1.0"

"""B200-native (sm_100a) forward of a Mixture-of-Experts FFN layer.

Route (gate GEMM, softmax, top-k, renormalise, load-balance loss) -> permute
(histogram, scan, stable counting sort, capacity drop) -> gather -> grouped
expert FFN on the tcgen05 tensor cores -> weighted combine, behind the C ABI
of libmoe_b200.so (include/moe_b200.h). Importing the package loads that
library; if it is not built the import fails.
"""
from . import _abi  # noqa: F401  (loads libmoe_b200.so or raises)
from ._abi import (MoeError, moe_capacity, moe_combine, moe_expert_ffn, moe_forward,  # noqa: F401
                   moe_forward_host, moe_forward_views, moe_gather, moe_get_device_error,
                   moe_permute, moe_route, moe_rows_max, moe_workspace_init)
from .layer import MoeLayer  # noqa: F401

"""B200 (sm_100a) hybrid sparse-linear attention: SLA2 routing, block-sparse
softmax branch (bf16, FP8 or INT8 Q/K), ReLU linear branch, alpha combine, PISA
exact-or-approximate mode (zero-order terms, optional global first-order term).

The compute path is the CUDA library ``libsla.so`` (C ABI in ``include/sla.h``);
``block_sparse_linear_proj_b200.sla`` is its ctypes binding.  Importing the
package does not load the library; the first call does, and fails loudly if it
is missing.
"""
from . import sla  # noqa: F401
from .sla import (SLA_LUT_COMPUTE, SLA_LUT_GIVEN, SLA_OUT_BF16, SLA_OUT_FP32,  # noqa: F401
                  SLA_SPARSE_BF16, SLA_SPARSE_FP8_E4M3, SLA_SPARSE_INT8, SlaError, params,
                  sla_check_device_status, cocluster_workspace, sla_cocluster,
                  sla_forward, sla_forward_coclustered, sla_forward_host, sla_permute_rows,
                  sla_pisa_cov_norms, sla_pisa_forward, sla_pisa_forward_host, sla_profile_enable,
                  sla_profile_read, sla_route,
                  sla_workspace_size, workspace)

__version__ = "0.1.0"

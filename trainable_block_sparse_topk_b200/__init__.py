"""SAS gated block-sparse causal attention for B200 (sm_100a).

The compute lives in libsas.so (CUDA kernels behind the C ABI of
include/sas.h). `binding` exposes the C entry points under their own names,
`api` adds output allocation and an autograd Function, and `synth` draws the
seeded synthetic workloads. Importing the package does not load the library;
the first call does, and it raises if the library has not been built.
"""
from .binding import (SAS_DT_BF16, SAS_DT_FP32, SAS_GATE_NONE, SAS_GATE_SOFTMAX, SAS_OP_BWD,  # noqa: F401
                      SAS_OP_DECODE, SAS_OP_FWD, SAS_OP_TOPK, SasError, make_desc, sas_block_topk,
                      sas_desc, sas_device_timeouts, sas_kernel_launches, sas_gated_attn_bwd, sas_gated_attn_fwd,
                      sas_sparse_decode, sas_status_string, sas_workspace_size)

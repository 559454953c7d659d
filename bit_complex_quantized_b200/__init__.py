"""B200-native PhaseQuant and multiplication-free complex GEMV/GEMM (libifq).

The compute path is the CUDA library libifq.so (include/ifq.h); this package
holds its ctypes binding (_lib), the in-tree build script (build) and the
seeded synthetic workload generator (workloads), and the host side of the
row split of a tensor across GPUs (shard).
"""
from ._lib import (  # noqa: F401
    EXPORTED,
    IFQ_DEV_NONFINITE,
    IFQ_DEV_TIMEOUT,
    IFQ_MAX_GEMV_BATCH,
    IFQ_MAX_GROUP,
    IFQ_MAX_STAGES,
    IFQ_QUANT_STATIC_SCRATCH_BYTES,
    GemvPlan,
    IfqError,
    LayerSet,
    LIB_PATH,
    ifq_dequantize,
    ifq_gemm,
    ifq_gemm_wait_limit,
    ifq_gemv,
    ifq_gemv_workspace_bytes,
    ifq_quantize_pack,
    ifq_quantize_finish,
    ifq_quantize_pack_static,
    ifq_quantize_stage,
    ifq_quantize_workspace_bytes,
    ifq_status_string,
    ifq_widely_linear_from_real,
    ifq_widely_linear_quantize_pack,
    ifq_widely_linear_quantize_workspace_bytes,
    load,
)

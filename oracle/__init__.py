"""Plain fp64 CPU oracle for PhaseQuant and the multiplication-free complex product.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may use it.  It shares no code with the CUDA library.

Sources, by page and section:
  * "Fairy2i write-up" (hotelren.com): §2.1 widely-linear transform,
    §3.1 phase rule, §3.2 axis scales, §4.1 recursive residual, §4.2 product.
  * "iFairy article" (bestcxt.com): §二.1 codebook, §二.2 multiplication-free GEMM.
  * "iFairy talk notes" (43b.com.cn): §2.2.2 phase rule, §2.3.1 x i = swap + negate,
    §2.1.3 rotary position code, §2.1.4 real-part attention score.
  * "iFairy article" §三: complex rotary position code as one complex multiply.
"""
from .phasequant import (  # noqa: F401
    CODEBOOK,
    widely_linear_from_real,
    widely_linear_planes_fp32,
    phase_code,
    phase_code_atan2,
    code_to_br_bi,
    quantize_stage,
    quantize_tensor,
    residual_after,
    pack_codes,
    unpack_codes,
    dequantize,
    dequantize_bf16,
    product,
    product_rows,
    tolerance_bound,
    rotate_outputs,
    score,
    near_boundary_mask,
    bf16_round,
    bf16_bits_to_f64,
)

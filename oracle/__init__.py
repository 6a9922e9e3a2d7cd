"""CPU oracle for the mixed-precision routed-expert layer.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The library's compute path
never imports this package, and this package never imports the library's
compute path: its one import from the package is the seeded input generators
(``mixed_precision_moe_b200.synth``), which hold none of the method's arithmetic.

The arithmetic lives in ``moe_oracle.c`` (plain C, IEEE binary64); this module
only builds it with gcc and marshals numpy arrays through ctypes.
"""
from .oracle import (  # noqa: F401
    BF16, INT8, INT4, build, num_threads, set_num_threads, bf16_to_double, fp16_to_double,
    fp16_from_float, quantize, dequantize, router_logits, route_topk, permute, grouped_ffn,
    combine, moe_layer, Expert, seeded_experts,
)

"""Float64 CPU oracle for the ISPA warmup path -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package. The CUDA library never calls it and shares no code with
it; the two meet only in the seeded input generator (``ispa_synth``).

Every function restates the definition it follows from "Towards
Memory-Efficient Autoregressive Video Generation via Instance-Specific
Parametric Absorption" (the Dutch technical summary, section 2, with the
identical Portuguese summary as a cross-check). All pins live in
``tests/test_oracle.py``; no function here is "parity unpinned".
"""
from .ispa_oracle import (  # noqa: F401
    branch_attention,
    dual_attention,
    local_attention,
    gram,
    default_lambda,
    absorb,
    reconstruction_error,
    streaming_layer,
    quantize_rows_int8,
    project_w8a8,
    rank_layers,
    warmup_layer,
    as_f64,
)

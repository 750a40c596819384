"""Float64 CPU oracle of the GPTQ layer quantizer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package.  The CUDA library never does, and the
two share no code: the only thing both sides consume is the seeded input
generator in ``workloads.py``.

Every function cites the passage of the GPTQ pages it restates (page title and
section).  Heavy loops live in ``gptq_oracle.c`` (plain C, float64, OpenMP only
across independent rows or matrix entries); this module holds the glue and the
steps that are one library call (a matrix product, an inverse, a stable sort).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, brute force, invariants or hand-computed examples; none
is "parity unpinned".
"""
from .gptq import (  # noqa: F401
    GPTQResult,
    act_order,
    bf16_round,
    damp_lambda,
    dead_columns,
    dequant_matmul,
    dequantize,
    eliminate,
    gptq_blocked,
    gptq_columns,
    gptq_columns_u,
    hessian,
    hessian_rows,
    inverse,
    n_groups,
    pack,
    prepare,
    proxy_loss,
    quant_params,
    quantize_code,
    quantize_layer,
    rtn,
    unpack,
    upper_factor,
    upper_factor_flip,
)

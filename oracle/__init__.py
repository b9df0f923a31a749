"""fp64 CPU oracle of the routed-MoE FFN layer.

TEST INFRASTRUCTURE ONLY: the test-suite, the package's smoke check and the
bench's CPU baseline / reference arm are its only users. The CUDA library
never imports, links or calls it.
"""

from .oracle import (  # noqa: F401
    OracleLayer,
    bf16_bits,
    bf16_from_double,
    build,
    combine,
    double_from_bf16,
    double_from_e2m1,
    double_from_e4m3,
    double_from_e8m0,
    expert_rows,
    expert_rows_fp4,
    forward_tokens,
    num_threads,
    permute,
    route,
    set_num_threads,
)

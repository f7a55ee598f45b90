"""CPU oracle of the top-k mixture-of-experts FFN layer (fp64, plain C).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline are the only callers.  The product path never imports this package
and shares no code with it.  See moe_oracle.c for the definition it follows.
"""
from .oracle import (  # noqa: F401
    build,
    lib,
    gelu_tanh,
    rmsnorm_plus_one,
    select_topk,
    route_weights,
    route,
    moe_forward,
    moe_forward_f32,
    build_f32,
    expert_ffn,
    weight_row,
    decode_bf16,
    decode_fp16,
    decode_e4m3,
    decode_e2m1,
    lmhead_stats,
    eb_accept,
    set_threads,
    get_threads,
)

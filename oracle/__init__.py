"""CPU oracle for the weight-only-quantized MoE forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may use it; the product path never does. It
shares no code with the CUDA path and imports nothing from it.

``qmoe_oracle.c`` states the operator's plain definition in fp64 (see its
header for the passages it follows). ``literal.py`` restates the whole
forward a second time in the most literal numpy, for tiny shapes.
"""
from .binding import (dequant, e2m1, forward, gated_act, linear_i8, num_threads, permute,  # noqa: F401
                      plain_act, quantize_i8, round_act, route, to_f64, unpack)

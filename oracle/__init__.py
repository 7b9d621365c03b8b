"""fp64 CPU oracle of the DeepSeekMoE layer forward -- TEST INFRASTRUCTURE.

Imported only by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs. The library under mixture_experts_layer_group_b200/ never
imports it and shares no code with it.

Pinned by tests/test_oracle_pins.py (printed parameter counts and team
counts, brute-force selection, segmentation and shared-fusion identities,
gate sums, dense ceiling, invariances). Output values of a full layer on
random weights are pinned only through those identities and invariants: the
pages print no worked numeric layer output.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import RouterCfg, Routing, TIE_EPS  # noqa: F401

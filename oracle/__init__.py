"""CPU oracle for the hashed embedding engine.

TEST INFRASTRUCTURE: imported only by tests/, __graft_entry__.smoke() and the
bench's CPU-baseline / reference arm.  The product package never imports it.
"""
from .oracle import Oracle, OPT_CODES, pack_keys, init_row, round_bf16, splitmix64_outputs  # noqa: F401

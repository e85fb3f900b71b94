"""CPU oracle for the packed-MXFP4 W4A16 top-4 MoE expert FFN.

TEST INFRASTRUCTURE ONLY. Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path
(``packed_mxfp4_w4a16_b200``) never imports, links or runs it.

Parity pins (each checked by ``tests/test_oracle_pins.py`` against something
other than the oracle itself): the E2M1 bit-field definition and the
printed value table, E8M0 powers of two, BF16 rounding against the binary32
routine and hand-worked ties, an independently unpacked dense brute force on
small shapes, closed forms of the model card arithmetic, top-k/softmax
invariants and brute force, and a hand-derived sequential-combine example;
for the NVFP4 and sym8 formats, their scale decodes against torch's float8 and
numpy's float16, dense brute forces and the exact reductions to the MXFP4
layer.
"""
from .oracle import *  # noqa: F401,F403

"""CPU oracle for the int6 QAT linear, the ReLU^2 MLP, the recurrent core and
the export quantizer.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline / reference leg may import this package.  The
product path (the CUDA library and its Python binding) never imports it, and
this package imports nothing from the product.

Quantizers are scalar C (qat_oracle.c, strict IEEE fp32); the dense algebra
is numpy float64 on the exact operand values.

Parity pins: every function here is checked by tests/test_oracle_pins.py
against closed forms, hand-derived examples, brute force or an independent
library routine.  No function is "parity unpinned".
"""
from .oracle import *  # noqa: F401,F403

"""Seeded synthetic workloads shared by the tests, the bench and the oracle checks.

This package draws inputs only (activations, weights, rotation parameters,
sign seeds) and encodes them in the storage formats the library consumes
(fp32, bf16 bit patterns, int8 codes with per-stage scales).  It holds none of
the rotation's arithmetic: no block construction, no stage application.
"""
from .synthetic import *  # noqa: F401,F403

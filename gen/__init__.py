"""Seeded synthetic input generators shared by the tests, the bench and the oracle checks."""
from .synthetic import (BLOCK, WORKLOADS, DecodeInputs, SynthInputs, Workload, load_plan,
                        make_custom, make_decode, make_inputs)

__all__ = ["BLOCK", "WORKLOADS", "DecodeInputs", "SynthInputs", "Workload", "load_plan",
           "make_custom", "make_decode", "make_inputs"]

"""Seeded synthetic input generators shared by the tests, the bench and the oracle checks."""
from .synthetic import (BLOCK, WORKLOADS, DashRouting, DecodeInputs, SynthInputs, Workload, load_plan,
                        make_custom, make_dash_routing, make_decode, make_inputs)

__all__ = ["BLOCK", "WORKLOADS", "DashRouting", "DecodeInputs", "SynthInputs", "Workload", "load_plan",
           "make_custom", "make_dash_routing", "make_decode", "make_inputs"]

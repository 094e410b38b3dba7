"""Seeded synthetic workloads shared by the tests, the bench and the oracle checks.

Data synthesis only; none of the indexer's arithmetic lives here.
"""
from .configs import WORKLOADS, Workload, workload
from .gen import Inputs, RopeInputs, construction_inputs, generate, rope_inputs, shrunk

__all__ = ["WORKLOADS", "Workload", "workload", "Inputs", "generate", "shrunk",
           "construction_inputs", "RopeInputs", "rope_inputs"]

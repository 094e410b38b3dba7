"""Seeded synthetic workloads shared by the tests, the bench and the oracle checks.

Data synthesis only; none of the indexer's arithmetic lives here.
"""
from .configs import WORKLOADS, Workload, workload
from .gen import Inputs, generate, shrunk, construction_inputs

__all__ = ["WORKLOADS", "Workload", "workload", "Inputs", "generate", "shrunk",
           "construction_inputs"]

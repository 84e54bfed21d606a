"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

Holds none of the Medusa method's arithmetic: only counter-based draws
(``gen``), the workload table (``workloads``) and, for the device, a CUDA
generator that restates the same definition (``device``).
"""

"""Seeded synthetic inputs (weights, prefix KV cache, noise, prefill embeddings).

Shared by the tests, the oracle runs and bench.py; holds none of the method's arithmetic.
"""
from . import gen, workloads  # noqa: F401

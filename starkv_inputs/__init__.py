"""Seeded synthetic inputs shared by the oracle's tests and the CUDA path's tests.

Holds random draws and workload shapes only, none of the method's arithmetic.
"""

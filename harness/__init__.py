"""Harness shared by the tests and bench.py: seeded synthetic inputs and
stand-in experts.  It holds none of the method's arithmetic and imports
neither the oracle nor the CUDA package."""

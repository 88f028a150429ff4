"""Seeded synthetic input generators shared by the CUDA path's tests/bench and the oracle."""

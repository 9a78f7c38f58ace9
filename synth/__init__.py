"""Seeded synthetic inputs shared by the oracle tests and the CUDA path."""

"""CUDA sources of libbi.so and the script that builds it (build.py)."""

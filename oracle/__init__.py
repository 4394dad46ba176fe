"""fp64 CPU oracle for the batch-invariant reduction kernels.

TEST INFRASTRUCTURE ONLY.  Imported by tests, the smoke check and the
benchmark's CPU-baseline leg; never by the product path.  See oracle.c for
what each function computes and which passage of the pages it follows.
"""

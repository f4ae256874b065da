"""fp64 CPU oracle of the Speed3R sparse global attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only tests/, the smoke check and the benchmark's
CPU-baseline leg import it. It shares no code with the CUDA library.
"""

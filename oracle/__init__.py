"""CPU oracle for the Gecko SCA + AWM forward (TEST INFRASTRUCTURE ONLY).

Only tests, the smoke check and the CPU-baseline leg of the benchmark import
this package.  It shares no code with the CUDA library.
"""

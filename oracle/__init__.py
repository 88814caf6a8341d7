"""CPU oracle for the LoReS decode step (test infrastructure only).

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg
import this package.  The product path never does.
"""

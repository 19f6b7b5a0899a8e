"""Float64 CPU oracle for the TTT inner-loop forward (test infrastructure only).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA path.
"""

"""CPU oracle for the SAGA + Atop-N decode step (test infrastructure only).

Only tests, the package smoke check and the benchmark's CPU-baseline leg may
import this package.
"""

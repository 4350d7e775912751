"""Float64 CPU oracle of the ETA decode step (test infrastructure only).

Only the test-suite, the package entry file's smoke check and the benchmark's
CPU-baseline / reference legs may import this package.
"""

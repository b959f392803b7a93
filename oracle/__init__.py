"""CPU oracle of the W4A16 + gated Error-Compensator layer.

Test infrastructure only: imported by the test suite, by the smoke check and
by the CPU-baseline leg of the benchmark, never by the library itself.
"""

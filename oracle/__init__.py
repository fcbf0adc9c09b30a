"""CPU oracle for the MiniKV hot path -- test infrastructure only.

Imported by the tests, the smoke check and the benchmark's CPU-baseline leg,
never by the product library.
"""

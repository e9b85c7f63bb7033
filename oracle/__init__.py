"""CPU oracle for paged KV-cache attention: test infrastructure only.

Imported by the tests, the smoke check and the benchmark's CPU-baseline leg;
never by the product path.
"""

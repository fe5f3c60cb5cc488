"""Float64 CPU oracle for the CSA2-over-FP4-KV hot path.

Test infrastructure only: imported by the tests, the smoke check and the bench's
CPU-baseline leg; never by the product library or its binding.
"""

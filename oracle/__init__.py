"""fp64 CPU oracle for attention-saliency KV-cache compaction.

Test infrastructure only: used by the test suite, the smoke check and the benchmark's
CPU-baseline leg, never by the product path.
"""

"""CPU oracle for SAS gated block-sparse attention.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg. The CUDA library (gated_block_sparse_sas_b200)
never imports it, and the two share no code.
"""

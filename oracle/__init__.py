"""fp64 CPU oracle for the attention forward pass (attn, attn_oracle.c) and its
backward (attn_bwd).

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only the test suite, the package smoke
check and the benchmark's CPU-baseline / reference arm may import it.  It
shares no code with the CUDA path (attention_forward_19_b200), and the CUDA
path never imports it.
"""

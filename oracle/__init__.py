"""fp64 CPU oracle of the Megatron-LM tensor-parallel layer.

Test infrastructure only: tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg may import it; the product path never does.
"""

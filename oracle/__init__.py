"""CPU oracle of the fused MoE FFN layer forward -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package. The product package never does.
"""

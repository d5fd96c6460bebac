"""CPU oracle of the routed-MoE layer -- test infrastructure only.

Only tests/, the package smoke check and bench.py's CPU-baseline leg may use it.
"""

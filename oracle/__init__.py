"""fp64 / exact-rational oracle of the SketchSSM decode path.

TEST INFRASTRUCTURE ONLY: used by tests/, __graft_entry__.smoke() and the
CPU-baseline legs of bench.py.  The ssm_decode_b200 library never imports it.
"""

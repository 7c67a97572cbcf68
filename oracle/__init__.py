"""CPU oracle for the MoE-layer forward -- test infrastructure only.

Imported by the tests, the smoke check and the benchmark's CPU baseline; never
by the library's CUDA path.
"""

"""MoonEP hot path on B200: online redundant-expert planning, fused
permute-dispatch, unpermute-combine, replica weight prefetch and replica
gradient reduction (and their backward pair and zero_copy = false copy-out),
as hand-written sm_100a CUDA behind a C ABI.

``load_balancing_plan_b200.moonep`` is the Python binding of the C ABI;
``load_balancing_plan_b200.views`` wraps receive-buffer views with their
lifetime check; ``load_balancing_plan_b200.inputs`` draws seeded synthetic
inputs.
"""
__all__ = ["moonep", "views", "inputs"]

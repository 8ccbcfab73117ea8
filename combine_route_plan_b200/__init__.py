"""B200-native rank-major MoE expert-parallel dispatch / combine.

The compute path is the C-ABI library ``libep_a2a.so`` (hand-written sm_100a
CUDA); :mod:`combine_route_plan_b200.ep_a2a` is its thin ctypes binding and
:mod:`combine_route_plan_b200.workloads` draws seeded synthetic inputs.
"""

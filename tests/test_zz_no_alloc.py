"""The allocation-free routing plan (ep_a2a_route_plan_noalloc) against the
CPU oracle and the workspace-based ep_a2a_dispatch.

Some callers cannot allocate device memory: their HBM is owned by an outer
allocator (a serving engine that reserves almost all of it for its own pools,
a host application that forbids plug-in libraries from calling cudaMalloc).
They cannot give ep_a2a_init a workspace holding the routing kernel's scratch,
so ep_a2a_route_plan_noalloc keeps that scratch in a fixed device array of the
library and takes only inputs and outputs.  This test calls it through the C
ABI, twice in a row on the same inputs and once more on another shape, and
checks every output against the oracle's routing plan and against what
ep_a2a_dispatch wrote (all integers, so the comparisons are exact); it also
checks that warm calls leave the device's allocated and free memory unchanged.
It lives in its own file, collected last, and passes alone in a fresh process
as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from combine_route_plan_b200 import workloads as W
import parity_util as U

pytestmark = pytest.mark.gpu

CANARY = 0xCD


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_route_plan_b200 import build
    build.build()
    from combine_route_plan_b200 import ep_a2a
    lib = ep_a2a.lib
    P = ctypes.c_void_p
    lib.ep_a2a_route_plan_noalloc.restype = ctypes.c_int
    lib.ep_a2a_route_plan_noalloc.argtypes = [
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        P, P, P, P, P, P, P, P, ctypes.c_int64, P]
    return ep_a2a


class Outputs:
    """Caller-owned output buffers in the layout ep_a2a_dispatch uses."""

    def __init__(self, w):
        ep, tpr, k = w.ep_size, w.tokens_per_rank, w.top_k
        slots = ep * tpr
        self.stride_plan = (k + 7) // 8 * 8
        self.plan_nd = torch.full((ep, tpr), CANARY, dtype=torch.uint8, device="cuda")
        self.plan_dst = torch.full((ep, tpr, self.stride_plan), CANARY, dtype=torch.uint8,
                                   device="cuda")
        self.counts = torch.full((ep, ep), -1, dtype=torch.int32, device="cuda")
        ids_bytes = slots * k * 4
        self.rank_stride = (ids_bytes + slots + 255) // 256 * 256
        self.recv = torch.full((ep, self.rank_stride), CANARY, dtype=torch.uint8, device="cuda")
        self.ids_bytes = ids_bytes

    def recv_ids(self, w):
        return self.recv[:, :self.ids_bytes].contiguous().view(torch.int32) \
            .view(w.ep_size, w.ep_size * w.tokens_per_rank, w.top_k)

    def recv_valid(self, w):
        return self.recv[:, self.ids_bytes:self.ids_bytes + w.ep_size * w.tokens_per_rank]


def _call_noalloc(ep, w, x, o, ids_dev):
    n = (ctypes.c_int32 * w.ep_size)(*[int(v) for v in x.local_num_tokens])
    mask = None
    if x.active_rank_mask is not None:
        words = [int(v) for v in x.active_rank_mask] + [0] * 4
        mask = ctypes.cast((ctypes.c_uint64 * 4)(*words[:4]), ctypes.c_void_p)
    recv_ids_ptr = o.recv.data_ptr()
    recv_valid_ptr = o.recv.data_ptr() + o.ids_bytes
    st = ep.lib.ep_a2a_route_plan_noalloc(
        w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank, -1,
        ctypes.c_void_p(ids_dev.data_ptr()), ctypes.cast(n, ctypes.c_void_p), mask,
        ctypes.c_void_p(o.plan_nd.data_ptr()), ctypes.c_void_p(o.plan_dst.data_ptr()),
        ctypes.c_void_p(o.counts.data_ptr()), ctypes.c_void_p(recv_ids_ptr),
        ctypes.c_void_p(recv_valid_ptr), o.rank_stride,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ep.OK, ep.lib.ep_a2a_last_error()


def _reference(ep, w, x):
    """What the existing workspace entry point writes for the same step."""
    comm = ep.EpA2A(w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank, w.hidden, [16],
                    enable_rank_mask=x.active_rank_mask is not None, workspace_fill=CANARY)
    d = comm.dispatch(x.token_selected_experts.cuda(), x.local_num_tokens, [], w.tokens_per_rank,
                      None, x.active_rank_mask)
    torch.cuda.synchronize()
    return comm, d


def _compare(w, o, d):
    torch.cuda.synchronize()
    assert torch.equal(o.plan_nd, d.plan_num_dst)
    assert torch.equal(o.plan_dst, d.plan_dst_ranks)
    assert torch.equal(o.counts, d.send_counts)
    assert torch.equal(o.recv_valid(w), d.recv_valid)
    assert torch.equal(o.recv_ids(w), d.recv_topk_ids)


def _compare_oracle(w, x, o):
    """Every output against the oracle's plan of the same step: plan rows, send
    counts, and each rank's valid bytes and received ids (the oracle leaves the
    rows of masked-off ranks at the canary, as the kernel does)."""
    torch.cuda.synchronize()
    plan = U.oracle_plan(w, x)
    k = w.top_k
    nd = plan.num_dst.copy()
    nd[nd < 0] = 0xFF
    U.assert_equal(o.plan_nd, nd.astype(np.uint8), "plan_num_dst")
    want = np.full(tuple(o.plan_dst.shape), 0xFF, np.uint8)
    ranks = plan.dst_ranks.copy()
    ranks[ranks < 0] = 0xFF
    want[:, :, :k] = ranks.astype(np.uint8)
    U.assert_equal(o.plan_dst, want, "plan_dst_ranks")
    U.assert_equal(o.counts, plan.send_counts, "send_counts")
    U.assert_equal(o.recv_valid(w), plan.recv_valid, "recv_valid")
    U.assert_equal(o.recv_ids(w), plan.recv_topk_ids, "recv_topk_ids")


def _device_memory():
    free, _ = torch.cuda.mem_get_info()
    return torch.cuda.memory_allocated(), torch.cuda.memory_reserved(), free


def test_noalloc_plan_matches_oracle_and_workspace_plan(ep):
    # wide EP with a rank mask and ragged token counts, at the full size
    w = W.C5
    x = W.make_inputs(w, with_expert_output=False)
    comm, d = _reference(ep, w, x)
    ids_dev = x.token_selected_experts.cuda()
    o = Outputs(w)
    _call_noalloc(ep, w, x, o, ids_dev)         # warm: the kernel's code is loaded
    for _ in range(2):                          # two calls in a row share the array
        torch.cuda.synchronize()
        before = _device_memory()
        _call_noalloc(ep, w, x, o, ids_dev)
        torch.cuda.synchronize()
        assert _device_memory() == before       # allocated, reserved and free bytes
        _compare(w, o, d)
        _compare_oracle(w, x, o)
    # a different shape after it: the array keeps the last call's contents
    w2 = W.scaled(W.C2, 100)
    x2 = W.make_inputs(w2, with_expert_output=False)
    comm2, d2 = _reference(ep, w2, x2)
    o2 = Outputs(w2)
    _call_noalloc(ep, w2, x2, o2, x2.token_selected_experts.cuda())
    _compare(w2, o2, d2)
    _compare_oracle(w2, x2, o2)
    comm.destroy()
    comm2.destroy()


def test_noalloc_rejects_too_many_ranks(ep):
    n = (ctypes.c_int32 * 65)(*([1] * 65))
    dummy = ctypes.c_void_p(16)
    st = ep.lib.ep_a2a_route_plan_noalloc(65, 260, 2, 4, -1, dummy, ctypes.cast(n, ctypes.c_void_p),
                                          None, dummy, dummy, dummy, dummy, dummy, 4096, None)
    assert st == ep.ERR_UNSUPPORTED
    assert b"64" in ep.lib.ep_a2a_last_error()


@pytest.mark.parametrize("valid_off,stride", [
    (0, 4096),            # recv_valid on top of recv_topk_ids
    (64, 4096),           # starts inside recv_topk_ids
    (-8, 4096),           # ends inside recv_topk_ids
    (2048, 2100),         # both fit, but not inside one stride
])
def test_noalloc_rejects_overlapping_outputs(ep, valid_off, stride):
    # ep 4, 16 tokens per rank, top_k 8: 2048 id bytes and 64 valid bytes per rank
    n = (ctypes.c_int32 * 4)(*([16] * 4))
    dummy = ctypes.c_void_p(1 << 20)
    ids = 1 << 24
    st = ep.lib.ep_a2a_route_plan_noalloc(4, 16, 8, 16, -1, dummy, ctypes.cast(n, ctypes.c_void_p),
                                          None, dummy, dummy, dummy, ctypes.c_void_p(ids),
                                          ctypes.c_void_p(ids + valid_off), stride, None)
    assert st == ep.ERR_INVALID_ARG

"""Run by test_checked_build.py in a child process whose EP_A2A_LIBRARY is
libep_a2a_checked.so (the library with its device index checks compiled in).

1. The checked build exports every entry point of include/ep_a2a.h and gives
   the oracle's results on ordinary inputs (dispatch, BF16 / FP8 / scaled FP8
   / expert-output combines), with a clean status.
2. Plan entries made out of range in the workspace after a dispatch (a
   destination rank >= ep_size; more destinations than a plan row holds) are
   reported by ep_a2a_get_status as EP_A2A_ERR_DEVICE_BOUNDS.  The corrupted
   entries are chosen so that every address they lead to still lies inside
   the caller's buffers (the expert rows are allocated for twice the ranks),
   so the check is observed without any access outside an allocation.
"""
import ctypes
import os
import re
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path[:0] = [ROOT, HERE]

import numpy as np  # noqa: E402
import torch  # noqa: E402

from combine_route_plan_b200 import ep_a2a  # noqa: E402
from combine_route_plan_b200 import workloads as W  # noqa: E402
import parity_util as U  # noqa: E402


def exports_every_declared_symbol():
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "ep_a2a.h")).read(),
                  flags=re.S)
    names = sorted(set(re.findall(r"\b(ep_a2a_[a-z0-9_]+)\s*\(", text)))
    lib = ctypes.CDLL(ep_a2a.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def parity(name):
    w = W.BY_NAME[name]
    x = W.make_inputs(w)
    run = U.Run(w, x)
    plan = U.oracle_plan(w, x)
    U.check_plan(run, plan, w)
    U.check_payloads(run, plan, w, x)
    U.check_eplb(run, w, x)
    U.check_combine(run, plan, w, x)
    init = U.oracle_out_init(w)
    comm, H = run.comm, w.hidden
    xo = x.expert_output

    def fresh():
        return torch.full((w.ep_size, w.tokens_per_rank, H), U.OUT_CANARY, dtype=torch.int16,
                          device="cuda").view(torch.bfloat16)
    out8, outs, oute = fresh(), fresh(), fresh()
    comm.combine(ep_a2a.quantize_e4m3(xo.cuda()), out8)
    codes, scales = ep_a2a.quantize_e4m3_rows(xo.cuda())
    comm.combine_scaled(codes, scales, outs)
    g = torch.Generator().manual_seed(w.seed)
    wts = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k), generator=g)
    y = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k, H), generator=g).to(torch.bfloat16)
    comm.combine_experts(wts.cuda(), y.cuda(), oute)
    torch.cuda.synchronize()
    assert comm.get_status() == ep_a2a.OK
    xq = U.oracle_quantize_big(U.to_np(xo), U.oracle_e4m3_table())
    oc, osc = U.oracle.quantize_e4m3_rows(U.to_np(xo), H)
    U.assert_equal(out8, U.oracle.combine(plan, xq, H, input_is_e4m3=True, out_init=init), "fp8")
    U.assert_equal(outs, U.oracle.combine_scaled(plan, oc, osc, H, out_init=init), "scaled")
    U.assert_equal(oute, U.oracle.combine_experts(plan, w.num_experts,
                                                  x.token_selected_experts.numpy(), wts.numpy(),
                                                  U.to_np(y), H, out_init=init), "experts")


def out_of_range_plan_entries_are_reported():
    w = W.C1                                   # ep 4, top_k 2: plan rows of 8 entries
    x = W.make_inputs(w)
    ep, tpr, H = w.ep_size, w.tokens_per_rank, w.hidden
    comm = ep_a2a.EpA2A(ep, w.num_experts, w.top_k, tpr, H, w.payload_row_bytes())
    ids = x.token_selected_experts.cuda()
    pays = [p.cuda() for p in x.payloads]
    # expert rows (and row scales) for 2 * ep ranks: rank 6's rows are in the buffer
    xb = torch.zeros((2 * ep, ep * tpr, H), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((2 * ep, ep * tpr, H), dtype=torch.float8_e4m3fn, device="cuda")
    sc = torch.ones((2 * ep, ep * tpr), dtype=torch.float32, device="cuda")
    calls = [lambda: comm.combine(xb[:ep]), lambda: comm.combine(q[:ep]),
             lambda: comm.combine_scaled(q[:ep], sc[:ep])]
    for corrupt in ("rank", "count"):
        for call in calls:
            d = comm.dispatch(ids, x.local_num_tokens, pays, tpr)
            torch.cuda.synchronize()
            if corrupt == "rank":
                d.plan_dst_ranks[0, 0, 0] = 2 * ep - 2      # a rank >= ep_size
            else:
                d.plan_dst_ranks[1, 0, :] = 0              # every entry a real rank ...
                d.plan_num_dst[1, 0] = d.plan_dst_ranks.shape[2] + 1   # ... one too many
            call()
            st = comm.get_status()
            assert st == ep_a2a.ERR_DEVICE_BOUNDS, (corrupt, st)
    # and a clean step afterwards
    comm.dispatch(ids, x.local_num_tokens, pays, tpr)
    comm.combine(x.expert_output.cuda())
    assert comm.get_status() == ep_a2a.OK


def main():
    assert os.path.basename(ep_a2a.LIB_PATH) == "libep_a2a_checked.so", ep_a2a.LIB_PATH
    exports_every_declared_symbol()
    for name in ("c1_ep4_tiny", "c2_ep8_decode", "c5_ep64_wide_masked"):
        parity(name)
    out_of_range_plan_entries_are_reported()
    print("checked build ok")


if __name__ == "__main__":
    main()

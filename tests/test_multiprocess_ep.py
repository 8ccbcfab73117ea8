"""Expert parallelism between real EP ranks: one process per rank.

Each test starts world_size processes (spawned, gloo over 127.0.0.1), each an
EP rank with its own window on the GPU; the windows are exchanged as CUDA IPC
handles, rows move as peer stores, and per-(source, destination) flags are
checked with bounded waits (ep_mp_* in include/ep_a2a.h).  Every rank checks
what it received and what its combine returned against the CPU oracle of the
whole step, element by element: received payload rows, ids, valid bytes,
EPLB rows and send counts bit-exact (rows nobody may write keep the window's
canary), the combine bit-exact.

The ranks never wait on one another inside a kernel: the caller's host
barrier separates each send phase from the receive phase, so a flag is
already set when its wait starts.  The failure test has one rank skip its
send; the peer's bounded wait runs out while the skipping rank sits at the
host barrier with no GPU work, and the peer reads EP_A2A_ERR_DEVICE_TIMEOUT
and keeps a usable context.
"""
import datetime
import multiprocessing as mp
import os
import socket
import traceback

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

CANARY = 0xCD
OUT_CANARY = -0x1112          # 0xEEEE as int16


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global_inputs(ep, E, k, tpr, H, rows, n, seed):
    """The whole step's inputs, identical on every rank (seeded)."""
    g = torch.Generator().manual_seed(seed)
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(ep * tpr)]) \
        .to(torch.int32).view(ep, tpr, k)
    ids[0, 0, 0] = -1                    # an id owned by no rank
    ids[ep - 1, 1, k - 1] = E            # the invalid id itself
    payloads = [torch.randint(0, 256, (ep, tpr, rb), generator=g, dtype=torch.int32)
                .to(torch.uint8) for rb in rows]
    stats = torch.randint(0, 4097, (ep, E), generator=g, dtype=torch.int32)
    xo = torch.randn((ep, ep * tpr, H), generator=g).to(torch.bfloat16)
    return ids, payloads, stats, xo


def _agree(ok: bool) -> bool:
    """Whether every rank's checks passed (gloo all-reduce).  Ranks agree before
    any rank starts the next phase, so that no rank leaves while a peer could
    still be writing into its window."""
    import torch.distributed as dist
    t = torch.tensor([0 if ok else 1], dtype=torch.int64)
    dist.all_reduce(t)
    return int(t.item()) == 0


def _checked(comm, fn):
    """Run the checks `fn`; if any rank's fail, every rank tears down cleanly
    (no kernel in flight, peer mappings closed) and this rank re-raises."""
    err = None
    try:
        fn()
    except Exception:
        err = traceback.format_exc()
    if not _agree(err is None):
        comm.destroy()
        raise AssertionError(err or "another rank's checks failed")


def _rank_main(rank, world, case):
    import oracle
    from combine_route_plan_b200 import ep_a2a, ep_mp
    ep = world
    E, k, tpr, H = 8 * ep, 4, 24, 128
    rows = [2 * H, 4 * k, 7]
    n = np.array([tpr, tpr - 3, 5, 0, 17, tpr, 1, 9][:ep], np.int32)
    mask = None
    if case == "masked":
        mask = np.array([(1 << ep) - 1 - (1 << 2)], np.uint64)     # rank 2 off
    ids, payloads, stats, xo = _global_inputs(ep, E, k, tpr, H, rows, n, seed=40 + ep)
    dev = torch.device("cuda", 0)
    comm = ep_mp.EpRank(None, rank, ep, E, k, tpr, H, rows, eplb_stats_num_experts=E,
                        enable_rank_mask=mask is not None, window_fill=CANARY)
    live = ep_mp.rank_is_live(mask, rank)

    if case == "timeout":
        # rank 1 skips its send; rank 0's wait for rank 1's flag runs out
        d = comm.dispatch(ids[rank].to(dev), int(n[rank]), [p[rank].to(dev) for p in payloads],
                          tpr, stats[rank].to(dev), mask, timeout_ns=50_000_000,
                          send=rank != 1, wait=rank == 0)
        def check_timeout():
            if rank != 0:
                return
            st = comm.get_status()
            assert st == ep_a2a.ERR_DEVICE_TIMEOUT, st
            assert comm.get_status() == ep_a2a.OK           # read and cleared
            y = torch.arange(1024, device=dev, dtype=torch.float32).sum()   # context usable
            assert float(y.item()) == 1023 * 1024 / 2
        _checked(comm, check_timeout)
        comm.destroy()
        return "timeout seen" if rank == 0 else "skipped"

    d = comm.dispatch(ids[rank].to(dev), int(n[rank]), [p[rank].to(dev) for p in payloads], tpr,
                      stats[rank].to(dev), mask)
    # the oracle of the whole step, this rank's slice
    plan = oracle.route(ep, E, k, tpr, ids.numpy(), n, mask,
                        recv_valid_init=np.full((ep, ep * tpr), CANARY, np.uint8),
                        recv_topk_ids_init=np.full((ep, ep * tpr, 4 * k), CANARY, np.uint8)
                        .view(np.int32))
    _checked(comm, lambda: _check_dispatch(comm, d, plan, live, rank, ep, tpr, k, rows, payloads,
                                           stats, mask))

    # combine: this rank returns its rows for the slots it received
    fp8 = case == "fp8"
    x = xo[rank].to(dev)
    if fp8:
        x = ep_a2a.quantize_e4m3(x)
    out = torch.full((tpr, H), OUT_CANARY, dtype=torch.int16, device=dev).view(torch.bfloat16)
    out = comm.combine(x, out, mask)

    def check_combine():
        if not live:
            return
        assert comm.get_status() == ep_a2a.OK
        bits = xo.view(torch.int16).numpy().view(np.uint16)
        if fp8:
            bits = oracle.quantize_e4m3(bits)
        want = oracle.combine(plan, bits, H, input_is_e4m3=fp8)
        assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), want[rank])
    _checked(comm, check_combine)
    comm.destroy()
    return "ok"


def _check_dispatch(comm, d, plan, live, rank, ep, tpr, k, rows, payloads, stats, mask):
    import oracle
    from combine_route_plan_b200 import ep_a2a
    st = comm.get_status()
    assert st == ep_a2a.OK, (st, ep_a2a.lib.ep_a2a_last_error())
    if live:
        assert np.array_equal(d.recv_valid.cpu().numpy(), plan.recv_valid[rank])
        assert np.array_equal(d.recv_topk_ids.cpu().numpy(), plan.recv_topk_ids[rank])
        assert np.array_equal(d.send_counts.cpu().numpy(), plan.send_counts[rank])
        nd = plan.num_dst[rank].copy()
        nd[nd < 0] = 0xFF
        assert np.array_equal(d.plan_num_dst.cpu().numpy(), nd.astype(np.uint8))
        for i, p in enumerate(payloads):
            want = oracle.dispatch_payload(plan, p.numpy(), only_dst=rank,
                                           recv_init=np.full((1, ep * tpr, rows[i]), CANARY,
                                                             np.uint8))
            assert np.array_equal(d.recv_payloads[i].cpu().numpy(), want.reshape(ep * tpr, -1)), i
        want_eplb = oracle.eplb_gather(ep, stats.numpy(), mask)
        assert np.array_equal(d.eplb_gathered_stats.cpu().numpy(), want_eplb[rank])


def _worker(rank, world, port, case, q):
    try:
        # the windows are exported over CUDA IPC, which needs plain cudaMalloc
        # allocations from torch's caching allocator
        os.environ.pop("PYTORCH_CUDA_ALLOC_CONF", None)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import torch.distributed as dist
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
        torch.cuda.set_device(0)
        q.put((rank, "ok", _rank_main(rank, world, case)))
    except Exception:
        q.put((rank, "fail", traceback.format_exc()))
    finally:
        try:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
        except Exception:
            pass


def _run(world, case):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_route_plan_b200 import build
    build.build()
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in ps:
        p.start()
    got = []
    try:
        for _ in ps:
            got.append(q.get(timeout=600))
    finally:
        for p in ps:
            p.join(timeout=120)
        for p in ps:
            if p.is_alive():
                p.kill()
    fails = [g for g in got if g[1] != "ok"]
    assert not fails, "\n".join(f"rank {r}: {msg}" for r, _, msg in fails)
    return {r: res for r, _, res in got}


@pytest.mark.parametrize("world", [2, 4])
def test_ranks_as_processes_bit_exact(world):
    res = _run(world, "bf16")
    assert all(v == "ok" for v in res.values())


def test_ranks_as_processes_fp8_combine():
    _run(2, "fp8")


def test_ranks_as_processes_with_a_masked_rank():
    _run(4, "masked")


def test_skipped_send_times_out_and_context_survives():
    res = _run(2, "timeout")
    assert res[0] == "timeout seen" and res[1] == "skipped"

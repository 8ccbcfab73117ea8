"""Host side of the multi-process EP ranks on CPU: world-size-2 gloo groups
exchange window handles and keep the phase barriers in step; the window size
and the entry points' argument checks run without a GPU."""
import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from combine_route_plan_b200 import build
    build.build()
    from combine_route_plan_b200 import ep_a2a, ep_mp
    return ep_a2a, ep_mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from combine_route_plan_b200 import ep_mp
    mine = bytes([rank]) * 64 + (256 * (rank + 1)).to_bytes(8, "little")
    got = ep_mp.exchange_handles(None, mine, world)
    dist.barrier()
    with open(os.path.join(out_dir, f"r{rank}.bin"), "wb") as f:
        f.write(b"".join(got))
    dist.destroy_process_group()


def test_handles_are_all_gathered_in_rank_order(tmp_path, lib):
    port = _free_port()
    mp.start_processes(_exchange_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    want = b"".join(bytes([r]) * 64 + (256 * (r + 1)).to_bytes(8, "little") for r in range(2))
    for r in range(2):
        assert (tmp_path / f"r{r}.bin").read_bytes() == want


def test_ipc_handle_layout(lib):
    _, ep_mp = lib
    assert ctypes.sizeof(ep_mp.IpcHandle) == 72
    assert ep_mp.IpcHandle.offset.offset == 64


def test_rank_liveness_from_mask(lib):
    _, ep_mp = lib
    mask = np.array([0b1011, 0, 1 << 3, 0], np.uint64)
    assert [ep_mp.rank_is_live(mask, r) for r in range(5)] == [True, True, False, True, False]
    assert ep_mp.rank_is_live(mask, 131) and not ep_mp.rank_is_live(mask, 130)
    assert ep_mp.rank_is_live(None, 7)


def test_window_size_grows_with_capacity_and_rows(lib):
    ep_a2a, ep_mp = lib
    base = ep_mp.ep_mp_window_size(ep_a2a.make_params(4, 16, 4, 24, 128, [256, 16]))
    more_tok = ep_mp.ep_mp_window_size(ep_a2a.make_params(4, 16, 4, 48, 128, [256, 16]))
    more_row = ep_mp.ep_mp_window_size(ep_a2a.make_params(4, 16, 4, 24, 128, [512, 16]))
    wider = ep_mp.ep_mp_window_size(ep_a2a.make_params(4, 16, 4, 24, 256, [256, 16]))
    assert more_tok > base and more_row > base and wider > base
    # at least the receive rows, ids, valid bytes and landing rows of ep * cap slots
    assert base >= 4 * 24 * (256 + 16 + 4 * 4 + 1 + 2 * 128)


def test_entry_points_reject_bad_arguments_on_the_host(lib):
    ep_a2a, ep_mp = lib
    p = ep_a2a.make_params(4, 16, 4, 24, 128, [256])
    peers = (ep_mp.IpcHandle * 4)()
    h = ctypes.c_void_p(0)
    L = ep_a2a.lib
    n = ep_mp.ep_mp_window_size(p)
    win = ctypes.c_void_p(1 << 20)
    assert L.ep_mp_init(ctypes.byref(p), 4, win, n, peers, None, ctypes.byref(h)) == \
        ep_a2a.ERR_INVALID_ARG                                   # rank out of range
    assert L.ep_mp_init(ctypes.byref(p), 0, ctypes.c_void_p(1 << 20 | 8), n, peers, None,
                        ctypes.byref(h)) == ep_a2a.ERR_INVALID_ARG  # unaligned window
    assert L.ep_mp_init(ctypes.byref(p), 0, win, n - 1, peers, None, ctypes.byref(h)) == \
        ep_a2a.ERR_INVALID_ARG                                   # window too small
    peers[1].offset = 8
    assert L.ep_mp_init(ctypes.byref(p), 0, win, n, peers, None, ctypes.byref(h)) == \
        ep_a2a.ERR_INVALID_ARG                                   # unaligned peer offset
    assert not h.value
    bad = ep_a2a.make_params(4, 18, 4, 24, 128, [256])          # E not a multiple of 4
    assert L.ep_mp_window_size(ctypes.byref(bad), ctypes.byref(ctypes.c_size_t())) == \
        ep_a2a.ERR_INVALID_ARG
    for fn, args in [("ep_mp_dispatch_wait", (None, 1000, None)),
                     ("ep_mp_combine_send", (None, None, 0, None)),
                     ("ep_mp_get_status", (None, None))]:
        assert getattr(L, fn)(*args) == ep_a2a.ERR_NOT_INITIALIZED
    assert L.ep_mp_destroy(ctypes.byref(ctypes.c_void_p(0))) == ep_a2a.OK

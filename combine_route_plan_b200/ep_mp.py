"""Expert parallelism between real EP ranks: one process per rank.

Thin binding of the ``ep_mp_*`` entry points of libep_a2a.so (declared in
include/ep_a2a.h) plus :class:`EpRank`, which owns one rank's window tensor
and does the host-side plumbing the library leaves to its caller: the
all-gather of the windows' CUDA IPC handles and the barriers that separate the
send and receive phases, over a ``torch.distributed`` process group (gloo).
Every byte of the path moves in the library's kernels.

The phases of one step, on every live rank (a masked-off rank only joins the
barriers)::

    dispatch  -> sync stream | barrier | dispatch_wait          (rows have landed)
    experts, combine_send -> sync stream | barrier | combine_finish
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence

import numpy as np
import torch

from . import ep_a2a as _a2a
from .ep_a2a import (DispatchResult, EpA2AError, Params, RANK_MASK_WORDS, _check, _stream_ptr,
                     lib, make_params)


class IpcHandle(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_uint8 * 64), ("offset", ctypes.c_int64)]


_P, _I32, _I64, _VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
for _name, (_res, _args) in {
    "ep_mp_window_size": (ctypes.c_int, [_P(Params), _P(ctypes.c_size_t)]),
    "ep_mp_export": (ctypes.c_int, [_VP, _P(IpcHandle)]),
    "ep_mp_init": (ctypes.c_int, [_P(Params), _I32, _VP, ctypes.c_size_t, _P(IpcHandle), _VP,
                                  _P(_VP)]),
    "ep_mp_dispatch": (ctypes.c_int, [_VP, _VP, _I32, _I32, _P(_VP), _P(_I64), _I32, _VP, _VP,
                                      _VP, _P(DispatchResult)]),
    "ep_mp_dispatch_wait": (ctypes.c_int, [_VP, _I64, _VP]),
    "ep_mp_combine_send": (ctypes.c_int, [_VP, _VP, ctypes.c_int, _VP]),
    "ep_mp_combine_finish": (ctypes.c_int, [_VP, _VP, ctypes.c_int, _I64, _VP]),
    "ep_mp_get_status": (ctypes.c_int, [_VP, _VP]),
    "ep_mp_destroy": (ctypes.c_int, [_P(_VP)]),
}.items():
    _fn = getattr(lib, _name)
    _fn.restype, _fn.argtypes = _res, _args


def ep_mp_window_size(params: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.ep_mp_window_size(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def ep_mp_export(window_ptr: int) -> bytes:
    h = IpcHandle()
    _check(lib.ep_mp_export(ctypes.c_void_p(window_ptr), ctypes.byref(h)))
    return bytes(h)


def exchange_handles(group, handle: bytes, world_size: int) -> List[bytes]:
    """All-gather every rank's exported window handle (host plumbing)."""
    import torch.distributed as dist
    got: List[Optional[bytes]] = [None] * world_size
    dist.all_gather_object(got, handle, group=group)
    return [bytes(g) for g in got]


def _mask_array(active_rank_mask):
    if active_rank_mask is None:
        return None
    words = [int(w) for w in np.asarray(active_rank_mask, dtype=np.uint64)] + [0] * RANK_MASK_WORDS
    return (ctypes.c_uint64 * RANK_MASK_WORDS)(*words[:RANK_MASK_WORDS])


def rank_is_live(active_rank_mask, r: int) -> bool:
    if active_rank_mask is None:
        return True
    return bool((int(np.asarray(active_rank_mask, dtype=np.uint64)[r // 64]) >> (r % 64)) & 1)


class RankDispatched:
    """Views of this rank's window after a dispatch (valid until the next one)."""

    def __init__(self, rank: "EpRank", res: DispatchResult, row_bytes: Sequence[int]):
        win = rank.window
        base = win.data_ptr()
        ep, k, tpr = rank.ep_size, rank.top_k, res.tokens_per_rank
        slots = ep * tpr

        def view(ptr, nbytes):
            return win[ptr - base: ptr - base + nbytes]
        self.tokens_per_rank = tpr
        self.recv_payloads = [view(res.recv_payloads[i], slots * rb).view(slots, rb)
                              for i, rb in enumerate(row_bytes)]
        self.recv_topk_ids = view(res.recv_topk_ids, slots * k * 4).view(torch.int32) \
            .view(slots, k)
        self.recv_valid = view(res.recv_valid, slots)
        self.eplb_gathered_stats = None
        if res.eplb_gathered_stats:
            ne = rank.eplb_stats_num_experts
            self.eplb_gathered_stats = view(res.eplb_gathered_stats, ep * ne * 4) \
                .view(torch.int32).view(ep, ne)
        self.send_counts = view(res.send_counts, ep * 4).view(torch.int32)
        self.plan_num_dst = view(res.plan_num_dst, tpr)
        ps = res.plan_stride
        self.plan_dst_ranks = view(res.plan_dst_ranks, tpr * ps).view(tpr, ps)


class EpRank:
    """This process's EP rank: a window tensor, the mapped peer windows, and the
    phase barriers over ``group`` (every rank of the group constructs one)."""

    def __init__(self, group, rank: int, ep_size: int, num_experts: int, top_k: int,
                 max_tokens_per_rank: int, hidden_size: int, payload_row_bytes: Sequence[int],
                 eplb_stats_num_experts: int = 0, enable_rank_mask: bool = False,
                 invalid_expert_id: int = -1, device=None, stream=None,
                 window_fill: Optional[int] = None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank, self.ep_size, self.top_k = rank, ep_size, top_k
        self.hidden_size = hidden_size
        self.eplb_stats_num_experts = eplb_stats_num_experts
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.params = make_params(ep_size, num_experts, top_k, max_tokens_per_rank, hidden_size,
                                  payload_row_bytes, eplb_stats_num_experts, enable_rank_mask,
                                  invalid_expert_id)
        nbytes = ep_mp_window_size(self.params)
        self.window = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        if window_fill is not None:     # tests: rows nobody may write keep this byte
            self.window.fill_(window_fill)
            torch.cuda.synchronize(self.device)
        handles = exchange_handles(group, ep_mp_export(self.window.data_ptr()), ep_size)
        peers = (IpcHandle * ep_size)()
        for r, hb in enumerate(handles):
            ctypes.memmove(ctypes.byref(peers[r]), hb, ctypes.sizeof(IpcHandle))
        self._h = ctypes.c_void_p(0)
        _check(lib.ep_mp_init(ctypes.byref(self.params), rank,
                              ctypes.c_void_p(self.window.data_ptr()), nbytes, peers,
                              ctypes.c_void_p(_stream_ptr(stream)), ctypes.byref(self._h)))
        self.barrier()              # every window is cleared before anyone sends
        self.last = None

    def barrier(self):
        self.dist.barrier(group=self.group)

    def _sync(self, stream):
        if stream is None:
            torch.cuda.current_stream(self.device).synchronize()
        elif isinstance(stream, torch.cuda.Stream):
            stream.synchronize()
        else:
            torch.cuda.synchronize(self.device)

    @property
    def handle(self) -> int:
        if not self._h.value:
            raise EpA2AError(_a2a.ERR_NOT_INITIALIZED, "handle destroyed")
        return self._h.value

    def dispatch(self, token_selected_experts: torch.Tensor, local_num_tokens: int,
                 payloads: Sequence[torch.Tensor], runtime_max_tokens_per_rank: int,
                 eplb_local_stats: Optional[torch.Tensor] = None, active_rank_mask=None,
                 timeout_ns: int = 1_000_000_000, stream=None, wait: bool = True,
                 send: bool = True):
        """Send this rank's tokens, then (after every rank has sent) check that
        every live rank's rows have arrived.  ``send=False`` joins the step's
        barriers without sending (a rank that skipped its send; failure tests).
        Returns the views of this rank's window, or None on a masked-off rank."""
        live = rank_is_live(active_rank_mask, self.rank)
        res = None
        if live and send:
            ids = token_selected_experts
            assert ids.is_cuda and ids.dtype == torch.int32 and ids.is_contiguous()
            rbs = [t[0].numel() * t.element_size() for t in payloads]
            ptrs = (ctypes.c_void_p * max(1, len(payloads)))(*[t.data_ptr() for t in payloads])
            rb = (ctypes.c_int64 * max(1, len(rbs)))(*rbs)
            res = DispatchResult()
            stats = eplb_local_stats.data_ptr() if eplb_local_stats is not None else 0
            _check(lib.ep_mp_dispatch(self.handle, ctypes.c_void_p(ids.data_ptr()),
                                      int(local_num_tokens), int(runtime_max_tokens_per_rank),
                                      ptrs, rb, len(payloads), ctypes.c_void_p(stats),
                                      _mask_array(active_rank_mask),
                                      ctypes.c_void_p(_stream_ptr(stream)), ctypes.byref(res)))
            self.last = (res, rbs)
        self._sync(stream)
        self.barrier()              # every rank's rows are in place
        if live and wait:
            _check(lib.ep_mp_dispatch_wait(self.handle, int(timeout_ns),
                                           ctypes.c_void_p(_stream_ptr(stream))))
        if not live or self.last is None:
            return None
        return RankDispatched(self, *self.last)

    def combine(self, expert_output: torch.Tensor, output: Optional[torch.Tensor] = None,
                active_rank_mask=None, timeout_ns: int = 1_000_000_000, stream=None):
        """Return this rank's rows (``expert_output`` [ep*tpr, hidden], bf16 or
        float8_e4m3fn) to their sources, then sum the rows of this rank's own
        tokens; returns bf16 [tpr, hidden] (None on a masked-off rank)."""
        live = rank_is_live(active_rank_mask, self.rank)
        x = expert_output
        dt = _a2a.COMBINE_BF16 if x.dtype == torch.bfloat16 else _a2a.COMBINE_FP8_E4M3
        if live:
            assert x.is_cuda and x.is_contiguous() and x.shape[-1] == self.hidden_size
            _check(lib.ep_mp_combine_send(self.handle, ctypes.c_void_p(x.data_ptr()), dt,
                                          ctypes.c_void_p(_stream_ptr(stream))))
        self._sync(stream)
        self.barrier()              # every rank's rows are back
        if not live:
            return None
        tpr = self.last[0].tokens_per_rank
        if output is None:
            output = torch.empty((tpr, self.hidden_size), dtype=torch.bfloat16, device=x.device)
        _check(lib.ep_mp_combine_finish(self.handle, ctypes.c_void_p(output.data_ptr()), dt,
                                        int(timeout_ns), ctypes.c_void_p(_stream_ptr(stream))))
        return output

    def get_status(self, stream=None) -> int:
        return lib.ep_mp_get_status(self.handle, ctypes.c_void_p(_stream_ptr(stream)))

    def destroy(self):
        """Unmap the peers' windows once every rank is done writing (barriers on
        both sides), then free this rank's window."""
        if not self._h.value:
            return
        torch.cuda.synchronize(self.device)
        self.barrier()
        _check(lib.ep_mp_destroy(ctypes.byref(self._h)))
        self.barrier()
        self.window = None

"""Thin ctypes binding of libep_a2a.so (declared in include/ep_a2a.h).

Argument marshalling only: every step of dispatch / combine runs in the CUDA
kernels of the library.  PyTorch supplies device memory (the workspace and the
caller's tensors) and streams.  There is no fallback: if the library is not
built, importing this module raises.

Low-level functions keep the C names (``ep_a2a_init``, ``ep_a2a_dispatch``,
...).  :class:`EpA2A` wraps one handle plus its workspace tensor and turns the
returned device pointers into zero-copy tensor views of the workspace.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# EP_A2A_LIBRARY selects another build of the same ABI, e.g. the checked build
# libep_a2a_checked.so (index checks compiled in); default: libep_a2a.so.
LIB_PATH = os.environ.get("EP_A2A_LIBRARY") or os.path.join(_HERE, "libep_a2a.so")

MAX_RANKS = 256
RANK_MASK_WORDS = 4
MAX_PAYLOADS = 8
MAX_TOP_K = 32

# ep_a2a_status
OK, ERR_INVALID_ARG, ERR_CAPACITY, ERR_UNSUPPORTED, ERR_CUDA, ERR_NOT_INITIALIZED, \
    ERR_NO_PLAN, ERR_DEVICE_TIMEOUT, ERR_DEVICE_BOUNDS = range(9)
COMBINE_BF16, COMBINE_FP8_E4M3 = 0, 1
OPT_COPY_PATH, OPT_COPY_CTAS_PER_SM, OPT_COPY_STAGES, OPT_COMBINE_THREADS, \
    OPT_BULK_MIN_ROW_BYTES, OPT_COMBINE_CTAS_PER_SM, OPT_COPY_CONSUMER_WARPS, \
    OPT_COPY_INTERLEAVE, OPT_VEC_UNROLL, OPT_VEC_CTAS_PER_SM, OPT_STORE_STREAMING, \
    OPT_PDL, OPT_VEC_THREADS_PER_TOKEN, OPT_COMBINE_PREFETCH, OPT_COPY_PREFETCH, \
    OPT_COMBINE_PIPELINE, OPT_COPY_VEC_BYTES, OPT_ROUTE_IN_COPY, \
    OPT_FP8_EXPERTS_KERNEL = range(19)


class EpA2AError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[{status}] {message}")
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [
        ("ep_size", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("max_tokens_per_rank", ctypes.c_int32),
        ("hidden_size", ctypes.c_int32),
        ("num_payloads", ctypes.c_int32),
        ("payload_row_bytes", ctypes.c_int64 * MAX_PAYLOADS),
        ("eplb_stats_num_experts", ctypes.c_int32),
        ("enable_rank_mask", ctypes.c_int32),
        ("invalid_expert_id", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class DispatchResult(ctypes.Structure):
    _fields_ = [
        ("tokens_per_rank", ctypes.c_int32),
        ("num_payloads", ctypes.c_int32),
        ("rank_stride_bytes", ctypes.c_int64),
        ("recv_payloads", ctypes.c_void_p * MAX_PAYLOADS),
        ("recv_topk_ids", ctypes.c_void_p),
        ("recv_valid", ctypes.c_void_p),
        ("eplb_gathered_stats", ctypes.c_void_p),
        ("send_counts", ctypes.c_void_p),
        ("plan_num_dst", ctypes.c_void_p),
        ("plan_dst_ranks", ctypes.c_void_p),
        ("plan_stride", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


KERNEL_NAMES = ["route_plan", "copy_bulk", "copy_vec", "combine", "copy_staged",
                "combine_experts", "combine_experts_fp8"]


class KernelTimes(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64 * 7), ("total_ms", ctypes.c_double * 7)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m combine_route_plan_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    st = ctypes.c_int
    sig = {
        "ep_a2a_workspace_size": (st, [P(Params), P(ctypes.c_size_t)]),
        "ep_a2a_init": (st, [P(Params), VP, ctypes.c_size_t, VP, P(VP)]),
        "ep_a2a_dispatch": (st, [VP, VP, VP, I32, P(VP), P(I64), I32, VP, VP, VP,
                                 P(DispatchResult)]),
        "ep_a2a_combine": (st, [VP, VP, ctypes.c_int, VP, VP]),
        "ep_a2a_quantize_e4m3": (st, [VP, VP, I64, VP]),
        "ep_a2a_combine_experts": (st, [VP, VP, VP, VP, VP]),
        "ep_a2a_combine_experts_fp8": (st, [VP, VP, VP, VP, VP]),
        "ep_a2a_combine_scaled": (st, [VP, VP, VP, VP, VP]),
        "ep_a2a_quantize_e4m3_rows": (st, [VP, VP, VP, I64, I32, VP]),
        "ep_a2a_allgather": (st, [I32, I32, VP, VP, P(VP), P(I64), I32, P(VP), I64, VP]),
        "ep_a2a_reduce_scatter": (st, [I32, I32, I32, VP, VP, VP, VP, VP]),
        "ep_a2a_get_status": (st, [VP, VP]),
        "ep_a2a_debug_wait_probe": (st, [VP, I64, VP]),
        "ep_a2a_set_option": (st, [VP, ctypes.c_int, I64]),
        "ep_a2a_destroy": (st, [P(VP)]),
        "ep_a2a_grow_params": (st, [P(Params), P(Params), P(Params), P(I32)]),
        "ep_a2a_set_combine_hidden": (st, [VP, I32]),
        "ep_a2a_profile_start": (st, [VP, I32]),
        "ep_a2a_profile_stop": (st, [VP, P(KernelTimes)]),
        "ep_a2a_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "ep_a2a_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status: int):
    if status != OK:
        raise EpA2AError(status, lib.ep_a2a_last_error().decode() or
                         lib.ep_a2a_status_string(status).decode())


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


# --------------------------------------------------------------------------- #
# C functions under their own names
# --------------------------------------------------------------------------- #

def ep_a2a_workspace_size(params: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.ep_a2a_workspace_size(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def ep_a2a_init(params: Params, workspace_ptr: int, workspace_bytes: int, stream=None) -> int:
    h = ctypes.c_void_p(0)
    _check(lib.ep_a2a_init(ctypes.byref(params), ctypes.c_void_p(workspace_ptr), workspace_bytes,
                           ctypes.c_void_p(_stream_ptr(stream)), ctypes.byref(h)))
    return h.value


def ep_a2a_dispatch(handle: int, token_selected_experts_ptr: int, local_num_tokens: Sequence[int],
                    runtime_max_tokens_per_rank: int, payload_ptrs: Sequence[int],
                    payload_row_bytes: Optional[Sequence[int]], eplb_local_stats_ptr: int = 0,
                    active_rank_mask: Optional[Sequence[int]] = None, stream=None) -> DispatchResult:
    n = (ctypes.c_int32 * len(local_num_tokens))(*[int(x) for x in local_num_tokens])
    ptrs = (ctypes.c_void_p * max(1, len(payload_ptrs)))(*[ctypes.c_void_p(p) for p in payload_ptrs])
    rb = None
    if payload_row_bytes is not None:
        rb = (ctypes.c_int64 * max(1, len(payload_row_bytes)))(*[int(x) for x in payload_row_bytes])
    mask = None
    if active_rank_mask is not None:
        words = [int(w) for w in active_rank_mask] + [0] * RANK_MASK_WORDS
        mask = (ctypes.c_uint64 * RANK_MASK_WORDS)(*words[:RANK_MASK_WORDS])
    res = DispatchResult()
    _check(lib.ep_a2a_dispatch(
        ctypes.c_void_p(handle), ctypes.c_void_p(token_selected_experts_ptr), n,
        int(runtime_max_tokens_per_rank), ptrs, rb, len(payload_ptrs),
        ctypes.c_void_p(eplb_local_stats_ptr or None),
        ctypes.cast(mask, ctypes.c_void_p) if mask is not None else None,
        ctypes.c_void_p(_stream_ptr(stream)), ctypes.byref(res)))
    return res


def ep_a2a_combine(handle: int, expert_output_ptr: int, dtype: int, output_ptr: int, stream=None):
    _check(lib.ep_a2a_combine(ctypes.c_void_p(handle), ctypes.c_void_p(expert_output_ptr),
                              int(dtype), ctypes.c_void_p(output_ptr),
                              ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_combine_experts(handle: int, topk_weights_ptr: int, expert_out_ptr: int,
                           output_ptr: int, stream=None):
    _check(lib.ep_a2a_combine_experts(ctypes.c_void_p(handle), ctypes.c_void_p(topk_weights_ptr),
                                      ctypes.c_void_p(expert_out_ptr), ctypes.c_void_p(output_ptr),
                                      ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_combine_experts_fp8(handle: int, topk_weights_ptr: int, expert_out_ptr: int,
                               output_ptr: int, stream=None):
    _check(lib.ep_a2a_combine_experts_fp8(ctypes.c_void_p(handle),
                                          ctypes.c_void_p(topk_weights_ptr),
                                          ctypes.c_void_p(expert_out_ptr),
                                          ctypes.c_void_p(output_ptr),
                                          ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_combine_scaled(handle: int, e4m3_ptr: int, scales_ptr: int, output_ptr: int,
                          stream=None):
    _check(lib.ep_a2a_combine_scaled(ctypes.c_void_p(handle), ctypes.c_void_p(e4m3_ptr),
                                     ctypes.c_void_p(scales_ptr), ctypes.c_void_p(output_ptr),
                                     ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_quantize_e4m3_rows(bf16_ptr: int, e4m3_ptr: int, scales_ptr: int, rows: int,
                              hidden: int, stream=None):
    _check(lib.ep_a2a_quantize_e4m3_rows(ctypes.c_void_p(bf16_ptr), ctypes.c_void_p(e4m3_ptr),
                                         ctypes.c_void_p(scales_ptr), int(rows), int(hidden),
                                         ctypes.c_void_p(_stream_ptr(stream))))


def _host_i32(values):
    arr = (ctypes.c_int32 * len(values))(*[int(v) for v in values])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def _host_mask(active_rank_mask):
    if active_rank_mask is None:
        return None, None
    words = [int(w) for w in np.asarray(active_rank_mask, dtype=np.uint64)] + [0] * RANK_MASK_WORDS
    arr = (ctypes.c_uint64 * RANK_MASK_WORDS)(*words[:RANK_MASK_WORDS])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def ep_a2a_allgather(ep_size: int, tokens_per_rank: int, local_num_tokens, payload_ptrs,
                     payload_row_bytes, recv_ptrs, recv_rank_stride_bytes: int,
                     active_rank_mask=None, stream=None):
    n_ptr, n_keep = _host_i32(local_num_tokens)
    m_ptr, m_keep = _host_mask(active_rank_mask)
    k = max(1, len(payload_ptrs))
    src = (ctypes.c_void_p * k)(*[ctypes.c_void_p(p) for p in payload_ptrs])
    dst = (ctypes.c_void_p * k)(*[ctypes.c_void_p(p) for p in recv_ptrs])
    rb = (ctypes.c_int64 * k)(*[int(b) for b in payload_row_bytes])
    _check(lib.ep_a2a_allgather(ep_size, tokens_per_rank, n_ptr, m_ptr, src, rb,
                                len(payload_ptrs), dst, int(recv_rank_stride_bytes),
                                ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_reduce_scatter(ep_size: int, tokens_per_rank: int, hidden: int, local_num_tokens,
                          x_ptr: int, out_ptr: int, active_rank_mask=None, stream=None):
    n_ptr, n_keep = _host_i32(local_num_tokens)
    m_ptr, m_keep = _host_mask(active_rank_mask)
    _check(lib.ep_a2a_reduce_scatter(ep_size, tokens_per_rank, hidden, n_ptr, m_ptr,
                                     ctypes.c_void_p(x_ptr), ctypes.c_void_p(out_ptr),
                                     ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_quantize_e4m3(bf16_ptr: int, e4m3_ptr: int, n: int, stream=None):
    _check(lib.ep_a2a_quantize_e4m3(ctypes.c_void_p(bf16_ptr), ctypes.c_void_p(e4m3_ptr), int(n),
                                    ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_get_status(handle: int, stream=None) -> int:
    """Raw status (does not raise): OK or ERR_DEVICE_TIMEOUT, ..."""
    return int(lib.ep_a2a_get_status(ctypes.c_void_p(handle), ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_debug_wait_probe(handle: int, limit_ns: int, stream=None):
    _check(lib.ep_a2a_debug_wait_probe(ctypes.c_void_p(handle), int(limit_ns),
                                       ctypes.c_void_p(_stream_ptr(stream))))


def ep_a2a_set_option(handle: int, option: int, value: int):
    _check(lib.ep_a2a_set_option(ctypes.c_void_p(handle), int(option), int(value)))


def ep_a2a_profile_start(handle: int, max_launches: int):
    _check(lib.ep_a2a_profile_start(ctypes.c_void_p(handle), int(max_launches)))


def ep_a2a_profile_stop(handle: int) -> dict:
    """{kernel name: (launches, total ms)} of the launches timed since start."""
    t = KernelTimes()
    _check(lib.ep_a2a_profile_stop(ctypes.c_void_p(handle), ctypes.byref(t)))
    return {name: (int(t.launches[i]), float(t.total_ms[i])) for i, name in enumerate(KERNEL_NAMES)}


def ep_a2a_destroy(handle_box: ctypes.c_void_p):
    _check(lib.ep_a2a_destroy(ctypes.byref(handle_box)))


def ep_a2a_grow_params(current: Params, request: Params):
    """(parameters serving both, True if they differ from ``current``)."""
    out, grown = Params(), ctypes.c_int32(0)
    _check(lib.ep_a2a_grow_params(ctypes.byref(current), ctypes.byref(request),
                                  ctypes.byref(out), ctypes.byref(grown)))
    return out, bool(grown.value)


def ep_a2a_set_combine_hidden(handle: int, hidden: int):
    _check(lib.ep_a2a_set_combine_hidden(ctypes.c_void_p(handle), int(hidden)))


def make_params(ep_size: int, num_experts: int, top_k: int, max_tokens_per_rank: int,
                hidden_size: int, payload_row_bytes: Sequence[int],
                eplb_stats_num_experts: int = 0, enable_rank_mask: bool = False,
                invalid_expert_id: int = -1) -> Params:
    p = Params()
    p.ep_size, p.num_experts, p.top_k = ep_size, num_experts, top_k
    p.max_tokens_per_rank, p.hidden_size = max_tokens_per_rank, hidden_size
    p.num_payloads = len(payload_row_bytes)
    for i, rb in enumerate(payload_row_bytes):
        p.payload_row_bytes[i] = int(rb)
    p.eplb_stats_num_experts = eplb_stats_num_experts
    p.enable_rank_mask = int(bool(enable_rank_mask))
    p.invalid_expert_id = invalid_expert_id
    p.reserved = 0
    return p


def ep_a2a_status_string(status: int) -> str:
    return lib.ep_a2a_status_string(int(status)).decode()


# --------------------------------------------------------------------------- #
# Convenience wrapper over torch tensors
# --------------------------------------------------------------------------- #

class Dispatched:
    """Workspace-backed views of one dispatch (valid until the next dispatch)."""

    def __init__(self, comm: "EpA2A", res: DispatchResult, row_bytes: List[int]):
        ws = comm.workspace
        base = ws.data_ptr()
        ep, k = comm.ep_size, comm.top_k
        tpr = res.tokens_per_rank
        stride = res.rank_stride_bytes
        slots = ep * tpr
        self.tokens_per_rank = tpr
        self.rank_stride_bytes = stride

        def per_rank(ptr, row_elems, dtype):
            """[ep, slots, row_elems] view of a per-rank array at byte pointer `ptr`."""
            esz = torch.tensor([], dtype=dtype).element_size()
            off = ptr - base
            nbytes_row = row_elems * esz
            v = torch.as_strided(ws, (ep, slots * nbytes_row), (stride, 1), off)
            return v.view(dtype).view(ep, slots, row_elems)

        self.recv_payloads = [per_rank(res.recv_payloads[i], rb, torch.uint8)
                              for i, rb in enumerate(row_bytes)]
        self.recv_topk_ids = per_rank(res.recv_topk_ids, k, torch.int32)
        self.recv_valid = per_rank(res.recv_valid, 1, torch.uint8).view(ep, slots)
        self.eplb_gathered_stats = None
        if res.eplb_gathered_stats:
            ne = comm.eplb_stats_num_experts
            off = res.eplb_gathered_stats - base
            v = torch.as_strided(ws, (ep, ep * ne * 4), (stride, 1), off)
            self.eplb_gathered_stats = v.view(torch.int32).view(ep, ep, ne)
        n_cnt = ep * ep * 4
        self.send_counts = ws[res.send_counts - base: res.send_counts - base + n_cnt] \
            .view(torch.int32).view(ep, ep)
        self.plan_num_dst = ws[res.plan_num_dst - base: res.plan_num_dst - base + slots] \
            .view(ep, tpr)
        ps = res.plan_stride
        self.plan_dst_ranks = ws[res.plan_dst_ranks - base: res.plan_dst_ranks - base + slots * ps] \
            .view(ep, tpr, ps)


class EpA2A:
    """One handle of the library plus its (torch-allocated) device workspace."""

    def __init__(self, ep_size: int, num_experts: int, top_k: int, max_tokens_per_rank: int,
                 hidden_size: int, payload_row_bytes: Sequence[int],
                 eplb_stats_num_experts: int = 0, enable_rank_mask: bool = False,
                 invalid_expert_id: int = -1, device=None, stream=None,
                 workspace_fill: Optional[int] = None):
        p = make_params(ep_size, num_experts, top_k, max_tokens_per_rank, hidden_size,
                        payload_row_bytes, eplb_stats_num_experts, enable_rank_mask,
                        invalid_expert_id)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self._workspace_fill = workspace_fill
        self._options = {}
        self._h = ctypes.c_void_p(0)
        self._create(p, stream)

    def _create(self, p: Params, stream):
        self.params = p
        self.ep_size, self.num_experts, self.top_k = p.ep_size, p.num_experts, p.top_k
        self.hidden_size = p.hidden_size
        self.payload_row_bytes = [int(p.payload_row_bytes[i]) for i in range(p.num_payloads)]
        self.eplb_stats_num_experts = p.eplb_stats_num_experts
        nbytes = ep_a2a_workspace_size(p)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        if self._workspace_fill is not None:
            self.workspace.fill_(self._workspace_fill)
        self._h = ctypes.c_void_p(ep_a2a_init(p, self.workspace.data_ptr(), nbytes, stream))
        for option, value in self._options.items():
            ep_a2a_set_option(self._h.value, option, value)
        self.combine_hidden = p.hidden_size
        self.last_tokens_per_rank = None

    def ensure_capacity(self, max_tokens_per_rank: Optional[int] = None,
                        hidden_size: Optional[int] = None,
                        payload_row_bytes: Optional[Sequence[int]] = None,
                        eplb_stats_num_experts: int = 0, enable_rank_mask: bool = False,
                        stream=None) -> bool:
        """Grow the handle to also serve this request (ep_a2a_grow_params); True if
        it was replaced.  Replacing synchronises the device, destroys the old handle
        and allocates a new workspace: earlier views and the plan are gone."""
        cur = self.params
        req = make_params(cur.ep_size, cur.num_experts, cur.top_k,
                          max_tokens_per_rank or cur.max_tokens_per_rank,
                          hidden_size or cur.hidden_size,
                          self.payload_row_bytes if payload_row_bytes is None
                          else payload_row_bytes,
                          eplb_stats_num_experts, enable_rank_mask, cur.invalid_expert_id)
        grown_params, grown = ep_a2a_grow_params(cur, req)
        if not grown:
            return False
        torch.cuda.synchronize(self.device)
        ep_a2a_destroy(self._h)
        self.workspace = None
        self._create(grown_params, stream)
        return True

    def _use_hidden(self, hidden: int):
        if hidden != self.combine_hidden:
            ep_a2a_set_combine_hidden(self.handle, hidden)
            self.combine_hidden = hidden

    @property
    def handle(self) -> int:
        if not self._h.value:
            raise EpA2AError(ERR_NOT_INITIALIZED, "handle destroyed")
        return self._h.value

    def set_option(self, option: int, value: int):
        ep_a2a_set_option(self.handle, option, value)
        self._options[option] = value

    def dispatch(self, token_selected_experts: torch.Tensor, local_num_tokens: Sequence[int],
                 payloads: Sequence[torch.Tensor], runtime_max_tokens_per_rank: Optional[int] = None,
                 eplb_local_stats: Optional[torch.Tensor] = None,
                 active_rank_mask=None, stream=None, views: bool = True):
        """token_selected_experts int32 [ep, tpr, k]; payloads each [ep, tpr, ...] (any dtype).

        Returns workspace-backed tensor views (:class:`Dispatched`), or the raw
        :class:`DispatchResult` when ``views`` is False (no per-call tensor setup)."""
        ids = token_selected_experts
        assert ids.is_cuda and ids.dtype == torch.int32 and ids.is_contiguous()
        tpr = ids.shape[1] if runtime_max_tokens_per_rank is None else runtime_max_tokens_per_rank
        ptrs, rbs = [], []
        for t in payloads:
            assert t.is_cuda and t.is_contiguous() and t.shape[0] == self.ep_size
            ptrs.append(t.data_ptr())
            rbs.append(t[0, 0].numel() * t.element_size() if t.dim() > 2 else t.element_size())
        stats_ptr = 0
        if eplb_local_stats is not None:
            assert eplb_local_stats.is_cuda and eplb_local_stats.dtype == torch.int32
            stats_ptr = eplb_local_stats.data_ptr()
        if active_rank_mask is not None:
            active_rank_mask = [int(w) for w in np.asarray(active_rank_mask, dtype=np.uint64)]
        if tpr > 0:
            assert ids.shape == (self.ep_size, tpr, self.top_k), ids.shape
            for t in payloads:
                assert t.shape[1] == tpr, t.shape
        if eplb_local_stats is not None:
            assert eplb_local_stats.shape == (self.ep_size, self.eplb_stats_num_experts)
        res = ep_a2a_dispatch(self.handle, ids.data_ptr(), local_num_tokens, tpr, ptrs, rbs,
                              stats_ptr, active_rank_mask, stream)
        self.last_tokens_per_rank = res.tokens_per_rank
        return Dispatched(self, res, rbs) if views else res

    def combine(self, expert_output: torch.Tensor, output: Optional[torch.Tensor] = None,
                tokens_per_rank: Optional[int] = None, stream=None) -> torch.Tensor:
        """expert_output [ep, ep*tpr, hidden] bf16 or float8_e4m3fn; returns bf16 [ep, tpr, hidden]."""
        x = expert_output
        assert x.is_cuda and x.is_contiguous()
        if x.dtype == torch.bfloat16:
            dt = COMBINE_BF16
        elif x.dtype in (torch.float8_e4m3fn, torch.uint8):
            dt = COMBINE_FP8_E4M3
        else:
            raise TypeError(f"combine input must be bf16 or float8_e4m3fn, got {x.dtype}")
        tpr = self.last_tokens_per_rank
        hidden = x.shape[-1] if x.dim() >= 2 else self.hidden_size
        if tpr is not None:
            assert x.numel() == self.ep_size * self.ep_size * tpr * hidden, x.shape
            self._use_hidden(hidden)
        if output is None:
            if tpr is None:
                tpr = tokens_per_rank if tokens_per_rank is not None else 1
            output = torch.empty((self.ep_size, tpr, hidden), dtype=torch.bfloat16,
                                 device=x.device)
        assert output.is_cuda and output.dtype == torch.bfloat16 and output.is_contiguous()
        if tpr is not None:
            assert output.numel() == self.ep_size * tpr * hidden, output.shape
        ep_a2a_combine(self.handle, x.data_ptr(), dt, output.data_ptr(), stream)
        return output

    def combine_experts(self, topk_weights: torch.Tensor, expert_output_per_slot: torch.Tensor,
                        output: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """topk_weights fp32 [ep, tpr, k]; expert_output_per_slot bf16 [ep, tpr, k, hidden];
        returns bf16 [ep, tpr, hidden] (see ep_a2a_combine_experts)."""
        tpr = self.last_tokens_per_rank
        assert tpr is not None, "combine needs a preceding dispatch"
        w, y = topk_weights, expert_output_per_slot
        assert w.is_cuda and w.dtype == torch.float32 and w.is_contiguous()
        assert w.numel() == self.ep_size * tpr * self.top_k, w.shape
        assert y.is_cuda and y.dtype == torch.bfloat16 and y.is_contiguous()
        hidden = y.shape[-1]
        assert y.numel() == self.ep_size * tpr * self.top_k * hidden, y.shape
        if output is None:
            output = torch.empty((self.ep_size, tpr, hidden), dtype=torch.bfloat16,
                                 device=y.device)
        assert output.is_cuda and output.dtype == torch.bfloat16 and output.is_contiguous()
        assert output.numel() == self.ep_size * tpr * hidden, output.shape
        self._use_hidden(hidden)
        ep_a2a_combine_experts(self.handle, w.data_ptr(), y.data_ptr(), output.data_ptr(), stream)
        return output

    def combine_experts_fp8(self, topk_weights: torch.Tensor, expert_output_per_slot: torch.Tensor,
                            output: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """As :meth:`combine_experts`, with each destination's row quantised to E4M3
        with one fp32 scale per row before the sum (ep_a2a_combine_experts_fp8)."""
        tpr = self.last_tokens_per_rank
        assert tpr is not None, "combine needs a preceding dispatch"
        w, y = topk_weights, expert_output_per_slot
        assert w.is_cuda and w.dtype == torch.float32 and w.is_contiguous()
        assert w.numel() == self.ep_size * tpr * self.top_k, w.shape
        assert y.is_cuda and y.dtype == torch.bfloat16 and y.is_contiguous()
        hidden = y.shape[-1]
        assert y.numel() == self.ep_size * tpr * self.top_k * hidden, y.shape
        if output is None:
            output = torch.empty((self.ep_size, tpr, hidden), dtype=torch.bfloat16,
                                 device=y.device)
        assert output.is_cuda and output.dtype == torch.bfloat16 and output.is_contiguous()
        assert output.numel() == self.ep_size * tpr * hidden, output.shape
        self._use_hidden(hidden)
        ep_a2a_combine_experts_fp8(self.handle, w.data_ptr(), y.data_ptr(), output.data_ptr(),
                                   stream)
        return output

    def combine_scaled(self, codes: torch.Tensor, row_scales: torch.Tensor,
                       output: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """codes E4M3 [ep, ep*tpr, hidden]; row_scales fp32 [ep, ep*tpr]; bf16 out."""
        tpr = self.last_tokens_per_rank
        assert tpr is not None, "combine needs a preceding dispatch"
        rows = self.ep_size * self.ep_size * tpr
        assert codes.is_cuda and codes.is_contiguous() and codes.element_size() == 1
        hidden = codes.shape[-1]
        assert codes.numel() == rows * hidden, codes.shape
        assert row_scales.is_cuda and row_scales.dtype == torch.float32
        assert row_scales.is_contiguous() and row_scales.numel() == rows, row_scales.shape
        if output is None:
            output = torch.empty((self.ep_size, tpr, hidden), dtype=torch.bfloat16,
                                 device=codes.device)
        assert output.is_cuda and output.dtype == torch.bfloat16 and output.is_contiguous()
        assert output.numel() == self.ep_size * tpr * hidden, output.shape
        self._use_hidden(hidden)
        ep_a2a_combine_scaled(self.handle, codes.data_ptr(), row_scales.data_ptr(),
                              output.data_ptr(), stream)
        return output

    def get_status(self, stream=None) -> int:
        return ep_a2a_get_status(self.handle, stream)

    def destroy(self):
        ep_a2a_destroy(self._h)          # idempotent; sets the handle to NULL

    def __del__(self):
        try:
            if getattr(self, "_h", None) is not None and self._h.value:
                lib.ep_a2a_destroy(ctypes.byref(self._h))
        except Exception:
            pass


def quantize_e4m3_rows(x_bf16: torch.Tensor, stream=None):
    """bf16 [..., hidden] -> (E4M3 codes as torch.float8_e4m3fn, fp32 scales [...])."""
    assert x_bf16.is_cuda and x_bf16.dtype == torch.bfloat16 and x_bf16.is_contiguous()
    hidden = x_bf16.shape[-1]
    rows = x_bf16.numel() // hidden
    codes = torch.empty(x_bf16.shape, dtype=torch.float8_e4m3fn, device=x_bf16.device)
    scales = torch.empty(x_bf16.shape[:-1], dtype=torch.float32, device=x_bf16.device)
    ep_a2a_quantize_e4m3_rows(x_bf16.data_ptr(), codes.data_ptr(), scales.data_ptr(), rows,
                              hidden, stream)
    return codes, scales


def quantize_e4m3(x_bf16: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """bf16 tensor -> E4M3 bytes (torch.float8_e4m3fn), by the library's kernel."""
    assert x_bf16.is_cuda and x_bf16.dtype == torch.bfloat16 and x_bf16.is_contiguous()
    if out is None:
        out = torch.empty(x_bf16.shape, dtype=torch.float8_e4m3fn, device=x_bf16.device)
    ep_a2a_quantize_e4m3(x_bf16.data_ptr(), out.data_ptr(), x_bf16.numel(), stream)
    return out

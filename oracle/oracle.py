"""ctypes loader for the plain-C oracle (``ep_a2a_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never imports, links or calls it, and it never imports the CUDA library.

All arrays are numpy arrays on the host.  The functions only marshal arguments;
every step of the computation is in the C file, which cites the page passages
it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_a2a_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libep_a2a_oracle.so")

# Plain IEEE arithmetic: no contraction into FMA, no fast-math reassociation.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (building the checker is not using it)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".{os.getpid()}.{time.time_ns()}.tmp"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.oracle_route.argtypes = [I, I, I, I, P, P, P, ctypes.c_int32, P, P, P, P, P]
        lib.oracle_route.restype = I
        lib.oracle_dispatch_payload.argtypes = [I, I, I, I64, P, P, P, P, I]
        lib.oracle_dispatch_payload.restype = None
        lib.oracle_eplb_gather.argtypes = [I, I, P, P, P]
        lib.oracle_eplb_gather.restype = None
        lib.oracle_combine.argtypes = [I, I, I, I, P, P, P, I, P, P, I64]
        lib.oracle_combine.restype = None
        lib.oracle_expert_reduce.argtypes = [I, I, I, I, I, P, P, P, P, P, P]
        lib.oracle_expert_reduce.restype = None
        lib.oracle_quantize_e4m3_rows.argtypes = [P, I64, I, P, P]
        lib.oracle_quantize_e4m3_rows.restype = None
        lib.oracle_combine_scaled.argtypes = [I, I, I, I, P, P, P, P, P]
        lib.oracle_combine_scaled.restype = None
        lib.oracle_allgather.argtypes = [I, I, I64, P, P, P, P]
        lib.oracle_allgather.restype = None
        lib.oracle_reduce_scatter.argtypes = [I, I, I, P, P, P, P]
        lib.oracle_reduce_scatter.restype = None
        lib.oracle_quantize_e4m3.argtypes = [P, P, I64]
        lib.oracle_quantize_e4m3.restype = None
        lib.oracle_bf16_from_f32.argtypes = [ctypes.c_float]
        lib.oracle_bf16_from_f32.restype = ctypes.c_uint16
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_e4m3_from_f32.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_from_f32.restype = ctypes.c_uint8
        lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f32.restype = ctypes.c_float
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _mask_words(active_rank_mask, ep_size):
    if active_rank_mask is None:
        return None
    m = np.ascontiguousarray(np.asarray(active_rank_mask, dtype=np.uint64))
    assert m.size * 64 >= ep_size
    return m


class RoutePlan:
    """Result of :func:`route` (host arrays)."""

    def __init__(self, ep_size, top_k, tokens_per_rank, num_dst, dst_ranks,
                 send_counts, recv_valid, recv_topk_ids):
        self.ep_size = ep_size
        self.top_k = top_k
        self.tokens_per_rank = tokens_per_rank
        self.num_dst = num_dst            # int32 [ep, tpr]; -1 = no token
        self.dst_ranks = dst_ranks        # int32 [ep, tpr, k]; ascending, -1 pad
        self.send_counts = send_counts    # int32 [ep(src), ep(dst)]
        self.recv_valid = recv_valid      # uint8 [ep(dst), ep*tpr]
        self.recv_topk_ids = recv_topk_ids  # int32 [ep(dst), ep*tpr, k]


def route(ep_size, num_experts, top_k, tokens_per_rank, token_selected_experts,
          local_num_tokens, active_rank_mask=None, invalid_expert_id=None,
          recv_valid_init=None, recv_topk_ids_init=None) -> RoutePlan:
    """Routing plan of every virtual rank (see ``oracle_route`` in the C file).

    ``recv_*_init`` give the prior contents of the receive arrays (rows of
    masked-off destinations keep them); by default they start as 0xAB canaries.
    """
    lib = _load()
    ep, k, tpr = ep_size, top_k, tokens_per_rank
    ids = np.ascontiguousarray(token_selected_experts, dtype=np.int32).reshape(ep, tpr, k)
    n = np.ascontiguousarray(local_num_tokens, dtype=np.int32).reshape(ep)
    mask = _mask_words(active_rank_mask, ep)
    inv = num_experts if invalid_expert_id is None else invalid_expert_id
    num_dst = np.empty((ep, tpr), np.int32)
    dst_ranks = np.empty((ep, tpr, k), np.int32)
    counts = np.empty((ep, ep), np.int32)
    if recv_valid_init is None:
        valid = np.full((ep, ep * tpr), 0xAB, np.uint8)
    else:
        valid = np.array(recv_valid_init, dtype=np.uint8, copy=True).reshape(ep, ep * tpr)
    if recv_topk_ids_init is None:
        rids = np.full((ep, ep * tpr, k), -0x54545455, np.int32)  # 0xABABABAB
    else:
        rids = np.array(recv_topk_ids_init, dtype=np.int32, copy=True).reshape(ep, ep * tpr, k)
    rc = lib.oracle_route(ep, num_experts, k, tpr, _ptr(ids), _ptr(n), _ptr(mask),
                          inv, _ptr(num_dst), _ptr(dst_ranks), _ptr(counts),
                          _ptr(valid), _ptr(rids))
    if rc != 0:
        raise ValueError("oracle_route: unsupported ep_size / num_experts")
    return RoutePlan(ep, k, tpr, num_dst, dst_ranks, counts, valid, rids)


def dispatch_payload(plan: RoutePlan, payload, recv_init=None, only_dst=-1):
    """Receive rows of one payload ``[ep, tpr, row_bytes]`` (any dtype, as bytes).

    Returns a uint8 array ``[ep, ep*tpr, row_bytes]`` (``[1, ...]`` when
    ``only_dst >= 0``).  Invalid rows keep ``recv_init`` (default 0xCD canary).
    """
    lib = _load()
    ep, tpr = plan.ep_size, plan.tokens_per_rank
    src = np.ascontiguousarray(payload).view(np.uint8).reshape(ep, tpr, -1)
    rb = src.shape[2]
    nd = 1 if only_dst >= 0 else ep
    if recv_init is None:
        recv = np.full((nd, ep * tpr, rb), 0xCD, np.uint8)
    else:
        recv = np.array(recv_init, dtype=np.uint8, copy=True).reshape(nd, ep * tpr, rb)
    lib.oracle_dispatch_payload(ep, plan.top_k, tpr, rb, _ptr(src), _ptr(plan.num_dst),
                                _ptr(plan.dst_ranks), _ptr(recv), int(only_dst))
    return recv


def eplb_gather(ep_size, eplb_local_stats, active_rank_mask=None, gathered_init=None):
    """``[ep(dst), ep(src), num_stats]`` int32; masked-off destinations keep ``gathered_init``."""
    lib = _load()
    stats = np.ascontiguousarray(eplb_local_stats, dtype=np.int32).reshape(ep_size, -1)
    ne = stats.shape[1]
    if gathered_init is None:
        out = np.full((ep_size, ep_size, ne), -0x32323233, np.int32)  # 0xCDCDCDCD
    else:
        out = np.array(gathered_init, dtype=np.int32, copy=True).reshape(ep_size, ep_size, ne)
    lib.oracle_eplb_gather(ep_size, ne, _ptr(stats), _ptr(_mask_words(active_rank_mask, ep_size)),
                           _ptr(out))
    return out


def combine(plan: RoutePlan, expert_output, hidden, input_is_e4m3=False,
            out_init=None, token_list=None):
    """bf16 bits ``uint16 [ep, tpr, hidden]`` (see ``oracle_combine``).

    ``expert_output`` holds bf16 bits (uint16) or E4M3 bytes (uint8), shaped
    ``[ep(dst), ep*tpr, hidden]``.  Rows of absent tokens keep ``out_init``
    (default 0xEEEE).  ``token_list`` (flat r*tpr+t) restricts the work.
    """
    lib = _load()
    ep, tpr = plan.ep_size, plan.tokens_per_rank
    dt = np.uint8 if input_is_e4m3 else np.uint16
    x = np.ascontiguousarray(expert_output).view(dt).reshape(ep, ep * tpr, hidden)
    if out_init is None:
        out = np.full((ep, tpr, hidden), 0xEEEE, np.uint16)
    else:
        out = np.array(out_init, dtype=np.uint16, copy=True).reshape(ep, tpr, hidden)
    if token_list is None:
        tl, nl = None, 0
    else:
        tl = np.ascontiguousarray(token_list, dtype=np.int64)
        nl = tl.size
    lib.oracle_combine(ep, plan.top_k, tpr, hidden, _ptr(plan.num_dst), _ptr(plan.dst_ranks),
                       _ptr(x), int(bool(input_is_e4m3)), _ptr(out), _ptr(tl), nl)
    return out


def expert_reduce(plan: RoutePlan, num_experts, token_selected_experts, topk_weights,
                  expert_out, hidden, z_init=None):
    """Each destination's combine row from per-(token, slot) expert outputs
    (see ``oracle_expert_reduce``): uint16 bf16 bits ``[ep, ep*tpr, hidden]``.

    ``expert_out`` holds bf16 bits shaped ``[ep, tpr, k, hidden]``; rows of z no
    token fills keep ``z_init`` (default 0xEEEE)."""
    lib = _load()
    ep, tpr, k = plan.ep_size, plan.tokens_per_rank, plan.top_k
    ids = np.ascontiguousarray(token_selected_experts, dtype=np.int32).reshape(ep, tpr, k)
    w = np.ascontiguousarray(topk_weights, dtype=np.float32).reshape(ep, tpr, k)
    y = np.ascontiguousarray(expert_out).view(np.uint16).reshape(ep, tpr, k, hidden)
    if z_init is None:
        z = np.full((ep, ep * tpr, hidden), 0xEEEE, np.uint16)
    else:
        z = np.array(z_init, dtype=np.uint16, copy=True).reshape(ep, ep * tpr, hidden)
    lib.oracle_expert_reduce(ep, num_experts, k, tpr, hidden, _ptr(plan.num_dst),
                             _ptr(plan.dst_ranks), _ptr(ids), _ptr(w), _ptr(y), _ptr(z))
    return z


def combine_experts(plan: RoutePlan, num_experts, token_selected_experts, topk_weights,
                    expert_out, hidden, out_init=None):
    """The combine of per-expert outputs: the expert reduction, then combine."""
    z = expert_reduce(plan, num_experts, token_selected_experts, topk_weights, expert_out,
                      hidden)
    return combine(plan, z, hidden, out_init=out_init)


def quantize_e4m3_rows(bf16_bits, hidden):
    """(E4M3 codes uint8 [rows, hidden], fp32 scales [rows]) of bf16 rows, one
    scale per row (see ``oracle_quantize_e4m3_rows``)."""
    lib = _load()
    x = np.ascontiguousarray(bf16_bits).view(np.uint16).reshape(-1, hidden)
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty(x.shape[0], np.float32)
    lib.oracle_quantize_e4m3_rows(_ptr(x), x.shape[0], hidden, _ptr(codes), _ptr(scales))
    return codes, scales


def combine_scaled(plan: RoutePlan, codes, row_scales, hidden, out_init=None):
    """Combine of E4M3 rows with one fp32 scale per row: bf16 bits [ep, tpr, hidden]."""
    lib = _load()
    ep, tpr = plan.ep_size, plan.tokens_per_rank
    x = np.ascontiguousarray(codes).view(np.uint8).reshape(ep, ep * tpr, hidden)
    sc = np.ascontiguousarray(row_scales, dtype=np.float32).reshape(ep, ep * tpr)
    if out_init is None:
        out = np.full((ep, tpr, hidden), 0xEEEE, np.uint16)
    else:
        out = np.array(out_init, dtype=np.uint16, copy=True).reshape(ep, tpr, hidden)
    lib.oracle_combine_scaled(ep, plan.top_k, tpr, hidden, _ptr(plan.num_dst),
                              _ptr(plan.dst_ranks), _ptr(x), _ptr(sc), _ptr(out))
    return out


def combine_experts_fp8(plan: RoutePlan, num_experts, token_selected_experts, topk_weights,
                        expert_out, hidden, out_init=None):
    """The low-precision combine of per-expert outputs with the quantisation on
    the sending side (flashinfer.moe_ep.NVLinkOneSidedConfig,
    use_low_precision_combine; flashinfer.moe_ep.NVLinkTwoSidedAlltoAll,
    combine()): each destination rank forms its row z_d from its own experts'
    weighted outputs (``expert_reduce``), quantises it to E4M3 with one fp32
    scale per row (``quantize_e4m3_rows``), and the rows are summed as decoded
    codes times their scales in ascending rank order (``combine_scaled``).
    The three steps in that order; nothing else."""
    z = expert_reduce(plan, num_experts, token_selected_experts, topk_weights, expert_out,
                      hidden)
    # the rows a destination sends are those of the tokens it received; only
    # they are quantised (rows are independent) and read by the combine
    rows = np.nonzero((np.asarray(plan.recv_valid) == 1).reshape(-1))[0]
    flat = z.reshape(-1, hidden)
    codes = np.zeros(flat.shape, np.uint8)
    scales = np.ones(flat.shape[0], np.float32)
    if rows.size:
        c, sc = quantize_e4m3_rows(np.ascontiguousarray(flat[rows]), hidden)
        codes[rows] = c
        scales[rows] = sc
    return combine_scaled(plan, codes.reshape(z.shape), scales.reshape(z.shape[:2]), hidden,
                          out_init=out_init)


def allgather(ep_size, tokens_per_rank, local_num_tokens, payload, active_rank_mask=None,
              recv_init=None):
    """Dense dispatch: uint8 ``[ep, ep*tpr, row_bytes]`` (see ``oracle_allgather``)."""
    lib = _load()
    ep, tpr = ep_size, tokens_per_rank
    src = np.ascontiguousarray(payload).view(np.uint8).reshape(ep, tpr, -1)
    rb = src.shape[2]
    n = np.ascontiguousarray(local_num_tokens, dtype=np.int32).reshape(ep)
    if recv_init is None:
        recv = np.full((ep, ep * tpr, rb), 0xCD, np.uint8)
    else:
        recv = np.array(recv_init, dtype=np.uint8, copy=True).reshape(ep, ep * tpr, rb)
    lib.oracle_allgather(ep, tpr, rb, _ptr(n), _ptr(_mask_words(active_rank_mask, ep)),
                         _ptr(src), _ptr(recv))
    return recv


def reduce_scatter(ep_size, tokens_per_rank, hidden, local_num_tokens, x, active_rank_mask=None,
                   out_init=None):
    """Dense combine: bf16 bits ``[ep, tpr, hidden]`` (see ``oracle_reduce_scatter``)."""
    lib = _load()
    ep, tpr = ep_size, tokens_per_rank
    xx = np.ascontiguousarray(x).view(np.uint16).reshape(ep, ep * tpr, hidden)
    n = np.ascontiguousarray(local_num_tokens, dtype=np.int32).reshape(ep)
    if out_init is None:
        out = np.full((ep, tpr, hidden), 0xEEEE, np.uint16)
    else:
        out = np.array(out_init, dtype=np.uint16, copy=True).reshape(ep, tpr, hidden)
    lib.oracle_reduce_scatter(ep, tpr, hidden, _ptr(n), _ptr(_mask_words(active_rank_mask, ep)),
                              _ptr(xx), _ptr(out))
    return out


def quantize_e4m3(bf16_bits):
    """E4M3 bytes of bf16 values (round to nearest even, saturate to +-448)."""
    lib = _load()
    x = np.ascontiguousarray(bf16_bits).view(np.uint16)
    out = np.empty(x.shape, np.uint8)
    lib.oracle_quantize_e4m3(_ptr(x), _ptr(out), x.size)
    return out


def bf16_from_f32(x: float) -> int:
    return int(_load().oracle_bf16_from_f32(float(x)))


def bf16_to_f32(h: int) -> float:
    return float(_load().oracle_bf16_to_f32(int(h)))


def e4m3_from_f32(x: float) -> int:
    return int(_load().oracle_e4m3_from_f32(float(x)))


def e4m3_to_f32(b: int) -> float:
    return float(_load().oracle_e4m3_to_f32(int(b)))


__all__ = ["build", "route", "dispatch_payload", "eplb_gather", "combine", "expert_reduce",
           "combine_experts", "quantize_e4m3_rows", "combine_scaled", "combine_experts_fp8",
           "allgather",
           "reduce_scatter",
           "quantize_e4m3", "bf16_from_f32", "bf16_to_f32", "e4m3_from_f32",
           "e4m3_to_f32", "RoutePlan"]

"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, then compare element by element."""
from __future__ import annotations

import numpy as np
import torch

import oracle

CANARY = 0xCD          # workspace fill: rows nobody may write keep it
OUT_CANARY = -0x1112   # 0xEEEE as int16: output rows of absent tokens keep it


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def bits_f32(bits_u16: np.ndarray) -> np.ndarray:
    return (np.asarray(bits_u16, np.uint32) << 16).view(np.float32)


def assert_equal(gpu: torch.Tensor, want: np.ndarray, what: str):
    """Bit-exact comparison on the GPU (large arrays), with the first mismatches."""
    g = gpu.contiguous().view(-1)
    w = torch.from_numpy(np.ascontiguousarray(want)).view(-1)
    if g.dtype != w.dtype:
        w = w.view(g.dtype) if g.element_size() == w.element_size() else w.to(g.dtype)
    w = w.to(g.device)
    assert g.numel() == w.numel(), (what, g.numel(), w.numel())
    if g.element_size() == 2:
        g, w = g.view(torch.int16), w.view(torch.int16)
    elif g.element_size() == 1:
        g, w = g.view(torch.uint8), w.view(torch.uint8)
    bad = (g != w).nonzero().view(-1)
    if bad.numel():
        idx = bad[:8].tolist()
        raise AssertionError(f"{what}: {bad.numel()} mismatches, first at {idx}: "
                             f"gpu {g[bad[:8]].tolist()} want {w[bad[:8]].tolist()}")


class Run:
    """One dispatch + combine through the C ABI."""

    def __init__(self, w, x, copy_path=None, options=None, capacity=None, fp8=False):
        from combine_route_plan_b200 import ep_a2a
        ep, tpr, k, E, H = w.ep_size, w.tokens_per_rank, w.top_k, w.num_experts, w.hidden
        self.comm = ep_a2a.EpA2A(ep, E, k, capacity or tpr, H, w.payload_row_bytes(),
                                 eplb_stats_num_experts=E if w.eplb else 0,
                                 enable_rank_mask=bool(w.masked_ranks), workspace_fill=CANARY)
        if copy_path is not None:               # None: the library's default path
            self.comm.set_option(ep_a2a.OPT_COPY_PATH, copy_path)
        for opt, val in (options or {}).items():
            self.comm.set_option(opt, val)
        self.ids = x.token_selected_experts.cuda()
        self.payloads = [p.cuda() for p in x.payloads]
        self.stats = x.eplb_local_stats.cuda() if x.eplb_local_stats is not None else None
        self.d = self.comm.dispatch(self.ids, x.local_num_tokens, self.payloads, tpr, self.stats,
                                    x.active_rank_mask)
        self.out = None
        if x.expert_output is not None:
            xo = x.expert_output.cuda()
            if fp8:
                self.xq = ep_a2a.quantize_e4m3(xo)
                del xo
                xo = self.xq
            self.out = torch.full((ep, tpr, H), OUT_CANARY, dtype=torch.int16,
                                  device="cuda").view(torch.bfloat16)
            self.comm.combine(xo, self.out)
            del xo
        torch.cuda.synchronize()
        assert self.comm.get_status() == ep_a2a.OK


def oracle_plan(w, x):
    ep, tpr = w.ep_size, w.tokens_per_rank
    return oracle.route(ep, w.num_experts, w.top_k, tpr, x.token_selected_experts.numpy(),
                        x.local_num_tokens, x.active_rank_mask,
                        recv_valid_init=np.full((ep, ep * tpr), CANARY, np.uint8),
                        recv_topk_ids_init=np.full((ep, ep * tpr, 4 * w.top_k), CANARY, np.uint8)
                        .view(np.int32))


def check_plan(run: Run, plan, w):
    d = run.d
    k = w.top_k
    nd = plan.num_dst.copy()
    nd[nd < 0] = 0xFF
    assert_equal(d.plan_num_dst, nd.astype(np.uint8), "plan_num_dst")
    want = np.full(d.plan_dst_ranks.shape, 0xFF, np.uint8)
    ranks = plan.dst_ranks.copy()
    ranks[ranks < 0] = 0xFF
    want[:, :, :k] = ranks.astype(np.uint8)
    assert_equal(d.plan_dst_ranks, want, "plan_dst_ranks")
    assert_equal(d.send_counts, plan.send_counts, "send_counts")
    assert_equal(d.recv_valid, plan.recv_valid, "recv_valid")
    assert_equal(d.recv_topk_ids, plan.recv_topk_ids, "recv_topk_ids")


def check_payloads(run: Run, plan, w, x):
    ep, tpr = w.ep_size, w.tokens_per_rank
    for i, p in enumerate(x.payloads):
        rb = p.shape[2]
        for dst in range(ep):
            want = oracle.dispatch_payload(plan, p.numpy(), only_dst=dst,
                                           recv_init=np.full((1, ep * tpr, rb), CANARY, np.uint8))
            assert_equal(run.d.recv_payloads[i][dst], want, f"payload {i} rank {dst}")


def check_eplb(run: Run, w, x):
    if x.eplb_local_stats is None:
        assert run.d.eplb_gathered_stats is None
        return
    ep = w.ep_size
    want = oracle.eplb_gather(ep, x.eplb_local_stats.numpy(), x.active_rank_mask,
                              gathered_init=np.full((ep, ep, 4 * w.num_experts), CANARY, np.uint8)
                              .view(np.int32))
    assert_equal(run.d.eplb_gathered_stats, want, "eplb_gathered_stats")


def oracle_out_init(w):
    return np.full((w.ep_size, w.tokens_per_rank, w.hidden), 0xEEEE, np.uint16)


def check_combine(run: Run, plan, w, x):
    want = oracle.combine(plan, to_np(x.expert_output), w.hidden, out_init=oracle_out_init(w))
    assert_equal(run.out, want, "combine")


def oracle_e4m3_table():
    return oracle.quantize_e4m3(np.arange(65536, dtype=np.uint32).astype(np.uint16))


def oracle_quantize_big(bf16_bits: np.ndarray, table: np.ndarray) -> np.ndarray:
    """The oracle's E4M3 encoder applied to every element (through its table of
    all 65536 bf16 inputs), in chunks to bound host memory."""
    flat = bf16_bits.reshape(-1)
    out = np.empty(flat.shape, np.uint8)
    step = 1 << 25
    for s in range(0, flat.size, step):
        out[s:s + step] = table[flat[s:s + step]]
    return out.reshape(bf16_bits.shape)


def valid_rows(plan) -> np.ndarray:
    """Flat indices d * (ep * tpr) + s of the receive rows a combine reads: rank
    d's row for slot s where d received the token (recv_valid == 1)."""
    return np.nonzero((np.asarray(plan.recv_valid) == 1).reshape(-1))[0]


def oracle_e4m3_rows_read(bf16_bits: np.ndarray, plan, table: np.ndarray) -> np.ndarray:
    """The oracle's E4M3 codes (through its table of every bf16 input) of the rows
    a combine reads; the other rows are 0 and never read."""
    H = bf16_bits.shape[-1]
    flat = bf16_bits.reshape(-1, H)
    idx = valid_rows(plan)
    out = np.zeros(flat.shape, np.uint8)
    out[idx] = table[flat[idx]]
    return out.reshape(bf16_bits.shape)


def oracle_row_quantize_read(bf16_bits: np.ndarray, plan, hidden: int):
    """oracle.quantize_e4m3_rows applied to the rows a combine reads (rows are
    independent); the other rows get codes 0 and scale 1 and are never read."""
    flat = bf16_bits.reshape(-1, hidden)
    idx = valid_rows(plan)
    codes = np.zeros(flat.shape, np.uint8)
    scales = np.ones(flat.shape[0], np.float32)
    if idx.size:
        c, sc = oracle.quantize_e4m3_rows(np.ascontiguousarray(flat[idx]), hidden)
        codes[idx] = c
        scales[idx] = sc
    return codes.reshape(bf16_bits.shape), scales.reshape(bf16_bits.shape[:-1])

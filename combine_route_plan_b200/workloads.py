"""Seeded synthetic workloads for rank-major MoE EP dispatch / combine.

This module only draws random inputs; it holds none of the dispatch / combine
arithmetic, so the CUDA path and the CPU oracle can both be fed from it.  All
draws use a torch CPU generator seeded with ``1000 + config_index``, so the
same config gives the same bytes on every machine.

The five workloads follow the shapes the pages discuss (DeepSeek-V3-like
hidden 7168, 256 experts, top_k 8; EP 8 / 16 / 64; BF16, MXFP8 and NVFP4
dispatch formats; an extra per-token payload; EPLB statistics; a rank mask):

  c1  ep 4,  E 8,   k 2, 16 tokens/rank, hidden 128 BF16          (tiny, exhaustive)
  c2  ep 8,  E 256, k 8, 128 tokens/rank, hidden 7168 BF16        (decode step)
  c3  ep 16, E 256, k 8, 512 tokens/rank, Zipf(1.2) routing,
      hidden 7168 as NVFP4 (run "nvfp4"), MXFP8 (run "mxfp8") or
      DeepSeekFp8 (run "dsfp8")                                   (quantized dispatch)
  c4  ep 8,  E 256, k 8, 4096 tokens/rank, hidden 7168 BF16, extra 64 B,
      EPLB stats, BF16 and FP8-E4M3 combine                        (prefill step)
  c5  ep 64, E 256, k 8, runtime max 64, local_num_tokens ~ U[1, 64],
      ranks 5, 17, 42 masked off                                   (wide EP)

Routing draws k distinct experts per token: uniformly (a random permutation
prefix, via the top-k of i.i.d. uniform keys) or, for c3, by Gumbel-top-k with
p(e) proportional to (e + 1)^-1.2 (popularity order = expert id).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int                    # 1-based config number; seed = 1000 + index
    ep_size: int
    num_experts: int
    top_k: int
    tokens_per_rank: int          # the step's runtime_max_tokens_per_rank
    hidden: int
    dispatch_format: str          # "bf16" | "nvfp4" | "mxfp8" | "dsfp8"
    routing: str = "uniform"      # "uniform" | "zipf"
    zipf_s: float = 1.2
    ragged_tokens: bool = False   # local_num_tokens ~ U[1, tokens_per_rank]
    extra_bytes: int = 0          # extra_payload_bytes_per_token
    eplb: bool = False
    masked_ranks: tuple = ()
    fp8_combine: bool = False     # also exercise the E4M3 combine

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def experts_per_rank(self) -> int:
        return self.num_experts // self.ep_size

    def payload_names(self) -> List[str]:
        if self.dispatch_format == "bf16":
            names = ["hidden"]
        else:
            names = ["hidden_q", "hidden_scale"]
        if self.extra_bytes:
            names.append("extra")
        names.append("topk_weights")
        return names

    def payload_row_bytes(self) -> List[int]:
        rows = []
        if self.dispatch_format == "bf16":
            rows.append(self.hidden * 2)
        elif self.dispatch_format == "nvfp4":
            rows += [self.hidden // 2, self.hidden // 16]
        elif self.dispatch_format == "mxfp8":
            rows += [self.hidden, self.hidden // 32]
        elif self.dispatch_format == "dsfp8":
            rows += [self.hidden, self.hidden // 128 * 4]
        else:
            raise ValueError(self.dispatch_format)
        if self.extra_bytes:
            rows.append(self.extra_bytes)
        rows.append(self.top_k * 4)
        return rows

    def mask_words(self) -> Optional[np.ndarray]:
        if not self.masked_ranks:
            return None
        words = np.zeros((self.ep_size + 63) // 64, np.uint64)
        for r in range(self.ep_size):
            if r not in self.masked_ranks:
                words[r // 64] |= np.uint64(1) << np.uint64(r % 64)
        return words


C1 = Workload("c1_ep4_tiny", 1, 4, 8, 2, 16, 128, "bf16")
C2 = Workload("c2_ep8_decode", 2, 8, 256, 8, 128, 7168, "bf16")
C3_NVFP4 = Workload("c3_ep16_zipf_nvfp4", 3, 16, 256, 8, 512, 7168, "nvfp4", routing="zipf")
C3_MXFP8 = Workload("c3_ep16_zipf_mxfp8", 3, 16, 256, 8, 512, 7168, "mxfp8", routing="zipf")
C3_DSFP8 = Workload("c3_ep16_zipf_dsfp8", 3, 16, 256, 8, 512, 7168, "dsfp8", routing="zipf")
C4 = Workload("c4_ep8_prefill", 4, 8, 256, 8, 4096, 7168, "bf16", extra_bytes=64,
              eplb=True, fp8_combine=True)
C5 = Workload("c5_ep64_wide_masked", 5, 64, 256, 8, 64, 7168, "bf16", ragged_tokens=True,
              masked_ranks=(5, 17, 42))

ALL = [C1, C2, C3_NVFP4, C3_MXFP8, C4, C5, C3_DSFP8]
BY_NAME = {w.name: w for w in ALL}


def scaled(w: Workload, tokens_per_rank: int, name: Optional[str] = None) -> Workload:
    """The same workload with another tokens_per_rank (for bounded samples)."""
    return dataclasses.replace(w, tokens_per_rank=tokens_per_rank,
                               name=name or f"{w.name}_tpr{tokens_per_rank}")


@dataclasses.dataclass
class Inputs:
    workload: Workload
    token_selected_experts: torch.Tensor   # int32 [ep, tpr, k]
    local_num_tokens: np.ndarray           # int32 [ep]
    payloads: List[torch.Tensor]           # each uint8 [ep, tpr, row_bytes]
    eplb_local_stats: Optional[torch.Tensor]  # int32 [ep, E]
    active_rank_mask: Optional[np.ndarray]    # uint64 words
    expert_output: Optional[torch.Tensor]     # bf16 [ep(dst), ep*tpr, hidden]


def _chunked_randn_bf16(shape, gen, chunk=1 << 26) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        flat[s:e] = torch.randn(e - s, generator=gen).to(torch.bfloat16)
    return out


def _route_ids(w: Workload, ntok: int, gen) -> torch.Tensor:
    E, k = w.num_experts, w.top_k
    out = torch.empty((ntok, k), dtype=torch.int32)
    step = 1 << 14
    if w.routing == "zipf":
        logp = -w.zipf_s * torch.log(torch.arange(1, E + 1, dtype=torch.float64))
    for s in range(0, ntok, step):
        e = min(ntok, s + step)
        u = torch.rand((e - s, E), generator=gen, dtype=torch.float64)
        if w.routing == "uniform":
            keys = u
        elif w.routing == "zipf":
            u = u.clamp_min(1e-300)
            keys = logp.unsqueeze(0) - torch.log(-torch.log(u))   # Gumbel-top-k
        else:
            raise ValueError(w.routing)
        out[s:e] = keys.topk(k, dim=1).indices.to(torch.int32)
    return out


_E2M1_GRID = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _encode_nvfp4(x: torch.Tensor):
    """[ntok, H] fp32 -> (packed E2M1 [ntok, H/2] u8, E4M3 block-16 scales [ntok, H/16] u8)."""
    ntok, H = x.shape
    blk = x.view(ntok, H // 16, 16)
    amax = blk.abs().amax(dim=2, keepdim=True).clamp_min(1e-12)
    scale = (amax / 6.0).clamp(max=448.0).to(torch.float8_e4m3fn)
    sdec = scale.to(torch.float32).clamp_min(2.0 ** -9)
    y = (blk / sdec).clamp(-6.0, 6.0)
    mag = y.abs().unsqueeze(-1)
    code = (mag - _E2M1_GRID).abs().argmin(dim=-1).to(torch.uint8)    # 0..7
    code = code | ((y < 0).to(torch.uint8) << 3)
    code = code.view(ntok, H)
    packed = code[:, 0::2] | (code[:, 1::2] << 4)
    return packed.contiguous(), scale.view(torch.uint8).view(ntok, H // 16).contiguous()


def _encode_mxfp8(x: torch.Tensor):
    """[ntok, H] fp32 -> (E4M3 elements [ntok, H] u8, UE8M0 block-32 scales [ntok, H/32] u8)."""
    ntok, H = x.shape
    blk = x.view(ntok, H // 32, 32)
    amax = blk.abs().amax(dim=2, keepdim=True).clamp_min(2.0 ** -100)
    e = torch.floor(torch.log2(amax)) - 8.0          # E4M3's largest binade is 2^8
    y = (blk / torch.exp2(e)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    scales = (e + 127.0).clamp(0, 254).to(torch.uint8).view(ntok, H // 32)
    return y.view(torch.uint8).view(ntok, H).contiguous(), scales.contiguous()


def _encode_dsfp8(x: torch.Tensor):
    """[ntok, H] fp32 -> (E4M3 elements [ntok, H] u8, fp32 block-128 scales [ntok, H/128 * 4] u8).

    DeepSeek-style FP8: one fp32 scale per 128 consecutive elements, amax / 448."""
    ntok, H = x.shape
    blk = x.view(ntok, H // 128, 128)
    scale = (blk.abs().amax(dim=2, keepdim=True) / 448.0).clamp_min(1e-30)
    y = (blk / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    scales = scale.to(torch.float32).view(ntok, H // 128).contiguous()
    return y.view(torch.uint8).view(ntok, H).contiguous(), scales.view(torch.uint8)


def make_inputs(w: Workload, with_expert_output: bool = True) -> Inputs:
    """Draw every input of one step of workload ``w``."""
    gen = torch.Generator().manual_seed(w.seed)
    ep, tpr, k, H = w.ep_size, w.tokens_per_rank, w.top_k, w.hidden
    ntok = ep * tpr

    ids = _route_ids(w, ntok, gen).view(ep, tpr, k).contiguous()
    if w.ragged_tokens:
        n = torch.randint(1, tpr + 1, (ep,), generator=gen).numpy().astype(np.int32)
    else:
        n = np.full(ep, tpr, np.int32)

    payloads: List[torch.Tensor] = []
    hid = torch.randn((ntok, H), generator=gen) if w.dispatch_format != "bf16" else None
    if w.dispatch_format == "bf16":
        h = _chunked_randn_bf16((ntok, H), gen)
        payloads.append(h.view(torch.uint8).view(ep, tpr, 2 * H))
    elif w.dispatch_format == "nvfp4":
        q, s = _encode_nvfp4(hid)
        payloads += [q.view(ep, tpr, -1), s.view(ep, tpr, -1)]
    elif w.dispatch_format == "mxfp8":
        q, s = _encode_mxfp8(hid)
        payloads += [q.view(ep, tpr, -1), s.view(ep, tpr, -1)]
    elif w.dispatch_format == "dsfp8":
        q, s = _encode_dsfp8(hid)
        payloads += [q.view(ep, tpr, -1), s.view(ep, tpr, -1)]
    del hid
    if w.extra_bytes:
        extra = torch.randint(0, 256, (ntok, w.extra_bytes), generator=gen, dtype=torch.int32)
        payloads.append(extra.to(torch.uint8).view(ep, tpr, w.extra_bytes))
    logits = torch.randn((ntok, k), generator=gen)
    weights = torch.softmax(logits, dim=1).to(torch.float32).contiguous()
    payloads.append(weights.view(torch.uint8).view(ep, tpr, 4 * k))

    stats = None
    if w.eplb:
        stats = torch.randint(0, 4097, (ep, w.num_experts), generator=gen, dtype=torch.int32)

    xo = None
    if with_expert_output:
        xo = _chunked_randn_bf16((ep, ep * tpr, H), gen)

    for p, rb in zip(payloads, w.payload_row_bytes()):
        assert p.shape == (ep, tpr, rb) and p.dtype == torch.uint8, (p.shape, rb)
    return Inputs(w, ids, n, [p.contiguous() for p in payloads], stats, w.mask_words(), xo)


def random_bytes_payload(ep: int, tpr: int, row_bytes: int, seed: int) -> torch.Tensor:
    """Arbitrary bit patterns (NaNs, -0, 0xFFFF words, ...) for byte-exactness checks."""
    gen = torch.Generator().manual_seed(seed)
    return torch.randint(0, 256, (ep, tpr, row_bytes), generator=gen,
                         dtype=torch.int32).to(torch.uint8)


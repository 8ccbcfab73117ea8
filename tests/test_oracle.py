"""Pins of the CPU oracle against facts the pages and the mathematics fix.

These run without a GPU.  Each test checks the oracle against something other
than itself: a hand-derived example, brute-force enumeration, a library
conversion routine, a closed form, an invariant, or a special case.
"""
import json
import math
import os
from itertools import permutations

import numpy as np
import pytest
import torch

from combine_route_plan_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(values):
    return torch.tensor(values, dtype=torch.float32).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def bits_to_f32(bits_u16):
    return (np.asarray(bits_u16, np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------- #
# Number formats
# --------------------------------------------------------------------------- #

def _special_f32():
    vals = [0.0, -0.0, 1.0, -1.0, 3.0e38, -3.4e38, float("inf"), float("-inf"),
            2.0 ** -126, 2.0 ** -130, -(2.0 ** -149), 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8,
            65504.0, 3.3895313892515355e38]
    # exact ties on the 16 dropped bits, with even and odd kept halves
    for upper in (0x3F80, 0x3F81, 0x4049, 0x7F7F, 0x0001, 0x8001):
        for lower in (0x7FFF, 0x8000, 0x8001):
            vals.append(np.array([(upper << 16) | lower], np.uint32).view(np.float32)[0])
    return np.array(vals, np.float32)


def test_bf16_round_matches_torch(oracle_mod):
    """fp32 -> bf16 nearest-even equals torch's conversion (a library routine)."""
    rng = np.random.default_rng(7)
    x = np.concatenate([_special_f32(),
                        rng.standard_normal(4000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-39).astype(np.float32),
                        rng.integers(0, 2 ** 32, 4000, dtype=np.uint64).astype(np.uint32)
                        .view(np.float32)])
    x = x[~np.isnan(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.bf16_from_f32(v) for v in x], np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(x[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]
    # NaN stays NaN
    assert math.isnan(oracle_mod.bf16_to_f32(oracle_mod.bf16_from_f32(float("nan"))))


def test_bf16_widen_is_exact(oracle_mod):
    for b in [0x0000, 0x8000, 0x3F80, 0xBF80, 0x0001, 0x7F7F, 0x7F80, 0xFF80]:
        ref = float(torch.tensor([b], dtype=torch.int16 if b < 0x8000 else torch.int32)
                    .to(torch.int16).view(torch.bfloat16).float())
        assert oracle_mod.bf16_to_f32(b) == ref or (math.isnan(ref))


def test_e4m3_decode_all_codes_match_torch(oracle_mod):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = np.array([oracle_mod.e4m3_to_f32(c) for c in range(256)], np.float32)
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(np.signbit(got[~both_nan]), np.signbit(ref[~both_nan]))
    assert np.array_equal(got[~both_nan], ref[~both_nan])
    assert set(np.nonzero(np.isnan(got))[0].tolist()) == {0x7F, 0xFF}
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0


def _e4m3_bruteforce(x: float) -> int:
    """Nearest finite E4M3 by exhaustive search; ties to the even code; saturating."""
    if math.isnan(x):
        return 0x7F
    sign = 0x80 if math.copysign(1.0, x) < 0 else 0
    a = min(abs(x), 448.0)
    best, best_d = None, None
    for c in range(0x7F):                   # 0x00..0x7E: all finite non-negative codes
        e, m = c >> 3, c & 7
        v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        d = abs(v - a)
        if best is None or d < best_d or (d == best_d and (c & 1) == 0):
            best, best_d = c, d
    return sign | best


def test_e4m3_encode_all_bf16_bruteforce(oracle_mod):
    """Every bf16 input: oracle encoder == exhaustive nearest search (and torch in range)."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = bits_to_f32(allbits)
    got = oracle_mod.quantize_e4m3(allbits)
    finite = ~np.isnan(f)
    # brute force on a stride of patterns covering every exponent, plus all near-saturation
    idx = np.concatenate([np.arange(0, 65536, 7), np.nonzero(np.abs(f) > 200)[0]])
    for i in np.unique(idx):
        if not finite[i]:
            assert got[i] in (0x7F,), (hex(allbits[i]), got[i])
            continue
        assert got[i] == _e4m3_bruteforce(float(f[i])), (f[i], hex(got[i]))
    inrange = finite & (np.abs(f) <= 448.0)
    ref = torch.from_numpy(f[inrange]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got[inrange], ref)
    # saturation (the satfinite reading): beyond 448, including infinities
    for v, code in [(449.0, 0x7E), (1e30, 0x7E), (float("inf"), 0x7E), (-float("inf"), 0xFE)]:
        assert oracle_mod.e4m3_from_f32(v) == code


# --------------------------------------------------------------------------- #
# Routing
# --------------------------------------------------------------------------- #

def _load_golden():
    with open(os.path.join(GOLDEN, "route_hand_example.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("case", ["no_mask", "mask_rank2_off"])
def test_route_hand_example(oracle_mod, case):
    g = _load_golden()
    ep, E, k, tpr = g["ep_size"], g["num_experts"], g["top_k"], g["tokens_per_rank"]
    exp = g[case]
    mask = np.array(exp["active_rank_mask"], np.uint64) if "active_rank_mask" in exp else None
    plan = oracle_mod.route(ep, E, k, tpr, np.array(g["token_selected_experts"], np.int32),
                            np.array(g["local_num_tokens"], np.int32), mask)
    assert plan.num_dst.tolist() == exp["num_dst"]
    assert plan.dst_ranks.tolist() == exp["dst_ranks"]
    assert plan.send_counts.tolist() == exp["send_counts"]
    ids = np.array(g["token_selected_experts"], np.int32).reshape(ep * tpr, k)
    for d, slots in enumerate(exp["valid_slots_per_dst"]):
        if slots is None:   # masked-off destination: untouched
            assert np.all(plan.recv_valid[d] == 0xAB)
            assert np.all(plan.recv_topk_ids[d] == -0x54545455)
            continue
        assert np.nonzero(plan.recv_valid[d] == 1)[0].tolist() == slots
        assert np.all((plan.recv_valid[d] == 0) | (plan.recv_valid[d] == 1))
        for s in range(ep * tpr):
            want = ids[s] if s in slots else np.full(k, E)
            assert plan.recv_topk_ids[d, s].tolist() == list(want)


def test_combine_hand_example(oracle_mod):
    g = _load_golden()
    ep, E, k, tpr, H = g["ep_size"], g["num_experts"], g["top_k"], g["tokens_per_rank"], \
        g["combine_hidden"]
    plan = oracle_mod.route(ep, E, k, tpr, np.array(g["token_selected_experts"], np.int32),
                            np.array(g["local_num_tokens"], np.int32))
    x = np.zeros((ep, ep * tpr, H), np.float32)
    for d in range(ep):
        for s in range(ep * tpr):
            x[d, s] = [2.0 ** d, -float(s)]
    x[:, 0, 1] = -0.0
    out = oracle_mod.combine(plan, bf16_bits(x.ravel()).reshape(x.shape), H)
    rows = g["combine_no_mask_expected"]["rows"]
    for r in range(ep):
        for t in range(tpr):
            if rows[r][t] is None:
                assert np.all(out[r, t] == 0xEEEE)
            else:
                assert out[r, t].tolist() == bf16_bits(rows[r][t]).tolist(), (r, t)


OWNER_E8_EP4 = [0, 0, 1, 1, 2, 2, 3, 3]   # written out by hand: e // (8 / 4)


def test_route_bruteforce_all_pairs_all_masks(oracle_mod):
    """ep 4, E 8, k 2: every ordered expert pair, every rank mask, every source rank."""
    pairs = list(permutations(range(8), 2))           # 56 ordered distinct pairs
    ep, E, k = 4, 8, 2
    tpr = len(pairs)
    ids = np.array([pairs for _ in range(ep)], np.int32)   # [ep, 56, 2]
    n = np.full(ep, tpr, np.int32)
    for m in range(1, 16):
        live = [bool(m >> r & 1) for r in range(ep)]
        plan = oracle_mod.route(ep, E, k, tpr, ids, n, np.array([m], np.uint64))
        for r in range(ep):
            for t, (a, b) in enumerate(pairs):
                if not live[r]:
                    assert plan.num_dst[r, t] == -1
                    continue
                want = sorted({OWNER_E8_EP4[a], OWNER_E8_EP4[b]} & {d for d in range(ep) if live[d]})
                assert plan.num_dst[r, t] == len(want)
                assert plan.dst_ranks[r, t, :len(want)].tolist() == want
                for d in range(ep):
                    if live[d]:
                        assert plan.recv_valid[d, r * tpr + t] == (d in want)
        # counts = per (src, dst) number of tokens
        for r in range(ep):
            for d in range(ep):
                want = 0
                if live[r] and live[d]:
                    want = sum(d in {OWNER_E8_EP4[a], OWNER_E8_EP4[b]} for a, b in pairs)
                assert plan.send_counts[r, d] == want


def test_out_of_range_ids_are_not_routed(oracle_mod):
    ids = np.array([[[-1, 8], [9, 3], [100, -7]]], np.int32).repeat(2, 0)
    plan = oracle_mod.route(2, 8, 2, 3, ids, np.array([3, 3], np.int32))
    assert plan.num_dst[0].tolist() == [0, 1, 0]
    assert plan.dst_ranks[0, 1].tolist() == [0, -1]


def _slot_payload(ep, tpr):
    """8-byte debug payload holding (src rank, token) as two int32."""
    p = np.zeros((ep, tpr, 2), np.int32)
    p[:, :, 0] = np.arange(ep)[:, None]
    p[:, :, 1] = np.arange(tpr)[None, :]
    return p


@pytest.mark.parametrize("w", [W.C1, W.C2, W.C5], ids=lambda w: w.name)
def test_dispatch_slot_index_and_once_per_rank(oracle_mod, w):
    """Each valid slot s of rank d holds the (src, t) with s = src*tpr + t; a
    token appears once per distinct live owning rank; invalid rows keep the canary."""
    x = W.make_inputs(w, with_expert_output=False)
    ep, tpr, k, E = w.ep_size, w.tokens_per_rank, w.top_k, w.num_experts
    ids = x.token_selected_experts.numpy()
    plan = oracle_mod.route(ep, E, k, tpr, ids, x.local_num_tokens, x.active_rank_mask)
    recv = oracle_mod.dispatch_payload(plan, _slot_payload(ep, tpr)).view(np.int32) \
        .reshape(ep, ep * tpr, 2)
    live = [True] * ep if x.active_rank_mask is None else \
        [bool(int(x.active_rank_mask[r // 64]) >> (r % 64) & 1) for r in range(ep)]
    epr = E // ep
    for d in range(ep):
        if not live[d]:
            assert np.all(plan.recv_valid[d] == 0xAB)
            continue
        for s in range(ep * tpr):
            r, t = divmod(s, tpr)
            owners = {int(e) // epr for e in ids[r, t] if 0 <= e < E}
            is_valid = live[r] and t < x.local_num_tokens[r] and d in owners
            assert plan.recv_valid[d, s] == is_valid
            if is_valid:
                assert recv[d, s].tolist() == [r, t]
                assert plan.recv_topk_ids[d, s].tolist() == ids[r, t].tolist()
            else:
                assert np.all(recv[d, s].view(np.uint8) == 0xCD)
                assert np.all(plan.recv_topk_ids[d, s] == E)
    # sum over destinations of valid == number of distinct live owners; counts agree
    nd = np.where(plan.num_dst < 0, 0, plan.num_dst)
    per_token = sum(plan.recv_valid[d].reshape(ep, tpr).astype(np.int64)
                    for d in range(ep) if live[d])
    assert np.array_equal(per_token, nd)
    assert np.array_equal(plan.send_counts.sum(1), nd.sum(1))


@pytest.mark.parametrize("w", [W.C1, W.C2, W.C5], ids=lambda w: w.name)
def test_combine_of_ones_counts_ranks(oracle_mod, w):
    """Dispatch all-ones rows, every rank returns 1.0: combine yields D(t) exactly."""
    ep, tpr, k, E, H = w.ep_size, w.tokens_per_rank, w.top_k, w.num_experts, 64
    x = W.make_inputs(w, with_expert_output=False)
    plan = oracle_mod.route(ep, E, k, tpr, x.token_selected_experts.numpy(),
                            x.local_num_tokens, x.active_rank_mask)
    ones = np.full((1, 1, H), 0x3F80, np.uint16).repeat(ep, 0).repeat(tpr, 1)
    recv = oracle_mod.dispatch_payload(plan, ones, recv_init=np.zeros(
        (ep, ep * tpr, 2 * H), np.uint8)).view(np.uint16).reshape(ep, ep * tpr, H)
    out = oracle_mod.combine(plan, recv, H)
    for r in range(ep):
        for t in range(tpr):
            nd = plan.num_dst[r, t]
            if nd < 0:
                assert np.all(out[r, t] == 0xEEEE)
            else:
                assert np.all(bits_to_f32(out[r, t]) == float(nd))


def test_ep1_is_identity(oracle_mod):
    """ep_size 1: dispatch is the identity copy and combine returns the row itself
    (bf16 -> fp32 -> +0 add -> bf16 is exact, -0 becomes +0)."""
    tpr, k, E, H = 37, 4, 8, 48
    rng = np.random.default_rng(3)
    ids = rng.integers(0, E, (1, tpr, k)).astype(np.int32)
    plan = oracle_mod.route(1, E, k, tpr, ids, np.array([tpr], np.int32))
    assert np.all(plan.num_dst == 1)
    data = rng.integers(0, 256, (1, tpr, 100)).astype(np.uint8)
    assert np.array_equal(oracle_mod.dispatch_payload(plan, data)[0], data[0])
    xb = bf16_bits(rng.standard_normal(tpr * H).astype(np.float32)).reshape(1, tpr, H)
    xb[0, 0, :4] = [0x8000, 0x0001, 0x7F7F, 0xFF7F]     # -0, min subnormal, +-max finite
    out = oracle_mod.combine(plan, xb, H)
    want = xb.copy()
    want[0, 0, 0] = 0x0000
    assert np.array_equal(out.reshape(1, tpr, H), want)


def test_all_experts_on_one_rank_is_identity(oracle_mod):
    ep, E, k, tpr, H = 4, 16, 4, 9, 32
    rng = np.random.default_rng(5)
    ids = np.zeros((ep, tpr, k), np.int32)
    for r in range(ep):
        for t in range(tpr):
            owner = rng.integers(0, ep)
            ids[r, t] = rng.choice(np.arange(owner * 4, owner * 4 + 4), k, replace=False)
    plan = oracle_mod.route(ep, E, k, tpr, ids, np.full(ep, tpr, np.int32))
    assert np.all(plan.num_dst == 1)
    x = bf16_bits(rng.standard_normal(ep * ep * tpr * H).astype(np.float32)) \
        .reshape(ep, ep * tpr, H)
    out = oracle_mod.combine(plan, x, H)
    for r in range(ep):
        for t in range(tpr):
            d = ids[r, t, 0] // 4
            assert np.array_equal(out[r, t], x[d, r * tpr + t])


# --------------------------------------------------------------------------- #
# Combine arithmetic: order, accumulator width, subnormals
# --------------------------------------------------------------------------- #

def _three_rank_plan(oracle_mod):
    # ep 3, E 3: token (r0, t0) selects experts 2, 0, 1 -> ranks {0, 1, 2}
    ids = np.array([[[2, 0, 1]], [[0, 0, 0]], [[0, 0, 0]]], np.int32)
    return oracle_mod.route(3, 3, 3, 1, ids, np.array([1, 0, 0], np.int32))


def _combine_three(oracle_mod, vals):
    plan = _three_rank_plan(oracle_mod)
    x = np.zeros((3, 3, 1), np.uint16)
    for d, v in enumerate(vals):
        x[d, 0, 0] = bf16_bits([v])[0]
    return bits_to_f32(oracle_mod.combine(plan, x, 1)[0, 0])[0]


def test_combine_adds_in_ascending_rank_order(oracle_mod):
    # ascending: (1 + 2^24) rounds to 2^24 (tie to even), then - 2^24 = 0
    # descending would give (-2^24 + 2^24) + 1 = 1
    assert _combine_three(oracle_mod, [1.0, 2.0 ** 24, -(2.0 ** 24)]) == 0.0


def test_combine_accumulates_in_fp32(oracle_mod):
    # fp32: 2^24 + 1 -> 2^24, then -2^24 -> 0.  An fp64 accumulator would give 1.
    assert _combine_three(oracle_mod, [2.0 ** 24, 1.0, -(2.0 ** 24)]) == 0.0
    # bf16 accumulation would lose 2^-8 twice; fp32 keeps 1 + 2^-7 (a bf16 value)
    assert _combine_three(oracle_mod, [1.0, 2.0 ** -8, 2.0 ** -8]) == 1.0 + 2.0 ** -7


def test_combine_keeps_subnormals(oracle_mod):
    # 2^-130 + 2^-130 + 0 = 2^-129 (flush-to-zero would give 0)
    assert _combine_three(oracle_mod, [2.0 ** -130, 2.0 ** -130, 0.0]) == 2.0 ** -129


def test_combine_rounds_once_nearest_even(oracle_mod):
    # 1 + 2^-8 is a tie between bf16 neighbours 1 and 1 + 2^-7: even -> 1.0;
    # 1 + 3*2^-8 ties between 1 + 2^-7 and 1 + 2^-6: even -> 1 + 2^-6
    assert _combine_three(oracle_mod, [1.0, 2.0 ** -8, 0.0]) == 1.0
    assert _combine_three(oracle_mod, [1.0, 2.0 ** -8, 2.0 ** -7]) == 1.0 + 2.0 ** -6


def test_combine_empty_set_is_positive_zero(oracle_mod):
    plan = oracle_mod.route(2, 4, 1, 1, np.array([[[3]], [[0]]], np.int32),
                            np.array([1, 1], np.int32), np.array([1], np.uint64))
    assert plan.num_dst[0, 0] == 0          # expert 3 -> rank 1, masked off
    out = oracle_mod.combine(plan, np.full((2, 2, 4), 0x7FC0, np.uint16), 4)
    assert np.all(out[0, 0] == 0x0000)
    assert np.all(out[1, 0] == 0xEEEE)      # masked-off source: untouched


# --------------------------------------------------------------------------- #
# Dense all-gather / reduce-scatter restatement
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("w", [W.C1, W.C2], ids=lambda w: w.name)
def test_matches_dense_allgather_reduce_scatter(oracle_mod, w):
    """vllm.distributed.device_communicators.all2all, AgRsAll2AllManager: dispatch as
    "all-gather every rank's rows, keep the owned ones", combine as "reduce-scatter of
    zero-padded rows".  Written here with another loop nest (rank d outermost,
    vectorised over tokens); it must agree bit for bit."""
    x = W.make_inputs(w)
    ep, tpr, k, E, H = w.ep_size, w.tokens_per_rank, w.top_k, w.num_experts, w.hidden
    ids = x.token_selected_experts.numpy()
    plan = oracle_mod.route(ep, E, k, tpr, ids, x.local_num_tokens)
    hid = x.payloads[0].numpy()
    recv = oracle_mod.dispatch_payload(plan, hid)
    gathered = hid.reshape(ep * tpr, -1)                       # all-gather
    owners = np.where((ids >= 0) & (ids < E), ids // (E // ep), -1).reshape(ep * tpr, k)
    exists = (np.arange(tpr)[None, :] < x.local_num_tokens[:, None]).reshape(-1)
    xo = x.expert_output.view(torch.int16).numpy().view(np.uint16)
    acc = np.zeros((ep * tpr, H), np.float32)
    for d in range(ep):
        keep = exists & (owners == d).any(axis=1)
        want = np.where(keep[:, None], gathered, np.uint8(0xCD))
        assert np.array_equal(recv[d], want)
        xd = np.where(keep[:, None], bits_to_f32(xo[d]), np.float32(0.0))
        acc = (acc + xd).astype(np.float32)                     # reduce over d, ascending
    dense = torch.from_numpy(acc).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out = oracle_mod.combine(plan, xo, H).reshape(ep * tpr, H)
    assert np.array_equal(out[exists], dense[exists])


# --------------------------------------------------------------------------- #
# EPLB gather and statistics of the routing
# --------------------------------------------------------------------------- #

def test_eplb_gather_rows_and_mask(oracle_mod):
    ep, ne = 5, 12
    stats = np.arange(ep * ne, dtype=np.int32).reshape(ep, ne) * 3 + 1
    g = oracle_mod.eplb_gather(ep, stats)
    for d in range(ep):
        assert np.array_equal(g[d], stats)          # row r = rank r's statistics
    mask = np.array([0b10111], np.uint64)           # rank 3 off
    g = oracle_mod.eplb_gather(ep, stats, mask)
    assert np.all(g[3] == -0x32323233)             # masked destination untouched
    for d in (0, 1, 2, 4):
        assert np.all(g[d, 3] == 0)
        for r in (0, 1, 2, 4):
            assert np.array_equal(g[d, r], stats[r])


def _dist_moments(ep, E, k, live):
    """Mean and variance of D (number of distinct live owners of k distinct uniform
    experts), by inclusion-exclusion over ranks."""
    epr = E // ep
    c = math.comb(E, k)
    p1 = 1 - math.comb(E - epr, k) / c
    p2 = 1 - 2 * math.comb(E - epr, k) / c + math.comb(E - 2 * epr, k) / c
    mean = live * p1
    var = live * p1 * (1 - p1) + live * (live - 1) * (p2 - p1 * p1)
    return mean, var


@pytest.mark.parametrize("w", [W.C2, W.C5, W.scaled(W.C4, 256)], ids=lambda w: w.name)
def test_mean_distinct_ranks_closed_form(oracle_mod, w):
    x = W.make_inputs(w, with_expert_output=False)
    ep, tpr = w.ep_size, w.tokens_per_rank
    plan = oracle_mod.route(ep, w.num_experts, w.top_k, tpr, x.token_selected_experts.numpy(),
                            x.local_num_tokens, x.active_rank_mask)
    live_src = [r for r in range(ep) if r not in w.masked_ranks]
    nd = np.concatenate([plan.num_dst[r, :x.local_num_tokens[r]] for r in live_src])
    mean, var = _dist_moments(ep, w.num_experts, w.top_k, ep - len(w.masked_ranks))
    assert abs(nd.mean() - mean) < 4 * math.sqrt(var / nd.size), (nd.mean(), mean)
    if w is W.C2:
        assert abs(mean - 5.295) < 1e-3          # the 5.295 quoted for EP 8, E 256, k 8


# --------------------------------------------------------------------------- #
# Weighted reduction over local experts (the combine's input) and its combine
# --------------------------------------------------------------------------- #

def test_expert_reduce_uses_one_rounding_per_term(oracle_mod):
    """Two slots owned by the same rank, worked by hand: with w0 = -(1 + 2^-7 +
    2^-20), y0 = 1, w1 = 1 + 2^-20, y1 = 1 + 2^-7 the exact sum is 2^-27.
    fmaf keeps it (the product w1*y1 = 1 + 2^-7 + 2^-20 + 2^-27 is never
    rounded on its own); a rounded product followed by an add would give 0."""
    ids = np.array([[[0, 1]], [[2, 3]]], np.int32)          # ep 2, E 4: experts 0, 1 -> rank 0
    plan = oracle_mod.route(2, 4, 2, 1, ids, np.array([1, 0], np.int32))
    w = np.zeros((2, 1, 2), np.float32)
    w[0, 0] = [-(1 + 2.0 ** -7 + 2.0 ** -20), 1 + 2.0 ** -20]
    y = np.zeros((2, 1, 2, 1), np.uint16)
    y[0, 0, :, 0] = bf16_bits([1.0, 1 + 2.0 ** -7])
    z = oracle_mod.expert_reduce(plan, 4, ids, w, y, 1)
    assert bits_to_f32(z[0, 0])[0] == 2.0 ** -27
    out = oracle_mod.combine_experts(plan, 4, ids, w, y, 1)
    assert bits_to_f32(out[0, 0])[0] == 2.0 ** -27


@pytest.mark.parametrize("w", [W.C1, W.C2, W.C5], ids=lambda w: w.name)
def test_combine_experts_matches_vectorised_restatement(oracle_mod, w):
    """Power-of-two weights make every product exact, so fmaf equals a plain
    multiply and add; the reduction and the combine are then restated with
    numpy fp32 arrays, looping over destination rank and slot and vectorising
    over tokens and columns."""
    H = 64
    x = W.make_inputs(w, with_expert_output=False)
    ep, tpr, k, E = w.ep_size, w.tokens_per_rank, w.top_k, w.num_experts
    rng = np.random.default_rng(11)
    ids = x.token_selected_experts.numpy()
    wts = (2.0 ** rng.integers(-3, 4, (ep, tpr, k))).astype(np.float32)
    wts *= np.where(rng.random((ep, tpr, k)) < 0.3, -1, 1).astype(np.float32)
    y = bf16_bits(rng.standard_normal(ep * tpr * k * H).astype(np.float32)).reshape(ep, tpr, k, H)
    plan = oracle_mod.route(ep, E, k, tpr, ids, x.local_num_tokens, x.active_rank_mask)
    got = oracle_mod.combine_experts(plan, E, ids, wts, y, H).reshape(ep * tpr, H)

    live = np.ones(ep, bool)
    for r in w.masked_ranks:
        live[r] = False
    owner = np.where((ids >= 0) & (ids < E), ids // (E // ep), -1).reshape(ep * tpr, k)
    exists = ((np.arange(tpr)[None, :] < x.local_num_tokens[:, None]) & live[:, None]).reshape(-1)
    yf = bits_to_f32(y.reshape(ep * tpr, k, H))
    wf = wts.reshape(ep * tpr, k)
    acc = np.zeros((ep * tpr, H), np.float32)
    for d in range(ep):
        if not live[d]:
            continue
        z = np.zeros((ep * tpr, H), np.float32)
        for j in range(k):
            sel = (owner[:, j] == d)[:, None]
            z = np.where(sel, (z + wf[:, j:j + 1] * yf[:, j, :]).astype(np.float32), z)
        zb = torch.from_numpy(z).to(torch.bfloat16).float().numpy()
        has = (owner == d).any(axis=1)[:, None]
        acc = np.where(has, (acc + zb).astype(np.float32), acc)
    want = torch.from_numpy(acc).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got[exists], want[exists])
    assert np.all(got[~exists] == 0xEEEE)


def test_expert_reduce_single_slot_is_the_weighted_row(oracle_mod):
    """top_k 1: every token's only destination gets bf16(w * y)."""
    ep, E, tpr, H = 4, 8, 20, 16
    rng = np.random.default_rng(2)
    ids = rng.integers(0, E, (ep, tpr, 1)).astype(np.int32)
    wts = rng.standard_normal((ep, tpr, 1)).astype(np.float32)
    y = bf16_bits(rng.standard_normal(ep * tpr * H).astype(np.float32)).reshape(ep, tpr, 1, H)
    plan = oracle_mod.route(ep, E, 1, tpr, ids, np.full(ep, tpr, np.int32))
    z = oracle_mod.expert_reduce(plan, E, ids, wts, y, H)
    for r in range(ep):
        for t in range(tpr):
            d = ids[r, t, 0] // 2
            # the fp64 product is exact; one fmaf onto +0 rounds it once to fp32,
            # then the row is rounded to bf16
            prod = wts[r, t, 0].astype(np.float64) * bits_to_f32(y[r, t, 0]).astype(np.float64)
            want = torch.from_numpy(prod.astype(np.float32)).to(torch.bfloat16) \
                .view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(z[d, r * tpr + t], want)


# --------------------------------------------------------------------------- #
# FP8 combine with one scale per row
# --------------------------------------------------------------------------- #

def test_row_quantize_with_amax_448_is_plain_e4m3(oracle_mod):
    """amax = 448 gives scale = inv = 1: the codes are plain E4M3 (torch's
    float8_e4m3fn conversion in range)."""
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((6, 64)) * 40).clip(-447, 447).astype(np.float32)
    x[:, 3] = 448.0
    xb = bf16_bits(x.ravel()).reshape(x.shape)
    codes, scales = oracle_mod.quantize_e4m3_rows(xb, 64)
    assert np.all(scales == 1.0)
    ref = torch.from_numpy(bits_to_f32(xb)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_row_quantize_is_invariant_to_powers_of_two(oracle_mod):
    rng = np.random.default_rng(6)
    x = bf16_bits(rng.standard_normal(8 * 96).astype(np.float32)).reshape(8, 96)
    c0, s0 = oracle_mod.quantize_e4m3_rows(x, 96)
    for m in (-20, -3, 5, 30):
        xm = bf16_bits((bits_to_f32(x) * np.float32(2.0 ** m)).ravel()).reshape(x.shape)
        cm, sm = oracle_mod.quantize_e4m3_rows(xm, 96)
        assert np.array_equal(cm, c0)
        assert np.all(sm == s0 * np.float32(2.0 ** m))


def test_row_quantize_error_bound_and_zero_rows(oracle_mod):
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((20, 128)) * rng.lognormal(0, 3, (20, 1))).astype(np.float32)
    x[5] = 0.0
    xb = bf16_bits(x.ravel()).reshape(x.shape)
    codes, scales = oracle_mod.quantize_e4m3_rows(xb, 128)
    assert scales[5] == 1.0 and np.all(codes[5] == 0)
    xf = bits_to_f32(xb).astype(np.float64)
    dec = np.vectorize(oracle_mod.e4m3_to_f32)(codes).astype(np.float64) * scales[:, None]
    # 3 mantissa bits: half an ulp is 2^-4 relative for normals; subnormal step 2^-9
    bound = np.maximum(2.0 ** -4 * np.abs(xf), 2.0 ** -10 * scales[:, None]) * (1 + 2.0 ** -20)
    assert np.all(np.abs(dec - xf) <= bound)


def test_combine_scaled_unit_scales_equal_plain_fp8(oracle_mod):
    w = W.C2
    x = W.make_inputs(w)
    plan = oracle_mod.route(w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank,
                            x.token_selected_experts.numpy(), x.local_num_tokens)
    q = oracle_mod.quantize_e4m3(x.expert_output.view(torch.int16).numpy().view(np.uint16))
    ones = np.ones((w.ep_size, w.ep_size * w.tokens_per_rank), np.float32)
    a = oracle_mod.combine_scaled(plan, q, ones, w.hidden)
    b = oracle_mod.combine(plan, q, w.hidden, input_is_e4m3=True)
    assert np.array_equal(a, b)


def test_combine_scaled_hand_example(oracle_mod):
    # token (0, 0) -> ranks {0, 1}; codes 1.0 (0x38) with scales 0.5 and 2: 0.5 + 2 = 2.5
    ids = np.array([[[0, 2]], [[0, 0]]], np.int32)
    plan = oracle_mod.route(2, 4, 2, 1, ids, np.array([1, 0], np.int32))
    codes = np.zeros((2, 2, 4), np.uint8)
    codes[0, 0, :] = 0x38
    codes[1, 0, :] = 0x38
    sc = np.array([[0.5, 1.0], [2.0, 1.0]], np.float32)
    out = oracle_mod.combine_scaled(plan, codes, sc, 4)
    assert np.all(bits_to_f32(out[0, 0]) == 2.5)


def test_combine_scaled_uses_fused_multiply_add(oracle_mod):
    """Rank 0's row: code -1.875 (0xBF) with scale 1; rank 1's row: 1.875 (0x3F)
    with scale 1 + 2^-23.  fmaf(1.875, 1 + 2^-23, -1.875) is exactly
    1.875 * 2^-23; rounding the product first would give 2^-22."""
    ids = np.array([[[0, 2]], [[0, 0]]], np.int32)
    plan = oracle_mod.route(2, 4, 2, 1, ids, np.array([1, 0], np.int32))
    codes = np.zeros((2, 2, 1), np.uint8)
    codes[0, 0, 0] = 0xBF
    codes[1, 0, 0] = 0x3F
    sc = np.array([[1.0, 1.0], [1.0 + 2.0 ** -23, 1.0]], np.float32)
    out = oracle_mod.combine_scaled(plan, codes, sc, 1)
    assert bits_to_f32(out[0, 0])[0] == 1.875 * 2.0 ** -23


# --------------------------------------------------------------------------- #
# Dense variant: all-gather dispatch, reduce-scatter combine
# --------------------------------------------------------------------------- #

def test_allgather_equals_dispatch_when_every_rank_is_an_owner(oracle_mod):
    """With top_k = ep_size and one expert of every rank per token, the
    rank-major dispatch sends each token to every rank: it must equal the
    all-gather (two different definitions of the same movement)."""
    ep, E, tpr, rb = 4, 16, 9, 24
    rng = np.random.default_rng(12)
    ids = np.zeros((ep, tpr, ep), np.int32)
    for r in range(ep):
        for t in range(tpr):
            ids[r, t] = rng.permutation([d * 4 + rng.integers(0, 4) for d in range(ep)])
    n = np.array([9, 3, 0, 7], np.int32)
    data = rng.integers(0, 256, (ep, tpr, rb)).astype(np.uint8)
    plan = oracle_mod.route(ep, E, ep, tpr, ids, n)
    assert np.all(plan.num_dst[plan.num_dst >= 0] == ep)
    assert np.array_equal(oracle_mod.dispatch_payload(plan, data),
                          oracle_mod.allgather(ep, tpr, n, data))
    mask = np.array([0b1011], np.uint64)
    plan = oracle_mod.route(ep, E, ep, tpr, ids, n, mask)
    assert np.array_equal(oracle_mod.dispatch_payload(plan, data),
                          oracle_mod.allgather(ep, tpr, n, data, mask))


@pytest.mark.parametrize("w", [W.C1, W.C5], ids=lambda w: w.name)
def test_reduce_scatter_equals_combine_of_zero_padded_rows(oracle_mod, w):
    """The reduce-scatter of rows that are +0.0 wherever the rank-major plan
    sends nothing equals the combine (adding +0.0 to an fp32 sum that is never
    -0.0 changes nothing)."""
    x = W.make_inputs(w)
    ep, tpr, H = w.ep_size, w.tokens_per_rank, w.hidden
    plan = oracle_mod.route(ep, w.num_experts, w.top_k, tpr, x.token_selected_experts.numpy(),
                            x.local_num_tokens, x.active_rank_mask)
    xo = x.expert_output.view(torch.int16).numpy().view(np.uint16).copy()
    for d in range(ep):
        if d in w.masked_ranks:
            continue
        xo[d][plan.recv_valid[d] != 1] = 0
    a = oracle_mod.reduce_scatter(ep, tpr, H, x.local_num_tokens, xo, x.active_rank_mask)
    b = oracle_mod.combine(plan, xo, H)
    assert np.array_equal(a, b)


def test_reduce_scatter_hand_example(oracle_mod):
    # 3 ranks, 1 token each, rank 1 masked off: out[r] = x[0][r] + x[2][r]
    x = np.zeros((3, 3, 2), np.float32)
    for d in range(3):
        for s in range(3):
            x[d, s] = [10.0 ** d, s + 0.5]
    xb = bf16_bits(x.ravel()).reshape(x.shape)
    out = oracle_mod.reduce_scatter(3, 1, 2, np.array([1, 1, 1], np.int32), xb,
                                    np.array([0b101], np.uint64))
    assert bits_to_f32(out[0, 0]).tolist() == [101.0, 1.0]
    assert bits_to_f32(out[2, 0]).tolist() == [101.0, 5.0]
    assert np.all(out[1, 0] == 0xEEEE)


def test_combine_experts_fp8_hand_example(oracle_mod):
    """The sender-side FP8 combine of per-expert outputs, worked by hand.

    ep 2, E 4 (rank 0 owns experts 0-1, rank 1 owns 2-3), top_k 2, one token of
    rank 0 with ids [0, 3] and weights [1, 0.5], hidden 2:
      y0 = [224, -3]       -> z_0 = bf16(1 * y0)   = [224, -3]
      y1 = [14, 1.1875]    -> z_1 = bf16(0.5 * y1) = [7, 0.59375]
    Row quantisation (one scale per row, amax / 448):
      z_0: amax 224, scale 0.5, inv 2   -> codes E4M3([448, -6]) = [448, -6]
      z_1: amax 7, scale 2^-6, inv 64   -> codes E4M3([448, 38]) = [448, 40]
           (38 lies halfway between 36 and 40; nearest-even picks 40)
    Combine, ascending rank, fma(decode, scale, acc) from +0:
      column 0: 448 * 0.5 = 224, then 224 + 448 * 2^-6 = 231
      column 1: -6 * 0.5 = -3,   then -3 + 40 * 2^-6 = -2.375
    The unquantised combine gives -2.40625 in column 1: the quantisation shows."""
    ids = np.array([[[0, 3]], [[0, 0]]], np.int32)
    n = np.array([1, 0], np.int32)
    plan = oracle_mod.route(2, 4, 2, 1, ids, n)
    w = np.array([[[1.0, 0.5]], [[0.0, 0.0]]], np.float32)
    y = np.zeros((2, 1, 2, 2), np.uint16)
    y[0, 0, 0] = bf16_bits([224.0, -3.0])
    y[0, 0, 1] = bf16_bits([14.0, 1.1875])
    out = oracle_mod.combine_experts_fp8(plan, 4, ids, w, y, 2)
    assert list(bits_to_f32(out[0, 0])) == [231.0, -2.375]
    plain = oracle_mod.combine_experts(plan, 4, ids, w, y, 2)
    assert list(bits_to_f32(plain[0, 0])) == [231.0, -2.40625]
    assert np.all(out[1] == 0xEEEE)          # rank 1 has no token: its row is untouched


def test_combine_experts_fp8_error_bound(oracle_mod):
    """Against the unquantised combine of the same expert outputs: each rank's
    row loses at most half an E4M3 step (2^-4 relative, or 2^-10 of its scale
    near zero) before the sum, so the result differs by at most the sum of those
    bounds plus the final bf16 rounding."""
    w = W.scaled(W.C2, 8)
    x = W.make_inputs(w, with_expert_output=False)
    ids = x.token_selected_experts.numpy()
    plan = oracle_mod.route(w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank, ids,
                            x.local_num_tokens)
    rng = np.random.default_rng(12)
    H = 64
    wts = rng.standard_normal((w.ep_size, w.tokens_per_rank, w.top_k)).astype(np.float32)
    y = bf16_bits(rng.standard_normal(w.ep_size * w.tokens_per_rank * w.top_k * H)
                  .astype(np.float32)).reshape(w.ep_size, w.tokens_per_rank, w.top_k, H)
    got = bits_to_f32(oracle_mod.combine_experts_fp8(plan, w.num_experts, ids, wts, y, H))
    z = oracle_mod.expert_reduce(plan, w.num_experts, ids, wts, y, H)
    zf = bits_to_f32(z).astype(np.float64)
    exact = np.zeros((w.ep_size, w.tokens_per_rank, H))
    bound = np.zeros_like(exact)
    tpr = w.tokens_per_rank
    for s in range(w.ep_size * tpr):
        r, t = divmod(s, tpr)
        for i in range(plan.num_dst[r, t]):
            d = plan.dst_ranks[r, t, i]
            row = zf[d, s]
            scale = np.abs(row).max() / 448.0
            exact[r, t] += row
            bound[r, t] += np.maximum(2.0 ** -4 * np.abs(row), 2.0 ** -10 * scale)
    bound = bound * (1 + 2.0 ** -10) + 2.0 ** -8 * np.abs(exact) + 1e-30
    assert np.all(np.abs(got - exact) <= bound)

"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep_a2a.h")


@pytest.fixture(scope="module")
def ep():
    from combine_route_plan_b200 import build
    build.build()
    from combine_route_plan_b200 import ep_a2a
    return ep_a2a


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_a2a_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for required in ["ep_a2a_init", "ep_a2a_dispatch", "ep_a2a_combine", "ep_a2a_destroy",
                     "ep_a2a_workspace_size", "ep_a2a_get_status"]:
        assert required in names


def _header_enum(prefix):
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return {m.group(1): int(m.group(2))
            for m in re.finditer(rf"\b{prefix}([A-Z0-9_]+)\s*=\s*(-?\d+)", text)}


def test_python_option_and_status_numbers_match_the_header(ep):
    opts = _header_enum("EP_A2A_OPT_")
    assert opts and sorted(opts.values()) == list(range(len(opts)))
    for name, value in opts.items():
        assert getattr(ep, "OPT_" + name) == value, name
    for name, value in _header_enum("EP_A2A_ERR_").items():
        assert getattr(ep, "ERR_" + name) == value, name


def test_library_exports_every_declared_symbol(ep):
    lib = ctypes.CDLL(ep.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def _params(ep, **kw):
    p = ep.Params()
    p.ep_size, p.num_experts, p.top_k = 8, 256, 8
    p.max_tokens_per_rank, p.hidden_size = 128, 7168
    rows = [14336, 32]
    p.num_payloads = len(rows)
    for i, r in enumerate(rows):
        p.payload_row_bytes[i] = r
    p.eplb_stats_num_experts = 0
    p.enable_rank_mask = 0
    p.invalid_expert_id = -1
    p.reserved = 0
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _ws_status(ep, p):
    n = ctypes.c_size_t(0)
    return ep.lib.ep_a2a_workspace_size(ctypes.byref(p), ctypes.byref(n)), n.value


def test_workspace_size_valid_and_monotone(ep):
    st, n = _ws_status(ep, _params(ep))
    assert st == ep.OK
    # at least every receive row of every rank: ep * (ep * cap) * row bytes
    assert n >= 8 * 8 * 128 * (14336 + 32 + 8 * 4 + 1)
    st2, n2 = _ws_status(ep, _params(ep, max_tokens_per_rank=256))
    assert st2 == ep.OK and n2 > n
    st3, n3 = _ws_status(ep, _params(ep, eplb_stats_num_experts=256))
    assert st3 == ep.OK and n3 > n


@pytest.mark.parametrize("field,value,status", [
    ("num_experts", 258, "ERR_INVALID_ARG"),        # not divisible by 4
    ("num_experts", 260, "ERR_INVALID_ARG"),        # not divisible by ep_size 8
    ("ep_size", 0, "ERR_UNSUPPORTED"),
    ("ep_size", 512, "ERR_UNSUPPORTED"),
    ("top_k", 0, "ERR_UNSUPPORTED"),
    ("top_k", 33, "ERR_UNSUPPORTED"),
    ("max_tokens_per_rank", 0, "ERR_INVALID_ARG"),
    ("hidden_size", 0, "ERR_INVALID_ARG"),
    ("num_payloads", 9, "ERR_UNSUPPORTED"),
    ("eplb_stats_num_experts", 128, "ERR_INVALID_ARG"),  # must cover all experts
    ("enable_rank_mask", 2, "ERR_INVALID_ARG"),
    ("reserved", 1, "ERR_INVALID_ARG"),
])
def test_workspace_size_rejects(ep, field, value, status):
    st, _ = _ws_status(ep, _params(ep, **{field: value}))
    assert st == getattr(ep, status)
    assert ep.lib.ep_a2a_last_error()


def test_zero_row_payload_rejected(ep):
    p = _params(ep)
    p.payload_row_bytes[1] = 0
    assert _ws_status(ep, p)[0] == ep.ERR_INVALID_ARG


def test_init_rejects_bad_workspace_before_touching_cuda(ep):
    p = _params(ep)
    _, n = _ws_status(ep, p)
    h = ctypes.c_void_p(0)
    assert ep.lib.ep_a2a_init(ctypes.byref(p), None, n, None, ctypes.byref(h)) == ep.ERR_INVALID_ARG
    assert ep.lib.ep_a2a_init(ctypes.byref(p), ctypes.c_void_p(4096 + 16), n, None,
                              ctypes.byref(h)) == ep.ERR_INVALID_ARG        # misaligned
    assert ep.lib.ep_a2a_init(ctypes.byref(p), ctypes.c_void_p(4096), n - 1, None,
                              ctypes.byref(h)) == ep.ERR_INVALID_ARG        # too small
    assert h.value is None


def test_calls_on_null_handle(ep):
    res = ep.DispatchResult()
    n = (ctypes.c_int32 * 8)(*([1] * 8))
    assert ep.lib.ep_a2a_dispatch(None, ctypes.c_void_p(16), n, 1, None, None, 0, None, None,
                                  None, ctypes.byref(res)) == ep.ERR_NOT_INITIALIZED
    assert ep.lib.ep_a2a_combine(None, ctypes.c_void_p(16), 0, ctypes.c_void_p(16),
                                 None) == ep.ERR_NOT_INITIALIZED
    assert ep.lib.ep_a2a_get_status(None, None) == ep.ERR_NOT_INITIALIZED
    assert ep.lib.ep_a2a_set_option(None, 0, 0) == ep.ERR_NOT_INITIALIZED


def test_destroy_is_idempotent_on_null(ep):
    box = ctypes.c_void_p(0)
    assert ep.lib.ep_a2a_destroy(ctypes.byref(box)) == ep.OK
    assert ep.lib.ep_a2a_destroy(ctypes.byref(box)) == ep.OK
    assert ep.lib.ep_a2a_destroy(None) == ep.OK


def test_quantize_argument_checks(ep):
    assert ep.lib.ep_a2a_quantize_e4m3(None, None, -1, None) == ep.ERR_INVALID_ARG
    assert ep.lib.ep_a2a_quantize_e4m3(None, None, 5, None) == ep.ERR_INVALID_ARG
    assert ep.lib.ep_a2a_quantize_e4m3(None, None, 0, None) == ep.OK      # nothing to do


def test_status_strings(ep):
    for s in range(8):
        assert ep.ep_a2a_status_string(s)
    assert "unknown" in ep.ep_a2a_status_string(99)


# --------------------------------------------------------------------------- #
# Capacity growth (vllm.distributed.device_communicators.all2all,
# FlashInferNVLinkOneSidedManager.initialize): a host-only rule, so tested here
# --------------------------------------------------------------------------- #

def _grow(ep, cur, req):
    out, grown = ep.Params(), ctypes.c_int32(-1)
    st = ep.lib.ep_a2a_grow_params(ctypes.byref(cur), ctypes.byref(req), ctypes.byref(out),
                                   ctypes.byref(grown))
    return st, out, grown.value


def _caps(p):
    return (p.max_tokens_per_rank, p.hidden_size,
            [p.payload_row_bytes[i] for i in range(p.num_payloads)],
            p.eplb_stats_num_experts, p.enable_rank_mask, p.invalid_expert_id)


def _with_rows(ep, rows, **kw):
    p = _params(ep, **kw)
    p.num_payloads = len(rows)
    for i in range(8):
        p.payload_row_bytes[i] = rows[i] if i < len(rows) else 0
    return p


def test_grow_keeps_a_handle_that_covers_the_request(ep):
    # the pages keep the communicator when tokens, hidden and dispatch bytes all fit
    cur = _with_rows(ep, [14336, 64, 32], max_tokens_per_rank=256)
    req = _with_rows(ep, [7168, 32], max_tokens_per_rank=128, hidden_size=4096)
    st, out, grown = _grow(ep, cur, req)
    assert st == ep.OK and grown == 0
    assert _caps(out) == (256, 7168, [14336, 64, 32], 0, 0, 256)   # id resolved to E


@pytest.mark.parametrize("req_kw,req_rows,want", [
    # more tokens: only the token capacity grows
    (dict(max_tokens_per_rank=512), [14336, 32], (512, 7168, [14336, 32])),
    # a larger hidden with a smaller dispatch format: hidden from the request,
    # row bytes from the current handle (the larger hidden sizes the combine, the
    # larger payload the dispatch)
    (dict(hidden_size=8192), [4096 + 512, 32], (128, 8192, [14336, 32])),
    # a smaller hidden with a larger payload (extra bytes): the reverse
    (dict(hidden_size=2048), [14336, 32, 64], (128, 7168, [14336, 32, 64])),
    # NVFP4 rows with scales (3584 + 448) against BF16 rows: positionwise maximum
    (dict(), [3584, 448, 32], (128, 7168, [14336, 448, 32])),
])
def test_grow_takes_the_larger_capacity(ep, req_kw, req_rows, want):
    cur = _with_rows(ep, [14336, 32])
    req = _with_rows(ep, req_rows, **req_kw)
    st, out, grown = _grow(ep, cur, req)
    assert st == ep.OK and grown == 1
    assert _caps(out)[:3] == want


@pytest.mark.parametrize("field,value", [("top_k", 4), ("num_experts", 128), ("ep_size", 4),
                                         ("invalid_expert_id", 7)])
def test_grow_rejects_a_different_layer_shape(ep, field, value):
    # one handle serves one top_k and one expert count (the pages assert both)
    cur = _params(ep)
    req = _params(ep, **{field: value})
    st, _, _ = _grow(ep, cur, req)
    assert st == ep.ERR_INVALID_ARG
    assert field.split("_")[0] in ep.lib.ep_a2a_last_error().decode()


def test_grow_validates_both_inputs(ep):
    st, _, _ = _grow(ep, _params(ep, hidden_size=0), _params(ep))
    assert st == ep.ERR_INVALID_ARG
    st, _, _ = _grow(ep, _params(ep), _params(ep, num_experts=250))
    assert st == ep.ERR_INVALID_ARG
    assert ep.lib.ep_a2a_grow_params(None, None, None, None) == ep.ERR_INVALID_ARG


def test_grow_turns_on_eplb_and_the_rank_mask(ep):
    cur = _params(ep)
    st, out, grown = _grow(ep, cur, _params(ep, eplb_stats_num_experts=256, enable_rank_mask=1))
    assert st == ep.OK and grown == 1
    assert (out.eplb_stats_num_experts, out.enable_rank_mask) == (256, 1)
    # -1 and E name the same invalid id
    st, out, grown = _grow(ep, _params(ep, invalid_expert_id=256), _params(ep))
    assert st == ep.OK and grown == 0


def test_grow_properties_on_random_requests(ep):
    """Over random layer sizes: the result covers both sides, takes every field
    from one of them, is the same either way round, is idempotent, and its
    workspace is at least as large as either side's."""
    rng = np.random.default_rng(7)
    for _ in range(300):
        sides = []
        for _s in range(2):
            n = int(rng.integers(0, 9))
            rows = [int(v) for v in rng.integers(1, 20000, n)]
            sides.append(_with_rows(ep, rows, max_tokens_per_rank=int(rng.integers(1, 5000)),
                                    hidden_size=int(rng.integers(1, 9000)),
                                    eplb_stats_num_experts=int(rng.integers(0, 2)) * 256,
                                    enable_rank_mask=int(rng.integers(0, 2))))
        a, b = sides
        st, ab, grown = _grow(ep, a, b)
        assert st == ep.OK
        st2, ba, _ = _grow(ep, b, a)
        assert st2 == ep.OK and _caps(ab) == _caps(ba)
        ca, cb, cg = _caps(a), _caps(b), _caps(ab)
        for i in (0, 1, 3, 4):
            assert cg[i] == max(ca[i], cb[i])
        ra, rb, rg = ca[2], cb[2], cg[2]
        assert len(rg) == max(len(ra), len(rb))
        for i, v in enumerate(rg):
            assert v == max(ra[i] if i < len(ra) else 0, rb[i] if i < len(rb) else 0)
        # the pages' dispatch-bytes rule: the grown rows hold either side's bytes
        assert sum(rg) >= max(sum(ra), sum(rb))
        assert grown == int(_caps(a)[:5] != cg[:5])
        for side in (a, b, ab):
            st, _, again = _grow(ep, ab, side)
            assert st == ep.OK and again == 0
        wa, wb, wg = (_ws_status(ep, p)[1] for p in (a, b, ab))
        assert wg >= max(wa, wb)


def test_checked_build_compiles_and_exports_every_symbol():
    """The checked build (device index checks compiled in) is the same ABI."""
    from combine_route_plan_b200 import build
    lib = ctypes.CDLL(build.build(checked=True))
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing

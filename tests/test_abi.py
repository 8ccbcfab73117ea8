"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

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

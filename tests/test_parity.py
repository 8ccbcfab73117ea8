"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle,
element by element, on the five synthetic workloads at full size and on edge
cases.  Dispatch, the plan, EPLB gather and the BF16 combine are bit-exact;
the FP8 combine is checked against the 2^-3 relative bar and, since both sides
take the same E4M3 decisions, also for bit-exactness."""
import functools
import gc

import numpy as np
import pytest
import torch

from combine_route_plan_b200 import workloads as W
import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_route_plan_b200 import build
    build.build()
    yield
    gc.collect()
    torch.cuda.empty_cache()


@functools.lru_cache(maxsize=8)
def _inputs(name):
    # every workload's inputs stay cached for the module (about 14 GB of host
    # memory at most), so tests that alternate between workloads draw each once
    return W.make_inputs(W.BY_NAME[name])


def _full_check(w, copy_path=None, options=None):
    x = _inputs(w.name)
    run = U.Run(w, x, copy_path=copy_path, options=options)
    plan = U.oracle_plan(w, x)
    U.check_plan(run, plan, w)
    U.check_payloads(run, plan, w, x)
    U.check_eplb(run, w, x)
    U.check_combine(run, plan, w, x)
    del run
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", [w.name for w in W.ALL])
def test_workload_bit_exact(name):
    _full_check(W.BY_NAME[name])


@pytest.mark.parametrize("name", ["c1_ep4_tiny", "c2_ep8_decode", "c5_ep64_wide_masked",
                                  "c4_ep8_prefill"])
def test_routing_inside_the_copy_bit_exact(name):
    """The vector copy kernel that also routes (one launch per dispatch; the
    default runs a separate routing kernel beside the copy): plan, counts, valid
    bytes, ids, EPLB rows, the combine, and the payload rows of the first and
    last destination ranks."""
    from combine_route_plan_b200 import ep_a2a
    w = W.BY_NAME[name]
    x = _inputs(w.name)
    run = U.Run(w, x, options={ep_a2a.OPT_ROUTE_IN_COPY: 1})
    plan = U.oracle_plan(w, x)
    U.check_plan(run, plan, w)
    U.check_eplb(run, w, x)
    U.check_combine(run, plan, w, x)
    ep, tpr = w.ep_size, w.tokens_per_rank
    for i, p in enumerate(x.payloads):
        rb = p.shape[2]
        for dst in sorted({0, ep - 1}):
            want = U.oracle.dispatch_payload(plan, p.numpy(), only_dst=dst,
                                             recv_init=np.full((1, ep * tpr, rb), U.CANARY,
                                                               np.uint8))
            U.assert_equal(run.d.recv_payloads[i][dst], want, f"payload {i} rank {dst}")
    del run
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,path", [
    (n, p) for n in ("c1_ep4_tiny", "c2_ep8_decode", "c5_ep64_wide_masked", "c3_ep16_zipf_nvfp4")
    for p in (0, 2)])
def test_bulk_copy_paths_bit_exact(name, path):
    """The two bulk-async copy paths (loads into shared memory + vector stores;
    bulk loads + bulk stores) on the workloads, next to the default vector path."""
    _full_check(W.BY_NAME[name], copy_path=path)


@pytest.mark.parametrize("path,stages,ctas,cw,inter", [
    (0, 0, 1, 8, 0), (0, 2, 1, 4, 1), (0, 3, 2, 16, 0), (0, 5, 3, 8, 1), (0, 32, 1, 8, 0),
    (0, 4, 4, 4, 1), (2, 2, 1, 8, 0), (2, 3, 2, 8, 1), (2, 4, 4, 8, 0), (2, 8, 1, 8, 1),
    (2, 16, 1, 8, 0), (2, 32, 1, 8, 1), (2, 5, 3, 8, 0),
])
def test_copy_tuning_does_not_change_results(path, stages, ctas, cw, inter):
    """Every copy path and staging configuration writes the same bytes."""
    from combine_route_plan_b200 import ep_a2a
    w = W.scaled(W.C2, 96)
    x = W.make_inputs(w, with_expert_output=False)
    run = U.Run(w, x, copy_path=path,
                options={ep_a2a.OPT_COPY_STAGES: stages, ep_a2a.OPT_COPY_CTAS_PER_SM: ctas,
                         ep_a2a.OPT_COPY_CONSUMER_WARPS: cw, ep_a2a.OPT_COPY_INTERLEAVE: inter})
    plan = U.oracle_plan(w, x)
    U.check_plan(run, plan, w)
    U.check_payloads(run, plan, w, x)


@pytest.mark.parametrize("unroll,ctas,streaming,tpt,rows", [
    (2, 1, 0, 32, [14336, 32]), (4, 8, 1, 64, [14336, 64, 32]), (8, 64, 0, 128, [14336, 32]),
    (8, 3, 1, 256, [100, 13, 16]), (2, 16, 1, 0, [7, 4096 + 8]), (4, 32, 1, 256, [14336, 32]),
    (4, 2, 0, 128, [1, 2, 4, 8, 16]),
])
def test_vector_copy_variants(unroll, ctas, streaming, tpt, rows):
    from combine_route_plan_b200 import ep_a2a
    w, x = _custom(8, 64, 8, 50, 32, rows, seed=unroll * 31 + ctas)
    run = U.Run(w, x, copy_path=1, options={ep_a2a.OPT_VEC_UNROLL: unroll,
                                            ep_a2a.OPT_VEC_CTAS_PER_SM: ctas,
                                            ep_a2a.OPT_STORE_STREAMING: streaming,
                                            ep_a2a.OPT_VEC_THREADS_PER_TOKEN: tpt})
    plan = U.oracle_plan(w, x)
    U.check_payloads(run, plan, w, x)


@pytest.mark.parametrize("name", ["c1_ep4_tiny", "c2_ep8_decode", "c5_ep64_wide_masked",
                                  "c3_ep16_zipf_nvfp4", "c3_ep16_zipf_mxfp8"])
def test_vector_copy_32_byte_accesses(name):
    """256-bit loads and stores where every row allows them (all-32 kernel),
    per-payload widths otherwise."""
    from combine_route_plan_b200 import ep_a2a
    _full_check(W.BY_NAME[name], options={ep_a2a.OPT_COPY_VEC_BYTES: 32})


@pytest.mark.parametrize("rows,shift", [([14336, 64, 32], 0), ([14336, 48], 0),
                                        ([4096 + 16, 32], 16), ([7, 96, 224], 0)])
def test_vector_copy_32_byte_mixed_rows(rows, shift):
    """Rows that are 32-byte multiples next to rows that are not, and sources
    that are only 16-byte aligned."""
    from combine_route_plan_b200 import ep_a2a
    ep, E, k, tpr, H = 8, 64, 8, 50, 32
    w, x = _custom(ep, E, k, tpr, H, rows, seed=sum(rows) % 1000 + shift)
    comm = ep_a2a.EpA2A(ep, E, k, tpr, H, rows, workspace_fill=U.CANARY)
    comm.set_option(ep_a2a.OPT_COPY_VEC_BYTES, 32)
    for tpt in (32, 256):
        comm.set_option(ep_a2a.OPT_VEC_THREADS_PER_TOKEN, tpt)
        srcs = []
        for p in x.payloads:
            buf = torch.empty(p.numel() + 64, dtype=torch.uint8, device="cuda")
            v = buf[shift: shift + p.numel()].view(p.shape)
            v.copy_(p.cuda())
            srcs.append(v)
        d = comm.dispatch(x.token_selected_experts.cuda(), x.local_num_tokens, srcs, tpr)
        torch.cuda.synchronize()
        plan = U.oracle_plan(w, x)
        for i, p in enumerate(x.payloads):
            for dst in range(ep):
                want = U.oracle.dispatch_payload(plan, p.numpy(), only_dst=dst, recv_init=np.full(
                    (1, ep * tpr, p.shape[2]), U.CANARY, np.uint8))
                U.assert_equal(d.recv_payloads[i][dst], want, f"payload {i} rank {dst} tpt {tpt}")


@pytest.mark.parametrize("name", ["c2_ep8_decode", "c5_ep64_wide_masked"])
def test_fp8_combines_with_16_byte_aligned_output(name):
    """The pipelined E4M3 combines store 32 bytes at once only into 32-byte
    aligned outputs; a 16-byte aligned output takes two 16-byte stores."""
    from combine_route_plan_b200 import ep_a2a
    w = W.BY_NAME[name]
    x = _inputs(w.name)
    run = U.Run(w, W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads,
                            x.eplb_local_stats, x.active_rank_mask, None))
    plan = U.oracle_plan(w, x)
    n = w.ep_size * w.tokens_per_rank * w.hidden
    xo = x.expert_output
    init = U.oracle_out_init(w)
    for shift in (8, 0):       # in bf16 elements: 16 and 0 bytes
        buf = torch.full((n + 16,), U.OUT_CANARY, dtype=torch.int16, device="cuda")
        out = buf[shift: shift + n].view(torch.bfloat16).view(w.ep_size, w.tokens_per_rank, w.hidden)
        run.comm.combine(ep_a2a.quantize_e4m3(xo.cuda()), out)
        torch.cuda.synchronize()
        xq = U.oracle_e4m3_rows_read(U.to_np(xo), plan, U.oracle_e4m3_table())
        U.assert_equal(out, U.oracle.combine(plan, xq, w.hidden, input_is_e4m3=True,
                                             out_init=init), f"fp8 shift {shift}")
        buf.fill_(U.OUT_CANARY)
        codes, scales = ep_a2a.quantize_e4m3_rows(xo.cuda())
        run.comm.combine_scaled(codes, scales, out)
        torch.cuda.synchronize()
        oc, osc = U.oracle_row_quantize_read(U.to_np(xo), plan, w.hidden)
        U.assert_equal(out, U.oracle.combine_scaled(plan, oc, osc, w.hidden, out_init=init),
                       f"scaled shift {shift}")


@pytest.mark.parametrize("rows", [[16], [4096 + 16, 32], [65536 + 16, 48]])
def test_staged_copy_row_sizes(rows):
    """Rows from one vector per token up to more than the staged kernel holds in
    registers (which then falls back to the vector copy)."""
    w, x = _custom(4, 16, 4, 40, 32, rows, seed=len(rows) * 7 + rows[0] % 97)
    run = U.Run(w, x)
    plan = U.oracle_plan(w, x)
    U.check_payloads(run, plan, w, x)


@pytest.mark.parametrize("name", ["c2_ep8_decode", "c5_ep64_wide_masked"])
def test_without_programmatic_dependent_launch(name):
    from combine_route_plan_b200 import ep_a2a
    _full_check(W.BY_NAME[name], options={ep_a2a.OPT_PDL: 0})


def test_cuda_graph_capture_and_replay():
    """Dispatch + combine captured into a CUDA graph give the oracle's result on
    every replay (new inputs are copied into the captured buffers between replays)."""
    from combine_route_plan_b200 import ep_a2a
    w = W.C2
    x = _inputs(w.name)
    comm = ep_a2a.EpA2A(w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank, w.hidden,
                        w.payload_row_bytes(), workspace_fill=U.CANARY)
    ids = x.token_selected_experts.cuda()
    pays = [p.cuda() for p in x.payloads]
    xo = x.expert_output.cuda()
    out = torch.empty((w.ep_size, w.tokens_per_rank, w.hidden), dtype=torch.bfloat16, device="cuda")

    def step():
        comm.dispatch(ids, x.local_num_tokens, pays, w.tokens_per_rank, views=False)
        comm.combine(xo, out)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    plan = U.oracle_plan(w, x)
    for _ in range(2):
        out.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        U.check_combine(type("R", (), {"out": out})(), plan, w, x)
    # new routing and rows through the same captured pointers
    ids.copy_(torch.roll(x.token_selected_experts, 1, dims=1).cuda())
    x3 = W.Inputs(w, torch.roll(x.token_selected_experts, 1, dims=1), x.local_num_tokens,
                  x.payloads, None, None, x.expert_output)
    g.replay()
    torch.cuda.synchronize()
    U.check_combine(type("R", (), {"out": out})(), U.oracle_plan(w, x3), w, x3)
    assert comm.get_status() == ep_a2a.OK


def test_cuda_graph_with_pipelined_combines():
    """Dispatch, the FP8 combine and the expert-output combine (pipelined
    kernels, L2 prefetch on) captured into one CUDA graph."""
    from combine_route_plan_b200 import ep_a2a
    w = W.C2
    x = _inputs(w.name)
    comm = ep_a2a.EpA2A(w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank, w.hidden,
                        w.payload_row_bytes(), workspace_fill=U.CANARY)
    comm.set_option(ep_a2a.OPT_COMBINE_PREFETCH, 1)
    ids = x.token_selected_experts.cuda()
    pays = [p.cuda() for p in x.payloads]
    xq = ep_a2a.quantize_e4m3(x.expert_output.cuda())
    g_ = torch.Generator().manual_seed(12)
    wts = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k), generator=g_)
    y = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k, w.hidden), generator=g_) \
        .to(torch.bfloat16)
    wts_d, y_d = wts.cuda(), y.cuda()
    out8 = torch.empty((w.ep_size, w.tokens_per_rank, w.hidden), dtype=torch.bfloat16,
                       device="cuda")
    oute = torch.empty_like(out8)

    def step():
        comm.dispatch(ids, x.local_num_tokens, pays, w.tokens_per_rank, views=False)
        comm.combine(xq, out8)
        comm.combine_experts(wts_d, y_d, oute)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    plan = U.oracle_plan(w, x)
    want8 = U.oracle.combine(plan, U.to_np(xq), w.hidden, input_is_e4m3=True)
    wante = U.oracle.combine_experts(plan, w.num_experts, x.token_selected_experts.numpy(),
                                     wts.numpy(), U.to_np(y), w.hidden)
    for _ in range(2):
        out8.fill_(0)
        oute.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        U.assert_equal(out8, want8, "fp8 combine in a graph")
        U.assert_equal(oute, wante, "expert combine in a graph")
    assert comm.get_status() == ep_a2a.OK


@pytest.mark.parametrize("prefetch,ctas", [(1, 4), (1, 12), (1, 128), (0, 8)])
def test_prefetch_options_do_not_change_results(prefetch, ctas):
    from combine_route_plan_b200 import ep_a2a
    for name in ("c2_ep8_decode", "c5_ep64_wide_masked"):
        _full_check(W.BY_NAME[name], options={ep_a2a.OPT_COMBINE_PREFETCH: prefetch,
                                              ep_a2a.OPT_COPY_PREFETCH: prefetch,
                                              ep_a2a.OPT_COMBINE_CTAS_PER_SM: ctas,
                                              ep_a2a.OPT_VEC_CTAS_PER_SM: min(ctas, 64)})
    w = W.C2
    x = _inputs(w.name)
    wts = x.payloads[-1].view(torch.float32).view(w.ep_size, w.tokens_per_rank, w.top_k)
    _check_combine_experts(w, x, _expert_outputs(w, seed=3), wts,
                           options={ep_a2a.OPT_COMBINE_PREFETCH: prefetch,
                                    ep_a2a.OPT_COMBINE_CTAS_PER_SM: ctas})


@pytest.mark.parametrize("threads,ctas", [(64, 0), (96, 3), (256, 64), (512, 1), (128, 1024),
                                          (0, 0)])
def test_combine_launch_shape_does_not_change_results(threads, ctas):
    from combine_route_plan_b200 import ep_a2a
    w = W.C2
    x = _inputs(w.name)
    run = U.Run(w, x, options={ep_a2a.OPT_COMBINE_THREADS: threads,
                               ep_a2a.OPT_COMBINE_CTAS_PER_SM: ctas})
    U.check_combine(run, U.oracle_plan(w, x), w, x)


@pytest.mark.parametrize("case", [
    ("c2_ep8_decode", None),
    ("c5_ep64_wide_masked", None),
    ("c1_ep4_tiny", None),
    ("mask", [0b10100101, 0, 0, 0]),       # tokens whose owners are all masked: +0
    ("odd", None),                          # hidden 40: FP8 rows take the element kernels
    ("wide_k", None),                       # top_k 16 over 16 ranks: not pipelined
])
@pytest.mark.parametrize("prefetch,threads", [(-1, 0), (2, 128), (0, 64)])
def test_pipelined_combines_match_the_oracle(case, prefetch, threads):
    """BF16, FP8, scaled-FP8 and expert-output combines with the two-deep
    pipelined kernels."""
    from combine_route_plan_b200 import ep_a2a
    name, mask = case
    if name in W.BY_NAME:
        w = W.BY_NAME[name]
        x = _inputs(w.name)
    elif name == "mask":
        w, x = _custom(8, 64, 6, 40, 64, [32], n=[40, 1, 0, 39, 17, 40, 2, 33], mask=mask, seed=8)
    elif name == "odd":
        w, x = _custom(4, 16, 4, 30, 40, [32], seed=19)
    else:
        w, x = _custom(16, 64, 16, 20, 64, [32], seed=23)
    opts = {ep_a2a.OPT_COMBINE_PIPELINE: 1, ep_a2a.OPT_COMBINE_PREFETCH: prefetch,
            ep_a2a.OPT_COMBINE_THREADS: threads}
    run = U.Run(w, W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads,
                            x.eplb_local_stats, x.active_rank_mask, None), options=opts)
    plan = U.oracle_plan(w, x)
    xo = x.expert_output
    H = w.hidden

    def fresh():
        return torch.full((w.ep_size, w.tokens_per_rank, H), U.OUT_CANARY, dtype=torch.int16,
                          device="cuda").view(torch.bfloat16)
    out, out8, outs = fresh(), fresh(), fresh()
    run.comm.combine(xo.cuda(), out)
    run.comm.combine(ep_a2a.quantize_e4m3(xo.cuda()), out8)
    codes, scales = ep_a2a.quantize_e4m3_rows(xo.cuda())
    run.comm.combine_scaled(codes, scales, outs)
    torch.cuda.synchronize()
    assert run.comm.get_status() == ep_a2a.OK
    init = U.oracle_out_init(w)
    xq = U.oracle_e4m3_rows_read(U.to_np(xo), plan, U.oracle_e4m3_table())
    oc, osc = U.oracle_row_quantize_read(U.to_np(xo), plan, H)
    U.assert_equal(out, U.oracle.combine(plan, U.to_np(xo), H, out_init=init), "bf16")
    U.assert_equal(out8, U.oracle.combine(plan, xq, H, input_is_e4m3=True, out_init=init), "fp8")
    U.assert_equal(outs, U.oracle.combine_scaled(plan, oc, osc, H, out_init=init), "scaled")
    g = torch.Generator().manual_seed(w.top_k + H)
    wts = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k), generator=g)
    y = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k, H), generator=g).to(torch.bfloat16)
    oute = fresh()
    run.comm.combine_experts(wts.cuda(), y.cuda(), oute)
    torch.cuda.synchronize()
    U.assert_equal(oute, U.oracle.combine_experts(plan, w.num_experts,
                                                  x.token_selected_experts.numpy(), wts.numpy(),
                                                  U.to_np(y), H, out_init=init), "experts")


@pytest.mark.parametrize("case,ctas", [
    (("c2_ep8_decode", None), 0),
    (("c2_ep8_decode", None), 3),
    (("c5_ep64_wide_masked", None), 0),
    (("c1_ep4_tiny", None), 1),
    (("c3_ep16_zipf_nvfp4", None), 0),
    (("mask", [0b10100101, 0, 0, 0]), 0),   # tokens whose owners are all masked: +0
    (("mask", [0b10100101, 0, 0, 0]), 1),
    (("short", None), 0),                   # hidden 40: rows shorter than a chunk
    (("short", None), 3),
])
def test_staged_combines_match_the_oracle(case, ctas):
    """BF16, FP8, scaled-FP8 and expert-output combines with the rows staged in
    shared memory by bulk-async copies (combine pipeline option 2), at 1 to 3
    CTAs per SM."""
    from combine_route_plan_b200 import ep_a2a
    name, mask = case
    if name in W.BY_NAME:
        w = W.BY_NAME[name]
        x = _inputs(w.name)
    elif name == "mask":
        w, x = _custom(8, 64, 6, 40, 64, [32], n=[40, 1, 0, 39, 17, 40, 2, 33], mask=mask, seed=8)
    else:
        w, x = _custom(4, 16, 4, 30, 40, [32], seed=19)
    opts = {ep_a2a.OPT_COMBINE_PIPELINE: 2, ep_a2a.OPT_COMBINE_CTAS_PER_SM: ctas}
    run = U.Run(w, W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads,
                            x.eplb_local_stats, x.active_rank_mask, None), options=opts)
    plan = U.oracle_plan(w, x)
    xo = x.expert_output
    H = w.hidden

    def fresh():
        return torch.full((w.ep_size, w.tokens_per_rank, H), U.OUT_CANARY, dtype=torch.int16,
                          device="cuda").view(torch.bfloat16)
    out, out8, outs = fresh(), fresh(), fresh()
    run.comm.combine(xo.cuda(), out)
    run.comm.combine(ep_a2a.quantize_e4m3(xo.cuda()), out8)
    codes, scales = ep_a2a.quantize_e4m3_rows(xo.cuda())
    run.comm.combine_scaled(codes, scales, outs)
    torch.cuda.synchronize()
    assert run.comm.get_status() == ep_a2a.OK
    init = U.oracle_out_init(w)
    xq = U.oracle_e4m3_rows_read(U.to_np(xo), plan, U.oracle_e4m3_table())
    oc, osc = U.oracle_row_quantize_read(U.to_np(xo), plan, H)
    U.assert_equal(out, U.oracle.combine(plan, U.to_np(xo), H, out_init=init), "bf16")
    U.assert_equal(out8, U.oracle.combine(plan, xq, H, input_is_e4m3=True, out_init=init), "fp8")
    U.assert_equal(outs, U.oracle.combine_scaled(plan, oc, osc, H, out_init=init), "scaled")
    g = torch.Generator().manual_seed(w.top_k + H + 1)
    wts = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k), generator=g)
    y = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k, H), generator=g).to(torch.bfloat16)
    oute = fresh()
    run.comm.combine_experts(wts.cuda(), y.cuda(), oute)
    torch.cuda.synchronize()
    assert run.comm.get_status() == ep_a2a.OK
    U.assert_equal(oute, U.oracle.combine_experts(plan, w.num_experts,
                                                  x.token_selected_experts.numpy(), wts.numpy(),
                                                  U.to_np(y), H, out_init=init), "experts")


def test_fp8_quantize_all_bf16_patterns():
    from combine_route_plan_b200 import ep_a2a
    table = U.oracle_e4m3_table()
    allbits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    for lead in (0, 1, 3, 8):        # misaligned starts and odd lengths take the scalar path
        src = torch.cat([torch.zeros(lead, dtype=torch.bfloat16), allbits]).cuda()[lead:]
        n = src.numel() - (lead % 3)
        out = torch.empty(n + 1, dtype=torch.uint8, device="cuda")[1:] if lead else \
            torch.empty(n, dtype=torch.uint8, device="cuda")
        ep_a2a.ep_a2a_quantize_e4m3(src.data_ptr(), out.data_ptr(), n)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        f = (np.arange(n, dtype=np.uint32) << 16).view(np.float32)
        nan = np.isnan(f)
        assert np.array_equal(got[~nan], table[:n][~nan]), f"quantize lead={lead}"
        assert np.all((got[nan] & 0x7F) == 0x7F)      # NaN stays NaN (its sign is not fixed)


@pytest.mark.parametrize("name", ["c4_ep8_prefill", "c2_ep8_decode", "c3_ep16_zipf_nvfp4",
                                  "c1_ep4_tiny", "c5_ep64_wide_masked"])
def test_fp8_combine(name):
    """The low-precision combine on every workload, at the library's default
    launch shape for its token count (8192 slots for the Zipf workload)."""
    w = W.BY_NAME[name]
    x = _inputs(w.name)
    run = U.Run(w, x, fp8=True)
    plan = U.oracle_plan(w, x)
    xq = U.oracle_e4m3_rows_read(U.to_np(x.expert_output), plan, U.oracle_e4m3_table())
    idx = torch.from_numpy(U.valid_rows(plan)).cuda()
    U.assert_equal(run.xq.view(-1, w.hidden).index_select(0, idx),
                   xq.reshape(-1, w.hidden)[U.valid_rows(plan)], "quantized rows the combine reads")
    want = U.oracle.combine(plan, xq, w.hidden, input_is_e4m3=True, out_init=U.oracle_out_init(w))
    got = U.to_np(run.out)
    exists = plan.num_dst >= 0
    gf = (got[exists].astype(np.uint32) << 16).view(np.float32)
    wf = (want[exists].astype(np.uint32) << 16).view(np.float32)
    rel = np.abs(gf.astype(np.float64) - wf) / np.maximum(np.abs(wf.astype(np.float64)), 1e-30)
    rel[(gf == wf)] = 0.0
    assert rel.max() <= 2.0 ** -3, rel.max()          # the stated bar
    U.assert_equal(run.out, want, "fp8 combine (bit-exact)")
    assert np.all(got[~exists] == 0xEEEE)


# --------------------------------------------------------------------------- #
# Edge cases
# --------------------------------------------------------------------------- #

def _custom(ep, E, k, tpr, H, rows, n=None, mask=None, seed=0, ids=None):
    """A workload-like object with arbitrary payload rows of random bytes."""
    g = torch.Generator().manual_seed(seed)
    if ids is None:
        ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(ep * tpr)]) \
            .to(torch.int32).view(ep, tpr, k)
    n = np.full(ep, tpr, np.int32) if n is None else np.asarray(n, np.int32)
    payloads = [W.random_bytes_payload(ep, tpr, rb, seed + 17 * i) for i, rb in enumerate(rows)]
    xo = torch.randn((ep, ep * tpr, H), generator=g).to(torch.bfloat16)

    class Cfg:
        pass
    w = Cfg()
    w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank, w.hidden = ep, E, k, tpr, H
    w.eplb = False
    w.masked_ranks = () if mask is None else tuple(r for r in range(ep)
                                                   if not (int(mask[r // 64]) >> (r % 64)) & 1)
    w.payload_row_bytes = lambda: list(rows)
    x = W.Inputs(w, ids.contiguous(), n, payloads, None,
                 None if mask is None else np.asarray(mask, np.uint64), xo)
    return w, x


@pytest.mark.parametrize("ep,E,k,tpr,H,rows", [
    (3, 12, 3, 37, 100, [1, 3, 13, 100]),          # odd rows: vector path, 1-byte vectors
    (5, 20, 5, 33, 24, [16, 48, 8, 4]),            # k not a power of two
    (16, 64, 16, 20, 64, [4096 + 16, 32]),         # 16 lanes per token
    (16, 64, 32, 9, 32, [64, 2]),                  # top_k 32: a whole warp per token
    (1, 8, 4, 50, 40, [272, 12]),                  # ep_size 1: identity
    (2, 4, 1, 64, 8, [16]),                        # top_k 1
    (4, 8, 2, 300, 128, [256, 8, 8]),              # several route blocks per rank, ragged tail
])
def test_edge_shapes(ep, E, k, tpr, H, rows):
    w, x = _custom(ep, E, k, tpr, H, rows, seed=ep * 100 + k)
    run = U.Run(w, x)
    plan = U.oracle_plan(w, x)
    U.check_plan(run, plan, w)
    U.check_payloads(run, plan, w, x)
    U.check_combine(run, plan, w, x)


def _mask_of(ep, live):
    words = [0, 0, 0, 0]
    for r in live:
        words[r // 64] |= 1 << (r % 64)
    return words


@pytest.mark.parametrize("case", [
    # the largest ep_size and top_k, one expert per rank
    dict(ep=256, E=256, k=32, tpr=4, H=64, rows=[32, 16]),
    # a mask spanning all four mask words, k 8 over 512 experts
    dict(ep=256, E=512, k=8, tpr=3, H=16, rows=[8],
         live=[0, 1, 63, 64, 100, 127, 128, 200, 254, 255]),
    # one token slot per rank, hidden 1 (element kernels), one-byte rows
    dict(ep=7, E=28, k=4, tpr=1, H=1, rows=[1]),
    # no rank has a token
    dict(ep=8, E=64, k=8, tpr=16, H=32, rows=[16], n=[0] * 8),
    # one live rank with tokens, the others empty or masked off
    dict(ep=8, E=64, k=8, tpr=16, H=32, rows=[16], n=[0, 0, 16, 0, 5, 0, 0, 0],
         live=[2, 5, 6]),
])
def test_extreme_shapes(case):
    """Maximum and degenerate sizes: every plan array, payload and the BF16,
    FP8 and expert-output combines against the oracle."""
    from combine_route_plan_b200 import ep_a2a
    ep, E, k, tpr, H, rows = (case[key] for key in ("ep", "E", "k", "tpr", "H", "rows"))
    mask = _mask_of(ep, case["live"]) if "live" in case else None
    w, x = _custom(ep, E, k, tpr, H, rows, n=case.get("n"), mask=mask, seed=ep + k + tpr)
    run = U.Run(w, x)
    plan = U.oracle_plan(w, x)
    U.check_plan(run, plan, w)
    U.check_payloads(run, plan, w, x)
    U.check_combine(run, plan, w, x)
    init = U.oracle_out_init(w)
    out8 = torch.full((ep, tpr, H), U.OUT_CANARY, dtype=torch.int16,
                      device="cuda").view(torch.bfloat16)
    run.comm.combine(ep_a2a.quantize_e4m3(x.expert_output.cuda()), out8)
    g = torch.Generator().manual_seed(ep * k)
    wts = torch.randn((ep, tpr, k), generator=g)
    y = torch.randn((ep, tpr, k, H), generator=g).to(torch.bfloat16)
    oute = torch.full((ep, tpr, H), U.OUT_CANARY, dtype=torch.int16,
                      device="cuda").view(torch.bfloat16)
    run.comm.combine_experts(wts.cuda(), y.cuda(), oute)
    torch.cuda.synchronize()
    assert run.comm.get_status() == ep_a2a.OK
    xq = U.oracle_quantize_big(U.to_np(x.expert_output), U.oracle_e4m3_table())
    U.assert_equal(out8, U.oracle.combine(plan, xq, H, input_is_e4m3=True, out_init=init), "fp8")
    U.assert_equal(oute, U.oracle.combine_experts(plan, E, x.token_selected_experts.numpy(),
                                                  wts.numpy(), U.to_np(y), H, out_init=init),
                   "experts")
    if "n" in case and not any(case["n"]):
        assert int(run.d.send_counts.sum()) == 0 and int(run.d.recv_valid.sum()) == 0


def test_misaligned_payload_pointers():
    ep, E, k, tpr, H = 4, 16, 4, 25, 64
    w, x = _custom(ep, E, k, tpr, H, [64, 32], seed=5)
    from combine_route_plan_b200 import ep_a2a
    comm = ep_a2a.EpA2A(ep, E, k, tpr, H, [64, 32], workspace_fill=U.CANARY)
    ids = x.token_selected_experts.cuda()
    shifted = []
    for i, p in enumerate(x.payloads):
        buf = torch.empty(p.numel() + 8, dtype=torch.uint8, device="cuda")
        v = buf[1 + 2 * i: 1 + 2 * i + p.numel()].view(p.shape)
        v.copy_(p.cuda())
        shifted.append(v)
    d = comm.dispatch(ids, x.local_num_tokens, shifted, tpr)
    torch.cuda.synchronize()
    plan = U.oracle_plan(w, x)
    for i, p in enumerate(x.payloads):
        for dst in range(ep):
            want = U.oracle.dispatch_payload(plan, p.numpy(), only_dst=dst, recv_init=np.full(
                (1, ep * tpr, p.shape[2]), U.CANARY, np.uint8))
            U.assert_equal(d.recv_payloads[i][dst], want, f"payload {i} rank {dst}")


def test_out_of_range_ids_and_duplicates():
    ep, E, k, tpr, H = 4, 16, 4, 8, 32
    ids = torch.tensor([[[-1, 16, 100, 3], [0, 1, 2, 3], [15, 15, 15, 15], [4, 8, 12, 0],
                         [-5, -5, 7, 7], [16, 17, 18, 19], [3, 2, 1, 0], [12, 9, 6, 3]]] * ep,
                       dtype=torch.int32)
    w, x = _custom(ep, E, k, tpr, H, [32], ids=ids, seed=9)
    run = U.Run(w, x)
    plan = U.oracle_plan(w, x)
    assert plan.num_dst[0].tolist() == [1, 1, 1, 4, 1, 0, 1, 4]
    U.check_plan(run, plan, w)
    U.check_payloads(run, plan, w, x)
    U.check_combine(run, plan, w, x)


@pytest.mark.parametrize("live", [[0], [3], [0, 5], list(range(1, 8))])
def test_rank_masks(live):
    ep, E, k, tpr, H = 8, 64, 6, 40, 64
    mask = [0, 0, 0, 0]
    for r in live:
        mask[0] |= 1 << r
    w, x = _custom(ep, E, k, tpr, H, [128, 24], n=[40, 1, 0, 39, 17, 40, 2, 33], mask=mask, seed=3)
    run = U.Run(w, x)
    plan = U.oracle_plan(w, x)
    U.check_plan(run, plan, w)
    U.check_payloads(run, plan, w, x)
    U.check_combine(run, plan, w, x)


def test_runtime_max_below_capacity_and_redispatch():
    """tokens_per_rank follows runtime_max_tokens_per_rank (slots src*tpr+t);
    a second dispatch on the same handle with another tpr fully replaces the plan."""
    from combine_route_plan_b200 import ep_a2a
    ep, E, k, H, cap = 8, 64, 4, 64, 96
    comm = ep_a2a.EpA2A(ep, E, k, cap, H, [64, 16], workspace_fill=U.CANARY)
    for tpr, seed in ((96, 1), (40, 2), (7, 3), (96, 4)):
        w, x = _custom(ep, E, k, tpr, H, [64, 16], n=[min(tpr, v) for v in
                                                         (tpr, 3, tpr, 0, 5, tpr - 1, 1, tpr)],
                       seed=seed)
        d = comm.dispatch(x.token_selected_experts.cuda(), x.local_num_tokens,
                          [p.cuda() for p in x.payloads], tpr if seed != 4 else 0)
        assert d.tokens_per_rank == tpr
        out = comm.combine(x.expert_output.cuda(), tokens_per_rank=tpr)
        torch.cuda.synchronize()
        plan = U.oracle_plan(w, x)
        nd = plan.num_dst.copy()
        nd[nd < 0] = 0xFF
        U.assert_equal(d.plan_num_dst, nd.astype(np.uint8), "plan_num_dst")
        U.assert_equal(d.recv_valid, plan.recv_valid, "recv_valid")
        U.assert_equal(d.recv_topk_ids, plan.recv_topk_ids, "recv_topk_ids")
        U.assert_equal(d.send_counts, plan.send_counts, "send_counts")
        want = U.oracle.combine(plan, U.to_np(x.expert_output), H,
                                out_init=U.to_np(out))  # absent rows: whatever out held
        exists = plan.num_dst >= 0
        got = U.to_np(out)
        assert np.array_equal(got[exists], want[exists])
        for i, p in enumerate(x.payloads):
            for dst in range(ep):
                g = d.recv_payloads[i][dst]
                pw = U.oracle.dispatch_payload(plan, p.numpy(), only_dst=dst)[0]
                valid = plan.recv_valid[dst] == 1
                U.assert_equal(g[torch.from_numpy(valid).cuda()], pw[valid], f"p{i} d{dst}")


def _check_valid_rows(d, plan, x, ep):
    """Plan arrays in full; payload rows where the plan says received."""
    nd = plan.num_dst.copy()
    nd[nd < 0] = 0xFF
    U.assert_equal(d.plan_num_dst, nd.astype(np.uint8), "plan_num_dst")
    U.assert_equal(d.recv_valid, plan.recv_valid, "recv_valid")
    U.assert_equal(d.recv_topk_ids, plan.recv_topk_ids, "recv_topk_ids")
    U.assert_equal(d.send_counts, plan.send_counts, "send_counts")
    for i, p in enumerate(x.payloads):
        for dst in range(ep):
            pw = U.oracle.dispatch_payload(plan, p.numpy(), only_dst=dst)[0]
            valid = plan.recv_valid[dst] == 1
            U.assert_equal(d.recv_payloads[i][dst][torch.from_numpy(valid).cuda()], pw[valid],
                           f"p{i} d{dst}")


def test_capacity_growth_serves_every_layer():
    """Layers of different sizes share one handle, grown on demand
    (vllm.distributed.device_communicators.all2all,
    FlashInferNVLinkOneSidedManager.initialize); every layer's dispatch and
    combine on the grown handle match the oracle, and options survive growth."""
    from combine_route_plan_b200 import ep_a2a
    ep, E, k = 4, 16, 4
    layers = [(24, 64, [128, 16]),
              (40, 32, [64, 16, 8]),      # more tokens, a smaller hidden, one more payload
              (16, 96, [256, 16]),        # a larger hidden and rows, fewer payloads
              (40, 64, [128, 16, 8])]     # fits
    comm = ep_a2a.EpA2A(ep, E, k, 24, 64, [128, 16], workspace_fill=U.CANARY)
    comm.set_option(ep_a2a.OPT_COMBINE_THREADS, 128)
    grew = []
    for i, (tpr, H, rows) in enumerate(layers):
        grew.append(comm.ensure_capacity(tpr, H, rows))
        w, x = _custom(ep, E, k, tpr, H, rows, n=[tpr, tpr - 3, 1, tpr], seed=40 + i)
        d = comm.dispatch(x.token_selected_experts.cuda(), x.local_num_tokens,
                          [p.cuda() for p in x.payloads], tpr)
        out = torch.full((ep, tpr, H), U.OUT_CANARY, dtype=torch.int16,
                         device="cuda").view(torch.bfloat16)
        comm.combine(x.expert_output.cuda(), out)
        torch.cuda.synchronize()
        assert comm.get_status() == ep_a2a.OK
        plan = U.oracle_plan(w, x)
        _check_valid_rows(d, plan, x, ep)
        U.assert_equal(out, U.oracle.combine(plan, U.to_np(x.expert_output), H,
                                             out_init=U.oracle_out_init(w)), f"combine {i}")
    assert grew == [False, True, True, False]
    assert (comm.params.max_tokens_per_rank, comm.params.hidden_size) == (40, 96)
    assert comm.payload_row_bytes == [256, 16, 8]
    assert comm._options[ep_a2a.OPT_COMBINE_THREADS] == 128


def test_combine_rows_shorter_than_the_handle_hidden():
    """A handle sized for hidden 128 combines rows of 64, 40 and 128 elements
    (BF16, FP8, expert outputs and scaled FP8), each matching the oracle."""
    from combine_route_plan_b200 import ep_a2a
    ep, E, k, tpr, Hcap = 4, 16, 4, 30, 128
    comm = ep_a2a.EpA2A(ep, E, k, tpr, Hcap, [32], workspace_fill=U.CANARY)
    for H in (64, 40, 128, 16):
        w, x = _custom(ep, E, k, tpr, H, [32], n=[30, 0, 17, 29], seed=60 + H)
        comm.dispatch(x.token_selected_experts.cuda(), x.local_num_tokens,
                      [p.cuda() for p in x.payloads], tpr)
        plan = U.oracle_plan(w, x)
        xo = x.expert_output
        out = comm.combine(xo.cuda())
        q = ep_a2a.quantize_e4m3(xo.cuda())
        out8 = comm.combine(q)
        g = torch.Generator().manual_seed(H)
        wts = torch.randn((ep, tpr, k), generator=g)
        y = torch.randn((ep, tpr, k, H), generator=g).to(torch.bfloat16)
        oute = comm.combine_experts(wts.cuda(), y.cuda())
        codes, scales = ep_a2a.quantize_e4m3_rows(xo.cuda())
        outs = comm.combine_scaled(codes, scales)
        torch.cuda.synchronize()
        assert comm.get_status() == ep_a2a.OK
        exists = plan.num_dst >= 0
        xq = U.oracle_quantize_big(U.to_np(xo), U.oracle_e4m3_table())
        oc, osc = U.oracle.quantize_e4m3_rows(U.to_np(xo), H)
        for got, want, what in [
                (out, U.oracle.combine(plan, U.to_np(xo), H), "bf16"),
                (out8, U.oracle.combine(plan, xq, H, input_is_e4m3=True), "fp8"),
                (oute, U.oracle.combine_experts(plan, E, x.token_selected_experts.numpy(),
                                                wts.numpy(), U.to_np(y), H), "experts"),
                (outs, U.oracle.combine_scaled(plan, oc, osc, H), "scaled")]:
            assert np.array_equal(U.to_np(got)[exists], want[exists]), (H, what)
    with pytest.raises(ep_a2a.EpA2AError) as e:
        ep_a2a.ep_a2a_set_combine_hidden(comm.handle, Hcap + 1)
    assert e.value.status == ep_a2a.ERR_CAPACITY
    with pytest.raises(ep_a2a.EpA2AError) as e:
        ep_a2a.ep_a2a_set_combine_hidden(comm.handle, 0)
    assert e.value.status == ep_a2a.ERR_INVALID_ARG


def test_counts_scratch_resets_between_calls():
    """Both routing paths leave the count accumulators and tickets at zero, so
    repeated dispatches, alternating between them, count afresh each time."""
    from combine_route_plan_b200 import ep_a2a
    w = W.scaled(W.C2, 64)
    x = W.make_inputs(w, with_expert_output=False)
    run = U.Run(w, x)
    plan = U.oracle_plan(w, x)
    for i in range(6):
        run.comm.set_option(ep_a2a.OPT_ROUTE_IN_COPY, i % 3 != 1)
        run.comm.dispatch(run.ids, x.local_num_tokens, run.payloads, w.tokens_per_rank)
        torch.cuda.synchronize()
        U.assert_equal(run.d.send_counts, plan.send_counts, "send_counts after repeat")


def test_nan_in_invalid_rows_never_reaches_output():
    w = W.C1
    x = W.make_inputs(w)
    plan = U.oracle_plan(w, x)
    xo = x.expert_output.clone()
    flat = xo.view(w.ep_size, -1, w.hidden)
    for d in range(w.ep_size):
        invalid = torch.from_numpy(plan.recv_valid[d] != 1)
        flat[d][invalid] = float("nan")
    x2 = W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads, None, None, xo)
    run = U.Run(w, x2)
    assert not torch.isnan(run.out.float()).any()
    U.check_combine(run, plan, w, x2)


def test_ones_combine_counts_destinations():
    w = W.C5
    x = _inputs(w.name)
    ones = torch.ones_like(x.expert_output)
    x2 = W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads[:0], None,
                  x.active_rank_mask, ones)
    run = U.Run(w, x2)
    plan = U.oracle_plan(w, x)
    got = run.out.float().cpu().numpy()
    for r in range(w.ep_size):
        for t in range(w.tokens_per_rank):
            if plan.num_dst[r, t] >= 0:
                assert np.all(got[r, t] == plan.num_dst[r, t])


# --------------------------------------------------------------------------- #
# Host validation that needs a live handle, and the bounded-wait status path
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("option,good,bad", [
    ("VEC_CTAS_PER_SM", [0, 1, 4, 64], [-1, 65]),
    ("COPY_PREFETCH", [-1, 0, 1], [-2, 2]),
    ("COMBINE_PREFETCH", [-1, 0, 1, 4], [-2, 5]),
    ("COMBINE_THREADS", [0, 64, 96, 128, 192, 512], [32, 100, 544]),
    ("COMBINE_CTAS_PER_SM", [0, 1, 1024], [-1, 1025]),
    ("VEC_THREADS_PER_TOKEN", [0, 32, 64, 128, 256], [16, 48, 512]),
    ("FP8_EXPERTS_KERNEL", [0, 1, 2], [-1, 3]),
])
def test_option_ranges(option, good, bad):
    """Every value an option documents is accepted and the ones outside are
    rejected with EP_A2A_ERR_INVALID_ARG, leaving the handle usable."""
    from combine_route_plan_b200 import ep_a2a
    comm = ep_a2a.EpA2A(4, 16, 2, 8, 32, [32])
    opt = getattr(ep_a2a, "OPT_" + option)
    for v in good:
        comm.set_option(opt, v)
    for v in bad:
        with pytest.raises(ep_a2a.EpA2AError) as e:
            comm.set_option(opt, v)
        assert e.value.status == ep_a2a.ERR_INVALID_ARG
    ids = torch.zeros((4, 8, 2), dtype=torch.int32, device="cuda")
    pay = torch.zeros((4, 8, 32), dtype=torch.uint8, device="cuda")
    comm.dispatch(ids, [8] * 4, [pay], 8)
    torch.cuda.synchronize()
    assert comm.get_status() == ep_a2a.OK


def test_dispatch_and_combine_validation():
    from combine_route_plan_b200 import ep_a2a
    ep, E, k, tpr, H = 4, 16, 2, 8, 32
    comm = ep_a2a.EpA2A(ep, E, k, tpr, H, [32], eplb_stats_num_experts=0)
    ids = torch.zeros((ep, tpr, k), dtype=torch.int32, device="cuda")
    pay = torch.zeros((ep, tpr, 32), dtype=torch.uint8, device="cuda")
    stats = torch.zeros((ep, E), dtype=torch.int32, device="cuda")
    xo = torch.zeros((ep, ep * tpr, H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ep_a2a.EpA2AError) as e:
        comm.combine(xo)
    assert e.value.status == ep_a2a.ERR_NO_PLAN

    def raw(handle=None, n=None, runtime=tpr, rb=(32,), stats_ptr=0, mask=None):
        return ep_a2a.ep_a2a_dispatch(handle or comm.handle, ids.data_ptr(),
                                      n if n is not None else [tpr] * ep, runtime,
                                      [pay.data_ptr()], list(rb), stats_ptr, mask)

    cases = [
        (dict(runtime=tpr + 1), ep_a2a.ERR_CAPACITY),
        (dict(n=[tpr + 1, 0, 0, 0]), ep_a2a.ERR_INVALID_ARG),
        (dict(n=[-1, 0, 0, 0]), ep_a2a.ERR_INVALID_ARG),
        (dict(mask=[0b1111]), ep_a2a.ERR_INVALID_ARG),          # mask without enable_rank_mask
        (dict(stats_ptr=stats.data_ptr()), ep_a2a.ERR_INVALID_ARG),  # EPLB not enabled
        (dict(rb=(48,)), ep_a2a.ERR_CAPACITY),                  # row above capacity
        (dict(rb=(0,)), ep_a2a.ERR_CAPACITY),
    ]
    for kw, status in cases:
        with pytest.raises(ep_a2a.EpA2AError) as e:
            raw(**kw)
        assert e.value.status == status, kw
    masked = ep_a2a.EpA2A(ep, E, k, tpr, H, [32], enable_rank_mask=True)
    with pytest.raises(ep_a2a.EpA2AError) as e:       # no live rank below ep_size
        raw(handle=masked.handle, mask=[0b10000])
    assert e.value.status == ep_a2a.ERR_INVALID_ARG
    comm.dispatch(ids, [1] * ep, [pay])
    comm.combine(xo)
    torch.cuda.synchronize()
    comm.destroy()
    comm.destroy()                                    # idempotent
    with pytest.raises(ep_a2a.EpA2AError) as e:
        comm.combine(xo)
    assert e.value.status == ep_a2a.ERR_NOT_INITIALIZED


def test_bounded_wait_reports_timeout_and_context_survives():
    from combine_route_plan_b200 import ep_a2a
    w = W.C1
    x = W.make_inputs(w)
    run = U.Run(w, x)
    ep_a2a.ep_a2a_debug_wait_probe(run.comm.handle, 20_000_000)     # 20 ms
    assert run.comm.get_status() == ep_a2a.ERR_DEVICE_TIMEOUT
    assert run.comm.get_status() == ep_a2a.OK                       # the word was cleared
    run2 = U.Run(w, x)                                               # context still usable
    plan = U.oracle_plan(w, x)
    U.check_plan(run2, plan, w)
    U.check_combine(run2, plan, w, x)


# --------------------------------------------------------------------------- #
# Combine of per-expert outputs (weighted local reduction fused into combine)
# --------------------------------------------------------------------------- #

def _expert_outputs(w, seed):
    """bf16 [ep, tpr, k, H] N(0,1) expert outputs, one row per (token, slot),
    drawn by a seeded CUDA generator (fast at the prefill size) and kept on the
    host, where the oracle reads them."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = (w.ep_size, w.tokens_per_rank, w.top_k, w.hidden)
    return torch.randn(shape, generator=g, device="cuda", dtype=torch.bfloat16).cpu()


def _check_combine_experts(w, x, y, wts, options=None):
    from combine_route_plan_b200 import ep_a2a
    run = U.Run(w, W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads,
                            x.eplb_local_stats, x.active_rank_mask, None), options=options)
    out = torch.full((w.ep_size, w.tokens_per_rank, w.hidden), U.OUT_CANARY, dtype=torch.int16,
                     device="cuda").view(torch.bfloat16)
    run.comm.combine_experts(wts.cuda(), y.cuda(), out)
    torch.cuda.synchronize()
    assert run.comm.get_status() == ep_a2a.OK
    plan = U.oracle_plan(w, x)
    want = U.oracle.combine_experts(plan, w.num_experts, x.token_selected_experts.numpy(),
                                    wts.numpy(), U.to_np(y), w.hidden,
                                    out_init=U.oracle_out_init(w))
    U.assert_equal(out, want, "combine of expert outputs")


@pytest.mark.parametrize("name", ["c1_ep4_tiny", "c2_ep8_decode", "c5_ep64_wide_masked",
                                  "c4_ep8_prefill", "c3_ep16_zipf_nvfp4"])
def test_combine_experts_bit_exact(name):
    w = W.BY_NAME[name]
    x = _inputs(w.name)
    wts = x.payloads[-1].view(torch.float32).view(w.ep_size, w.tokens_per_rank, w.top_k)
    y = _expert_outputs(w, seed=w.seed + 77)
    _check_combine_experts(w, x, y, wts)


@pytest.mark.parametrize("ep,E,k,tpr,H", [
    (3, 12, 3, 37, 100),     # hidden not a multiple of 8: element path
    (16, 64, 16, 20, 64),    # top_k above 8: element path
    (4, 16, 5, 33, 40),      # top_k 5, vector path
    (8, 64, 8, 40, 64),
])
def test_combine_experts_edge_shapes(ep, E, k, tpr, H):
    w, x = _custom(ep, E, k, tpr, H, [16], seed=ep * 13 + k)
    g = torch.Generator().manual_seed(k)
    wts = torch.randn((ep, tpr, k), generator=g)
    y = torch.randn((ep, tpr, k, H), generator=g).to(torch.bfloat16)
    _check_combine_experts(w, x, y, wts)


def test_combine_experts_with_masks_and_invalid_ids():
    ep, E, k, tpr, H = 8, 64, 6, 40, 64
    mask = [0b10110111, 0, 0, 0]
    w, x = _custom(ep, E, k, tpr, H, [32], n=[40, 1, 0, 39, 17, 40, 2, 33], mask=mask, seed=21)
    ids = x.token_selected_experts.clone()
    ids[0, :5, 0] = -3
    ids[1, 0, 1] = 64
    x = W.Inputs(w, ids, x.local_num_tokens, x.payloads, None, x.active_rank_mask, None)
    g = torch.Generator().manual_seed(5)
    wts = torch.randn((ep, tpr, k), generator=g)
    y = torch.randn((ep, tpr, k, H), generator=g).to(torch.bfloat16)
    _check_combine_experts(w, x, y, wts)


# --------------------------------------------------------------------------- #
# Low-precision combine of per-expert outputs, quantised on the sending side
# --------------------------------------------------------------------------- #

def _check_combine_experts_fp8(w, x, y, wts, options=None):
    from combine_route_plan_b200 import ep_a2a
    run = U.Run(w, W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads,
                            x.eplb_local_stats, x.active_rank_mask, None), options=options)
    out = torch.full((w.ep_size, w.tokens_per_rank, w.hidden), U.OUT_CANARY, dtype=torch.int16,
                     device="cuda").view(torch.bfloat16)
    run.comm.combine_experts_fp8(wts.cuda(), y.cuda(), out)
    torch.cuda.synchronize()
    assert run.comm.get_status() == ep_a2a.OK
    plan = U.oracle_plan(w, x)
    want = U.oracle.combine_experts_fp8(plan, w.num_experts, x.token_selected_experts.numpy(),
                                        wts.numpy(), U.to_np(y), w.hidden,
                                        out_init=U.oracle_out_init(w))
    U.assert_equal(out, want, "sender-side FP8 combine of expert outputs")
    return out, plan, want


@pytest.mark.parametrize("name", ["c1_ep4_tiny", "c2_ep8_decode", "c5_ep64_wide_masked",
                                  "c3_ep16_zipf_nvfp4", "c4_ep8_prefill"])
def test_combine_experts_fp8_bit_exact(name):
    w = W.BY_NAME[name]
    x = _inputs(w.name)
    wts = x.payloads[-1].view(torch.float32).view(w.ep_size, w.tokens_per_rank, w.top_k)
    y = _expert_outputs(w, seed=w.seed + 91)
    out, plan, want = _check_combine_experts_fp8(w, x, y, wts)
    # the stated bar against the same oracle, element by element (bit-exact
    # already implies it; kept as the figure the bar is quoted on)
    exists = plan.num_dst >= 0
    g = U.bits_f32(U.to_np(out)[exists]).astype(np.float64)
    o = U.bits_f32(want[exists]).astype(np.float64)
    rel = np.abs(g - o) / np.maximum(np.abs(o), 1e-30)
    rel[g == o] = 0.0
    assert rel.max() <= 2.0 ** -3


@pytest.mark.parametrize("ep,E,k,tpr,H", [
    (3, 12, 3, 37, 100),     # hidden not a multiple of 8: element kernel
    (16, 64, 16, 20, 64),    # top_k above 8: element kernel
    (4, 16, 5, 33, 40),      # top_k 5, shared-memory kernel
    (8, 64, 8, 40, 64),
    (2, 8, 8, 16, 8192),     # the widest rows of the shared-memory kernel at two ranks
])
def test_combine_experts_fp8_edge_shapes(ep, E, k, tpr, H):
    w, x = _custom(ep, E, k, tpr, H, [16], seed=ep * 17 + k)
    g = torch.Generator().manual_seed(k + 3)
    wts = torch.randn((ep, tpr, k), generator=g)
    y = (torch.randn((ep, tpr, k, H), generator=g) *
         torch.exp(torch.randn((ep, tpr, k, 1), generator=g) * 2)).to(torch.bfloat16)
    _check_combine_experts_fp8(w, x, y, wts)


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("case", ["c2_ep8_decode", "c5_ep64_wide_masked", (4, 16, 5, 33, 40),
                                  (2, 8, 8, 16, 8192), (4, 16, 4, 20, 7168 + 256)])
def test_combine_experts_fp8_other_kernels(case, kernel):
    """The two other kernels of the sender-side FP8 expert combine: a cluster per
    token with one column vector per thread and the rows z_d in registers (1),
    and one CTA per token with the whole rows in shared memory (2); the default
    splits each token over a cluster with the rows of each slice in shared
    memory."""
    from combine_route_plan_b200 import ep_a2a
    if isinstance(case, str):
        w = W.BY_NAME[case]
        x = _inputs(w.name)
        wts = x.payloads[-1].view(torch.float32).view(w.ep_size, w.tokens_per_rank, w.top_k)
        y = _expert_outputs(w, seed=w.seed + 93)
    else:
        ep, E, k, tpr, H = case
        w, x = _custom(ep, E, k, tpr, H, [16], seed=ep * 19 + k)
        g = torch.Generator().manual_seed(k + 5)
        wts = torch.randn((ep, tpr, k), generator=g)
        y = torch.randn((ep, tpr, k, H), generator=g).to(torch.bfloat16)
    _check_combine_experts_fp8(w, x, y, wts, options={ep_a2a.OPT_FP8_EXPERTS_KERNEL: kernel})


def test_combine_experts_fp8_masks_invalid_ids_and_zero_rows():
    ep, E, k, tpr, H = 8, 64, 6, 40, 64
    mask = [0b10110111, 0, 0, 0]
    w, x = _custom(ep, E, k, tpr, H, [32], n=[40, 1, 0, 39, 17, 40, 2, 33], mask=mask, seed=29)
    ids = x.token_selected_experts.clone()
    ids[0, :5, 0] = -3
    ids[1, 0, 1] = 64
    x = W.Inputs(w, ids, x.local_num_tokens, x.payloads, None, x.active_rank_mask, None)
    g = torch.Generator().manual_seed(9)
    wts = torch.randn((ep, tpr, k), generator=g)
    wts[3, :4] = 0.0                 # rows z_d of zeros: scale and inverse 1
    y = torch.randn((ep, tpr, k, H), generator=g).to(torch.bfloat16)
    _check_combine_experts_fp8(w, x, y, wts)


# --------------------------------------------------------------------------- #
# FP8 combine with one scale per row
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("hidden,rows", [(7168, 4096), (100, 333), (16, 7), (8192, 64)])
def test_quantize_rows_matches_oracle(hidden, rows):
    from combine_route_plan_b200 import ep_a2a
    g = torch.Generator().manual_seed(hidden + rows)
    x = torch.randn((rows, hidden), generator=g) * torch.exp(torch.randn((rows, 1), generator=g) * 3)
    x[rows // 2] = 0.0
    xb = x.to(torch.bfloat16)
    codes, scales = ep_a2a.quantize_e4m3_rows(xb.cuda())
    torch.cuda.synchronize()
    oc, osc = U.oracle.quantize_e4m3_rows(U.to_np(xb), hidden)
    U.assert_equal(codes.view(torch.uint8), oc, "row codes")
    U.assert_equal(scales, osc, "row scales")


@pytest.mark.parametrize("name", ["c2_ep8_decode", "c5_ep64_wide_masked", "c1_ep4_tiny",
                                  "c3_ep16_zipf_nvfp4", "c4_ep8_prefill"])
def test_combine_scaled_bit_exact(name):
    from combine_route_plan_b200 import ep_a2a
    w = W.BY_NAME[name]
    x = _inputs(w.name)
    run = U.Run(w, W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads,
                            x.eplb_local_stats, x.active_rank_mask, None))
    xo = x.expert_output
    codes, scales = ep_a2a.quantize_e4m3_rows(xo.cuda())
    out = torch.full((w.ep_size, w.tokens_per_rank, w.hidden), U.OUT_CANARY, dtype=torch.int16,
                     device="cuda").view(torch.bfloat16)
    run.comm.combine_scaled(codes, scales, out)
    torch.cuda.synchronize()
    assert run.comm.get_status() == ep_a2a.OK
    plan = U.oracle_plan(w, x)
    oc, osc = U.oracle_row_quantize_read(U.to_np(xo), plan, w.hidden)
    want = U.oracle.combine_scaled(plan, oc, osc, w.hidden, out_init=U.oracle_out_init(w))
    U.assert_equal(out, want, "scaled fp8 combine")
    # against the unquantized bf16 combine: E4M3 keeps 3 mantissa bits per term
    ref = U.oracle.combine(plan, U.to_np(xo), w.hidden)
    exists = plan.num_dst >= 0
    got = U.bits_f32(U.to_np(out)[exists]).astype(np.float64)
    exact = U.bits_f32(ref[exists]).astype(np.float64)
    absx = np.abs(U.bits_f32(U.to_np(xo))).max()
    assert np.max(np.abs(got - exact)) <= 8 * 2.0 ** -4 * absx


def test_combine_scaled_odd_hidden():
    from combine_route_plan_b200 import ep_a2a
    ep, E, k, tpr, H = 4, 16, 4, 30, 40
    w, x = _custom(ep, E, k, tpr, H, [16], seed=31)
    run = U.Run(w, W.Inputs(w, x.token_selected_experts, x.local_num_tokens, x.payloads, None,
                            None, None))
    codes, scales = ep_a2a.quantize_e4m3_rows(x.expert_output.cuda())
    out = run.comm.combine_scaled(codes, scales)
    torch.cuda.synchronize()
    oc, osc = U.oracle.quantize_e4m3_rows(U.to_np(x.expert_output), H)
    plan = U.oracle_plan(w, x)
    want = U.oracle.combine_scaled(plan, oc, osc, H)
    exists = plan.num_dst >= 0
    assert np.array_equal(U.to_np(out)[exists], want[exists])


# --------------------------------------------------------------------------- #
# Dense variant: all-gather dispatch, reduce-scatter combine
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("name", ["c1_ep4_tiny", "c2_ep8_decode", "c5_ep64_wide_masked"])
def test_dense_allgather_and_reduce_scatter(name):
    from combine_route_plan_b200 import ep_a2a
    w = W.BY_NAME[name]
    x = _inputs(w.name)
    ep, tpr, H = w.ep_size, w.tokens_per_rank, w.hidden
    rows = w.payload_row_bytes()
    offs, off = [], 0
    for rb in rows:
        offs.append(off)
        off += (ep * tpr * rb + 255) // 256 * 256
    stride = off
    recv = torch.full((ep, stride), U.CANARY, dtype=torch.uint8, device="cuda")
    pays = [p.cuda() for p in x.payloads]
    ep_a2a.ep_a2a_allgather(ep, tpr, x.local_num_tokens, [p.data_ptr() for p in pays], rows,
                            [recv.data_ptr() + o for o in offs], stride, x.active_rank_mask)
    xo = x.expert_output.cuda()
    out = torch.full((ep, tpr, H), U.OUT_CANARY, dtype=torch.int16, device="cuda") \
        .view(torch.bfloat16)
    ep_a2a.ep_a2a_reduce_scatter(ep, tpr, H, x.local_num_tokens, xo.data_ptr(), out.data_ptr(),
                                 x.active_rank_mask)
    torch.cuda.synchronize()
    for i, (p, rb) in enumerate(zip(x.payloads, rows)):
        want = U.oracle.allgather(ep, tpr, x.local_num_tokens, p.numpy(), x.active_rank_mask)
        got = recv[:, offs[i]:offs[i] + ep * tpr * rb]
        U.assert_equal(got, want, f"allgather payload {i}")
    want = U.oracle.reduce_scatter(ep, tpr, H, x.local_num_tokens, U.to_np(x.expert_output),
                                   x.active_rank_mask)
    U.assert_equal(out, want, "reduce_scatter")


def test_reduce_scatter_element_path():
    from combine_route_plan_b200 import ep_a2a
    ep, tpr, H = 3, 10, 100
    g = torch.Generator().manual_seed(3)
    xo = torch.randn((ep, ep * tpr, H), generator=g).to(torch.bfloat16)
    n = [10, 4, 0]
    out = torch.full((ep, tpr, H), U.OUT_CANARY, dtype=torch.int16, device="cuda") \
        .view(torch.bfloat16)
    ep_a2a.ep_a2a_reduce_scatter(ep, tpr, H, n, xo.cuda().data_ptr(), out.data_ptr())
    torch.cuda.synchronize()
    U.assert_equal(out, U.oracle.reduce_scatter(ep, tpr, H, n, U.to_np(xo)), "reduce_scatter")

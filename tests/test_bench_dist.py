"""The N > 1 path of bench.py on CPU: world-size-2 gloo groups.

bench.py runs one independent replica per GPU and reports the max over ranks
of the timed region; these tests exercise that harness (barriers, the max
reduction, rank-0-only output) without a GPU."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import time
    import bench
    dist = bench.init_group("gloo", timeout_s=60)
    sleep_s = 0.01 * (rank + 1)          # rank 1 is the slower one
    ms = bench.run_timed(lambda: time.sleep(sleep_s), steps=5, warmup=3,
                         timer=bench.WallTimer(), dist=dist)
    mx = bench.reduce_max(float(rank * 10 + 1), dist)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"ms": ms, "max": mx}, f)
    dist.destroy_process_group()


def test_run_timed_takes_the_max_over_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0 = json.load(open(tmp_path / "r0.json"))
    r1 = json.load(open(tmp_path / "r1.json"))
    assert r0["ms"] == r1["ms"]                 # both ranks report the same (max) time
    assert r0["ms"] >= 5 * 20.0 * 0.95          # at least the slow rank's 5 x 20 ms
    assert r0["max"] == r1["max"] == 11.0


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1",
           "--ref-budget-s", "2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                       # rank 0 alone prints
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "tokens/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_algorithmic_bytes_of_the_prefill_step():
    sys.path.insert(0, ROOT)
    import bench
    from combine_route_plan_b200 import workloads as W
    w = W.C4
    n_tok, sum_d = 32768, 173434
    b = bench.algorithmic_bytes(w, n_tok, sum_d, live=8, fp8=False)
    rb = 14336 + 64 + 32
    assert b.copy == n_tok * rb + sum_d * rb
    assert b.combine == sum_d * 7168 * 2 + n_tok * 7168 * 2
    b8 = bench.algorithmic_bytes(w, n_tok, sum_d, live=8, fp8=True)
    assert b8.combine == sum_d * 7168 + n_tok * 7168 * 2


def test_all_cores_oracle_baseline_runs_spawned_processes():
    sys.path.insert(0, ROOT)
    import bench
    from combine_route_plan_b200 import workloads as W
    rec = bench.cpu_baseline_all_cores(W.C1, 0.5, tokens_per_rank=16, procs=2)
    assert rec["cores"] == 2 and rec["kind"] == "oracle" and rec["value"] > 0
    assert "2 single-threaded processes" in rec["sample"]


def test_algorithmic_bytes_of_the_expert_output_combine():
    sys.path.insert(0, ROOT)
    import bench
    from combine_route_plan_b200 import workloads as W
    w = W.C4
    n_tok, sum_d, slots = 32768, 173434, 32768 * 8
    b = bench.algorithmic_bytes(w, n_tok, sum_d, live=8, fp8=False, live_slots=slots)
    # one bf16 row per (token, slot), the ids and weights, one bf16 output row
    assert b.combine == slots * 7168 * 2 + n_tok * 8 * 8 + n_tok * 7168 * 2
    assert b.step == b.copy + b.combine + b.route


def test_kernel_sources_hash_ignores_comments_only():
    sys.path.insert(0, ROOT)
    import bench
    code = "__global__ void k(int* p) { p[0] = 1; }\n"
    commented = ("// a comment\n/* a block\n   comment */\n__global__ void k(int* p) {\n"
                 "  p[0] = 1;  // trailing\n}\n")
    assert bench._code_only(code) == bench._code_only(commented)
    assert bench._code_only(code) != bench._code_only(code.replace("1;", "2;"))


def test_committed_traffic_only_for_the_sources_it_was_taken_on(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    assert bench.committed_traffic("copy_vec", "c4_ep8_prefill") == (
        rec["kernels"]["copy_vec"]["dram_bytes_per_launch"]
        if rec["sources_hash"] == bench.kernel_sources_hash() else None)
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda: "0" * 16)
    assert bench.committed_traffic("copy_vec", "c4_ep8_prefill") is None
    assert bench.committed_traffic("copy_vec", "c2_ep8_decode") is None


def test_l2_note_says_which_rule_the_timing_meets():
    sys.path.insert(0, ROOT)
    import bench
    l2 = 126 << 20
    assert bench.l2_note(True, 10 ** 8, l2).startswith("512 MB L2 flush")
    assert bench.l2_note(False, 5_938_896_128, l2).startswith("inputs larger than L2")
    assert bench.l2_note(False, 185_000_000, l2).startswith("no flush, warm L2")

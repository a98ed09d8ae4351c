"""Host-side logic of bench.py on CPU: byte accounting, request sampling, the
reference (oracle) arm, and the max/sum-over-ranks reductions with two gloo
ranks."""
import json
import os
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_kv_flight_b200 import workloads  # noqa: E402


def test_metric_bytes_by_hand():
    # two requests, L = 0 and 15 -> n = 1 and 16 tokens; Hkv 2, d 64, bf16
    kv = 2 * 2 * (1 + 16) * 64 * 2
    qo = 2 * 2 * 8 * 64 * 2
    assert bench.metric_bytes([0, 15], 8, 2, 64, 16, False) == kv + qo
    # E4M3: one byte per element plus two fp32 scales per attended (page, kv head)
    kv8 = 2 * 2 * (1 + 16) * 64 * 1
    scales = 2 * (1 + 1) * 2 * 4
    assert bench.metric_bytes([0, 15], 8, 2, 64, 16, True) == kv8 + qo + scales


def test_metric_bytes_with_several_new_tokens_by_hand():
    # L = 0 and 15 with 3 new tokens each -> 3 and 18 tokens read once per
    # (request, kv head); q and out for 3 tokens per request
    kv = 2 * 2 * (3 + 18) * 64 * 2
    qo = 2 * 2 * 3 * 8 * 64 * 2
    assert bench.metric_bytes([0, 15], 8, 2, 64, 16, False, q_len=3) == kv + qo


def test_full_step_bytes_by_hand():
    # L = 0 and 15 -> 1 and 16 attended tokens over 1 and 1 pages (P 16); Hq 8, Hkv 2, d 64
    metric = bench.metric_bytes([0, 15], 8, 2, 64, 16, False)
    rope = 2 * (2 * 8 * 64 * 2          # q read and written back
                + 2 * 2 * 64 * 2        # k_new, v_new read
                + 2 * 2 * 64 * 2        # k, v rows written (bf16)
                + 4)                    # the landing page's block-table entry
    index = (1 + 1) * 4 + 2 * 2 * 4     # attended pages' entries; seq_lens read by both kernels
    assert bench.full_step_bytes([0, 15], 8, 2, 64, 16, False) == metric + rope + index
    # E4M3: one byte per stored element, plus the landing page's two scales per kv head
    metric8 = bench.metric_bytes([0, 15], 8, 2, 64, 16, True)
    rope8 = 2 * (2 * 8 * 64 * 2 + 2 * 2 * 64 * 2 + 2 * 2 * 64 * 1 + 4 + 2 * 2 * 4)
    assert bench.full_step_bytes([0, 15], 8, 2, 64, 16, True) == metric8 + rope8 + index
    # several new tokens: L = 15 with 3 new -> 18 tokens over 2 pages
    m3 = bench.metric_bytes([15], 8, 2, 64, 16, False, q_len=3)
    r3 = 3 * (2 * 8 * 64 * 2 + 2 * 2 * 64 * 2 + 2 * 2 * 64 * 2 + 4)
    assert bench.full_step_bytes([15], 8, 2, 64, 16, False, q_len=3) == m3 + r3 + 2 * 4 + 2 * 4


def test_full_step_bytes_stay_near_the_metric_on_every_workload():
    for name in workloads.CONFIG_NAMES:
        w = workloads.make(name)
        by, full = bench.workload_bytes(w), bench.full_step_bytes(w.seq_lens, w.Hq, w.Hkv, w.d, w.P, w.kv_fp8,
                                                                  w.q_len)
        assert by < full < 1.1 * by + 64 * 1024, name


def test_host_cpu_reports_a_model_and_thread_count():
    info = bench.host_cpu()
    assert isinstance(info["cpu_model"], str) and info["cpu_model"]
    assert info["host_threads"] >= 1


def test_llama8b_bytes_near_the_recipe_estimate():
    w_lens = workloads.draw_lengths("llama8b", np.random.default_rng(workloads.config_seed("llama8b")))
    by = bench.metric_bytes(w_lens, 32, 8, 128, 32, False)
    assert 4.5e8 < by < 6.5e8


def test_sample_requests_respects_budget():
    w = workloads.make("tiny")
    picks = bench.sample_requests(w, 100)
    assert picks == [0]                      # at least one request
    picks = bench.sample_requests(w, 10**9)
    assert picks == list(range(w.batch))


def test_reference_arm_prints_one_json_line_on_cpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                        "tiny", "--steps", "3", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=600, check=True)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["cpu_baseline"]["host_threads"] >= 1 and d["cpu_baseline"]["cpu_model"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    # the config object is the workload's, the same one the GPU arm prints
    assert d["config"] == bench.workload_config(workloads.make("tiny"), "tiny", 1)


def test_reference_sample_cuts_a_request_that_exceeds_the_step_budget():
    """A step budget below one request (long contexts: one request of 32k-128k
    tokens x 8 kv heads times 1000 steps would run for an hour) cuts the
    sampled request to the cached tokens that fit, at least one page."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                        "tiny", "--steps", "3", "--warmup", "3", "--ref-budget", "8"], capture_output=True,
                       text=True, env=env, timeout=600, check=True)
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    w = workloads.make("tiny")                     # first request: 17 cached tokens, page 16, Hkv 2
    assert "cut to its first 16 cached tokens" in d["cpu_baseline"]["sample"]
    assert d["metric_bytes_per_step_sampled"] == bench.metric_bytes([16], w.Hq, w.Hkv, w.d, w.P, w.kv_fp8)


def test_default_suite_ends_on_the_largest_workload():
    assert bench.DEFAULT_CONFIG == "suite"
    sizes = {n: bench.workload_bytes(workloads.make(n)) for n in bench.SUITE}
    assert bench.SUITE[-1] == "longctx" and sizes["longctx"] == max(sizes.values())
    assert {"llama8b", "hetero70b", "fp8", "spec4"} <= set(bench.SUITE)


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(1.5 + rank)
        sm = bench.sum_over_ranks(10.0 * (rank + 1))
        bench.barrier()
        q.put((rank, mx, sm))
    finally:
        dist.destroy_process_group()


def test_rank_reductions_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [2.5, 2.5]
    assert [r[2] for r in res] == [30.0, 30.0]


def test_reference_arm_under_torchrun_prints_once_from_rank_zero():
    """Launched like the multi-GPU runs (torchrun, two ranks), the reference
    arm runs on rank 0 alone: one JSON line, every rank exits 0."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    port = 29700 + (os.getpid() % 200)
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port),
                        os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=600, check=True)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0


def test_one_gpu_suite_runs_each_workload_in_its_own_process(monkeypatch, capsys):
    # the children's command lines carry the parent's flags, each workload's
    # name and its CPU-baseline budget (short before the last line); their
    # JSON lines are passed on in order
    import subprocess
    calls = []

    class Done:
        def __init__(self, cmd):
            self.returncode = 0
            self.stdout = "noise\n" + json.dumps({"workload": cmd[cmd.index("--config") + 1]}) + "\n"

    def fake_run(cmd, stdout=None, text=None):
        calls.append(cmd)
        return Done(cmd)

    monkeypatch.setattr(subprocess, "run", fake_run)
    assert bench.main(["--steps", "7", "--warmup", "4", "--no-e2e"]) == 0
    assert [c[c.index("--config") + 1] for c in calls] == list(bench.SUITE)
    budgets = [float(c[c.index("--cpu-budget") + 1]) for c in calls]
    assert budgets[:-1] == [5.0] * (len(calls) - 1) and budgets[-1] == 20.0
    for c in calls:
        assert c[c.index("--steps") + 1] == "7" and c[c.index("--warmup") + 1] == "4" and "--no-e2e" in c
    out = [json.loads(ln)["workload"] for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert out == list(bench.SUITE)

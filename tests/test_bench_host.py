"""Host-side checks of bench.py (no GPU): the multi-rank aggregation over a real
two-rank gloo group, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench
    try:
        q.put((rank, bench.max_over_ranks(1.5 + rank, world, "cpu")))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    """Each rank's per-step time goes in, every rank gets the slowest one back."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == {0: 2.5, 1: 2.5}


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25


def _run_bench(args, env_extra=None, timeout=600):
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout, env=env)


def test_reference_arm_json_line():
    """--impl reference times the oracle and prints one JSON line of the contract."""
    r = _run_bench(["--impl", "reference", "--workload", "tiny_t8_int4_f32", "--steps", "2",
                    "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny_t8_int4_f32"


def test_reference_arm_other_ranks_print_nothing():
    """Under torchrun only rank 0 runs the reference arm; the others exit 0 quietly."""
    r = _run_bench(["--impl", "reference", "--workload", "tiny_t8_int4_f32", "--steps", "1",
                    "--warmup", "1"], env_extra={"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_algorithmic_figures():
    """The roofline's algorithmic bytes and flops, against figures worked out by
    hand for the GLM-shaped layer (H 6144, I 2048, top-8, int4)."""
    sys.path.insert(0, ROOT)
    import bench
    from quantized_routed_expert_tc_b200 import workloads as W
    wl = W.GLM_DECODE_T1
    # one expert: gate + up = 4096 rows x (3072 code bytes + 4 scale bytes),
    # down = 6144 rows x (1024 + 4)
    assert wl.expert_bytes() == 4096 * 3076 + 6144 * 1028 == 18_915_328
    # T = 1: 8 routed experts + the shared one, gate/up rows only
    assert bench.gateup_weight_bytes(wl, 8) == 9 * 4096 * 3076 == 113_393_664
    assert bench.gateup_weight_bytes(wl.with_(wbits=8), 8) == 9 * 4096 * 6148
    assert bench.gateup_weight_bytes(wl.with_(wbits=2), 8) == 9 * 4096 * 1540
    # 2048-token prefill: (2048 * 8 + 2048) rows of tokens x 4096 weight rows x 6144 inputs, 2 flops each
    pf = W.GLM_PREFILL_T2048_BF16
    assert bench.tc_gateup_flops(pf, 2048) == 2 * 18432 * 4096 * 6144 == 927_712_935_936
    assert bench.uses_tensor_cores(pf) and not bench.uses_tensor_cores(wl)


def test_code_hash_covers_the_default_build_only():
    """The kernel hash that keys recorded traffic ignores comments and the lines
    that exist only in bounds-checked builds, and nothing else."""
    sys.path.insert(0, ROOT)
    import bench
    src = "int a = 1;  // note\n/* block */\nQRX_CHECK_OR(a < 2, return);\n#include \"qrx_check.cuh\"\n\nint b = a;\n"
    assert bench._code_only(src) == "int a = 1;\nint b = a;"
    assert bench._code_only("int a = 2;\nint b = a;") != bench._code_only(src)


def test_parity_sample_against_the_baseline_reference():
    """The bench's parity sample: the CPU-baseline leg returns the oracle's result on
    the GPU arm's first batch, and parity_sample compares the GPU rows with it."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from quantized_routed_expert_tc_b200 import workloads as W
    from quantized_routed_expert_tc_b200.layer import activations, expert_f32, router_weights
    wl = W.TINY
    x0 = activations(wl, batch=0)
    cpu, ref = bench.cpu_baseline(wl, 0.05, first=x0)
    assert cpu["kind"] == "oracle" and cpu["value"] > 0
    idx_o, w_o, out_o = ref
    # the reference is the oracle's layer on that very batch
    Wr, bias = router_weights(wl)
    ex = {e: oracle.quantize_expert(*expert_f32(wl, e), wl.wbits) for e in range(wl.n_experts)}
    sh = oracle.quantize_expert(*expert_f32(wl, wl.n_experts), wl.wbits)
    i2, _, o2 = oracle.moe_forward(wl, x0, Wr, bias, ex, sh)
    assert np.array_equal(i2, idx_o) and np.array_equal(o2, out_o)

    same = bench.parity_sample(ref, idx_o, out_o)
    assert same["ok"] and same["max_err_ratio"] == 0.0 and same["rows_compared"] == wl.T
    # GPU rows beyond the oracle's slice are ignored
    longer = np.vstack([out_o, np.full((5, wl.hidden), 1e9, np.float32)])
    idx_longer = np.vstack([idx_o, np.zeros((5, wl.top_k), np.int32)])
    assert bench.parity_sample(ref, idx_longer, longer)["ok"]
    # an error above the tolerance fails
    bad = out_o.copy()
    bad[1, 3] += 0.01 * np.abs(out_o).max()
    r = bench.parity_sample(ref, idx_o, bad)
    assert not r["ok"] and 9e-3 < r["max_err_ratio"] < 1.1e-2
    # a token whose selection differs is counted and left out
    idx_bad = idx_o.copy()
    idx_bad[1, 0] = (idx_bad[1, 0] + 1) % wl.n_experts
    r = bench.parity_sample(ref, idx_bad, bad)
    assert r["ok"] and r["selection_differs"] == 1 and r["rows_compared"] == wl.T - 1


def test_readme_bench_commands_parse(monkeypatch):
    """Every `python bench.py ...` line of the README parses with the bench's own
    argument parser, and every workload it names exists."""
    import shlex
    sys.path.insert(0, ROOT)
    import bench
    from quantized_routed_expert_tc_b200 import workloads as W
    with open(os.path.join(ROOT, "README.md"), encoding="utf-8") as f:
        lines = [ln.split("#")[0].strip() for ln in f if ln.strip().startswith("python bench.py")]
    assert len(lines) >= 5
    for ln in lines:
        argv = shlex.split(ln)[1:]
        monkeypatch.setattr(sys, "argv", argv)
        args = bench.parse()
        assert args.workload in W.ALL, ln

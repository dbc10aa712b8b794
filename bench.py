#!/usr/bin/env python
"""Benchmark of the routed-MoE layer forward on B200.

Default workload: the GLM-5.2-shaped MoE layer (hidden 6144, 256 routed experts
plus one shared expert, intermediate 2048, sigmoid group-limited top-8 router),
one decode token per step, packed int4 experts with per-row f32 scales, f32
activations.  A step is one full layer forward (route, permute, gate/up +
SwiGLU, down, combine) through the C ABI on one batch of synthetic input that
is already resident in HBM.  Inputs rotate through distinct token batches and
L2 is flushed between steps outside the timed events.

  python bench.py [--gpus N --steps K --warmup W] [--impl qrx|reference]

--impl reference times the CPU oracle (the plain reference implementation) on
the host cores on the same workload.  N > 1: one process per GPU under
torchrun, each an independent replica (the layer does not shard), value =
tokens of all ranks / max over ranks of the per-step time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed-MoE layer tokens/s; int4 expert-weight GB/s vs HBM peak"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["qrx", "reference"], default="qrx")
    ap.add_argument("--workload", default="glm_decode_t1_int4_f32")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling case: fewer routed experts (same per-launch work at T=1)")
    ap.add_argument("--topp", type=float, default=0.0,
                    help="adaptive expert top-p (0: off) applied inside the layer")
    ap.add_argument("--kernel", choices=["requant_fp8"], default=None,
                    help="measure one auxiliary kernel instead of the layer")
    ap.add_argument("--union-stats", action="store_true",
                    help="union sizes of correlated verify batches (router + permutation)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling case: another token count per step")
    ap.add_argument("--no-settle", action="store_true",
                    help="skip the 1 s clock-settle loop (for ncu launch counting)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0
TC_MIN_T = 256          # tokens from which bf16 x int4 batches run on the tensor cores


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (the slowest rank's time); x itself on
    one rank.  device: where the collective's tensor lives (cuda for NCCL)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def uses_tensor_cores(wl) -> bool:
    """Whether the library takes the tcgen05 path for this workload's expert FFN."""
    return wl.afmt == 2 and wl.wbits == 4 and wl.T >= TC_MIN_T


def uses_decode_gemv(wl) -> bool:
    """One-token calls: the decode GEMV (k_gemv2), with the selection and the
    permutation fused into its gate/up launch and the combine into its down."""
    return not uses_tensor_cores(wl) and wl.T == 1


def uses_mma_gemv(wl) -> bool:
    """Calls of 2..64 tokens over int4 / int8 weights, or int2 weights with f32 /
    bf16 activations: the multi-token GEMV on tensor cores (k_gmma)."""
    return not uses_tensor_cores(wl) and 2 <= wl.T <= 64 and (wl.wbits in (4, 8) or
                                                               (wl.wbits == 2 and wl.afmt != 1))


def gemv_kernel(wl) -> str:
    return "k_gemv2" if uses_decode_gemv(wl) else ("k_gmma" if uses_mma_gemv(wl) else "k_ffn_gemv")


def launches_per_call(wl) -> int:
    """Library kernels per layer call (top-p and usage add none):
    one token: logits, gate/up (+ selection, permutation), down (+ combine) = 3;
    2..32 tokens: logits, selection + permutation, gate/up, down, combine = 5
    (64 tokens: selection and permutation apart, 6); tensor-core engine:
    logits, selection, permutation, token gather, gate/up, down, combine = 7;
    other GEMV shapes: activation records, logits, selection, permutation,
    gate/up, h records, down, combine = 8."""
    if uses_tensor_cores(wl):
        return 7
    if uses_decode_gemv(wl):
        return 3
    if uses_mma_gemv(wl):
        return 5 if wl.T <= 32 else 6
    return 8


def dtype_label(wl) -> str:
    """The arithmetic the expert FFN computes in.  GEMV engines: exact int32 sums
    of int8 activation digits times the packed codes -- f32 / bf16 activations as
    three int8 digit planes of a 22-bit fixed point (one power-of-two scale per
    row in the decode and multi-token GEMVs, per 32-block in the older GEMV
    engine), Q8_0 as its
    int8 codes with f32 block scales; the tensor-core engine: bf16 x bf16 -> f32."""
    if uses_tensor_cores(wl):
        return "bf16"
    w = f"int{wl.wbits}"
    mma = ", tensor-core mma" if uses_mma_gemv(wl) else ""
    if wl.afmt == 1:
        return f"int8 (Q8_0) x {w} -> int32{mma}"
    src = "bf16" if wl.afmt == 2 else "f32"
    return f"int8x3 digit planes (22-bit fixed point of {src}) x {w} -> int32{mma}"


# How the dominant kernel's duration is taken: events placed between the layer's
# kernels on the launching stream would stop the launches overlapping inside the
# timed steps, so they go in a second loop over the same batches and weights.
ROOFLINE_TIMING = ("CUDA events around the gate/up launch on the launching stream, in a loop of "
                   "the same workload run after the timed steps (qrx_moe_forward_profiled), "
                   "mean over up to 50 launches, L2 flushed between steps")


def gateup_weight_bytes(wl, n_union):
    """Algorithmic bytes of one gate/up launch: each union expert and the shared
    expert read once, 2I rows of H codes plus one f32 scale each."""
    return (n_union + 1) * (2 * wl.inter * (wl.hidden * wl.wbits // 8 + 4))


def tc_gateup_flops(wl, T: int) -> float:
    """Algorithmic flops of one tensor-core gate/up launch: 2 per weight x token
    product, over every assignment plus the shared expert's T tokens, for the
    2I gate and up rows of H inputs."""
    return 2.0 * (T * wl.top_k + T) * (2 * wl.inter) * wl.hidden


def tensor_peak():
    """Dense bf16 tensor peak (burst: the kernel is timed between its own events)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (burst)"
    return FALLBACK_BF16_TFLOPS, "fallback"


def _code_only(text: str) -> str:
    """The code the measured (default) build compiles: the source without // and
    /* */ comments, blank lines, and the lines that exist only for bounds-checked
    builds (QRX_CHECK_OR / QRX_CHECK_ONLY and the qrx_check.cuh include, which
    expand to nothing without -DQRX_CHECK).  Edits to any of those leave the
    compiled kernel, and so its measured traffic, unchanged."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines
                     if ln.strip() and not re.search(r"qrx_check", ln, flags=re.I))


def kernel_source_hash(kernel: str = "k_gemv2_gateup") -> str:
    """Hash of a kernel's code (comments excluded): traffic figures apply only to it."""
    h = hashlib.sha256()
    files = ("k_ffn_tc.cuh", "qrx_dev.cuh") if kernel.startswith("k_ffn_tc") else \
        ("k_gemv2.cuh", "qrx_dev.cuh") if kernel.startswith("k_gemv2") else \
        ("k_gmma.cuh", "k_gemv2.cuh", "qrx_dev.cuh") if kernel.startswith("k_gmma") else \
        ("k_ffn_gemv.cuh", "qrx_dev.cuh")
    for f in files:
        with open(os.path.join(ROOT, "quantized_routed_expert_tc_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    rec = d.get(kernel, {}).get(workload)
    if not rec or rec.get("source_sha") != kernel_source_hash(kernel):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                p = [v.strip() for v in line.split(",")]
                if len(p) >= 9 and p[1].replace(".", "").isdigit():
                    rows.append(p)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, wl):
    """The CPU oracle on the host cores: one batch (or a bounded slice of it) per step."""
    import numpy as np
    import oracle
    from quantized_routed_expert_tc_b200.layer import activations, expert_f32, router_weights

    Wr, bias = router_weights(wl)
    npool = min(max(args.steps, 1), 4)
    ts = oracle_slice(wl)
    xs = [activations(wl, batch=b)[:ts] for b in range(npool)]
    needed = set()
    for x in xs:
        r = oracle.router(wl, x, Wr, bias)
        needed.update(int(e) for e in np.unique(r["idx"]))
    experts = {e: oracle.quantize_expert(*expert_f32(wl, e), wl.wbits) for e in sorted(needed)}
    shared = oracle.quantize_expert(*expert_f32(wl, wl.n_experts), wl.wbits)
    for i in range(args.warmup if args.warmup < 2 else 1):
        oracle.moe_forward(wl, xs[i % npool], Wr, bias, experts, shared, topp=args.topp)
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        oracle.moe_forward(wl, xs[i % npool], Wr, bias, experts, shared, topp=args.topp)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = ts / (ms / 1e3)
    cores = oracle.max_threads()
    sample = (f"{npool} distinct {wl.T}-token batches cycled over {args.steps} steps" if ts == wl.T else
              f"the first {ts} tokens of {npool} distinct {wl.T}-token batches, cycled over "
              f"{args.steps} steps (tokens/s extrapolated linearly)")
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": workload_config(wl, args.topp),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def run_requant(args):
    """FP8 (128x128 block scales) -> packed int4 rows over the gate/up and down
    matrices of 16 GLM-shaped experts (HBM-bound): bytes = FP8 read + codes and
    scales written, per launch; CUDA events, L2 flushed between launches."""
    import numpy as np
    import torch
    from quantized_routed_expert_tc_b200 import build as qbuild, qrx
    qbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nexp, H, I, bits = 16, 6144, 2048, 4
    mats = [(nexp * 2 * I, H), (nexp * H, I)]          # stacked w13 rows, stacked w2 rows
    gen = torch.Generator(device=dev).manual_seed(1234)
    bufs = []
    for rows, K in mats:
        w8 = torch.randint(0, 126, (rows, K), dtype=torch.uint8, device=dev, generator=gen)
        bs = torch.rand(((rows + 127) // 128, (K + 127) // 128), device=dev, generator=gen) * 1e-2 + 1e-4
        q = torch.empty((rows, K * bits // 8), dtype=torch.uint8, device=dev)
        sc = torch.empty(rows, dtype=torch.float32, device=dev)
        bufs.append((w8, bs, q, sc))
    nbytes = sum(w8.numel() + q.numel() + 4 * sc.numel() + 4 * bs.numel() for w8, bs, q, sc in bufs)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    def once():
        for w8, bs, q, sc in bufs:
            qrx.qrx_requant_fp8(w8, bs, bits, q, sc, stream)
    for _ in range(args.warmup):
        once()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        once()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    rc = qrx.qrx_last_error()
    if rc != qrx.QRX_OK:
        raise RuntimeError(qrx.qrx_strerror(rc))
    ms = float(np.median(times))
    peak, kind = peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    print(json.dumps({"metric": "FP8 128x128-block -> per-row int4 requantisation GB/s",
                      "value": gbs, "unit": "GB/s", "ms_per_call": ms, "steps": args.steps,
                      "config": {"experts": nexp, "matrices": [list(m) for m in mats], "bits": bits},
                      "roofline": {"kernel": "k_requant_fp8", "bound": "hbm", "achieved": gbs,
                                   "peak": peak, "peak_kind": kind, "unit": "GB/s",
                                   "frac": gbs / peak, "bytes_per_call": nbytes},
                      "gpu_launches": 2 * args.steps}))


def run_union_stats(args):
    """Expert-union size of verify batches whose tokens share router input structure
    (token i = sqrt(rho) z + sqrt(1 - rho) z_i), through qrx_route + qrx_permute at
    the GLM shape: loads per forward = union + 1 (shared expert)."""
    import numpy as np
    import torch
    from quantized_routed_expert_tc_b200 import build as qbuild, qrx, workloads as W
    from quantized_routed_expert_tc_b200.layer import activations_correlated, router_weights
    qbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = W.GLM_DECODE_T1
    Wr_np, bias_np = router_weights(base)
    Wr, bias = torch.from_numpy(Wr_np).to(dev), torch.from_numpy(bias_np).to(dev)
    rows = []
    for rho in (0.0, 0.5, 0.8, 0.9, 0.95, 1.0):
        for T in (1, 2, 3, 4, 8, 16):
            wl = base.with_(T=T)
            c = qrx.cfg_of(wl)
            ws = qrx.workspace(c, T, dev)
            idx = torch.empty((T, wl.top_k), dtype=torch.int32, device=dev)
            w = torch.empty((T, wl.top_k), dtype=torch.float32, device=dev)
            perm = qrx.Perm.empty(T, wl.top_k, wl.n_experts)
            nus = []
            for b in range(32):
                x = torch.from_numpy(activations_correlated(wl, T, rho, batch=b)).to(dev)
                qrx.qrx_route(c, x, Wr, bias, idx, w, ws)
                qrx.qrx_permute(c, idx, perm)
                nus.append(int(perm.n_union.item()))
            nu = float(np.mean(nus))
            rows.append({"rho": rho, "T": T, "n_union_mean": nu, "loads_per_forward": nu + 1,
                         "loads_per_token_if_all_accepted": (nu + 1) / T})
    print(json.dumps({"metric": "verify-batch expert union (GLM shape, 32 batches each)",
                      "rows": rows}))


def workload_config(wl, topp: float = 0.0):
    from quantized_routed_expert_tc_b200 import workloads as W
    extra = {"expert_top_p": topp} if topp else {}
    return {**extra, "workload": wl.name, "tokens_per_step": wl.T, "hidden": wl.hidden,
            "routed_experts": wl.n_experts, "shared_experts": 1, "inter": wl.inter,
            "top_k": wl.top_k, "n_group": wl.n_group, "topk_group": wl.topk_group,
            "weights": f"int{wl.wbits} per-row f32 scale",
            "activations": W.AFMT_NAMES[wl.afmt], "parallelism": "replicas",
            "l2": "flushed between steps (256 MiB write outside the timed events); "
                  "inputs rotate over distinct token batches"}


# ----------------------------------------------------------------------------- CPU baseline
ORACLE_SLICE = 64   # largest token batch the oracle times whole


def oracle_slice(wl):
    """Tokens per oracle call: the whole batch up to ORACLE_SLICE tokens, else a slice
    of that many (the oracle's cost grows with tokens x experts per token, so its
    tokens/s on a slice stands for the batch; the sample text says so)."""
    return wl.T if wl.T <= ORACLE_SLICE else ORACLE_SLICE


def cpu_baseline(wl, seconds: float, topp: float = 0.0, first=None):
    """The oracle timed on the host cores over two batches (or their first
    oracle_slice(wl) tokens).  `first`, when given, is the first batch (the GPU
    arm's batch 0); the oracle's result on it is returned beside the timing, as
    (idx, w, out), for the parity sample."""
    import numpy as np
    import oracle
    from quantized_routed_expert_tc_b200.layer import activations, expert_f32, router_weights

    Wr, bias = router_weights(wl)
    ts = oracle_slice(wl)
    xs = [activations(wl, batch=1000 + b)[:ts] for b in range(2)]
    if first is not None:
        xs[0] = first[:ts]
    needed = set()
    for x in xs:
        needed.update(int(e) for e in np.unique(oracle.router(wl, x, Wr, bias)["idx"]))
    experts = {e: oracle.quantize_expert(*expert_f32(wl, e), wl.wbits) for e in sorted(needed)}
    shared = oracle.quantize_expert(*expert_f32(wl, wl.n_experts), wl.wbits)
    n, t_total, ref = 0, 0.0, None
    while t_total < seconds or n < 2:
        t0 = time.perf_counter()
        res = oracle.moe_forward(wl, xs[n % 2], Wr, bias, experts, shared, topp=topp)
        t_total += time.perf_counter() - t0
        if n == 0:
            ref = res
        n += 1
        if n >= 200:
            break
    what = f"{ts} token(s)" if ts == wl.T else \
        f"the first {ts} tokens of the {wl.T}-token batch (tokens/s extrapolated linearly)"
    return {"value": n * ts / t_total, "unit": "tokens/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{n} layer forwards of {what} over 2 distinct batches "
                      f"({t_total:.1f} s of CPU time)"}, ref


def parity_sample(ref, idx_gpu, out_gpu, tol: float = 1e-3) -> dict:
    """The timed configuration against the oracle on one batch: `ref` = the
    oracle's (idx, w, out) on the batch's first tokens, `idx_gpu` / `out_gpu` the
    GPU layer's result on the whole batch (a token's output depends on that token
    alone).  Tokens whose expert selection differs (a near-tie resolved the other
    way) are counted and left out of the error."""
    import numpy as np
    idx_o, _, out_o = ref
    ts = idx_o.shape[0]
    same = np.all(np.asarray(idx_gpu)[:ts] == idx_o, axis=1)
    got = np.asarray(out_gpu, dtype=np.float64)[:ts][same]
    want = out_o.astype(np.float64)[same]
    scale = float(np.abs(want).max()) if want.size else 0.0
    err = float(np.abs(got - want).max() / scale) if scale > 0 else 0.0
    return {"tokens": int(ts), "rows_compared": int(same.sum()),
            "selection_differs": int((~same).sum()), "max_err_ratio": err, "tolerance": tol,
            "ok": bool(err <= tol and same.any())}


# ----------------------------------------------------------------------------- GPU arm
def run_qrx(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from quantized_routed_expert_tc_b200 import build as qbuild, qrx
    from quantized_routed_expert_tc_b200.layer import GpuLayer, activations, to_device_act

    qbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    glay = GpuLayer(wl, device=dev)
    cfg = qrx.cfg_of(wl)
    T, H, k = wl.T, wl.hidden, wl.top_k
    npool = 16
    xs_np = [activations(wl, batch=rank * 1000 + b) for b in range(npool)]
    xs = [to_device_act(wl, x, dev) for x in xs_np]
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    out = torch.empty((T, H), dtype=torch.float32, device=dev)
    ws = qrx.workspace(cfg, T, dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB > L2
    stream = torch.cuda.current_stream(dev)

    # union size per pool batch (for the algorithmic bytes of each step)
    unions = []
    for x in xs:
        qrx.qrx_moe_forward(cfg, x, glay.Wr, glay.bias, glay.routed[wl.wbits],
                            glay.shared[wl.wbits], idx, w, out, ws, topp=args.topp)
        unions.append(int(torch.unique(idx[idx >= 0]).numel()))
    torch.cuda.synchronize(dev)
    rc = qrx.qrx_last_error()
    if rc != qrx.QRX_OK:
        raise RuntimeError(f"device error before timing: {qrx.qrx_strerror(rc)}")

    def step(i, ev0, ev1):
        flush.zero_()
        ev0.record(stream)
        qrx.qrx_moe_forward(cfg, xs[i % npool], glay.Wr, glay.bias, glay.routed[wl.wbits],
                            glay.shared[wl.wbits], idx, w, out, ws, stream, topp=args.topp)
        ev1.record(stream)

    def step_profiled(i, evs):
        flush.zero_()
        qrx.qrx_moe_forward_profiled(cfg, xs[i % npool], glay.Wr, glay.bias,
                                     glay.routed[wl.wbits], glay.shared[wl.wbits], idx, w, out,
                                     ws, evs, stream, topp=args.topp)

    sampler = ClockSampler(local_rank)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(args.warmup):
        step(i, e0, e1)
    t_settle = time.perf_counter()
    i = 0
    while not args.no_settle and time.perf_counter() - t_settle < 1.0:   # clocks settle
        step(i, e0, e1)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_push("timed")
    for i in range(args.steps):
        step(i, *evs[i])
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total = np.array([a.elapsed_time(z) for a, z in evs])        # ms per step
    ms_step = max_over_ranks(float(total.mean()), world, dev)
    rc = qrx.qrx_last_error()
    if rc != qrx.QRX_OK:
        raise RuntimeError(f"device error during timing: {qrx.qrx_strerror(rc)}")

    # stage breakdown (events between the kernels; a separate, untimed-for-value loop)
    nprof = min(args.steps, 50)
    pevs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(nprof)]
    for i in range(nprof):
        step_profiled(i, pevs[i])
    torch.cuda.synchronize(dev)
    per = np.array([[pevs[i][j].elapsed_time(pevs[i][j + 1]) for j in range(6)]
                    for i in range(nprof)])          # ms per stage per step

    # algorithmic bytes: each union expert and the shared expert read once
    nu = np.array([unions[i % npool] for i in range(nprof)], dtype=np.float64)
    exp_bytes = wl.expert_bytes()
    gateup_bytes = gateup_weight_bytes(wl, nu)
    gu_ms = per[:, 3]          # the gate/up kernel alone (stage 3)
    achieved = float((gateup_bytes / (gu_ms / 1e3)).mean() / 1e9)
    peak, peak_kind = peaks()
    tc = uses_tensor_cores(wl)
    if tc:
        gateup_flops = tc_gateup_flops(wl, T)
        tc_achieved = gateup_flops / float(gu_ms.mean() / 1e3) / 1e12
        tc_peak, tc_peak_kind = tensor_peak()
    nu_all = np.array([unions[i % npool] for i in range(args.steps)], dtype=np.float64)
    weight_gbs = float(((nu_all + 1) * exp_bytes).mean() / (ms_step / 1e3) / 1e9)
    gv_kernel = gemv_kernel(wl)
    traffic = recorded_traffic("k_ffn_tc_gateup" if tc else f"{gv_kernel}_gateup", wl.name)

    e2e = None
    if not args.no_e2e:
        xh = [torch.from_numpy(x).pin_memory() if wl.afmt != 2 else
              torch.from_numpy(x.view(np.int16)).pin_memory() for x in xs_np]
        oh = torch.empty((T, H), dtype=torch.float32).pin_memory()
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(min(args.warmup, 3)):
            qrx.qrx_moe_forward_hostio(cfg, xh[i % npool], glay.Wr, glay.bias,
                                       glay.routed[wl.wbits], glay.shared[wl.wbits], oh, ws, stream)
        for i in range(args.steps):
            flush.zero_()
            es[i][0].record(stream)
            qrx.qrx_moe_forward_hostio(cfg, xh[i % npool], glay.Wr, glay.bias,
                                       glay.routed[wl.wbits], glay.shared[wl.wbits], oh, ws, stream)
            es[i][1].record(stream)
        torch.cuda.synchronize(dev)
        e_ms = float(np.mean([a.elapsed_time(z) for a, z in es]))
        e_ms = max_over_ranks(e_ms, world, dev)
        xbytes = T * H * (2 if wl.afmt == 2 else 4)
        e2e = {"value": T * world / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": xbytes,
               "d2h_bytes_per_step": T * H * 4, "ms_per_step": e_ms}

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the timed call once more on batch 0, checked against the oracle on its first tokens
        qrx.qrx_moe_forward(cfg, xs[0], glay.Wr, glay.bias, glay.routed[wl.wbits],
                            glay.shared[wl.wbits], idx, w, out, ws, stream, topp=args.topp)
        torch.cuda.synchronize(dev)
        rc = qrx.qrx_last_error()
        if rc != qrx.QRX_OK:
            raise RuntimeError(f"device error in the parity sample: {qrx.qrx_strerror(rc)}")
        idx0, out0 = idx.cpu().numpy(), out.cpu().numpy()
        cpu, ref = cpu_baseline(wl, args.cpu_seconds, args.topp, first=xs_np[0])
        parity = parity_sample(ref, idx0, out0)

    if rank == 0:
        stages = ["act_records", "router", "permute", "gateup", "down", "combine"]
        launches_per_step = launches_per_call(wl)
        line = {
            "metric": METRIC, "value": T * world / (ms_step / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_label(wl),
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights quantised by the "
                    "library; no trained weights)",
            "config": workload_config(wl, args.topp),
            "weight_gbs": weight_gbs,
            "weight_gbs_frac_of_measured_hbm": weight_gbs / peak,
            "weight_gbs_frac_of_8tbs": weight_gbs / SPEC_HBM_GBS,
            "n_union_mean": float(nu.mean()),
            # routed slots per routed expert read, T*k / n_union (slots dropped by top-p counted)
            "reuse_ratio": float(np.mean(T * k / nu)),
            "stage_us": {s: float(per[:, j].mean() * 1e3) for j, s in enumerate(stages)},
            "stage_note": "from qrx_moe_forward_profiled: events between kernels disable the "
                          "launch overlap, so the stages sum to more than ms_per_step" +
                          ("; one-token calls fuse the selection and permutation into gate/up "
                           "and the combine into down" if uses_decode_gemv(wl) else ""),
            "roofline": ({"kernel": "k_ffn_tc (gate/up + SwiGLU, tcgen05)", "bound": "tensor",
                          "achieved": tc_achieved, "peak": tc_peak, "unit": "TFLOP/s",
                          "frac": tc_achieved / tc_peak, "peak_kind": tc_peak_kind,
                          "traffic": traffic, "algorithmic_flops_per_launch": gateup_flops,
                          "timing": ROOFLINE_TIMING,
                          "weight_bytes_per_launch": float(gateup_bytes.mean()),
                          "weight_gbs": achieved}
                         if tc else
                         {"kernel": f"{gv_kernel} (gate/up + SwiGLU)", "bound": "hbm",
                          "achieved": achieved, "peak": peak, "unit": "GB/s",
                          "frac": achieved / peak, "peak_kind": peak_kind,
                          "traffic": traffic, "timing": ROOFLINE_TIMING,
                          "algorithmic_bytes_per_launch": float(gateup_bytes.mean())}),
            "cpu_baseline": cpu,
            "parity_sample": parity,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line))


def main():
    args = parse()
    from quantized_routed_expert_tc_b200 import workloads as W
    wl = W.ALL[args.workload]
    if args.experts:
        wl = wl.with_(name=f"{wl.name}_e{args.experts}", n_experts=args.experts)
    if args.tokens:
        wl = wl.with_(name=f"{wl.name}_t{args.tokens}", T=args.tokens)
    if args.topp:
        wl = wl.with_(name=f"{wl.name}_topp{args.topp:g}")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.kernel == "requant_fp8":
        if rank == 0:
            run_requant(args)
        return
    if args.union_stats:
        if rank == 0:
            run_union_stats(args)
        return
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_qrx(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the MoE layer with zero-computation experts on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl reference]

One step = one pass of the whole layer (router + top-k, dispatch, grouped
SwiGLU expert GEMMs, combine) over one batch of seeded synthetic tokens. The
default workload is the largest fixed single-GPU layer, the bf16
large-expert-count layer (T=8192, d=6144, 256 routed experts of width 2048 +
64 zero experts, top-12, fp32 router, about 30 % of routing slots on zero
experts); ``--config decode`` and the others select the remaining workloads.
Prints one JSON line.

Under torchrun each rank runs its own replica on its own batch (seed + rank):
the layer is data-parallel over tokens with no exchange, so scaling is weak
and the only collectives are the timing barrier and the max over ranks.

``--impl reference`` times the CPU oracle (fp64, OpenMP) on a bounded sample
of the same workload on this machine's host cores; rank 0 only.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_synth import get_config, make_inputs, make_tokens, torch_dtype  # noqa: E402

METRIC = "MoE-layer tokens/s; grouped-GEMM % bf16 TC peak; router/dispatch/combine GB/s"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


KERNEL_SOURCES = ("expert_ffn.cu", "sm100_ptx.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "grouped_gemm_tc_traffic.json")


def kernel_source_digest():
    """Digest of the expert-GEMM sources; a recorded ncu traffic figure is only
    reported while the kernel it was taken on is unchanged."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "expert_routing_dispatch_router_b200", "csrc",
                               name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(config_name, units):
    """ncu dram bytes (read + write) of one gate/up + down launch pair, scaled
    from the recorded capture by the touched experts, or None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f)
    entry = rec.get(config_name)
    if not entry or entry.get("source_digest") != kernel_source_digest():
        return None
    return entry["dram_bytes_per_touched_expert"] * units


def workload_name(sh):
    return (f"{sh.name}: T={sh.T}, d={sh.d}, {sh.n_routed} routed experts (SwiGLU, "
            f"F={sh.ffn}) + {sh.n_zero} zero experts, top-{sh.top_k}, "
            f"{sh.act_dtype} activations/weights, fp32 router, routing={sh.routing}")


def run_config(sh, seed, world):
    """The `config` object of the JSON line; both arms print the same one."""
    w_bytes = sh.n_routed * 3 * sh.ffn * sh.d * (2 if sh.act_dtype == "bf16" else 4)
    return {"workload": workload_name(sh), "seed": seed,
            "l2": "inputs larger than L2: the touched expert weights (up to "
                  f"{w_bytes / 1e9:.2f} GB) stream from HBM every step",
            "parallelism": f"replicas{world}"}


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


# --------------------------------------------------------- reference (CPU) --
def run_reference(args, sh):
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = make_inputs(sh, args.seed)
    cores = oracle.num_threads()
    # the oracle runs its tokens in parallel, one per thread: by default a
    # step samples one token per host thread, so every core has work
    sample = min(sh.T, args.ref_tokens if args.ref_tokens else cores)
    toks = torch.arange(sample, dtype=torch.int32).numpy()

    def step():
        oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down,
                     sh.n_routed, sh.top_k, sh.routed_scale, tokens=toks)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = args.steps * sample / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(sh, args.seed, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"per step: whole layer on the first {sample} of "
                                   f"{sh.T} tokens (fp64 oracle, OpenMP)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(sh, inp, budget_s=12.0):
    """The oracle, as it stands, on this host's cores: whole layer over the
    batch, repeated until about budget_s seconds of CPU work."""
    import oracle
    cores = oracle.num_threads()
    n_tok = sh.T if sh.T <= 256 else 256
    toks = torch.arange(n_tok, dtype=torch.int32).numpy()
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down,
                     sh.n_routed, sh.top_k, sh.routed_scale, tokens=toks)
        done += n_tok
        if time.perf_counter() - t0 >= budget_s or done >= 64 * n_tok:
            break
    dt = time.perf_counter() - t0
    # the same on one core, on a few tokens (about 3 s)
    n1 = min(n_tok, 4)
    oracle.set_num_threads(1)
    try:
        done1, t1 = 0, time.perf_counter()
        while done1 == 0 or (time.perf_counter() - t1 < 3.0 and done1 < 64 * n1):
            oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down,
                         sh.n_routed, sh.top_k, sh.routed_scale, tokens=toks[:n1])
            done1 += n1
        dt1 = time.perf_counter() - t1
    finally:
        oracle.set_num_threads(cores)
    return {"value": done / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"whole layer (fp64) on {n_tok} of {sh.T} tokens, repeated "
                      f"{done // n_tok}x ({dt:.1f} s)",
            "single_core": {"value": done1 / dt1, "unit": "tokens/s",
                            "sample": f"{n1} tokens, repeated {done1 // n1}x ({dt1:.1f} s)"}}


# -------------------------------------------------------------- GPU path --
def graph_time_ms(fn, reps):
    """Device time per call of fn, captured `reps` times in one CUDA graph so
    host launch overhead does not hide the kernels' own duration."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    g.replay()
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / reps
    del g
    return ms


def event_time_ms(fn, reps, stream):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(reps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / reps


def run_gpu(args, sh):
    import expert_routing_dispatch_router_b200 as moe
    from expert_routing_dispatch_router_b200 import replicas

    pre = replicas.rank_info()
    local = pre.local
    torch.cuda.set_device(local)
    info = replicas.init("nccl", 120.0, torch.device("cuda", local))
    world, rank = info.world, info.rank
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    pk = peaks()

    # one model (router and expert weights of the base seed); every rank
    # routes its own batch of tokens
    inp = make_inputs(sh, args.seed)
    inp.x = make_tokens(sh, replicas.batch_seed(args.seed, info))
    d = inp.to(dev)
    ls = moe.LayerShape(sh.T, sh.d, sh.n_routed, sh.n_zero, sh.top_k, sh.ffn,
                        torch_dtype(sh.act_dtype), sh.routed_scale)
    ws = moe.alloc_workspace(ls, dev)
    out = torch.empty(sh.T, sh.d, dtype=d.x.dtype, device=dev)
    counts = torch.empty(sh.E, dtype=torch.int32, device=dev)

    def step():
        moe.layer_forward(ls, d.x, d.w_router, d.bias, d.w_gate, d.w_up, d.w_down, ws,
                          out=out, counts=counts)

    step()
    torch.cuda.synchronize()
    err = moe.read_device_error(ws)
    if err != 0:
        raise RuntimeError(f"device error {err} in the first step")
    c = counts.cpu()
    R = int(c[: sh.n_routed].sum())
    U = int((c[: sh.n_routed] > 0).sum())

    sampler = ClockSampler(local)
    sampler.start()
    # warm-up: W steps, and at least ~1.5 s so the clock sampler sees load
    t_end = time.time() + 1.5
    n = 0
    while n < args.warmup or time.time() < t_end:
        step()
        n += 1
        if n % 64 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    # the timed steps are replays of a CUDA graph holding G layer calls (G
    # divides K), as a serving loop would issue them: no host launch gaps
    G = max(g for g in range(1, min(args.steps, 25) + 1) if args.steps % g == 0)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        for _ in range(G):
            step()
    graph.replay()
    torch.cuda.synchronize()
    replicas.barrier(info)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps // G):
        graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    del graph
    replicas.barrier(info)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = replicas.max_over_ranks(start.elapsed_time(end), info, dev)
    ms_per_step = ms / args.steps
    value = replicas.job_throughput(sh.T, args.steps, info, ms)

    # ---- end to end through the host-buffer entry point
    # A serving loop double-buffers: two lanes, each with its own stream,
    # workspace and pinned x/out buffers, and the steps alternate between
    # them. Every step still copies its x in and its out back; the copies of
    # one lane overlap the kernels of the other. The single-lane figure
    # (each step's copies in series with its kernels) is reported beside it.
    lanes = []
    for _ in range(2):
        lanes.append({"stream": torch.cuda.Stream(dev),
                      "ws": moe.alloc_workspace(ls, dev),
                      "x": inp.x.clone().pin_memory(),
                      "out": torch.empty(sh.T, sh.d, dtype=d.x.dtype).pin_memory()})

    def step_host(ln):
        moe.layer_forward_host(ls, ln["x"], d.w_router, d.bias, d.w_gate, d.w_up, d.w_down,
                               ln["ws"], ln["out"], stream=ln["stream"])

    def capture_host(n_lanes):
        # a CUDA graph of G host-entry calls; with two lanes it holds two
        # independent chains, forked from and joined back to the capture stream
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        with torch.cuda.graph(g, stream=cap):
            for ln in lanes[:n_lanes]:
                ln["stream"].wait_stream(cap)
            for i in range(G):
                step_host(lanes[i % n_lanes])
            for ln in lanes[:n_lanes]:
                cap.wait_stream(ln["stream"])
        return g

    for _ in range(max(args.warmup, 3)):
        for ln in lanes:
            step_host(ln)
    torch.cuda.synchronize()
    e2e_ms = {}
    for n_lanes in (1, 2):
        hgraph = capture_host(n_lanes)
        hgraph.replay()
        torch.cuda.synchronize()
        replicas.barrier(info)
        e2e_ms[n_lanes] = replicas.max_over_ranks(
            event_time_ms(hgraph.replay, args.steps // G, stream) / G, info, dev)
        del hgraph
    for ln in lanes:
        assert torch.equal(ln["out"], out.cpu()), \
            "host entry point disagrees with device entry point"
    act_b = sh.T * sh.d * d.x.element_size()

    # ---- per-stage timings (staged calls, same inputs), rank 0 only
    comp = {}
    roof = None
    if rank == 0:
        reps = 50
        idx, gate = moe.route(ls, d.x, d.w_router, d.bias, ws)
        t_route = graph_time_ms(lambda: moe.route(ls, d.x, d.w_router, d.bias, ws), reps)
        cnt, offs, row_tok, slot_row, x_perm = moe.dispatch(ls, d.x, idx, ws)
        t_disp = graph_time_ms(lambda: moe.dispatch(ls, d.x, idx, ws), reps)
        y_perm = moe.expert_ffn(ls, x_perm, offs, d.w_gate, d.w_up, d.w_down, ws)
        t_ffn = graph_time_ms(lambda: moe.expert_ffn(ls, x_perm, offs, d.w_gate, d.w_up,
                                                     d.w_down, ws, y_perm=y_perm), reps)
        out_c = torch.empty_like(out)
        t_comb = graph_time_ms(lambda: moe.combine(ls, d.x, y_perm, idx, gate, slot_row,
                                                   out=out_c), reps)
        t_graph = graph_time_ms(step, reps)
        es = d.x.element_size()
        Tk = sh.T * sh.top_k
        b_route = sh.T * sh.d * es + sh.E * sh.d * 4 + sh.E * 4 + Tk * 8
        b_disp = 2 * Tk * 4 + Tk * 4 * 2 + 2 * R * sh.d * es
        b_ffn = U * 3 * sh.ffn * sh.d * es
        n_zero_tok = int(((idx >= sh.n_routed).any(dim=1)).sum())
        b_comb = R * sh.d * es + n_zero_tok * sh.d * es + sh.T * sh.d * es + Tk * 12
        flops_ffn = 6.0 * R * sh.d * sh.ffn
        hbm = pk["hbm_gbs"]

        def gbs(b, ms):
            g = b / ms / 1e6
            return {"ms": ms, "gbs": g, "frac_of_measured_hbm": g / hbm,
                    "frac_of_8tbs": g / 8000.0}

        flops_router = 2.0 * sh.T * sh.d * sh.E
        # whole layer against its own ceiling: the larger of its FLOPs at the
        # bf16 peak and its algorithmic bytes at the HBM peak
        b_layer = b_route + b_ffn + sh.T * sh.d * es * 2
        t_floor_ms = max((flops_ffn + flops_router) / (pk["bf16_tflops"] * 1e9),
                         b_layer / (hbm * 1e6))
        comp = {
            "router_topk": gbs(b_route, t_route),
            "dispatch": gbs(b_disp, t_disp),
            "expert_ffn": {"ms": t_ffn, "gbs": b_ffn / t_ffn / 1e6,
                           "tflops": flops_ffn / t_ffn / 1e9,
                           "tensor_frac_of_measured_bf16": flops_ffn / t_ffn / 1e9
                           / pk["bf16_tflops"],
                           "tensor_frac_of_2250_spec": flops_ffn / t_ffn / 1e9 / 2250.0},
            "combine": gbs(b_comb, t_comb),
            "layer_graph": {"ms": t_graph, "tokens_per_s": sh.T / (t_graph / 1e3),
                            "roofline_frac": t_floor_ms / t_graph},
            "R": R, "U": U,
        }
        # the bound is whichever ceiling is lower for this batch: weight bytes
        # at the HBM copy peak, or FLOPs at the bf16 peak (burst: the call is
        # timed alone)
        if flops_ffn / (pk["bf16_tflops"] * 1e12) > b_ffn / (pk["hbm_gbs"] * 1e9):
            ach = flops_ffn / t_ffn / 1e9
            roof = {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                    "traffic": measured_traffic(sh.name, U),
                    "kernel": "moe_expert_ffn: grouped GEMM gate/up + down (+ plan)",
                    "algorithmic_flops": flops_ffn,
                    "peak_source": pk["source"] + " bf16_tflops (burst cuBLAS GEMM)",
                    # the FFN call runs back to back for hundreds of ms under
                    # the power cap: its fraction of the sustained figure too
                    "peak_sustained": pk["bf16_tflops_sustained"],
                    "frac_of_sustained": ach / pk["bf16_tflops_sustained"]}
        else:
            ach = b_ffn / t_ffn / 1e6
            roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / pk["hbm_gbs"], "traffic": None,
                    "kernel": "moe_expert_ffn: grouped_gemm_tc gate/up + down (+ plan)",
                    "algorithmic_bytes": b_ffn,
                    "peak_source": pk["source"] + " hbm_gbs (burst copy)"}
            roof["traffic"] = measured_traffic(sh.name, U)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": sh.act_dtype, "data": "synthetic",
            "config": run_config(sh, args.seed, world),
            "launch": f"CUDA graph of {G} layer calls, replayed {args.steps // G} times",
            "touched_experts": {"U": U, "weight_bytes": U * 3 * sh.ffn * sh.d * 2},
            "e2e": {"value": replicas.job_throughput(sh.T, 1, info, e2e_ms[2]), "unit": "tokens/s",
                    "launch": f"CUDA graph of {G} host-entry calls alternating between two "
                              "streams and workspaces (copies included)",
                    "single_lane_value": replicas.job_throughput(sh.T, 1, info, e2e_ms[1]),
                    "h2d_bytes_per_step": act_b, "d2h_bytes_per_step": act_b},
            "gpu_launches": args.steps * moe.launch_count(ls),
            "roofline": roof,
            "components": comp,
            "clocks": clocks,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(sh, inp)
        print(json.dumps(line), flush=True)
    replicas.finalize(info)


def make_parser():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="large_e",
                    help="workload name; on one GPU a comma-separated list runs each in "
                         "turn in one process (one JSON line each), e.g. the sweep points")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="tokens per reference step (default: one per host thread)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap


def main():
    args = make_parser().parse_args()
    if args.warmup < 3:
        args.warmup = 3
    names = [n for n in args.config.split(",") if n]
    if len(names) > 1 and (args.impl == "reference" or int(os.environ.get("WORLD_SIZE", "1")) > 1):
        raise SystemExit("a list of workloads runs on one GPU, ours only")
    for name in names:
        sh = get_config(name)
        if args.impl == "reference":
            run_reference(args, sh)
        else:
            run_gpu(args, sh)


if __name__ == "__main__":
    main()

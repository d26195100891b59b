"""Benchmark of the KDA core on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--train]

One step = one kda_chunk_fwd over the grouped-value-head training-shape
workload (B=4, H=16, HV=32, T=8192, Dk=Dv=128, chunk=64, bf16 activations,
q/k L2-norm, beta sigmoid and bounded gate in-kernel), inputs resident in HBM.
Rank 0 prints ONE JSON line with the throughput in token-heads/s, its fraction
of the BF16 tensor-core and HBM rooflines, the end-to-end number through the
Python API with host buffers, the decode step (B=256, H=HV=32, D=128, fp32
state, 512 consecutive steps) in GB/s, the segmented KCP pass, the layer
prologue / epilogue kernels in GB/s, and the FP64 oracle timed on the host
cores as a reported baseline.

The extras include the training path (forward keeping the per-chunk states,
then kda_chunk_bwd) at the same workload, each timed on the device; --train is
accepted for compatibility and changes nothing.

Multi-GPU (torchrun): every rank runs its own batch of the same workload (weak
scaling, no collective on the data path); the time is the max over ranks.
--impl reference times the FP64 oracle (the only reference this method has)
on rank 0 on a bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk_kda fwd tokens·heads/s + % bf16 TC peak; kda_step decode HBM GB/s"
# DRAM bytes (read + write) per launch from ncu captures of the current kernels
# (profiles/chunk_tc_kernel_gva_b1.md: one B=1 launch, 32 chains, scaled by 4 to
# the 128 chains of the B=4 launch; profiles/step_kernel_decode_bf16.md).
CHUNK_TC_TRAFFIC_B4 = 4 * (201.954816e6 + 50.557440e6)   # ncu dram read + write of one B=1 launch, x4 chains
STEP_TRAFFIC = 545.3e6 + 480.8e6
UNIT = "tokens·heads/s"
NOMINAL_HBM_GBS = 8000.0      # B200 HBM3e, nominal (the measured copy peak is the roofline)
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # CUDA-core FP32: SMs x FMA lanes x 2 x max clock


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured (MEASURED_PEAKS.json)"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback (MEASURED_PEAKS.json absent: earlier copy/cuBLAS measurement on B200)"}


def chunk_flops_per_token_head(Dk, Dv, C):
    # 6 Dk Dv (W S, (Q Gamma) S, K^T U) + C (3 Dk + 2 Dv) (A_kk, A_qk, W, Ut, A_qk U) + C^2/3 (solve)
    return 6 * Dk * Dv + C * (3 * Dk + 2 * Dv) + C * C / 3.0


def chunk_bytes(w):
    """Algorithmic HBM bytes of one kda_chunk_fwd: every input read once, o written once,
    initial/final state once per chain."""
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T
    b = ntok * w.H * w.Dk * es * 2            # q, k
    b += ntok * w.HV * w.Dv * es * 2          # v, o
    b += ntok * w.HV * w.Dk * es              # g (raw z)
    b += ntok * w.HV * es                     # beta
    b += w.B * w.HV * w.Dk * w.Dv * 4 * (1 + (1 if w.s0_std is not None else 0))  # S_T (+S0)
    return b


def decode_bytes(w):
    es = 2 if w.dtype == "bf16" else 4
    b = 2 * w.B * w.HV * w.Dk * w.Dv * 4      # state read + write
    b += w.B * w.H * w.Dk * es * 2 + w.B * w.HV * (w.Dv * 2 + w.Dk + 1) * es   # q,k,v,o,z,beta
    return b


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during a timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        # the raw samples; KDA_CLOCKS_DIR keeps them somewhere chosen (default: the temp directory)
        self.path = os.path.join(os.environ.get("KDA_CLOCKS_DIR", tempfile.gettempdir()),
                                 "clocks_bench_%d.csv" % os.getpid())

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


def dist_setup(n, backend="nccl"):
    """Rank/world from the torchrun environment; one process group per job.

    Ranks shard the work by batch (each runs its own independent batch of the
    workload, seeded by rank_seed), so the only collectives are the timing
    barrier and the max-over-ranks reduction."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=timedelta(seconds=300), **kw)
    return world, rank, local


def rank_seed(w, rank):
    """Seed of rank `rank`'s batch: every rank draws an independent batch."""
    return w.seed + 1000 * rank


def whole_job_value(units_per_rank, world, ms):
    """Throughput of the whole job: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / (ms * 1e-3)


def max_over_ranks(x, world, device):
    """Max of a host float over the ranks (on `device`: cuda for NCCL, cpu for gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device):
    import torch
    if world > 1:
        import torch.distributed as dist
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


def cpu_baseline(w):
    """Time the FP64 oracle, as it stands, on the host cores: the whole
    workload w (every chain, every token) generated on the CPU with the same
    recipe, so no sampling is needed; the oracle parallelises over chains."""
    import oracle
    import torch
    import workloads

    def f64(t):
        return None if t is None else t.to(torch.float64).numpy()

    inp = workloads.chunk_inputs(w)
    arrays = [f64(inp[n]) for n in ("q", "k", "v", "g", "beta")]
    kw = dict(A_log=f64(inp["A_log"]), dt_bias=f64(inp["dt_bias"]), S0=f64(inp["S0"]))
    del inp
    t0 = time.perf_counter()
    oracle.kda_fwd(*arrays, **kw)
    dt = time.perf_counter() - t0
    return {"value": w.token_heads / dt, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "FP64 oracle on the whole B=%d,HV=%d,T=%d workload (%d chains, %.1f s wall)"
                      % (w.B, w.HV, w.T, w.B * w.HV, dt)}


def oracle_chunk_timing(w, T_override=None):
    """The FP64 oracle on a whole chunk workload (or its first T_override
    tokens of every chain), wall time on the host cores."""
    import oracle
    import torch
    import workloads

    def f64(t):
        return None if t is None else t.to(torch.float64).numpy()

    ws = w if T_override is None else workloads.workload(w.name, T=T_override)
    inp = workloads.chunk_inputs(ws)
    arrays = [f64(inp[n]) for n in ("q", "k", "v", "g", "beta")]
    kw = dict(A_log=f64(inp["A_log"]), dt_bias=f64(inp["dt_bias"]), S0=f64(inp["S0"]))
    del inp
    t0 = time.perf_counter()
    oracle.kda_fwd(*arrays, **kw)
    dt = time.perf_counter() - t0
    return {"value": ws.token_heads / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "seconds": dt,
            "sample": "FP64 oracle, whole B=%d HV=%d T=%d pass (%d chains)" % (ws.B, ws.HV, ws.T, ws.B * ws.HV)}


def oracle_decode_timing(w, n_steps=8):
    """The FP64 oracle on n_steps consecutive decode steps of the whole batch."""
    import oracle
    import torch
    import workloads

    def f64(t):
        return None if t is None else t.to(torch.float64).numpy()

    S = f64(workloads.decode_state(w))
    steps = [workloads.decode_step_inputs(w, i) for i in range(n_steps)]
    t0 = time.perf_counter()
    for d in steps:
        S, _ = oracle.kda_step(S, *(f64(d[n]) for n in ("q", "k", "v", "g", "beta")), A_log=f64(d["A_log"]))
    dt = (time.perf_counter() - t0) / n_steps
    return {"value": decode_bytes(w) / dt / 1e9, "unit": "GB/s", "ms_per_step": dt * 1e3,
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "FP64 oracle, %d consecutive steps of the whole B=%d HV=%d batch" % (n_steps, w.B, w.HV)}


def run_reference(args):
    """--impl reference: the FP64 oracle on rank 0, one bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    import oracle
    import workloads
    w = workloads.workload("gva_bf16")
    # Only the sampled slice is generated: the first value heads of batch row 0.
    cores = oracle.num_threads()
    nh = min(w.HV, max(2, cores))
    T_s = 1024
    ws = workloads.workload("gva_bf16", B=1, T=T_s)
    inp = workloads.chunk_inputs(ws)

    def f64(t):
        return None if t is None else t.to(torch.float64).numpy()

    hq = max(1, nh // (w.HV // w.H))
    arrays = (f64(inp["q"][:, :, :hq]), f64(inp["k"][:, :, :hq]), f64(inp["v"][:, :, :nh]),
              f64(inp["g"][:, :, :nh]), f64(inp["beta"][:, :, :nh]))
    kw = dict(A_log=f64(inp["A_log"][:nh]), dt_bias=f64(inp["dt_bias"][:nh]))
    for _ in range(args.warmup):
        oracle.kda_fwd(*arrays, **kw)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.kda_fwd(*arrays, **kw)
    dt = (time.perf_counter() - t0) / args.steps
    value = nh * T_s / dt
    sample = "FP64 oracle, %d value heads x %d tokens of the B=4,HV=32,T=8192 workload per step" % (nh, T_s)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "gva_bf16: B=4 H=16 HV=32 T=8192 Dk=Dv=128 chunk=64 (sampled)",
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def time_launches(fn, n, stream):
    """n launches of fn with CUDA events around each one on `stream`; returns ms per launch."""
    import torch
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    evs[0].record(stream)
    for i in range(n):
        fn(i)
        evs[i + 1].record(stream)
    evs[-1].synchronize()
    return [evs[i].elapsed_time(evs[i + 1]) for i in range(n)]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--decode-steps", type=int, default=512)
    ap.add_argument("--no-extras", action="store_true", help="only the headline workload")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing")
    ap.add_argument("--batch", type=int, default=None,
                    help="override B of the headline workload (small cases for profiling)")
    ap.add_argument("--train", action="store_true",
                    help="(kept for compatibility: the training path is always timed with the extras)")
    ap.add_argument("--only", default=None, choices=["small", "decode", "kcp", "layer", "train"],
                    help="run one extra entry alone and print its object (for profiling one kernel; "
                         "not the result line)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    args.warmup = max(args.warmup, 3)

    import torch
    import gated_delta_rule_157_b200 as kda
    import workloads

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    pk = peaks()

    if args.only:
        entries = {
            "small": lambda: bench_small_configs(args, kda, workloads, dev, stream, pk, world, rank),
            "decode": lambda: bench_decode(args, kda, workloads, dev, stream, pk, world, rank),
            "kcp": lambda: bench_kcp(args, kda, workloads, dev, stream, world, rank),
            "layer": lambda: bench_layer(args, kda, dev, stream, pk, world),
            "train": lambda: bench_train(args, kda, workloads, dev, stream, world, rank),
        }
        res = entries[args.only]()
        if rank == 0:
            print(json.dumps({"entry": args.only, **res}), flush=True)
        return 0

    # ---------------- headline: chunked forward, B=4 HV=32 T=8192 -------------
    w = workloads.workload("gva_bf16")
    if args.batch is not None:
        w = workloads.workload("gva_bf16", B=args.batch)
    inp = workloads.chunk_inputs(w, seed=rank_seed(w, rank), device=dev)
    o = torch.empty((w.B, w.T, w.HV, w.Dv), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((w.B, w.HV, w.Dk, w.Dv), dtype=torch.float32, device=dev)

    def step(_i):
        kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                          A_log=inp["A_log"], dt_bias=inp["dt_bias"], S0=inp["S0"],
                          chunk=w.chunk, algo=args.algo, o=o, S_T=S_T, stream=stream)

    for i in range(args.warmup):
        step(i)
    kda.kda_device_status(stream)
    clocks = Clocks(local)
    barrier(world, dev)
    clocks.start()
    per = time_launches(step, args.steps, stream)
    barrier(world, dev)
    clk = clocks.stop()
    kda.kda_device_status(stream)
    ms_local = sum(per) / len(per)
    ms = max_over_ranks(ms_local, world, dev)
    units = w.token_heads
    value = whole_job_value(units, world, ms)
    flops = units * chunk_flops_per_token_head(w.Dk, w.Dv, w.chunk)
    nbytes = chunk_bytes(w)
    achieved_gbs = nbytes / (ms_local * 1e-3) / 1e9
    tflops = flops / (ms_local * 1e-3) / 1e12

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "gva_bf16: B=%d H=16 HV=32 T=8192 Dk=Dv=128 chunk=64 per GPU, " % w.B +
                                   "bf16 q/k/v/z/beta, fp32 state; l2norm, beta sigmoid, gate in-kernel",
                       "algo": args.algo, "l2": "inputs larger than L2 (%.2f GB read per step)"
                                                % (nbytes / 1e9),
                       "parallelism": "dp%d (independent batches per GPU)" % world},
            "tc_peak_frac": tflops / pk["bf16_tflops"],
            "useful_tflops": tflops,
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved_gbs / pk["hbm_gbs"],
                         "traffic": CHUNK_TC_TRAFFIC_B4 if (w.B == 4 and args.algo != "simt") else None,
                         "traffic_unit": "bytes per launch (ncu dram read + write)",
                         "kernel": "kda_chunk_fwd (%s)" % args.algo,
                         "peak_source": pk["source"] + ", hbm_gbs burst"},
            "gpu_launches": args.steps}
    if clk is not None:
        line["clocks"] = clk

    # ---------------- end to end through the API with host buffers ------------
    # Every step copies its inputs in from pinned host memory, runs the chunk
    # forward and copies o and S_T out.  Three streams and two buffer sets
    # form a pipeline: step i+1's inputs go in (host to device) while step i
    # computes and its results come out (device to host, the other direction
    # of the link).  The time is the span from the first copy in to the last
    # copy out, divided by the steps.
    host = {n: inp[n].cpu().pin_memory() for n in ("q", "k", "v", "g", "beta")}
    dev_in = [{n: torch.empty_like(inp[n]) for n in host} for _ in range(2)]
    d_o, d_S = [o, torch.empty_like(o)], [S_T, torch.empty_like(S_T)]
    h_o = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
    h_S = [torch.empty(S_T.shape, dtype=S_T.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = h_o[0].numel() * h_o[0].element_size() + h_S[0].numel() * h_S[0].element_size()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        """n pipelined steps; returns ms from the first copy in to the last copy out."""
        torch.cuda.synchronize(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev_done[b])          # step i-2 has read these inputs
            with torch.cuda.stream(s_in):
                for name in host:
                    dev_in[b][name].copy_(host[name], non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])         # step i-2's results are out
            kda.kda_chunk_fwd(dev_in[b]["q"], dev_in[b]["k"], dev_in[b]["v"], dev_in[b]["g"],
                              dev_in[b]["beta"], A_log=inp["A_log"], dt_bias=inp["dt_bias"], S0=inp["S0"],
                              chunk=w.chunk, algo=args.algo, o=d_o[b], S_T=d_S[b], stream=stream)
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                h_o[b].copy_(d_o[b], non_blocking=True)
                h_S[b].copy_(d_S[b], non_blocking=True)
            ev_out[b].record(s_out)
        t1.record(s_out)
        t1.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(2)
    barrier(world, dev)
    n_e2e = max(3, min(args.steps, 10))
    ms_total = e2e_run(n_e2e)
    barrier(world, dev)
    ms_e2e = max_over_ranks(ms_total / n_e2e, world, dev)
    line["e2e"] = {"value": whole_job_value(units, world, ms_e2e), "unit": UNIT,
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "ms_per_step": ms_e2e, "steps": n_e2e, "api": "gated_delta_rule_157_b200.kda_chunk_fwd",
                   "pipeline": "inputs of step i+1 copied in while step i computes and its o, S_T are "
                               "copied out (three streams, two buffer sets)"}
    del host, dev_in, d_o, d_S, h_o, h_S

    if not args.no_extras:
        line["small"] = bench_small_configs(args, kda, workloads, dev, stream, pk, world, rank)
        line["decode"] = bench_decode(args, kda, workloads, dev, stream, pk, world, rank)
        line["kcp"] = bench_kcp(args, kda, workloads, dev, stream, world, rank)
        line["layer"] = bench_layer(args, kda, dev, stream, pk, world)
        line["train"] = bench_train(args, kda, workloads, dev, stream, world, rank)
        line["gpu_launches_extras"] = {"small": line["small"]["launches"],
                                       "decode": line["decode"]["launches"],
                                       "kcp": line["kcp"]["launches"],
                                       "layer": line["layer"]["launches"],
                                       "train": line["train"]["launches"]}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["kcp"]["cpu_baseline_unsegmented"] = oracle_chunk_timing(workloads.workload("kcp_bf16"))
            line["decode"]["cpu_baseline"] = oracle_decode_timing(workloads.workload("decode_bf16"))

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()
    return 0


def bench_small_configs(args, kda, workloads, dev, stream, pk, world, rank):
    """tiny_fp32 (B=1 H=HV=2 T=64 D=16 chunk 16, fp32: the SIMT kernel) and
    prefill_bf16 (B=1 H=HV=16 T=4096 D=128 chunk 64, bf16, S0 ~ N(0, 0.02):
    16 chains, so 16 of the 148 SMs work), each timed over consecutive
    launches with inputs resident."""
    out, launches = {}, 0
    for name in ("tiny_fp32", "prefill_bf16"):
        w = workloads.workload(name)
        inp = workloads.chunk_inputs(w, seed=rank_seed(w, rank), device=dev)
        o = torch_empty_like_o(w, dev)

        def step(_i):
            kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], A_log=inp["A_log"],
                              dt_bias=inp["dt_bias"], S0=inp["S0"], chunk=w.chunk, o=o, stream=stream)

        for i in range(args.warmup):
            step(i)
        barrier(world, dev)
        k = max(5, min(args.steps, 20))
        per = time_launches(step, k, stream)
        barrier(world, dev)
        ms_local = sum(per) / len(per)
        ms = max_over_ranks(ms_local, world, dev)
        e = {"workload": "%s: B=%d H=%d HV=%d T=%d Dk=Dv=%d chunk=%d %s" % (name, w.B, w.H, w.HV, w.T, w.Dk,
                                                                         w.chunk, w.dtype),
             "value": whole_job_value(w.token_heads, world, ms), "unit": UNIT, "ms_per_step": ms,
             "launches": k, "chains": w.B * w.HV}
        if name == "prefill_bf16":
            tfl = w.token_heads * chunk_flops_per_token_head(w.Dk, w.Dv, w.chunk) / (ms_local * 1e-3) / 1e12
            gbs = chunk_bytes(w) / (ms_local * 1e-3) / 1e9
            e["tc_peak_frac"] = tfl / pk["bf16_tflops"]
            e["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / pk["hbm_gbs"], "traffic": None}
            e["occupancy"] = "%d chains on 148 SMs: one CTA per chain" % (w.B * w.HV)
            # the same forward with each sequence cut into segments run in
            # parallel (states-only pass with transitions, compose, output pass)
            nseg = kda.seq_segments(w.B, w.HV, w.T, w.chunk,
                                    torch_sm_count(dev))

            def step_sp(_i):
                kda.kda_chunk_fwd_seqpar(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                         A_log=inp["A_log"], dt_bias=inp["dt_bias"], S0=inp["S0"],
                                         chunk=w.chunk, segments=nseg)

            for i in range(args.warmup):
                step_sp(i)
            barrier(world, dev)
            per_sp = time_launches(step_sp, k, stream)
            barrier(world, dev)
            ms_sp_local = sum(per_sp) / len(per_sp)
            ms_sp = max_over_ranks(ms_sp_local, world, dev)
            tfl_sp = w.token_heads * chunk_flops_per_token_head(w.Dk, w.Dv, w.chunk) / (ms_sp_local * 1e-3) / 1e12
            e["seqpar"] = {"segments": nseg, "ms_per_step": ms_sp,
                           "value": whole_job_value(w.token_heads, world, ms_sp), "unit": UNIT,
                           "tc_peak_frac": tfl_sp / pk["bf16_tflops"], "speedup": ms / ms_sp,
                           "launches": 3 * k, "api": "gated_delta_rule_157_b200.kda_chunk_fwd_seqpar"}
            launches += 3 * k
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            e["cpu_baseline"] = oracle_chunk_timing(w)
        out[name] = e
        launches += k
        del inp, o
    out["launches"] = launches
    return out


def torch_sm_count(dev):
    import torch
    return torch.cuda.get_device_properties(dev).multi_processor_count


def torch_empty_like_o(w, dev):
    import torch
    return torch.empty((w.B, w.T, w.HV, w.Dv), dtype=w.torch_dtype, device=dev)


def bench_decode(args, kda, workloads, dev, stream, pk, world, rank):
    """512 consecutive decode steps of B=256, H=HV=32, D=128 against a resident fp32 state."""
    import torch
    w = workloads.workload("decode_bf16")
    S = workloads.decode_state(w, seed=rank_seed(w, rank), device=dev)
    n = args.decode_steps
    steps = [workloads.decode_step_inputs(w, i, seed=rank_seed(w, rank), device=dev)
             for i in range(n)]
    o = torch.empty((w.B, w.HV, w.Dv), dtype=torch.bfloat16, device=dev)

    def step(i):
        d = steps[i % n]
        kda.kda_step(S, d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"], o=o,
                     stream=stream)

    for i in range(args.warmup):
        step(i)
    barrier(world, dev)
    per = time_launches(step, n, stream)
    barrier(world, dev)
    ms_local = sum(per) / len(per)
    ms = max_over_ranks(ms_local, world, dev)
    nb = decode_bytes(w)
    gbs = nb / (ms_local * 1e-3) / 1e9
    return {"workload": "decode_bf16: B=256 H=HV=32 Dk=Dv=128, fp32 state, %d consecutive steps" % n,
            "value": world * nb / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": STEP_TRAFFIC,
                         "traffic_unit": "bytes per launch (ncu dram read + write)", "kernel": "kda_step"},
            "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
            "launches": n, "l2": "state 512 MiB > L2"}


def bench_kcp(args, kda, workloads, dev, stream, world, rank):
    """Segmented forward of B=1, HV=16, T=65536 as 8 segments of 8192: segments
    with transitions (one batched launch), the combine, and the rerun for o."""
    import torch
    w = workloads.workload("kcp_bf16")
    inp = workloads.chunk_inputs(w, seed=rank_seed(w, rank), device=dev)
    L = w.T // w.n_seg
    seg = {n: inp[n].view(w.n_seg, L, *inp[n].shape[2:]) for n in ("q", "k", "v", "g", "beta")}
    o = torch.empty((w.n_seg, L, w.HV, w.Dv), dtype=torch.bfloat16, device=dev)
    S_loc = torch.empty((w.n_seg, w.HV, w.Dk, w.Dv), dtype=torch.float32, device=dev)
    M_loc = torch.empty((w.n_seg, w.HV, w.Dk, w.Dk), dtype=torch.float32, device=dev)
    S_in = torch.empty((w.n_seg + 1, w.HV, w.Dk, w.Dv), dtype=torch.float32, device=dev)
    S_init = inp["S0"].view(w.HV, w.Dk, w.Dv)

    def step(_i):
        kda.kda_chunk_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"], A_log=inp["A_log"],
                          chunk=w.chunk, algo=args.algo, S_T=S_loc, M_T=M_loc,
                          output_transition=True, output_o=False, stream=stream)
        kda.kda_compose(M_loc, S_loc, S_init, S_in=S_in, stream=stream)
        kda.kda_chunk_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"], A_log=inp["A_log"],
                          S0=S_in[:w.n_seg], chunk=w.chunk, algo=args.algo, o=o,
                          output_final_state=False, stream=stream)

    for i in range(args.warmup):
        step(i)
    barrier(world, dev)
    k = max(3, min(args.steps, 10))
    per = time_launches(step, k, stream)
    barrier(world, dev)
    ms = max_over_ranks(sum(per) / len(per), world, dev)
    return {"workload": "kcp_bf16: B=1 H=HV=16 T=65536 as 8 x 8192, Dk=Dv=128",
            "value": whole_job_value(w.token_heads, world, ms), "unit": UNIT, "ms_per_step": ms,
            "launches": 3 * k}


def bench_train(args, kda, workloads, dev, stream, world, rank):
    """Training path at the headline workload (or --batch): kda_chunk_fwd
    keeping the per-chunk states (the tensor-core kernel for this shape) and
    kda_chunk_bwd, timed apart; throughput in token-heads per second of
    forward + backward."""
    import torch
    w = workloads.workload("gva_bf16") if args.batch is None else workloads.workload("gva_bf16", B=args.batch)
    inp = workloads.chunk_inputs(w, seed=rank_seed(w, rank), device=dev)
    g = torch.Generator(device=dev).manual_seed(17 + rank)
    dout = torch.randn((w.B, w.T, w.HV, w.Dv), device=dev, generator=g).to(torch.bfloat16)
    S_ch = torch.empty((w.B, w.HV, -(-w.T // w.chunk), w.Dk, w.Dv), device=dev)
    o = torch.empty((w.B, w.T, w.HV, w.Dv), dtype=torch.bfloat16, device=dev)

    def fwd(_i):
        kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], A_log=inp["A_log"],
                          dt_bias=inp["dt_bias"], S0=inp["S0"], chunk=w.chunk, o=o, S_chunks=S_ch,
                          output_final_state=False, algo=args.algo, stream=stream)

    def bwd(_i):
        kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S_ch, dout, None,
                          A_log=inp["A_log"], dt_bias=inp["dt_bias"], chunk=w.chunk, stream=stream)

    out = {"workload": "gva_bf16 B=%d: forward with chunk states (algo %s) + backward (fp32; A/P products "
                       "on the tensor cores, the rest on the CUDA cores)" % (w.B, args.algo),
           "launches": 0}
    # kernels per call: the forward is one launch; the backward three (chunk
    # kernel, L2-norm and gate/parameter passes) after the output zeroing
    n_kernels = {"forward_with_states": 1, "backward": 3}
    for name, fn in (("forward_with_states", fwd), ("backward", bwd)):
        for i in range(max(1, min(args.warmup, 2))):
            fn(i)
        kda.kda_device_status(stream)
        barrier(world, dev)
        k = max(3, min(args.steps, 5))
        per = time_launches(fn, k, stream)
        barrier(world, dev)
        kda.kda_device_status(stream)
        out[name] = {"ms_per_step": max_over_ranks(sum(per) / len(per), world, dev)}
        out["launches"] += k * n_kernels[name]
    ms = out["forward_with_states"]["ms_per_step"] + out["backward"]["ms_per_step"]
    out["value"] = whole_job_value(w.token_heads, world, ms)
    out["unit"] = UNIT
    # The backward runs on the CUDA cores in fp32: its roofline is the FP32 FMA
    # rate (148 SMs x 128 lanes x 2 x 1965 MHz), counted on twice the forward's
    # useful FLOPs (the usual count for the gradient of a product chain).
    ms_b = out["backward"]["ms_per_step"]
    tfl = 2 * w.token_heads * chunk_flops_per_token_head(w.Dk, w.Dv, w.chunk) / (ms_b * 1e-3) / 1e12
    out["backward"]["roofline"] = {"bound": "alu", "achieved": tfl, "peak": FP32_FMA_TFLOPS, "unit": "TFLOP/s",
                                   "frac": tfl / FP32_FMA_TFLOPS, "traffic": None,
                                   "flops": "2 x forward useful FLOPs"}
    return out


def bench_layer(args, kda, dev, stream, pk, world):
    """Layer prologue (short convolution + SiLU (+ per-head L2 norm) of q, k, v)
    and epilogue (RMSNorm + sigmoid gate of o) at the headline shapes (B=4,
    T=8192, H=16 q/k heads, HV=32 value heads, 128 channels).  Both stream
    bf16 in and out once: bytes = 2 B x (elements read + elements written)."""
    import torch
    g = torch.Generator(device=dev).manual_seed(5)
    B, T, H, HV, D = 4, 8192, 16, 32, 128
    xq = torch.randn((B, T, H * D), device=dev, generator=g).to(torch.bfloat16)
    xk = torch.randn((B, T, H * D), device=dev, generator=g).to(torch.bfloat16)
    xv = torch.randn((B, T, HV * D), device=dev, generator=g).to(torch.bfloat16)
    wq, wk = (torch.randn((H * D, 4), device=dev, generator=g) * 0.5 for _ in range(2))
    wv = torch.randn((HV * D, 4), device=dev, generator=g) * 0.5
    yq, yk, yv = torch.empty_like(xq), torch.empty_like(xk), torch.empty_like(xv)
    o = torch.randn((B * T, HV, D), device=dev, generator=g).to(torch.bfloat16)
    gate = torch.randn((B * T, HV, D), device=dev, generator=g).to(torch.bfloat16)
    yo = torch.empty_like(o)

    def pro(_i):
        kda.kda_short_conv(xq, wq, head_dim=D, y=yq, stream=stream)
        kda.kda_short_conv(xk, wk, head_dim=D, y=yk, stream=stream)
        kda.kda_short_conv(xv, wv, y=yv, stream=stream)

    def epi(_i):
        kda.kda_output_gate(o, gate, y=yo, stream=stream)

    out = {"workload": "B=4 T=8192: prologue of q, k (16 x 128 channels, head L2 norm) and "
                       "v (32 x 128); epilogue of o (32 heads x 128)", "launches": 0}
    for name, fn, nbytes, nl in (("prologue", pro, 2 * 2 * (xq.numel() + xk.numel() + xv.numel()), 3),
                                 ("epilogue", epi, 2 * 3 * o.numel(), 1)):
        for i in range(args.warmup):
            fn(i)
        barrier(world, dev)
        k = max(3, min(args.steps, 10))
        per = time_launches(fn, k, stream)
        barrier(world, dev)
        ms_local = sum(per) / len(per)
        ms = max_over_ranks(ms_local, world, dev)
        gbs = nbytes / (ms_local * 1e-3) / 1e9
        out[name] = {"ms_per_step": ms, "value": world * nbytes / (ms * 1e-3) / 1e9, "unit": "GB/s",
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": gbs / pk["hbm_gbs"], "traffic": None}}
        out["launches"] += nl * k
    return out


if __name__ == "__main__":
    sys.exit(main())

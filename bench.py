#!/usr/bin/env python
"""Benchmark of the linear-logp operator on B200.

One step = the whole hot path on one batch: the forward (fused LM-head GEMM
+ online logsumexp / entropy + target gather, then the fixed-order combine)
and the backward (per vocab chunk: logits recompute + dlogits, dHidden GEMM,
dW GEMM).  Default workload: the RL actor step, 8 ragged sequences
concatenated (T = 5980 for seed 3), H=4096, V=151936, bf16, tau = 1.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one process per GPU, weak scaling: every rank
processes its own batch against the same (replicated) W; there is no
data-path collective (rows are independent).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "linear-logp fwd+bwd tokens/s at H4096 V151936 bf16; % of BF16 TC peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_rl_actor_step.json")


def kernel_sources_sha256():
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "invariant_lm_head_gemm_b200", "csrc", "*"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic():
    """DRAM bytes per launch (read + write) of the forward and backward kernels
    from the committed ncu capture, or (None, None) once the kernel sources
    differ from the ones that capture measured."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None, None
    if t.get("csrc_sha256") != kernel_sources_sha256():
        return None, None
    tot = lambda k: t[k]["dram_read_bytes"] + t[k]["dram_write_bytes"]
    return tot("forward"), tot("backward")


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, tag=""):
        self.index = index
        self.proc = None
        # the raw samples (the summary goes into the JSON line); directory from
        # RLK_CLOCKS_DIR, else the system's temporary directory
        import tempfile
        out_dir = os.environ.get("RLK_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, "clocks_rank%d%s.csv" % (index, tag))

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
        return False

    def summary(self):
        if self.proc is None:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        except OSError:
            return None
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# Nominal dense bf16 tensor throughput per SM per clock (4096 bf16 FMAs): 148 SMs
# at 1965 MHz give 2.38 PFLOP/s, the datasheet's 2.25 PFLOP/s at ~1.86 GHz.
FLOPS_PER_SM_CLOCK = 8192.0
MAX_SM_MHZ = 1965.0


def clock_fields(ms, clk, tflops, n_sms):
    """Clock-normalised figures of a kernel timed while `clk` sampled the SM
    clock: its cycles per launch at the median clock, the time it would take at
    the maximum clock, and its throughput as a fraction of the tensor peak at
    the clock it ran at (comparable across boxes whose power-capped clocks
    differ)."""
    if not clk or not clk.get("sm_mhz"):
        return {"sm_mhz": None}
    mhz = clk["sm_mhz"]
    return {"sm_mhz": mhz, "clock_samples": clk.get("samples"),
            "mcycles_per_launch": ms * mhz / 1e3,
            "ms_at_%dMHz" % MAX_SM_MHZ: ms * mhz / MAX_SM_MHZ,
            "frac_at_clock": tflops / (n_sms * FLOPS_PER_SM_CLOCK * mhz * 1e6 / 1e12)}


def aggregate(ms_local, tokens_local):
    """Across ranks: the slowest rank's step time and the tokens all ranks
    processed (weak scaling: value = tokens / max time)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms_local), float(tokens_local)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms_local], dtype=torch.float64, device=dev)
    n = torch.tensor([tokens_local], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), float(n.item())


def rl_inputs(rank):
    from invariant_lm_head_gemm_b200 import workloads as wl
    w = wl.rl_step(3 + 1000 * rank, with_weight=False)
    W = wl.make_weight(3, wl.QWEN_V, wl.QWEN_H)
    return w, W


def cpu_baseline(w, W, rows=8):
    """The fp64 oracle, as it stands, on a bounded sample of rows of the same
    workload (forward + backward), on this host's cores."""
    import oracle
    oracle.build()
    idx = np.linspace(0, w.T - 1, rows).astype(np.int64)
    t0 = time.perf_counter()
    oracle.forward(w.hidden[idx], W, w.targets[idx], w.temperature)
    oracle.backward(w.hidden[idx], W, w.targets[idx], w.temperature, w.dlogp[idx],
                    w.dentropy[idx])
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d of %d rows of the RL actor step (H=4096, V=151936), fp64 C oracle "
                      "forward + backward, %.1f s" % (rows, w.T, dt)}


def cpu_oracle_sides(w, W):
    """The oracle timed beside the other two measured paths: the forward of a
    single row (the decode shape, T = 1) against the full head, and one
    transition step at the report's first shape."""
    import oracle
    from oracle import transition as tro
    from invariant_lm_head_gemm_b200 import workloads as wlm
    oracle.build()
    t0 = time.perf_counter()
    oracle.forward(w.hidden[:1], W, w.targets[:1], w.temperature)
    t_dec = time.perf_counter() - t0
    B, n = wlm.TRANSITION_SHAPES[0]
    tw = wlm.transition_case(0, B, n)
    t0 = time.perf_counter()
    tro.transition_sample(tw.x, tw.v, tw.eps, tw.a, tw.c, tw.s)
    t_tr = time.perf_counter() - t0
    return ({"us_per_call": 1e6 * t_dec, "cores": oracle.num_threads(), "kind": "oracle",
             "sample": "fp64 C oracle forward of 1 row (H=4096, V=151936)"},
            {"us_per_call": 1e6 * t_tr, "cores": 1, "kind": "oracle",
             "sample": "fp64 numpy oracle, one sampling step at B3 x 257x96"})


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w, W = rl_inputs(0)
    import oracle
    oracle.build()
    rows_per_step = args.ref_rows
    rng = np.random.default_rng(0)

    def step():
        idx = np.sort(rng.choice(w.T, rows_per_step, replace=False))
        oracle.forward(w.hidden[idx], W, w.targets[idx], w.temperature)
        oracle.backward(w.hidden[idx], W, w.targets[idx], w.temperature, w.dlogp[idx],
                        w.dentropy[idx])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = rows_per_step * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Gaussian, bf16-rounded)",
        "config": config_dict(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": "%d random rows of the RL actor step per step "
                                   "(fwd + bwd, fp64 C oracle)" % rows_per_step},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w, world):
    return {"workload": "rl_actor_step: 8 ragged sequences (lengths U[256,1024], seed 3), "
                        "fwd+bwd, H=4096, V=151936, bf16, tau=1",
            "T_per_rank": int(w.T), "H": 4096, "V": 151936, "temperature": 1.0,
            "seq_lens": [int(x) for x in w.seq_lens], "parallelism": "dp%d" % world,
            "l2": "inputs larger than L2: all of W (1.245 GB) is read every step"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from invariant_lm_head_gemm_b200 import binding

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w, W_host = rl_inputs(rank)
    T, H, V = w.T, w.H, w.V

    def to_dev_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    W = to_dev_bf16(W_host)
    hid = to_dev_bf16(w.hidden)
    tg = torch.from_numpy(w.targets).to(dev)
    dl = torch.from_numpy(w.dlogp).to(dev)
    de = torch.from_numpy(w.dentropy).to(dev)
    ws = binding.make_workspace(T, H, V, True, dev)
    logp = torch.empty(T, device=dev)
    ent = torch.empty(T, device=dev)
    lse = torch.empty(T, device=dev)
    dH = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    dW = torch.empty(V, H, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # N > 1: the data-parallel exchange of dW (deterministic reduce-scatter:
    # NCCL all-to-all of vocab slices, then the rank-ordered sum).  Overlapped
    # (default): the backward publishes each vocab chunk's completion and the
    # exchange runs a group of chunks at a time on a second stream, each group
    # waiting on the device for its chunks; "after": one exchange once the
    # backward is done.
    use_rs = world > 1 and not args.no_dw_reduce
    overlap = use_rs and args.dw_exchange == "overlap"
    chunk = binding.bwd_chunk_width(V)
    groups = -(-(-(-V // chunk)) // args.dw_group_chunks)
    if use_rs:
        from invariant_lm_head_gemm_b200 import dp
        per = -(-V // world)
        rs_recv = torch.empty(world, per, H, dtype=torch.float32, device=dev)
        # a rank's rows of the group-wise exchange exceed V / world by at most
        # one per group
        rs_out = torch.empty(per + groups, H, dtype=torch.float32, device=dev)
        comm = torch.cuda.Stream(dev)
        words = torch.zeros(-(-V // chunk), dtype=torch.int32, device=dev)
        seq = [0]

    def backward(h, t, l_, e_, dlp, den, out):
        """The backward and, for N > 1, the dW exchange it feeds."""
        if not use_rs:
            binding.rlk_linear_logp_bwd(h, W, t, 1.0, l_, e_, dlp, den, ws, out=out)
        elif overlap:
            stream.wait_stream(comm)       # the last exchange has read dW
            seq[0] += 1
            binding.rlk_linear_logp_bwd_signal(h, W, t, 1.0, l_, e_, dlp, den, ws, out, words,
                                               seq[0])
            dp.reduce_scatter_dw_overlapped(out[1], chunk, chunk_done=words, seq=seq[0],
                                            group_chunks=args.dw_group_chunks, stream=comm,
                                            recv=rs_recv.view(-1), out=rs_out)
        else:
            binding.rlk_linear_logp_bwd(h, W, t, 1.0, l_, e_, dlp, den, ws, out=out)
            dp.reduce_scatter_dw(out[1], rs_recv, rs_out)

    def join_exchange():
        if overlap:
            stream.wait_stream(comm)

    def step():
        binding.rlk_linear_logp_fwd(hid, W, tg, 1.0, ws, out=(logp, ent, lse))
        backward(hid, tg, lse, ent, dl, de, (dH, dW))

    def barrier():
        if world > 1:
            dist.barrier()

    # ---------------------------------------------------------------- decode-shaped forward
    # Rollout scoring / decode: the first T rows of the batch against the same
    # W (1.245 GB, far above L2, so every call streams W from HBM).  Bound by
    # HBM: algorithmic bytes = W + hidden rows + targets + outputs.  Timed as
    # CUDA-graph replays of one captured call, the way a decode loop runs it
    # (an eager call at these sizes is bound by the host's launch work; its
    # time is reported too), before the long GEMM steps drive the clocks down
    # to the power cap.  One untimed pass over the sizes first.
    def decode_us(Td):
        h_d, t_d = hid[:Td].contiguous(), tg[:Td].contiguous()
        outs = tuple(torch.empty(Td, device=dev) for _ in range(3))

        def call():
            binding.rlk_linear_logp_fwd(h_d, W, t_d, 1.0, ws, out=outs)

        call()
        torch.cuda.synchronize()
        e_a = torch.cuda.Event(enable_timing=True)
        e_b = torch.cuda.Event(enable_timing=True)
        e_a.record(stream)
        for _ in range(10):
            call()
        e_b.record(stream)
        torch.cuda.synchronize()
        eager = 1e3 * e_a.elapsed_time(e_b) / 10
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            call()
        for _ in range(3):
            graph.replay()
        e_a.record(stream)
        for _ in range(20):
            graph.replay()
        e_b.record(stream)
        torch.cuda.synchronize()
        return 1e3 * e_a.elapsed_time(e_b) / 20, eager

    decode_rows = (1, 4, 16, 64, 128, 192, 256)
    for Td in decode_rows:
        decode_us(Td)
    dec_us = [decode_us(Td) for Td in decode_rows]
    dec_gbs = [(V * H * 2 + Td * (H * 2 + 8 + 12)) / (u * 1e-6) / 1e9
               for Td, (u, _) in zip(decode_rows, dec_us)]
    decode = {"kernel": "decode_fwd_kernel (T <= 256: operands swapped, 128 vocab rows per CTA, "
                        "N = T padded to 16/32; single-CTA MMA for N <= 32, CTA-pair MMA "
                        "(M = 256) from N = 64) + combine; larger T: the pair kernel",
              "bound": "hbm", "unit": "GB/s", "timing": "CUDA-graph replay, 20 calls",
              "rows": list(decode_rows), "us_per_call": [u for u, _ in dec_us],
              "eager_us_per_call": [e for _, e in dec_us], "achieved": dec_gbs,
              "frac": [g / peaks()[0]["hbm_gbs"] for g in dec_gbs]}

    # ---------------------------------------------------------------- diffusion transition step
    # The report's three transition shapes; one sampling step (reads x, v,
    # eps; writes mean, prev_sample, logp: 20 bytes per element).  A sampler
    # loop captured whole: 20 steps in one CUDA graph, replayed 10 times.  At
    # these sizes (1.5-31 MB per step) launch gaps still set much of the time.
    from invariant_lm_head_gemm_b200 import workloads as wl
    wlm = wl
    trans = {"kernel": "transition_kernel (one launch per step)", "bound": "hbm",
             "unit": "GB/s", "timing": "CUDA graph of 20 steps, replayed 10 times", "shapes": [],
             "us_per_call": [], "achieved": [], "frac": []}
    for i, (Bt, nt) in enumerate(wlm.TRANSITION_SHAPES):
        tw = wlm.transition_case(i, Bt, nt)
        tx, tv, te, ta, tc, tsd = (torch.from_numpy(np.ascontiguousarray(q)).to(dev)
                                   for q in (tw.x, tw.v, tw.eps, tw.a, tw.c, tw.s))
        t_ws = binding.transition_workspace(Bt, nt, dev)
        t_out = (torch.empty_like(tx), torch.empty_like(tx), torch.empty(Bt, device=dev))
        binding.rlk_transition_sample(tx, tv, te, ta, tc, tsd, out=t_out, workspace=t_ws)
        tg_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tg_graph, capture_error_mode="thread_local"):
            for _ in range(20):
                binding.rlk_transition_sample(tx, tv, te, ta, tc, tsd, out=t_out, workspace=t_ws)
        for _ in range(2):
            tg_graph.replay()
        ta0 = torch.cuda.Event(enable_timing=True)
        ta1 = torch.cuda.Event(enable_timing=True)
        ta0.record(stream)
        for _ in range(10):
            tg_graph.replay()
        ta1.record(stream)
        torch.cuda.synchronize()
        t_us = 1e3 * ta0.elapsed_time(ta1) / 200
        t_gbs = (20 * Bt * nt + 16 * Bt) / (t_us * 1e-6) / 1e9
        trans["shapes"].append([Bt, nt])
        trans["us_per_call"].append(t_us)
        trans["achieved"].append(t_gbs)
        trans["frac"].append(t_gbs / peaks()[0]["hbm_gbs"])
        del tg_graph

    # ---------------------------------------------------------------- dense GEMM (LoRA-gate shapes)
    # The batch-invariant dense GEMM on the report's LoRA-gate shapes (y[T,N] =
    # x[T,K] . W[N,K]^T, fp32 out).  A CUDA graph of 20 calls that cycle
    # through enough copies of x and W to exceed L2 (so W streams from HBM as
    # it would in a model), replayed 5 times.  Bound per shape: the larger of
    # the tensor time (2TNK at the burst peak) and the HBM time (x, W and y).
    gemm = {"kernel": "T <= 224: decode_fwd_kernel store mode (operands swapped; 64 W rows per "
                      "CTA for T <= 128 and N <= 8192, else 128); larger T: "
                      "pair_kernel<kModeGemm> (256 x 256 pair tiles); fp32 out",
            "timing": "CUDA graph of 20 calls over rotating copies (> L2), replayed 5 times",
            "shapes": [], "us_per_call": [], "tflops": [], "gbs": [], "bound": [], "frac": []}
    for (gN, gK, gT) in ((512, 384, 70), (2048, 1024, 257), (5120, 5120, 33)):
        w_bytes = 2 * (gN + gT) * gK
        ncopy = max(2, -(-256 * 2 ** 20 // w_bytes))
        gx = [torch.randn(gT, gK, device=dev).to(torch.bfloat16) for _ in range(ncopy)]
        gw = [(torch.randn(gN, gK, device=dev) / gK ** 0.5).to(torch.bfloat16) for _ in range(ncopy)]
        gy = torch.empty(gT, gN, device=dev)
        g_ws = torch.zeros(int(binding.lib().rlk_gemm_workspace_bytes()), dtype=torch.uint8,
                           device=dev)
        binding.rlk_gemm_bf16_f32(gx[0], gw[0], out=gy, workspace=g_ws)
        g_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_graph, capture_error_mode="thread_local"):
            for i in range(20):
                binding.rlk_gemm_bf16_f32(gx[i % ncopy], gw[i % ncopy], out=gy, workspace=g_ws)
        g_graph.replay()
        ga0 = torch.cuda.Event(enable_timing=True)
        ga1 = torch.cuda.Event(enable_timing=True)
        ga0.record(stream)
        for _ in range(5):
            g_graph.replay()
        ga1.record(stream)
        torch.cuda.synchronize()
        g_us = 1e3 * ga0.elapsed_time(ga1) / 100
        g_flops = 2.0 * gT * gN * gK
        g_bytes = w_bytes + 4 * gT * gN
        t_tensor = g_flops / (peaks()[0]["bf16_tflops"] * 1e12) * 1e6
        t_hbm = g_bytes / (peaks()[0]["hbm_gbs"] * 1e9) * 1e6
        gemm["shapes"].append("N%d K%d T%d" % (gN, gK, gT))
        gemm["us_per_call"].append(g_us)
        gemm["tflops"].append(g_flops / (g_us * 1e-6) / 1e12)
        gemm["gbs"].append(g_bytes / (g_us * 1e-6) / 1e9)
        gemm["bound"].append("tensor" if t_tensor > t_hbm else "hbm")
        gemm["frac"].append(max(t_tensor, t_hbm) / g_us)
        del g_graph, gx, gw
    gemm["device_error_flags"] = binding.rlk_read_device_error(g_ws)

    # ---------------------------------------------------------------- device-resident
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.nvtx.range_push("rl_step_timed")   # lets ncu capture just this region
        e0.record(stream)
        for _ in range(args.steps):
            step()
        join_exchange()
        e1.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max, tokens_all = aggregate(ms, T)
    flags = binding.rlk_read_device_error(ws)

    # ---------------------------------------------------------------- each pass alone
    # Per-call CUDA events; the SM clock is sampled over each loop (at least
    # ~0.6 s of calls, so that the 100 ms sampler sees several samples).
    def per_call_ms(fn, n, tag):
        for _ in range(3):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        torch.cuda.synchronize()
        with ClockSampler(local, tag) as c:
            for a, b in ev:
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev), c.summary()

    def calls_for(ms_guess, n_min):
        return max(n_min, int(600.0 / ms_guess) + 1)

    fwd_ms, fwd_clk = per_call_ms(lambda: binding.rlk_linear_logp_fwd(hid, W, tg, 1.0, ws,
                                                                      out=(logp, ent, lse)),
                                  calls_for(5.5, args.steps), "_fwd")
    bwd_ms, bwd_clk = per_call_ms(lambda: binding.rlk_linear_logp_bwd(hid, W, tg, 1.0, lse, ent,
                                                                      dl, de, ws, out=(dH, dW)),
                                  calls_for(18.0, args.steps), "_bwd")

    # ---------------------------------------------------------------- the T = 4096 target point
    # Forward + backward at T = 4096, H = 4096, V = 151936 (Qwen-shaped rows:
    # hidden RMS-normalised, per-row dlogp ~ N(0,1), dentropy = 0.001) against
    # the same W; and the forward alone on the same rows (the Qwen3-8B-shaped
    # LM-head forward workload).  Device-resident inputs, W read every call.
    tp_w = wl.target_point(2, with_weight=False)
    T4 = tp_w.T
    hid4 = to_dev_bf16(tp_w.hidden)
    tg4 = torch.from_numpy(tp_w.targets).to(dev)
    dl4 = torch.from_numpy(tp_w.dlogp).to(dev)
    de4 = torch.from_numpy(tp_w.dentropy).to(dev)
    outs4 = tuple(torch.empty(T4, device=dev) for _ in range(3))
    dH4 = torch.empty(T4, H, dtype=torch.bfloat16, device=dev)

    def step4():
        binding.rlk_linear_logp_fwd(hid4, W, tg4, 1.0, ws, out=outs4)
        binding.rlk_linear_logp_bwd(hid4, W, tg4, 1.0, outs4[2], outs4[1], dl4, de4, ws,
                                    out=(dH4, dW))

    t4_ms, t4_clk = per_call_ms(step4, calls_for(17.0, args.steps), "_t4096")
    q_ms, q_clk = per_call_ms(lambda: binding.rlk_linear_logp_fwd(hid4, W, tg4, 1.0, ws,
                                                                  out=outs4),
                              calls_for(4.0, args.steps), "_qwen_fwd")
    del hid4, dH4

    # ---------------------------------------------------------------- one rank of TP = 8
    # Vocab-parallel: rank 0's shard (W rows [0, 24576)) on the same batch;
    # kernels only (the exchange needs the other ranks).
    from invariant_lm_head_gemm_b200 import tp as tpmod
    tp_world = 8
    align = tpmod.shard_alignment(V)
    s0, s1 = tpmod.shard_rows(V, tp_world, 0, align)
    W_s = W[s0:s1]
    Gs = -(-(s1 - s0) // binding.fwd_split_width())
    tp_part = [torch.empty(T, Gs, device=dev) for _ in range(3)]
    tp_yt = torch.empty(T, device=dev)
    R = -(-T // tp_world)
    cps = -(-(s1 - s0) // binding.bwd_chunk_width(V))
    tp_dh = torch.empty(tp_world, cps, R, H, device=dev)
    tp_dW = torch.empty(s1 - s0, H, device=dev)
    tp_f, _ = per_call_ms(lambda: binding.rlk_linear_logp_fwd_shard(hid, W_s, tg, V, s0, 1.0,
                                                                    tp_part, tp_yt, ws),
                          args.steps, "_tpf")
    tp_b, _ = per_call_ms(lambda: binding.rlk_linear_logp_bwd_shard(
        hid, W_s, tg, V, s0, 1.0, lse, ent, dl, de, tp_dh, R, dW_shard=tp_dW, workspace=ws),
        args.steps, "_tpb")
    tp_line = {"tp": tp_world, "shard_rows": s1 - s0, "fwd_shard_ms": tp_f, "bwd_shard_ms": tp_b,
               "tflops": 8.0 * T * H * (s1 - s0) / ((tp_f + tp_b) * 1e-3) / 1e12,
               "note": "rank 0's kernels on one GPU; the all-gathers / all-to-all are not "
                       "included; with 8192-row shard alignment the largest TP = 8 shard holds "
                       "1.29x the mean, which caps TP = 8 at 6.2x one GPU"}
    del tp_dh, tp_dW

    # ---------------------------------------------------------------- end to end, host buffers
    # Every step copies its inputs (hidden, targets, dlogp, dentropy) from
    # pinned host memory and reads its results (logp, entropy and dHidden, which
    # feeds the layer below) back to pinned host memory, all inside the timed
    # region; dW stays on the device for the optimiser.  Inputs and results are
    # double-buffered: the copies run on a second stream, step i+1's inputs and
    # step i-1's results moving while step i computes (events keep a buffer set
    # from being reused before its step and its read-back are done).
    host_in = (torch.from_numpy(w.hidden.view(np.int16)).view(torch.bfloat16).pin_memory(),
               torch.from_numpy(w.targets).pin_memory(),
               torch.from_numpy(w.dlogp).pin_memory(),
               torch.from_numpy(w.dentropy).pin_memory())
    dev_in = [(hid, tg, dl, de), tuple(torch.empty_like(t) for t in (hid, tg, dl, de))]
    res = [torch.empty(2, T, dtype=torch.float32, device=dev) for _ in range(2)]
    dH_set = [dH, torch.empty_like(dH)]
    out_h = [torch.empty(2, T, dtype=torch.float32).pin_memory() for _ in range(2)]
    dH_h = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]

    def copy_in(k):
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(freed[k])      # set k's last step and read-back are done
            for d, h in zip(dev_in[k], host_in):
                d.copy_(h, non_blocking=True)
            copied[k].record(copy_stream)

    def run_set(k):
        stream.wait_event(copied[k])
        h_k, t_k, l_k, e_k = dev_in[k]
        binding.rlk_linear_logp_fwd(h_k, W, t_k, 1.0, ws, out=(res[k][0], res[k][1], lse))
        backward(h_k, t_k, lse, res[k][1], l_k, e_k, (dH_set[k], dW))
        computed[k].record(stream)
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(computed[k])
            out_h[k].copy_(res[k], non_blocking=True)
            dH_h[k].copy_(dH_set[k], non_blocking=True)
            freed[k].record(copy_stream)

    def e2e_steps(n, start_event=None):
        if start_event is not None:
            copy_stream.wait_event(start_event)
        copy_in(0)
        for i in range(n):
            if i + 1 < n:
                copy_in((i + 1) % 2)
            run_set(i % 2)
        join_exchange()
        stream.wait_event(freed[(n - 1) % 2])     # the last read-back is inside the region

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    barrier()
    ee0 = torch.cuda.Event(enable_timing=True)
    ee1 = torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    e2e_steps(args.steps, ee0)
    ee1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms, _ = aggregate(ee0.elapsed_time(ee1) / args.steps, T)
    h2d = T * H * 2 + T * 8 + T * 4 + T * 4
    d2h = 2 * T * 4 + T * H * 2

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, W_host, rows=args.cpu_rows)
        decode["cpu_oracle"], trans["cpu_oracle"] = cpu_oracle_sides(w, W_host)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    pk, src = peaks()
    fwd_traffic, bwd_traffic = measured_traffic()
    flops_tok = 8.0 * H * V
    step_tflops = flops_tok * tokens_all / world / (ms_max * 1e-3) / 1e12
    fwd_tflops = 2.0 * T * H * V / (fwd_ms * 1e-3) / 1e12
    bwd_tflops = 6.0 * T * H * V / (bwd_ms * 1e-3) / 1e12
    t4_tflops = flops_tok * T4 / (t4_ms * 1e-3) / 1e12
    q_tflops = 2.0 * T4 * H * V / (q_ms * 1e-3) / 1e12
    # fwd pair kernel, combine, bwd pair kernel (+ the ordered sums of dW: one
    # per chunk group when overlapped, one otherwise)
    launches_per_step = 3 + ((groups if overlap else 1) if use_rs else 0)
    value = tokens_all / (ms_max * 1e-3)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded Gaussian, bf16-rounded; stands in for Qwen3-8B hidden "
                "states / LM head and DAPO-Math-17k rollouts)",
        "config": config_dict(w, world),
        "tflops_per_gpu": step_tflops,
        "pct_of_bf16_peak": {"burst": step_tflops / pk["bf16_tflops"],
                             "sustained": step_tflops / pk["bf16_tflops_sustained"],
                             "datasheet_2250": step_tflops / 2250.0, "peaks": src},
        "roofline": dict({"kernel": "backward: one persistent pair-kernel launch (logits "
                                    "recompute + dlogits, dHidden and dW GEMMs), timed alone",
                          "bound": "tensor", "achieved": bwd_tflops, "peak": pk["bf16_tflops"],
                          "unit": "TFLOP/s", "frac": bwd_tflops / pk["bf16_tflops"],
                          "frac_of_sustained": bwd_tflops / pk["bf16_tflops_sustained"],
                          "traffic": bwd_traffic, "peak_source": src + " burst bf16",
                          "flops_per_launch": 6.0 * T * H * V, "ms_per_launch": bwd_ms},
                         **clock_fields(bwd_ms, bwd_clk, bwd_tflops, n_sms)),
        "fwd_roofline": dict({"kernel": "forward: pair-kernel GEMM + online logsumexp/entropy + "
                                        "target gather, with its combine, timed alone",
                              "bound": "tensor", "achieved": fwd_tflops,
                              "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": fwd_tflops / pk["bf16_tflops"],
                              "traffic": fwd_traffic, "peak_source": src + " burst bf16",
                              "flops_per_launch": 2.0 * T * H * V, "ms_per_launch": fwd_ms},
                             **clock_fields(fwd_ms, fwd_clk, fwd_tflops, n_sms)),
        "step_roofline": dict({"bound": "tensor", "achieved": step_tflops,
                               "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                               "frac": step_tflops / pk["bf16_tflops_sustained"],
                               "flops_per_token": flops_tok,
                               "peak_source": src + " sustained bf16", "ms_per_step": ms_max},
                              **clock_fields(ms_max, clk.summary(), step_tflops, n_sms)),
        "target_T4096": dict({"workload": "fwd+bwd, T=4096 Qwen-shaped rows (RMS-normalised "
                                          "hidden, seed 2), H=4096, V=151936, tau=1",
                              "tokens_per_s": T4 / (t4_ms * 1e-3), "ms_per_step": t4_ms,
                              "achieved": t4_tflops, "unit": "TFLOP/s",
                              "frac": t4_tflops / pk["bf16_tflops"],
                              "frac_of_sustained": t4_tflops / pk["bf16_tflops_sustained"],
                              "target_tokens_per_s": 0.6 * pk["bf16_tflops"] * 1e12 / flops_tok},
                             **clock_fields(t4_ms, t4_clk, t4_tflops, n_sms)),
        "qwen_fwd": dict({"workload": "Qwen3-8B-shaped LM-head forward only: T=4096 "
                                      "(RMS-normalised hidden), H=4096, V=151936, tau=1",
                          "tokens_per_s": T4 / (q_ms * 1e-3), "ms_per_call": q_ms,
                          "achieved": q_tflops, "unit": "TFLOP/s",
                          "frac": q_tflops / pk["bf16_tflops"],
                          "target_tokens_per_s": 0.6 * pk["bf16_tflops"] * 1e12 / (2.0 * H * V)},
                         **clock_fields(q_ms, q_clk, q_tflops, n_sms)),
        "cpu_baseline": cpu,
        "e2e": {"value": tokens_all / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "copies": "pinned host buffers every step: hidden, targets, dlogp, dentropy in; "
                          "logp, entropy and dHidden back; dW stays on the device for the "
                          "optimiser; inputs and results double-buffered, copies on a second "
                          "stream overlapping the neighbouring steps' compute"},
        "gpu_launches": launches_per_step * args.steps,
        "dw_exchange": {"included": bool(use_rs),
                        "kind": "deterministic reduce-scatter of dW: NCCL all-to-all of "
                                "vocab-row slices, then the rank-ordered sum (rlk_sum_ordered)",
                        "overlapped": bool(overlap),
                        "groups": int(groups) if overlap else (1 if use_rs else 0),
                        "bytes_sent_per_rank": (int((world - 1) * -(-V // world) * H * 4)
                                                if use_rs else 0)},
        "decode_fwd": decode,
        "transition": trans,
        "dense_gemm": gemm,
        "tp_shard": dict(tp_line, frac=tp_line["tflops"] / pk["bf16_tflops"],
                         peak=pk["bf16_tflops"]),
        "clocks": clk.summary(),
        "device_error_flags": flags,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_profile(args):
    """A few calls of one pass (fwd or fwd+bwd) on a smaller seeded case, for
    ncu captures; prints nothing that is a benchmark number."""
    import torch

    from invariant_lm_head_gemm_b200 import binding
    from invariant_lm_head_gemm_b200 import workloads as wl

    if args.profile == "cublas":
        # The library GEMM beside the pair kernel for a like-for-like capture:
        # torch.matmul (cuBLAS) bf16 at the forward's shape, hidden . W^T
        # (T x V x H), and at 8192^3.  Nothing of the operator runs here.
        dev = torch.device("cuda", 0)
        T, H, V = args.T, 4096, args.V
        g = torch.Generator(device="cpu").manual_seed(5)
        hid = torch.randn(T, H, generator=g).to(torch.bfloat16).to(dev)
        W = (0.02 * torch.randn(V, H, generator=g)).to(torch.bfloat16).to(dev)
        a = torch.randn(8192, 8192, generator=g).to(torch.bfloat16).to(dev)
        for _ in range(args.iters):
            hid @ W.t()
            a @ a
        torch.cuda.synchronize()
        print("profile case done: cublas T=%d H=%d V=%d and 8192^3, iters=%d" % (
            T, H, V, args.iters))
        return 0
    if args.profile == "transition":
        B, n = wl.TRANSITION_SHAPES[1]
        tw = wl.transition_case(1, B, n)
        dev = torch.device("cuda", 0)
        tx, tv, te, ta, tc, ts = (torch.from_numpy(np.ascontiguousarray(q)).to(dev)
                                  for q in (tw.x, tw.v, tw.eps, tw.a, tw.c, tw.s))
        ws = binding.transition_workspace(B, n, dev)
        for _ in range(args.iters):
            binding.rlk_transition_sample(tx, tv, te, ta, tc, ts, workspace=ws)
        torch.cuda.synchronize()
        print("profile case done: transition B=%d n=%d iters=%d flags=%d" % (
            B, n, args.iters, binding.rlk_read_device_error(ws)))
        return 0
    T, H, V = args.T, 4096, args.V
    hidden, targets = wl.make_rows(5, T, H, V)
    W = wl.make_weight(5, V, H)
    dev = torch.device("cuda", 0)

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    hid, Wd = bf(hidden), bf(W)
    tg = torch.from_numpy(targets).to(dev)
    dl = torch.ones(T, device=dev)
    de = torch.full((T,), 1e-3, device=dev)
    ws = binding.make_workspace(T, H, V, True, dev)
    for _ in range(args.iters):
        logp, ent, lse = binding.rlk_linear_logp_fwd(hid, Wd, tg, 1.0, ws)
        if args.profile == "bwd":
            binding.rlk_linear_logp_bwd(hid, Wd, tg, 1.0, lse, ent, dl, de, ws)
    torch.cuda.synchronize()
    print("profile case done: %s T=%d H=%d V=%d iters=%d flags=%d" % (
        args.profile, T, H, V, args.iters, binding.rlk_read_device_error(ws)))
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=48)
    ap.add_argument("--ref-rows", type=int, default=48,
                    help="rows of the RL step the reference arm (the fp64 oracle) runs per step")
    ap.add_argument("--dw-exchange", choices=["overlap", "after"], default="overlap",
                    help="N > 1: overlap the dW exchange with the backward (chunk groups on a "
                         "second stream) or run it after the backward")
    ap.add_argument("--dw-group-chunks", type=int, default=4,
                    help="vocab chunks per group of the overlapped dW exchange")
    ap.add_argument("--no-dw-reduce", action="store_true",
                    help="N > 1: leave out the deterministic dW reduce-scatter from the step")
    ap.add_argument("--profile", choices=["fwd", "bwd", "transition", "cublas"], default=None,
                    help="run a small case for an ncu capture instead of the benchmark")
    ap.add_argument("--T", type=int, default=2048, help="rows of the --profile case")
    ap.add_argument("--V", type=int, default=32768, help="vocab of the --profile case")
    ap.add_argument("--iters", type=int, default=3, help="calls in the --profile case")
    args = ap.parse_args()
    if args.profile:
        return run_profile(args)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark of the latent-KV chunk attention hot path on B200.

One step = one denoising pass of one chunk through one Wan2.1-T2V-1.3B-shaped
latent attention layer: cache append (down-projection + ring write), window
3D-RoPE, query absorption, and chunk attention with the fused W_uv
up-projection -- N_q = 4680 queries x 12 heads over N_k = 32760 keys.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun) are replicas: every
rank runs its own independent rollout; the timed region is bracketed by a
barrier and CUDA synchronisation, and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from latent_kv_attention_down_b200 import synth  # noqa: E402

METRIC = "MLA chunk-attention TFLOP/s and query tokens/s, Wan-1.3B layer shape, 1×B200"
WORKLOAD = synth.WAN
N_LAYER_SETS = 12  # distinct layer buffers cycled through: ~1 GB of inputs, far above the 126 MB L2


def step_flops(d=WORKLOAD):
    """Algorithmic FLOPs of one step (absorbed form)."""
    nq, nk = d.n_queries, d.window_tokens
    attn = 2 * nq * nk * d.n_heads * (2 * d.d_latent + d.d_rope)
    append = 2 * nq * d.d_model * (d.d_latent + d.d_rope)
    absorb = 2 * nq * d.n_heads * d.d_nope * d.d_latent
    uv = 2 * nq * d.n_heads * d.d_latent * d.d_head
    return {"attention": attn, "append": append, "q_absorb": absorb, "w_uv": uv,
            "total": attn + append + absorb + uv}


def dense_flops(d=WORKLOAD):
    nq, nk = d.n_queries, d.window_tokens
    return {"attention": 2 * nq * nk * d.n_heads * (2 * d.d_head),
            "append": 2 * nq * d.d_model * (d.d_latent + d.d_rope) + 2 * nq * d.n_heads * d.d_latent * (d.d_nope + d.d_head)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j["hbm_gbs"], j["bf16_tflops"], j.get("bf16_tflops_sustained", j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def profiled_traffic(kernel_file, summary):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken on
    the current source of the kernel (its sha256 is recorded beside it)."""
    path = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "latent_kv_attention_down_b200", "csrc", kernel_file)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    text = open(path).read()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_b):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is busy."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- replicas

def max_over_ranks_of(v: float, dist=None, device="cpu") -> float:
    """The largest of every rank's v (every rank gets it); v itself without a process group."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job rate of independent replicas: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms_per_step_max * 1e-3)


# ----------------------------------------------------------------------------- CPU oracle baseline

def oracle_sample(n_queries=256, heads=None, seed=0):
    """Time the fp64 oracle on a bounded sample of the workload: the full
    32760-key window built from x (down-projection, per-head reconstruction,
    3D-RoPE, softmax) for ``n_queries`` query tokens of the chunk, all heads."""
    import oracle.vmla_oracle as O
    d = WORKLOAD
    w = synth.weights(d, 0, seed)
    frame_x = {}
    for c in range(d.window_frames // d.chunk_frames):
        x = synth.activations(d, 0, c, base_seed=seed)[0]
        for k in range(d.chunk_frames):
            frame_x[c * d.chunk_frames + k] = x[k * d.tokens_per_frame:(k + 1) * d.tokens_per_frame]
    last = d.window_frames // d.chunk_frames - 1
    q = synth.queries(d, 0, last, base_seed=seed)[0]
    rows = np.arange(n_queries)
    t0 = time.perf_counter()
    c, r, kpos, torg = O.window_latents(frame_x, d.window_frames, d.window_frames, w.w_down, d.d_latent,
                                        d.grid_h, d.grid_w)
    qpos = O.chunk_query_positions(last * d.chunk_frames, d.chunk_frames, torg, d.grid_h, d.grid_w)
    O.chunk_attention(c, r, kpos, q, qpos, w.w_uk, w.w_uv, d_nope=d.d_nope, rope_pairs=d.rope_pairs,
                      query_rows=rows, heads=heads)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(n_queries=256):
    secs = oracle_sample(n_queries)
    per_query = step_flops()["total"] / WORKLOAD.n_queries
    return {"value": n_queries * per_query / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle", "query_tokens_per_s": n_queries / secs, "seconds": round(secs, 2),
            "sample": f"fp64 numpy oracle, {n_queries} of the 4680 query tokens x 12 heads over the full "
                      f"32760-key window, window built from x (down-projection, per-head K/V, 3D-RoPE, softmax); "
                      f"TFLOP/s credited at the GPU step's FLOPs per query token"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    n = 128
    times = []
    for _ in range(args.warmup_ref):
        oracle_sample(n)
    for _ in range(args.steps_ref):
        times.append(oracle_sample(n))
    secs = sum(times) / len(times)
    per_query = step_flops()["total"] / WORKLOAD.n_queries
    value = n * per_query / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps_ref, "warmup": args.warmup_ref, "ms_per_step": secs * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "wan1.3b-layer: N_q=4680 (sampled 128), N_k=32760, n_h=12, d_c=192, d_rope=32"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{n} query tokens x 12 heads over the full window per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def run_ours(args, rank, world, local_rank):
    import torch
    from latent_kv_attention_down_b200 import api
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    d = WORKLOAD
    L = N_LAYER_SETS
    cfg = api.config_from_dims(d, layers=L)
    m = api.LatentKVAttention(cfg).allocate(device=dev, design=api.DESIGN_RECON_ONCE, dense=args.dense)
    bf = torch.bfloat16
    seed = 1000 * rank
    wts = [synth.weights(d, l, seed) for l in range(L)]
    W = [tuple(torch.from_numpy(a).to(dev, bf) for a in (w.w_down, w.w_uk, w.w_uv)) for w in wts]
    chunks = d.window_frames // d.chunk_frames
    first = (chunks - 1) * d.chunk_frames
    # fill every layer's 21-frame window (the fill activations are shared by the layers), then give each
    # layer set its own chunk activations, queries and output for the timed passes
    for c in range(chunks):
        x = torch.from_numpy(synth.activations(d, 0, c, base_seed=seed)).to(dev, bf)
        for l in range(L):
            m.append(l, x, W[l][0], c * d.chunk_frames, d.chunk_frames)
            if args.dense:
                m.dense_append(l, x, W[l][0], W[l][1], W[l][2], c * d.chunk_frames, d.chunk_frames)
    xs, qs, outs = [], [], []
    for l in range(L):
        xs.append(torch.from_numpy(synth.activations(d, l, chunks - 1, pass_=1, base_seed=seed)).to(dev, bf))
        qs.append(torch.from_numpy(synth.queries(d, l, chunks - 1, base_seed=seed)).to(dev, bf))
        outs.append(torch.empty((1, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32, device=dev))
    torch.cuda.synchronize()
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"

    def step_with(design):
        def step(i):
            l = i % L
            m.append(l, xs[l], W[l][0], first, d.chunk_frames)
            m.attention(l, qs[l], W[l][1], W[l][2], outs[l], first, d.chunk_frames, design)
        return step

    # the headline step: the design the library's AUTO takes at this window (reconstruct-once)
    step = step_with(api.DESIGN_AUTO)

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(v):
        return max_over_ranks_of(v, dist, dev)

    def timed(fn, steps, warmup, profile=False):
        for i in range(warmup):
            fn(i)
        torch.cuda.synchronize()
        barrier()
        if profile:
            m.profile(True)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        s0.record()
        for i in range(steps):
            fn(warmup + i)
        s1.record()
        torch.cuda.synchronize()
        barrier()
        return s0.elapsed_time(s1)

    def kernel_ms(names):
        """Per-launch milliseconds of each profiled stage (CUDA events around each launch)."""
        out = {}
        for k in names:
            tot, n = m.profile_read(k)
            out[k] = {"ms_per_launch": tot / max(n, 1), "launches": n}
        return out

    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(visible.split(",")[local_rank] if visible else local_rank)
    clocks.start()
    time.sleep(0.3)
    ms = timed(step, args.steps, args.warmup)  # bare: no per-stage events inside the timed loop
    clk = clocks.stop()
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    ms_step = max_over_ranks(ms / args.steps)
    F = step_flops()
    value = replica_throughput(F["total"], ms_step, world) / 1e12
    tokens = replica_throughput(d.n_queries, ms_step, world)
    # the per-kernel breakdown of the same step, from a second pass with CUDA events around each launch
    timed(step, args.steps, 3, profile=True)
    per_kernel = kernel_ms(("append", "rope", "q_absorb", "reconstruct_once", "dense_attention", "attention"))
    m.profile(False)
    auto_design = "recon_once" if per_kernel["dense_attention"]["launches"] else "absorbed"
    per_kernel = {k: v for k, v in per_kernel.items() if v["launches"]}
    launches_per_step = sum(v["launches"] for v in per_kernel.values()) / args.steps

    # the absorbed design's step and kernel, timed the same way (bare, then profiled)
    asteps = max(10, args.steps)
    ms_abs = max_over_ranks(timed(step_with(api.DESIGN_ABSORBED), asteps, 3) / asteps)
    timed(step_with(api.DESIGN_ABSORBED), asteps, 3, profile=True)
    abs_kernels = kernel_ms(("append", "rope", "q_absorb", "attention"))
    m.profile(False)

    # ------------------------------------------------ end to end from pinned host memory
    xh = [xs[l].cpu().pin_memory() for l in range(2)]
    qh = [qs[l].cpu().pin_memory() for l in range(2)]
    oh = [torch.empty(outs[0].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    xd, qd, od = torch.empty_like(xs[0]), torch.empty_like(qs[0]), torch.empty_like(outs[0])

    def e2e_step(i):
        l = i % 2
        m.step_host(l, xh[l], qh[l], oh[l], W[l][0], W[l][1], W[l][2], xd, qd, od, first, d.chunk_frames,
                    api.DESIGN_AUTO)

    e2e_steps = max(10, args.steps // 4)
    ms_e2e = max_over_ranks(timed(e2e_step, e2e_steps, 3) / e2e_steps)
    h2d = xh[0].numel() * 2 + qh[0].numel() * 2
    d2h = oh[0].numel() * 4

    # ------------------------------------------------ dense per-head comparison on the same box
    dense = None
    if args.dense:
        def dense_step(i):
            l = i % L
            m.dense_append(l, xs[l], W[l][0], W[l][1], W[l][2], first, d.chunk_frames)
            m.dense_attention(l, qs[l], outs[l], first, d.chunk_frames)
        dsteps = max(10, args.steps // 4)
        ms_d = timed(dense_step, dsteps, 3, profile=True)
        da_ms, da_n = m.profile_read("dense_attention")
        dap_ms, dap_n = m.profile_read("dense_append")
        m.profile(False)
        DF = dense_flops()
        dense = {"ms_per_step": max_over_ranks(ms_d / dsteps),
                 "attention_ms": da_ms / max(da_n, 1), "append_ms": dap_ms / max(dap_n, 1),
                 "attention_tflops": DF["attention"] / (da_ms / max(da_n, 1) * 1e-3) / 1e12,
                 "cache_scalars_per_token": 2 * d.n_heads * d.d_head, "window_read_bytes": d.window_tokens * 2 * d.n_heads * d.d_head * 2}

    # ------------------------------------------------ design (b): per-head K/V rebuilt inside every key tile
    DF = dense_flops()
    tsteps = max(10, args.steps // 4)
    ms_t = max_over_ranks(timed(step_with(api.DESIGN_RECONSTRUCT), tsteps, 3) / tsteps)
    timed(step_with(api.DESIGN_RECONSTRUCT), tsteps, 3, profile=True)
    tk = kernel_ms(("append", "rope", "q_absorb", "attention_reconstruct"))
    m.profile(False)
    rt_attn_ms = tk["attention_reconstruct"]["ms_per_launch"]
    recon_in_tile = {"ms_per_step": ms_t, "tflops_effective": world * F["total"] / (ms_t * 1e-3) / 1e12,
                     "kernels_ms": {k: v["ms_per_launch"] for k, v in tk.items()},
                     "attention_tflops_issued": (DF["attention"] + 2 * d.window_tokens * d.d_latent * 224 *
                                                 d.n_heads * ((d.n_queries + 127) // 128)) / (rt_attn_ms * 1e-3) / 1e12}

    # ------------------------------------------------ roofline of the dominant kernel (attention)
    hbm, tc_burst, tc_sust, src = load_peaks()
    # the kernel runs inside a timed loop of args.steps chunk steps: past half a second of continuous
    # load the GPU sits at its power cap, so the sustained figure is the matching denominator
    long_run = ms_step * args.steps >= 500.0
    peak = tc_sust if long_run else tc_burst
    peak_source = f"{src} bf16 dense, cuBLAS, " + (
        f"sustained (the kernel runs inside {ms_step * args.steps / 1e3:.1f} s of continuous load)"
        if long_run else "burst (timed region under half a second)")

    def tensor_roofline(kernel, launch_ms, flops, traffic):
        achieved = flops / (launch_ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": peak_source, "frac_of_burst": achieved / tc_burst,
                "frac_of_sustained": achieved / tc_sust, "traffic": traffic, "kernel": kernel,
                "launch_ms": launch_ms, "algorithmic_flops_per_launch": flops}

    if auto_design == "recon_once":
        # d_head = 128 attention over the window's per-head K/V: 2 * N_q * N_k * n_h * (128 + 128) FLOPs
        roofline = tensor_roofline("attn_tc_kernel<128,true,false,32,true>", per_kernel["dense_attention"]["ms_per_launch"],
                                   DF["attention"], profiled_traffic("attn_tc.cu", "attn_per_head_wan_layer.md"))
    else:
        roofline = tensor_roofline("attn_tc_kernel<192,false,false,32>", per_kernel["attention"]["ms_per_launch"],
                                   F["attention"], profiled_traffic("attn_tc.cu", "attn_absorbed_wan_layer.md"))
    absorbed_roofline = tensor_roofline("attn_tc_kernel<192,false,false,32>", abs_kernels["attention"]["ms_per_launch"],
                                        F["attention"], profiled_traffic("attn_tc.cu", "attn_absorbed_wan_layer.md"))
    # HBM-bound kernels: algorithmic bytes per launch
    nq, nk = d.n_queries, d.window_tokens
    append_bytes = nq * d.d_model * 2 + (d.d_latent + d.d_rope) * d.d_model * 2 + nq * (d.d_latent + d.d_rope) * 2
    absorbed_bytes = {"append": append_bytes,
                      "rope": 2 * nk * d.d_rope * 2,
                      "q_absorb": nq * d.n_heads * d.d_head * 2 + d.n_heads * d.d_nope * d.d_latent * 2 +
                      nq * d.n_heads * (d.d_latent + d.d_rope) * 2}
    recon_bytes = {"append": append_bytes,
                   # bf16 queries in, fp16 per-head queries (positional part rotated) out
                   "per_head_queries": 2 * nq * d.n_heads * d.d_head * 2,
                   # latents and positional keys in, 2 * n_h * 128 fp16 scalars per key out
                   "reconstruct_once": nk * (d.d_latent + d.d_rope) * 2 + nk * 2 * d.n_heads * d.d_head * 2}

    def with_bytes(ks, alg):
        for k, b in alg.items():
            if k in ks:
                ks[k]["algorithmic_bytes"] = b
                ks[k]["gbs"] = b / (ks[k]["ms_per_launch"] * 1e-3) / 1e9
                ks[k]["frac_of_hbm"] = ks[k]["gbs"] / hbm
        add_copy_reference(ks, dev)
        return ks

    # the kernels of the headline step (reconstruct-once names its stage-2 kernel for what it does)
    kernels = {("per_head_queries" if auto_design == "recon_once" and k == "q_absorb" else k): dict(v)
               for k, v in per_kernel.items()}
    kernels = with_bytes(kernels, recon_bytes if auto_design == "recon_once" else absorbed_bytes)
    if "per_head_queries" in kernels:
        # launched on the handle's side stream beside the reconstruction: its event time spans the
        # overlap, not the kernel alone
        kernels["per_head_queries"]["overlapped_with"] = "reconstruct_once"
    abs_kernels = with_bytes({k: dict(v) for k, v in abs_kernels.items()}, absorbed_bytes)

    workload = ("wan1.3b-layer chunk step: append 3 frames + attention with the design AUTO takes "
                + ("(recon-once: per-head queries, the window's per-head K/V rebuilt once with its window-relative "
                   "RoPE, d_head=128 attention)" if auto_design == "recon_once"
                   else "(absorbed: window RoPE, q-absorb, attention with fused W_uv)")
                + "; N_q=4680, N_k=32760, n_h=12, d_c=192, d_rope=32, batch 1")
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload, "design": auto_design,
                       "global_batch": world, "seq_len": nk, "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2: {L} layer buffer sets cycled",
                       "flops": "effective: 2*N_q*N_k*n_h*(2*d_c + d_rope) + append + q-absorb + W_uv per step, "
                                "the same numerator for every design"},
            "query_tokens_per_s": tokens, "roofline": roofline, "kernels": kernels,
            "e2e": {"value": world * F["total"] / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms_e2e,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "vmla_chunk_step_host (pinned host x, q -> device, append, attention, out -> host), AUTO"},
            "gpu_launches": int(round(launches_per_step * args.steps)), "clocks": clk}
    line["designs"] = {"auto": auto_design,
                       "absorbed": {"ms_per_step": ms_abs, "tflops_effective": world * F["total"] / (ms_abs * 1e-3) / 1e12,
                                    "kernels": abs_kernels, "roofline": absorbed_roofline},
                       "reconstruct_in_tile": recon_in_tile}
    if args.legs:
        line["legs"] = {"batch8": batch8_leg(m_timed=timed, dev=dev, hbm=hbm, tc=tc_burst, seed=seed),
                        "hbm_saturation": saturation_leg(dev=dev, hbm=hbm, tc=tc_burst, seed=seed),
                        "latent_width": width_leg(m_timed=timed, dev=dev, tc=tc_burst, seed=seed),
                        "sink_window": sink_leg(dev=dev, tc=tc_burst, seed=seed),
                        "folded_output_mixer": folded_leg(dev=dev, tc=tc_burst, seed=seed),
                        "query_latent": qlatent_leg(dev=dev, seed=seed),
                        "rotary_split": rotary_leg(dev=dev, tc=tc_burst, seed=seed)}
    if dense:
        line["dense"] = dense
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_queries)
    if rank == 0:
        print(json.dumps(line), flush=True)
    m.close()


def _pool_fill(m, d, pool, xp, W, layer, chunks):
    for c in range(chunks):
        m.append(layer, pool.activations(layer, c, 0, pool=xp), W[0], c * d.chunk_frames, d.chunk_frames)


def copy_gbs(nbytes, dev, reps=15):
    """What a plain device copy achieves on the same traffic (nbytes/2 read + nbytes/2 written),
    timed like the kernels: CUDA events around each launch, sources cycled through more than
    the L2 so every copy reads HBM; median of `reps`."""
    import torch
    half = max(int(nbytes) // 2 // 16 * 16, 16)
    nbuf = max(2, -(-512 * 2 ** 20 // half))
    src = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(nbuf)]
    dst = torch.empty(half, dtype=torch.uint8, device=dev)
    times = []
    for i in range(reps + 3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src[i % nbuf])
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            times.append(e0.elapsed_time(e1))
    del src, dst
    times.sort()
    return 2 * half / (times[len(times) // 2] * 1e-3) / 1e9


def add_copy_reference(kernels, dev):
    """Attach to every HBM-bound kernel entry the same-size copy rate and the kernel's fraction of it."""
    for e in kernels.values():
        if "algorithmic_bytes" in e:
            c = copy_gbs(e["algorithmic_bytes"], dev)
            e["copy_same_bytes_gbs"] = c
            e["frac_of_same_size_copy"] = e["gbs"] / c


def batch8_leg(m_timed, dev, hbm, tc, seed):
    return batch_leg(8, dev, hbm, tc, seed, steps=20, auto=True)


def saturation_leg(dev, hbm, tc, seed):
    """The HBM-bound kernels at batch 64 (one append moves 1.06 GB, one RoPE pass 268 MB, one
    q-absorb 2.5 GB), where launch and pipeline ramp no longer hide their streaming rate."""
    return batch_leg(64, dev, hbm, tc, seed, steps=3)


def batch_leg(batch, dev, hbm, tc, seed, steps, auto=False):
    """The same layer at batch B: B independent rings, B*4680 queries per call; two layer sets
    alternate so inputs stay above L2.  The absorbed design's step gives the HBM-bound kernels
    (append, RoPE, q-absorb); with `auto` the step AUTO runs (reconstruct-once at d_c 192) is timed
    too."""
    import torch
    from latent_kv_attention_down_b200 import api
    d = WORKLOAD.replace(batch=batch)
    L = 2
    m = api.LatentKVAttention(api.config_from_dims(d, layers=L)).allocate(device=dev)
    pool = synth.FramePool(d, base_seed=seed)
    bf = torch.bfloat16
    xp = torch.from_numpy(pool.x).to(dev, bf)
    qp = torch.from_numpy(pool.q).to(dev, bf)
    W = [tuple(torch.from_numpy(a).to(dev, bf) for a in (w.w_down, w.w_uk, w.w_uv))
         for w in (synth.weights(d, l, seed) for l in range(L))]
    chunks = d.window_frames // d.chunk_frames
    first = (chunks - 1) * d.chunk_frames
    for l in range(L):
        _pool_fill(m, d, pool, xp, W[l], l, chunks)
    xs = [pool.activations(l, chunks - 1, 1, pool=xp) for l in range(L)]
    qs = [pool.queries(l, chunks - 1, 1, pool=qp) for l in range(L)]
    out = torch.empty((d.batch, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32, device=dev)
    del xp, qp

    def step(i):
        l = i % L
        m.append(l, xs[l], W[l][0], first, d.chunk_frames)
        m.attention(l, qs[l], W[l][1], W[l][2], out, first, d.chunk_frames, api.DESIGN_ABSORBED)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    m.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(3 + i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    k = {n: m.profile_read(n) for n in ("append", "rope", "q_absorb", "attention")}
    m.profile(False)
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    F = step_flops(WORKLOAD)
    B = d.batch
    nq, nk = d.n_queries, d.window_tokens
    alg = {"append": B * nq * d.d_model * 2 + (d.d_latent + d.d_rope) * d.d_model * 2 + B * nq * (d.d_latent + d.d_rope) * 2,
           "rope": B * 2 * nk * d.d_rope * 2,
           "q_absorb": B * nq * d.n_heads * d.d_head * 2 + d.n_heads * d.d_nope * d.d_latent * 2 +
           B * nq * d.n_heads * (d.d_latent + d.d_rope) * 2}
    res = {"workload": f"wan1.3b-layer chunk step at batch {B} ({B} rings, N_q={B * nq} per call, "
                       f"N_k={nk} per sample)",
           "ms_per_step": ms, "tflops": B * F["total"] / (ms * 1e-3) / 1e12,
           "query_tokens_per_s": B * nq / (ms * 1e-3), "kernels": {}}
    for n, (t, c) in k.items():
        per = t / max(c, 1)
        e = {"ms_per_launch": per}
        if n in alg:
            e["algorithmic_bytes"] = alg[n]
            e["gbs"] = alg[n] / (per * 1e-3) / 1e9
            e["frac_of_hbm"] = e["gbs"] / hbm
        else:
            e["tflops"] = B * F["attention"] / (per * 1e-3) / 1e12
            e["frac_of_bf16_peak"] = e["tflops"] / tc
        res["kernels"][n] = e
    if auto:
        def step_auto(i):
            l = i % L
            m.append(l, xs[l], W[l][0], first, d.chunk_frames)
            m.attention(l, qs[l], W[l][1], W[l][2], out, first, d.chunk_frames, api.DESIGN_AUTO)

        for i in range(3):
            step_auto(i)
        torch.cuda.synchronize()
        m.profile(True)
        e0.record()
        for i in range(steps):
            step_auto(3 + i)
        e1.record()
        torch.cuda.synchronize()
        ms_a = e0.elapsed_time(e1) / steps
        ka = {n: m.profile_read(n) for n in ("append", "reconstruct_once", "dense_attention")}
        m.profile(False)
        st, flags = m.device_status()
        assert st == 0, f"device status {st} flags {flags:#x}"
        if ka["dense_attention"][1]:
            att = ka["dense_attention"][0] / ka["dense_attention"][1]
            rec = ka["reconstruct_once"][0] / max(ka["reconstruct_once"][1], 1)
            res["auto"] = {"design": "recon_once", "ms_per_step": ms_a,
                           "tflops": B * F["total"] / (ms_a * 1e-3) / 1e12,
                           "query_tokens_per_s": B * nq / (ms_a * 1e-3),
                           "attention_ms": att, "reconstruct_once_ms": rec,
                           "attention_tflops_issued": B * dense_flops()["attention"] / (att * 1e-3) / 1e12,
                           "frac_of_bf16_peak": B * dense_flops()["attention"] / (att * 1e-3) / 1e12 / tc}
    m.close()
    add_copy_reference(res["kernels"], dev)
    return res


def sink_leg(dev, tc, seed, steps=50):
    """The pages' long-horizon context: one sink frame + six recent frames (10920 keys),
    window-relative RoPE, after 12 chunks; one chunk step (append + attention) timed."""
    import torch
    from latent_kv_attention_down_b200 import api
    d = synth.WAN_SINK
    L = 8
    m = api.LatentKVAttention(api.config_from_dims(d, layers=L)).allocate(device=dev)
    pool = synth.FramePool(d, base_seed=seed)
    bf = torch.bfloat16
    xp = torch.from_numpy(pool.x).to(dev, bf)
    qp = torch.from_numpy(pool.q).to(dev, bf)
    W = [tuple(torch.from_numpy(a).to(dev, bf) for a in (w.w_down, w.w_uk, w.w_uv))
         for w in (synth.weights(d, l, seed) for l in range(L))]
    chunks = 12
    for l in range(L):
        for c in range(chunks):
            m.append(l, pool.activations(l, c, 0, pool=xp), W[l][0], c * d.chunk_frames, d.chunk_frames)
    first = (chunks - 1) * d.chunk_frames
    xs = [pool.activations(l, chunks - 1, 1, pool=xp) for l in range(L)]
    qs = [pool.queries(l, chunks - 1, 1, pool=qp) for l in range(L)]
    out = torch.empty((1, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32, device=dev)

    def step(i):
        l = i % L
        m.append(l, xs[l], W[l][0], first, d.chunk_frames)
        m.attention(l, qs[l], W[l][1], W[l][2], out, first, d.chunk_frames, api.DESIGN_ABSORBED)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    m.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    at_ms, at_n = m.profile_read("attention")
    m.profile(False)
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    nk = d.window_tokens
    attn_flops = 2 * d.n_queries * nk * d.n_heads * (2 * d.d_latent + d.d_rope)
    att = at_ms / max(at_n, 1)

    # the design AUTO takes here (reconstruct-once at d_c 192)
    def step_auto(i):
        l = i % L
        m.append(l, xs[l], W[l][0], first, d.chunk_frames)
        m.attention(l, qs[l], W[l][1], W[l][2], out, first, d.chunk_frames, api.DESIGN_AUTO)

    for i in range(3):
        step_auto(i)
    torch.cuda.synchronize()
    m.profile(True)
    e0.record()
    for i in range(steps):
        step_auto(i)
    e1.record()
    torch.cuda.synchronize()
    ms_a = e0.elapsed_time(e1) / steps
    da_ms, da_n = m.profile_read("dense_attention")
    m.profile(False)
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    m.close()
    res = {"workload": "wan1.3b-layer, 1 sink frame + 6 recent frames (N_k=10920), window-relative RoPE, "
                       "chunk 12; the absorbed design's step", "ms_per_step": ms,
           "query_tokens_per_s": d.n_queries / (ms * 1e-3),
           "attention_ms": att, "attention_tflops": attn_flops / (att * 1e-3) / 1e12,
           "frac_of_bf16_peak": attn_flops / (att * 1e-3) / 1e12 / tc}
    if da_n:
        dflops = 2 * d.n_queries * nk * d.n_heads * 256
        res["auto"] = {"design": "recon_once", "ms_per_step": ms_a, "query_tokens_per_s": d.n_queries / (ms_a * 1e-3),
                       "attention_ms": da_ms / da_n, "attention_tflops_issued": dflops / (da_ms / da_n * 1e-3) / 1e12,
                       "frac_of_bf16_peak": dflops / (da_ms / da_n * 1e-3) / 1e12 / tc}
    return res


def folded_leg(dev, tc, seed, steps=50):
    """W_uv folded into the output mixer: the chunk step with out = sum_h (W_O,h W_uv,h) o~_h
    (absorbed attention + one K = 12 x 192 GEMM to d_model = 1536 columns)."""
    import torch
    from latent_kv_attention_down_b200 import api
    d = WORKLOAD
    L = 4
    m = api.LatentKVAttention(api.config_from_dims(d, layers=L)).allocate(device=dev)
    pool = synth.FramePool(d, base_seed=seed)
    bf = torch.bfloat16
    xp = torch.from_numpy(pool.x).to(dev, bf)
    qp = torch.from_numpy(pool.q).to(dev, bf)
    ws = [synth.weights(d, l, seed) for l in range(L)]
    W = [tuple(torch.from_numpy(a).to(dev, bf) for a in (w.w_down, w.w_uk, w.w_uv, w.w_o)) for w in ws]
    folds = []
    for l in range(L):
        f = torch.empty(d.d_model, d.n_heads * d.d_latent, dtype=bf, device=dev)
        m.fold_output_weights(W[l][3], W[l][2], f)
        folds.append(f)
    chunks = d.window_frames // d.chunk_frames
    for l in range(L):
        for c in range(chunks):
            m.append(l, pool.activations(l, c, 0, pool=xp), W[l][0], c * d.chunk_frames, d.chunk_frames)
    first = (chunks - 1) * d.chunk_frames
    xs = [pool.activations(l, chunks - 1, 1, pool=xp) for l in range(L)]
    qs = [pool.queries(l, chunks - 1, 1, pool=qp) for l in range(L)]
    out = torch.empty((1, d.n_queries, d.d_model), dtype=torch.float32, device=dev)

    def step(i):
        l = i % L
        m.append(l, xs[l], W[l][0], first, d.chunk_frames)
        m.attention_folded(l, qs[l], W[l][1], folds[l], out, first, d.chunk_frames)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    m.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    k = {n: m.profile_read(n) for n in ("attention", "folded_mixer")}
    m.profile(False)
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    gemm_ms = k["folded_mixer"][0] / max(k["folded_mixer"][1], 1)
    gemm_flops = 2 * 2 * d.n_queries * d.d_model * d.n_heads * d.d_latent  # rounded part + residual
    m.close()
    return {"workload": "wan1.3b-layer chunk step with W_O W_uv folded (K=2304, d_out=1536)", "ms_per_step": ms,
            "attention_ms": k["attention"][0] / max(k["attention"][1], 1), "mixer_gemm_ms": gemm_ms,
            "mixer_gemm_tflops": gemm_flops / (gemm_ms * 1e-3) / 1e12}


def qlatent_leg(dev, seed, steps=50):
    """The content path absorbed into the query latent: the chunk step whose absorbed queries
    come from c_Q (d_q = 768) by one K = 768 GEMM per head instead of W_uk,h^T q_nope."""
    import torch
    from latent_kv_attention_down_b200 import api
    d = WORKLOAD
    L = 4
    m = api.LatentKVAttention(api.config_from_dims(d, layers=L)).allocate(device=dev)
    pool = synth.FramePool(d, base_seed=seed)
    bf = torch.bfloat16
    xp = torch.from_numpy(pool.x).to(dev, bf)
    ws = [synth.weights(d, l, seed) for l in range(L)]
    W = [tuple(torch.from_numpy(a).to(dev, bf) for a in (w.w_down, w.w_uk, w.w_uv)) for w in ws]
    qabs = []
    for l in range(L):
        w_uq, w_qr = synth.query_latent_weights(d, l, seed)
        f = torch.empty(d.n_heads, d.d_latent + d.d_rope, d.d_q, dtype=bf, device=dev)
        m.fold_query_weights(torch.from_numpy(w_uq).to(dev, bf), torch.from_numpy(w_qr).to(dev, bf), W[l][1], f)
        qabs.append(f)
    chunks = d.window_frames // d.chunk_frames
    for l in range(L):
        for c in range(chunks):
            m.append(l, pool.activations(l, c, 0, pool=xp), W[l][0], c * d.chunk_frames, d.chunk_frames)
    first = (chunks - 1) * d.chunk_frames
    xs = [pool.activations(l, chunks - 1, 1, pool=xp) for l in range(L)]
    cqs = [torch.from_numpy(synth.query_latents(d, l, chunks - 1, 1, seed)).to(dev, bf) for l in range(L)]
    out = torch.empty((1, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32, device=dev)

    def step(i):
        l = i % L
        m.append(l, xs[l], W[l][0], first, d.chunk_frames)
        m.attention_qlatent(l, cqs[l], qabs[l], W[l][2], out, first, d.chunk_frames)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    m.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    k = {n: m.profile_read(n) for n in ("q_absorb", "attention")}
    m.profile(False)
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    q_ms = k["q_absorb"][0] / max(k["q_absorb"][1], 1)
    q_flops = 2 * d.n_queries * d.n_heads * (d.d_latent + d.d_rope) * d.d_q
    m.close()
    return {"workload": "wan1.3b-layer chunk step, absorbed queries from c_Q (d_q=768)", "ms_per_step": ms,
            "query_gemm_ms": q_ms, "query_gemm_tflops": q_flops / (q_ms * 1e-3) / 1e12,
            "attention_ms": k["attention"][0] / max(k["attention"][1], 1)}


def width_leg(m_timed, dev, tc, seed, widths=(64, 128, 192, 256, 384, 512)):
    """Latent width sweep on the Wan layer: attention time of every built design
    and of the dense per-head cache for the same seeded x and q."""
    import torch
    from latent_kv_attention_down_b200 import api
    res = {}
    steps = 10
    bf = torch.bfloat16
    for dc in widths:
        d = WORKLOAD.replace(d_latent=dc)
        L = 2
        m = api.LatentKVAttention(api.config_from_dims(d, layers=L)).allocate(device=dev, design=api.DESIGN_RECON_ONCE,
                                                                              dense=True)
        pool = synth.FramePool(d, base_seed=seed)
        xp = torch.from_numpy(pool.x).to(dev, bf)
        qp = torch.from_numpy(pool.q).to(dev, bf)
        W = [tuple(torch.from_numpy(a).to(dev, bf) for a in (w.w_down, w.w_uk, w.w_uv))
             for w in (synth.weights(d, l, seed) for l in range(L))]
        chunks = d.window_frames // d.chunk_frames
        first = (chunks - 1) * d.chunk_frames
        for l in range(L):
            for c in range(chunks):
                x = pool.activations(l, c, 0, pool=xp)
                m.append(l, x, W[l][0], c * d.chunk_frames, d.chunk_frames)
                m.dense_append(l, x, W[l][0], W[l][1], W[l][2], c * d.chunk_frames, d.chunk_frames)
        qs = [pool.queries(l, chunks - 1, 0, pool=qp) for l in range(L)]
        out = torch.empty((1, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32, device=dev)
        F = step_flops(d)
        entry = {"absorbed_flops": F["attention"], "dense_flops": dense_flops(d)["attention"]}
        designs = [("recon_once", api.DESIGN_RECON_ONCE), ("dense", None)]
        if dc <= 256:
            designs.append(("absorbed", api.DESIGN_ABSORBED))
        if dc <= 192:
            designs.append(("reconstruct_in_tile", api.DESIGN_RECONSTRUCT))
        for name, design in designs:
            def call(i):
                l = i % L
                if design is None:
                    m.dense_attention(l, qs[l], out, first, d.chunk_frames)
                else:
                    m.attention(l, qs[l], W[l][1], W[l][2], out, first, d.chunk_frames, design)
            for i in range(3):
                call(i)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(steps):
                call(i)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
            entry[name] = {"ms_per_call": ms, "tflops_effective": F["attention"] / (ms * 1e-3) / 1e12}
        st, flags = m.device_status()
        assert st == 0, f"device status {st} flags {flags:#x}"
        res[str(dc)] = entry
        m.close()
        del xp, qp, W, qs, out, m
        torch.cuda.empty_cache()
    return res


def rotary_leg(dev, tc, seed, splits=((112, 16, (4, 2, 2)), (96, 32, (6, 5, 5)), (64, 64, (12, 10, 10)),
                                      (32, 96, (16, 16, 16)))):
    """d_head 128 split into content/rotary dims 112/16, 96/32, 64/64 and 32/96 on the Wan layer (d_c
    192, full window): one chunk step per split and design -- the absorbed design, reconstruct-once
    (AUTO's choice) and the dense per-head cache -- with the attention kernel's time and rate."""
    import torch
    from latent_kv_attention_down_b200 import api
    res = {}
    steps = 20
    bf = torch.bfloat16
    for dn, dr, pairs in splits:
        d = WORKLOAD.replace(d_nope=dn, d_rope=dr, rope_pairs=pairs)
        L = 2
        m = api.LatentKVAttention(api.config_from_dims(d, layers=L)).allocate(device=dev, design=api.DESIGN_RECON_ONCE,
                                                                             dense=True)
        pool = synth.FramePool(d, base_seed=seed)
        xp = torch.from_numpy(pool.x).to(dev, bf)
        qp = torch.from_numpy(pool.q).to(dev, bf)
        W = [tuple(torch.from_numpy(a).to(dev, bf) for a in (w.w_down, w.w_uk, w.w_uv))
             for w in (synth.weights(d, l, seed) for l in range(L))]
        chunks = d.window_frames // d.chunk_frames
        first = (chunks - 1) * d.chunk_frames
        for l in range(L):
            _pool_fill(m, d, pool, xp, W[l], l, chunks)
            for c in range(chunks):
                m.dense_append(l, pool.activations(l, c, 0, pool=xp), W[l][0], W[l][1], W[l][2], c * d.chunk_frames,
                               d.chunk_frames)
        xs = [pool.activations(l, chunks - 1, 1, pool=xp) for l in range(L)]
        qs = [pool.queries(l, chunks - 1, 1, pool=qp) for l in range(L)]
        out = torch.empty((1, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32, device=dev)
        F, DF = step_flops(d), dense_flops(d)
        per = {}
        for name, design, stage, flops in (("absorbed", api.DESIGN_ABSORBED, "attention", F["attention"]),
                                           ("recon_once", api.DESIGN_RECON_ONCE, "dense_attention", DF["attention"]),
                                           ("dense", None, "dense_attention", DF["attention"])):
            def step(i):
                l = i % L
                if design is None:
                    m.dense_append(l, xs[l], W[l][0], W[l][1], W[l][2], first, d.chunk_frames)
                    m.dense_attention(l, qs[l], out, first, d.chunk_frames)
                else:
                    m.append(l, xs[l], W[l][0], first, d.chunk_frames)
                    m.attention(l, qs[l], W[l][1], W[l][2], out, first, d.chunk_frames, design)
            for i in range(3):
                step(i)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(steps):
                step(3 + i)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
            m.profile(True)
            for i in range(steps):
                step(3 + steps + i)
            at, n = m.profile_read(stage)
            m.profile(False)
            st, flags = m.device_status()
            assert st == 0, f"device status {st} flags {flags:#x}"
            att = at / max(n, 1)
            per[name] = {"ms_per_step": ms, "attention_ms": att,
                         "tflops_effective": F["total"] / (ms * 1e-3) / 1e12,
                         "attention_tflops_issued": flops / (att * 1e-3) / 1e12,
                         "frac_of_bf16_peak": flops / (att * 1e-3) / 1e12 / tc}
        res[f"{dn}/{dr}"] = per
        m.close()
        del xp, qp, W, xs, qs, out, m
        torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-dense", dest="dense", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-legs", dest="legs", action="store_false",
                    help="skip the batch-8 and latent-width legs")
    ap.add_argument("--cpu-queries", type=int, default=4096)
    ap.add_argument("--steps-ref", type=int, default=None)
    ap.add_argument("--warmup-ref", type=int, default=None)
    args = ap.parse_args()
    args.steps_ref = args.steps_ref if args.steps_ref is not None else min(args.steps, 5)
    args.warmup_ref = args.warmup_ref if args.warmup_ref is not None else min(args.warmup, 1)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

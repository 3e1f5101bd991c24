"""Benchmark of the MoE split-LoRA expert block, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config gpt-oss-20b]

One step = route -> permute -> gate_up + SwiGLU -> down -> weighted combine ->
weighted dY gather -> down / gate_up backward -> LoRA gradients -> dX combine,
all through the C ABI on one stream.  Inputs are seeded synthetic tensors of
the gpt-oss-20b-shaped layer (T = 8192 tokens, H = I = 2880, 32 experts,
top-4, LoRA r = 16, s = 2) resident in HBM before the timed region.

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs an
independent replica (the block has no exchange step on one layer): weak
scaling, time = max over ranks.  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_expert_grouped_softmax_b200 import synthetic as S  # noqa: E402
from moe_expert_grouped_softmax_b200 import workload as WL  # noqa: E402

METRIC = "MoE-LoRA block fwd+bwd tokens/s and TFLOP/s (% BF16 tensor peak) on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def kernel_src_hash():
    """Hash of the kernel sources (csrc + header): ncu counters taken with
    other sources do not describe the kernels being timed."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_expert_grouped_softmax_b200", "csrc")
    for f in sorted(os.listdir(csrc)) + ["../../include/moe_lora.h"]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload):
    """Per-launch DRAM bytes (read + write) from profiles/roofline_traffic.txt,
    or {} when they were taken on other kernel sources or another workload."""
    p = os.path.join(ROOT, "profiles", "roofline_traffic.txt")
    if not os.path.exists(p):
        return {}
    kv = {}
    for line in open(p):
        line = line.split("#")[0].strip()
        if "=" in line:
            k, v = (x.strip() for x in line.split("=", 1))
            kv[k] = v
    if kv.get("src_sha256") != kernel_src_hash() or kv.get("workload") != workload:
        return {}
    return {k: float(v) for k, v in kv.items() if k not in ("src_sha256", "workload")}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, dev):
    """Max of the float x over all ranks of the default process group (every
    rank calls it with its own x); x itself without a group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(T, steps, ws, ms_total):
    """Whole-job throughput: every rank processes T tokens per step (weak
    scaling); ms_total is the slowest rank's total time of the timed steps."""
    return T * steps * ws / (ms_total / 1e3)


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi (every 50 ms,
    into a file) and keeps the samples taken inside [t_begin, t_end]."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None
        self.t_begin = self.t_end = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(1.0)  # let the sampler come up before the timed span

    def stop(self):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        import datetime as dt
        sm, mx, pw, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        lines = open(self.path).read().splitlines() if self.path else []
        for l in lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = dt.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, mxx = float(f[1]), float(f[2])
            except ValueError:
                continue
            if self.t_begin is not None and not (self.t_begin - 0.06 <= ts <= self.t_end + 0.06):
                continue
            sm.append(clk)
            mx = mxx
            try:
                pw.append(float(f[3]))
            except ValueError:
                pass
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if self.path:
            os.unlink(self.path)
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
               "reasons": sorted(reasons), "samples": len(sm)}
        if pw:
            out["power_w_max"] = max(pw)
        return out


# ---------------------------------------------------------------------------
def run_ours(args, cfg):
    import torch.distributed as dist
    from moe_expert_grouped_softmax_b200 import ops

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if args.cta_pairs >= 0:
        ops.set_cta_pairs(bool(args.cta_pairs))
    dev = torch.device("cuda", local)

    T, H, I, E, k, r, s = (cfg[x] for x in ("T", "H", "I", "E", "k", "r", "s"))
    R = T * k
    inp = S.make_inputs(cfg)
    W = [inp[n].to(dev) for n in ("W1", "A1", "B1", "W2", "A2", "B2")]
    X, logits, dY = (inp[n].to(dev) for n in ("X", "logits", "dY"))
    blk = ops.MoeBlock(T, H, I, E, k, r, s, device=dev, full_ft=args.full_ft,
                       train_router=args.train_router)
    Wr = None
    if args.train_router:   # router weights of the trained-router variant
        g = torch.Generator().manual_seed(cfg["seed"] + 77)
        Wr = (torch.randn(E, H, generator=g) * 0.05).to(torch.bfloat16).to(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if ws > 1:
            dist.barrier()

    for _ in range(args.warmup):
        blk.step(X, logits, dY, W, Wr)
    torch.cuda.synchronize()
    st = ops.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    # kernels the library launches per step (host-side count of one eager step)
    l0 = ops.kernel_launches()
    blk.step(X, logits, dY, W, Wr)
    per_step = ops.kernel_launches() - l0
    use_graph = args.launch == "graph"
    if use_graph:
        # one CUDA graph of the whole step, replayed: the same kernels with the
        # same arguments, launched together
        blk.capture(X, logits, dY, W, Wr)
        torch.cuda.synchronize()

    K = args.steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    clk = Clocks(local)
    clk.start()
    barrier()
    torch.cuda.synchronize()
    clk.t_begin = time.time()
    for i in range(K):
        flush.zero_()                      # L2 flush, outside the timed span
        ev0[i].record(stream)
        if use_graph:
            blk.replay()
        else:
            blk.step(X, logits, dY, W, Wr)
        ev1[i].record(stream)
    launches = per_step * K
    torch.cuda.synchronize()
    clk.t_end = time.time()
    barrier()
    clk.stop()
    timed_s = clk.t_end - clk.t_begin
    st = ops.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timed steps")
    ms_steps = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    ms_total = float(sum(ms_steps))
    # per-kernel durations: the same steps again with a CUDA event pair around
    # every launch on the launching stream (kept out of the headline timing
    # above, which they would slow down).  With graph launch the step is
    # captured once more with the events as record nodes and replayed, so
    # that no host launch gap falls inside a kernel's event pair; eager
    # launch records them around each eager launch.
    durations = {kind: [] for kind in ops.PROF_KINDS}
    barrier()
    if use_graph:
        ops.profile_enable(True)
        pgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pgraph):
            blk.step(X, logits, dY, W, Wr)
        torch.cuda.synchronize()
        for i in range(K):
            flush.zero_()
            pgraph.replay()
            torch.cuda.synchronize()
            for kind in ops.PROF_KINDS:
                durations[kind] += ops.profile_collect(kind)
        ops.profile_enable(False)
        del pgraph
    else:
        ops.profile_enable(True)
        for i in range(K):
            flush.zero_()
            blk.step(X, logits, dY, W, Wr)
        torch.cuda.synchronize()
        for kind in ops.PROF_KINDS:   # collect before the hook is switched off
            durations[kind] = ops.profile_collect(kind)
        ops.profile_enable(False)
    kern = {}
    for kind, d in durations.items():
        if d:
            kern[kind] = {"launches": len(d), "avg_ms": float(np.mean(d)),
                          "total_ms": float(np.sum(d))}
    st = ops.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timed steps")
    ms_total = max_over_ranks(ms_total, dev)

    # ---- end to end through the public API with host buffers: every step
    # copies its X, logits and dY from pinned host memory and reads back Y,
    # dX and the four LoRA gradients.  Copies run on their own streams so that
    # step i's inputs and step i-1's results move while step i computes
    # (two block instances, double-buffered).
    e2e = None
    if not args.no_e2e:
        blocks = [blk, ops.MoeBlock(T, H, I, E, k, r, s, device=dev, full_ft=args.full_ft,
                                    train_router=args.train_router)]
        hin = [(X.cpu().pin_memory(), logits.cpu().pin_memory(), dY.cpu().pin_memory())
               for _ in range(2)]
        din = [(torch.empty_like(X), torch.empty_like(logits), torch.empty_like(dY))
               for _ in range(2)]

        def outs(b):
            return [b.Y, b.dX, b.dA1, b.dB1, b.dA2, b.dB2]

        hout = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs(b)]
                for b in blocks]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        comp = torch.cuda.current_stream()
        ev = {n: [torch.cuda.Event() for _ in range(2)]
              for n in ("fwd_in", "bwd_in", "fwd_done", "in_free", "done", "out_free")}

        def run_e2e(nsteps):
            # per block b (two, alternating steps): X and logits upload -> forward;
            # dY upload (overlapping the forward) -> backward; Y download
            # (overlapping the backward), then dX and the gradients
            for i in range(nsteps):
                b = i & 1
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev["in_free"][b])
                    din[b][0].copy_(hin[b][0], non_blocking=True)
                    din[b][1].copy_(hin[b][1], non_blocking=True)
                    ev["fwd_in"][b].record(s_in)
                    din[b][2].copy_(hin[b][2], non_blocking=True)
                    ev["bwd_in"][b].record(s_in)
                comp.wait_event(ev["fwd_in"][b])
                if i >= 2:
                    comp.wait_event(ev["out_free"][b])
                if use_graph:
                    blocks[b].replay_forward()
                else:
                    blocks[b].forward(din[b][0], din[b][1], W, Wr)
                ev["fwd_done"][b].record(comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev["fwd_done"][b])
                    hout[b][0].copy_(outs(blocks[b])[0], non_blocking=True)
                comp.wait_event(ev["bwd_in"][b])
                if use_graph:
                    blocks[b].replay_backward()
                else:
                    blocks[b].backward(din[b][2], W, Wr)
                ev["in_free"][b].record(comp)
                ev["done"][b].record(comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev["done"][b])
                    for o, h in zip(outs(blocks[b])[1:], hout[b][1:]):
                        h.copy_(o, non_blocking=True)
                    ev["out_free"][b].record(s_out)

        if use_graph:
            # each block's forward and backward captured on its own input buffers
            for b in range(2):
                blocks[b].capture_parts(din[b][0], din[b][1], din[b][2], W, Wr)
            torch.cuda.synchronize()
        run_e2e(max(2, args.warmup))
        torch.cuda.synchronize()
        barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        comp.wait_event(t0)
        s_out.wait_event(t0)
        run_e2e(K)
        s_in.wait_stream(s_out)
        s_in.wait_stream(comp)
        t1.record(s_in)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(float(t0.elapsed_time(t1)), dev)
        h2d = sum(h.numel() * h.element_size() for h in hin[0])
        d2h = sum(h.numel() * h.element_size() for h in hout[0])
        e2e = {"value": job_tokens_per_s(T, K, ws, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / K,
               "note": "pinned host buffers; copies on two streams overlap the "
                       "neighbouring steps' compute (double-buffered; dY's upload "
                       "overlaps the forward, Y's download the backward)"
                       + ("; dW1, dW2 stay on the device (an optimizer step would "
                          "consume them there)" if args.full_ft else "")}
        st = ops.device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} after end-to-end steps")

    counts = blk.counts.cpu().numpy()
    return dict(ms_total=ms_total, ms_steps=ms_steps, kern=kern, e2e=e2e,
                clocks=clk.summary(), counts=counts, ws=ws, rank=rank,
                launches=launches, timed_s=timed_s)


_CPU_INPUTS = {}


def cpu_oracle_sample(cfg, n_tok):
    """Times the fp64 oracle (as it stands) on the first n_tok tokens of the
    workload (same weights, same routing rule).  Returns (seconds, threads)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        threads = os.cpu_count() or 1
    key = (cfg["name"], n_tok)
    if key not in _CPU_INPUTS:
        inp = S.make_inputs(cfg)
        _CPU_INPUTS[key] = (
            inp["X"][:n_tok].float().numpy(), inp["logits"][:n_tok].numpy(),
            inp["dY"][:n_tok].float().numpy(),
            [inp[n].float().numpy() for n in ("W1", "A1", "B1", "W2", "A2", "B2")])
    X, L, dY, Wt = _CPU_INPUTS[key]
    t0 = time.perf_counter()
    Y, ctx = O.block_forward(X, L, cfg["k"], *Wt, cfg["s"])
    O.block_backward(dY, ctx)
    return time.perf_counter() - t0, threads


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="gpt-oss-20b", choices=list(S.CONFIGS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--launch", choices=["graph", "eager"], default="graph",
                    help="timed steps as replays of one captured CUDA graph of the step "
                         "(default) or as eager launches")
    ap.add_argument("--extra-configs", default="qwen3-30b-a3b,gpt-oss-20b-long",
                    help="comma-separated configs also measured in the same run "
                         "(device-timed steps only); empty for none")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=128)
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (small cases for profiler captures)")
    ap.add_argument("--full-ft", action="store_true",
                    help="full fine-tuning: also the base-weight gradients dW1, dW2")
    ap.add_argument("--train-router", action="store_true",
                    help="trained router: logits = X Wr^T and its backward in the step")
    ap.add_argument("--cta-pairs", type=int, default=-1,
                    help="1: grouped GEMMs on CTA pairs, 0: single CTAs, "
                         "-1: library default")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    cfg = S.make_config(args.config)
    if args.tokens:
        cfg["T"] = args.tokens
    T, H, I, E, k, r = (cfg[x] for x in ("T", "H", "I", "E", "k", "r"))
    R = T * k
    flops = WL.block_flops(T, H, I, E, k, r, full_ft=args.full_ft,
                           train_router=args.train_router)["total"]
    pk = peaks()
    workload = WORKLOADS[args.config]
    if args.full_ft:
        workload += ", full fine-tuning (base-weight gradients too)"
    if args.train_router:
        workload += ", trained router (logits GEMM and router backward in the step)"
    config = {"workload": workload, "T": T, "H": H, "I": I, "E": E, "top_k": k,
              "lora_r": r, "lora_s": cfg["s"], "logits": cfg["logits"],
              "parallelism": "replicas", "l2": "256 MiB memset before each step, "
              "outside the timed span",
              "launch": ("one CUDA graph of the whole step, replayed" if args.launch == "graph"
                         else "eager launches"),
              "kernel_timing": ("CUDA event pairs as record nodes of a second graph of the "
                                "step, replayed K times after the timed steps"
                                if args.launch == "graph" else
                                "CUDA event pairs around each eager launch, K more steps")}
    ws, rank, _ = dist_env()

    if args.impl == "reference":
        if rank != 0:
            return
        n_tok = max(8, min(T, args.cpu_sample_tokens // 2))
        secs = []
        threads = 1
        for i in range(args.warmup + args.steps):
            dt, threads = cpu_oracle_sample(cfg, n_tok)
            if i >= args.warmup:
                secs.append(dt)
        tot = float(sum(secs))
        val = n_tok * len(secs) / tot
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * tot / len(secs), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads,
                                 "kind": "oracle",
                                 "sample": f"first {n_tok} tokens of the layer per step "
                                           f"(all {E} experts' weights), fwd+bwd"},
                "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch.distributed as dist
    if ws > 1:
        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(dev)
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=300))
    res = run_ours(args, cfg)
    main_rec = analyse(res, cfg, args, pk, flops)
    # the other target shapes, measured in the same run (device-timed steps,
    # no end-to-end or CPU legs): same step, same timing rules
    extras = {}
    for name in [c for c in args.extra_configs.split(",") if c] if not args.tokens else []:
        if name == args.config:
            continue
        ecfg = S.make_config(name)
        eargs = argparse.Namespace(**{**vars(args), "no_e2e": True})
        torch.cuda.empty_cache()
        eres = run_ours(eargs, ecfg)
        ef = WL.block_flops(*(ecfg[x] for x in ("T", "H", "I", "E", "k", "r")),
                            full_ft=args.full_ft, train_router=args.train_router)["total"]
        rec = analyse(eres, ecfg, eargs, pk, ef)
        extras[name] = {"workload": WORKLOADS[name], "T": ecfg["T"], "H": ecfg["H"],
                        "I": ecfg["I"], "E": ecfg["E"], "top_k": ecfg["k"],
                        "lora_r": ecfg["r"], "logits": ecfg["logits"], **rec}
    if ws > 1:
        dist.destroy_process_group()
    if res["rank"] != 0:
        return
    cpu = None
    if not args.no_cpu_baseline:
        n_tok = args.cpu_sample_tokens
        dt, threads = cpu_oracle_sample(cfg, n_tok)
        cpu = {"value": n_tok / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"first {n_tok} tokens of the layer (all {E} experts' weights), "
                         f"fwd+bwd, {dt:.1f} s"}
        # the same oracle on one host thread, on a quarter of that sample
        try:
            from threadpoolctl import threadpool_limits
            n1 = max(8, n_tok // 4)
            with threadpool_limits(limits=1):
                dt1, _ = cpu_oracle_sample(cfg, n1)
            cpu["single_thread"] = {"value": n1 / dt1, "unit": "tokens/s", "cores": 1,
                                    "sample": f"first {n1} tokens, fwd+bwd, {dt1:.1f} s"}
        except ImportError:  # pragma: no cover
            pass
    line = {"metric": METRIC, "value": main_rec["value"], "unit": "tokens/s",
            "n_gpus": res["ws"], "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": main_rec["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": config,
            "tflops": main_rec["tflops"], "frac_of_bf16_peak": main_rec["frac_of_bf16_peak"],
            "flops_per_step": flops, "roofline": main_rec["roofline"],
            "gemm_kernels": main_rec["gemm_kernels"], "hbm_kernels": main_rec["hbm_kernels"],
            "kernels": main_rec["kernels"], "cpu_baseline": cpu, "e2e": res["e2e"],
            "gpu_launches": res["launches"], "clocks": main_rec["clocks"],
            "routing": main_rec["routing"], "configs": extras}
    print(json.dumps(line), flush=True)


def pick_peak(pk, clocks, timed_s):
    """The bf16 tensor peak a kernel's fraction is taken against: the burst
    figure (cuBLAS timed alone), unless this run's own clock record shows a
    seconds-long timed region held down by the power cap, where the
    sustained figure is the matching one."""
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    if capped and timed_s >= 2.0 and "bf16_tflops_sustained" in pk:
        return pk["bf16_tflops_sustained"], (
            f"{pk['source']} sustained bf16 ({timed_s:.1f} s timed region, sw_power_cap active)")
    return pk["bf16_tflops"], f"{pk['source']} burst bf16 (cuBLAS bf16 8192^3, best of 10)"


def analyse(res, cfg, args, pk, flops):
    """Per-step throughput and the per-kernel roofline figures of one run."""
    from moe_expert_grouped_softmax_b200 import ops
    T, H, I, E, k, r = (cfg[x] for x in ("T", "H", "I", "E", "k", "r"))
    R = T * k
    K = args.steps
    ms_per_step = res["ms_total"] / K
    tokens_s = job_tokens_per_s(T, K, res["ws"], res["ms_total"])
    tflops = flops / (ms_per_step / 1e3) / 1e12
    kern = res["kern"]
    clocks = res["clocks"]
    # GEMMs that ran on CTA pairs take their rank-r products from the rank
    # pass, whose FLOPs are then not the GEMM's (the library reports its
    # choice per GEMM: gate_up fwd K = H, down fwd K = I, down bwd K = H,
    # gate_up bwd K = 2I)
    pairs = tuple(ops.uses_cta_pairs(R, E, kr) for kr in (H, I, H, 2 * I))
    gemm_flops = WL.gemm_flops(R, H, I, r, pairs=pairs)
    gemm_names = ("gate_up_fwd", "down_fwd", "down_bwd", "gate_up_bwd", "base_grad")
    dom = max((kk for kk in kern if kk in gemm_names),
              key=lambda kk: kern[kk]["total_ms"], default=None)
    traffic = measured_traffic(cfg["name"] if not args.tokens else "")
    peak, peak_src = pick_peak(pk, clocks, res.get("timed_s", 0.0))
    burst = pk["bf16_tflops"]
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    clk_scale = (smax / sm) if (sm and smax) else None
    roof = None
    gemm_roof = {}
    for kk in gemm_names:
        if kk not in kern:
            continue
        a = gemm_flops[kk] / (kern[kk]["avg_ms"] / 1e3) / 1e12
        gemm_roof[kk] = {"TFLOP_s": a, "frac_of_burst": a / burst,
                         "frac_of_sustained": a / pk.get("bf16_tflops_sustained", burst),
                         "frac_clock_normalised": (a * clk_scale / burst) if clk_scale else None,
                         "flops_per_launch": gemm_flops[kk], "avg_ms": kern[kk]["avg_ms"],
                         "traffic": traffic.get(kk)}
    if dom is not None:
        g = gemm_roof[dom]
        roof = {"kernel": dom, "bound": "tensor", "achieved": g["TFLOP_s"], "peak": peak,
                "unit": "TFLOP/s", "frac": g["TFLOP_s"] / peak, "traffic": traffic.get(dom),
                "peak_source": peak_src, "frac_of_burst_peak": g["frac_of_burst"],
                "frac_of_sustained_peak": g["frac_of_sustained"],
                "frac_clock_normalised": g["frac_clock_normalised"],
                "clock_note": "frac_clock_normalised = achieved x sm_max_mhz / median "
                              "sm_mhz of this run's samples, over the burst peak",
                "flops_per_launch": gemm_flops[dom]}
    hb = WL.hbm_bytes(T, H, E, k)
    hb["lora_grad"] = R * (H + 2 * I + I + H) * 2 + 4 * r * R * 2 + E * r * (3 * H + 3 * I) * 2
    # rank-r passes (one per GEMM that runs on CTA pairs): each streams U
    # [R, K] and the factor [E, K, r] and writes [R, r] twice; mean bytes
    # per launch over the passes of one step
    rank_k = [kr for kr, p in zip((H, I, H, 2 * I), pairs) if p]
    if rank_k:
        hb["rank_down"] = sum(R * kr * 2 + E * r * kr * 2 + 2 * R * r * 2
                              for kr in rank_k) // len(rank_k)
    mem = {}
    for kk in ("permute", "unpermute", "route", "lora_grad", "rank_down"):
        if kk in kern and kk in hb:
            # permute / unpermute run twice per step with the same bytes
            gbs = hb[kk] / (kern[kk]["avg_ms"] / 1e3) / 1e9
            mem[kk] = {"GB_s": gbs, "frac_of_measured_hbm": gbs / pk["hbm_gbs"],
                       "frac_of_8TBs": gbs / 8000.0, "bytes_per_launch": hb[kk],
                       "avg_ms": kern[kk]["avg_ms"], "traffic": traffic.get(kk)}
    return {"value": tokens_s, "ms_per_step": ms_per_step, "tflops": tflops,
            "frac_of_bf16_peak": tflops / burst, "roofline": roof,
            "gemm_kernels": gemm_roof, "hbm_kernels": mem, "kernels": kern,
            "clocks": clocks, "timed_s": res.get("timed_s"),
            "routing": S.routing_stats(res["counts"]), "steps": K}


WORKLOADS = {"gpt-oss-20b": "gpt-oss-20b-shaped MoE layer fwd+bwd",
             "qwen3-30b-a3b": "Qwen3-30B-A3B-shaped MoE layer fwd+bwd",
             "gpt-oss-20b-long": "long-context gpt-oss-20b-shaped MoE layer fwd+bwd",
             "deepseek-v3": "DeepSeek-V3-shaped MoE layer fwd+bwd",
             "tiny": "tiny MoE block fwd+bwd"}


if __name__ == "__main__":
    main()

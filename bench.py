"""Benchmark of the NVFP4 paged-KV hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--T 1|6] [--impl native|reference]

Workload: the long-context agentic batch -- 3 sequences with 330000,
420000 and 470000 cached tokens, 24 query / 4 KV heads, head_dim 256, NVFP4
KV in random page order -- decoding T=1 token each (T=6 for MTP verify).
One step = quantise-append this step's K/V rows + split-K decode attention +
combine, i.e. one attention layer of one decode iteration.  Inputs are
synthetic (seeded N(0,1) bf16, four K channels x10) and resident in HBM;
the 1.4 GB pool is larger than L2, so no flush is needed between steps.

Metric: NVFP4 KV-read GB/s = algorithmic KV bytes of the step (every
visible cached token, K and V, every kv-head, read once) / step time, with
decode tokens/s (B*T query tokens per layer-call / step time) beside it.

The same JSON line carries, as sub-objects measured after the timed
region: the T=6 verify on the same pool, page spill / restore through a
pinned arena, the chunked prefill (TFLOP/s), the fused RoPE + append, a
decode step replayed from a CUDA Graph, and the decode over a K8V4 cache
(the last three are guarded: a failure is reported in its own object).

Launched with torchrun for N > 1: every rank runs its own replica of the
workload (the path has no cross-GPU exchange); the reported value is the
bytes of all ranks over the max-over-ranks time.

--impl reference runs the float64 CPU oracle on a bounded sample of the
same workload on this machine's host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 KV-read GB/s (% of HBM peak) and decode tokens/s at 3x~470k ctx"
FALLBACK_HBM_GBS = 6650.0
REF_BUDGET_S = 90.0  # oracle seconds of a whole --impl reference run
# Rotary embedding for the fused RoPE + append line: the scaling factor of the
# pages' 555k-context example; the base is this library's reading (the pages
# give none).
ROPE_SCALE = 2.12
ROPE_BASE = 1.0e7
DATASHEET_HBM_GBS = 8000.0
DATASHEET_BF16_TFLOPS = 2250.0  # dense

# DRAM traffic of one decode-attention launch, from one ncu capture of the
# kernel built from the sources whose SHA-256 (of their concatenation, in this
# order) is recorded here (profiles/decode_qk4_long_ctx_3x60k_T1.md: 3 x 60000
# cached tokens, T=1, 24/4 heads, d 256).  Traffic grows with the KV bytes
# attended, so it is scaled by them to the benchmarked workload; it applies
# only to that kernel, and once any of its sources changes the figure no
# longer applies and is reported null.
DECODE_CAPTURE = {
    "kernel": "decode_qk4",
    "sources": ["nvfp4_quantized_kv_b200/csrc/decode_qk4.cu",
                "nvfp4_quantized_kv_b200/csrc/sm100.cuh",
                "nvfp4_quantized_kv_b200/csrc/nvkv_common.cuh",
                "include/nvkv.h"],
    "sha256": "cc497b3949b877049093e0c373fdab8f332cd7d4eeca000e7c4e2d88e85a02cb",
    "dram_bytes_read": 207595776,
    "dram_bytes_write": 3718912,
    "kv_bytes": 207363456,
}


def sources_sha256(paths):
    """SHA-256 of the concatenated files (None when one is missing)."""
    h = hashlib.sha256()
    try:
        for rel in paths:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return h.hexdigest()


def decode_traffic(kv_bytes, kernel):
    """DRAM bytes (read + write) of one decode launch attending kv_bytes, or
    None when the kernel or its sources differ from the captured ones."""
    if kernel != DECODE_CAPTURE["kernel"] or not DECODE_CAPTURE["sha256"]:
        return None
    if sources_sha256(DECODE_CAPTURE["sources"]) != DECODE_CAPTURE["sha256"]:
        return None
    per_byte = (DECODE_CAPTURE["dram_bytes_read"] + DECODE_CAPTURE["dram_bytes_write"]) / \
        DECODE_CAPTURE["kv_bytes"]
    return per_byte * kv_bytes


def bf16_peak():
    """Dense 16-bit tensor-core peak (f16 and bf16 MMAs run at the same rate)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(gpu_index), "-lms", "200"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(x: float, device) -> float:
    """The largest value of x over all ranks (the slowest rank's time); x on
    a single process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample(wl, rows_max=6, ctx_cap=None, kv=None):
    """Time the float64 oracle on one (sequence 0, kv-head 0) pair: all its
    query rows over its visible cache (the first ctx_cap positions when
    capped; kv = the pre-generated rows of those positions).  Returns (GB/s
    in the metric's unit, seconds, threads, description)."""
    import oracle
    b, h = 0, 0
    kv_len = int(wl.kv_lens[b]) if ctx_cap is None else min(int(wl.kv_lens[b]), ctx_cap)
    k, v = kv if kv is not None else wl.kv_rows(b, 0, kv_len)
    q = wl.queries()
    G = wl.group
    jobs = []
    for t in range(wl.T):
        for g in range(G):
            n_vis = min(wl.query_position(b, t) + 1, kv_len)
            jobs.append((k, v, h, n_vis, q[b * wl.T + t, h * G + g]))
    jobs = jobs[:rows_max]
    threads = os.cpu_count() or 1
    oracle.lib()  # build / load outside the timed region
    t0 = time.perf_counter()
    oracle.attention_rows(jobs, wl.num_kv_heads, wl.head_dim, wl.sm_scale, threads)
    dt = time.perf_counter() - t0
    kv_bytes = kv_len * wl.head_dim * 2 * (1 / 2 + 1 / 16)  # one kv-head, K and V, NVFP4
    desc = (f"sequence 0 ({kv_len} of {int(wl.kv_lens[b])} tokens), kv-head 0, {len(jobs)} query "
            f"rows (all rows of that pair), float64 oracle, {min(threads, len(jobs))} threads busy")
    return kv_bytes / dt / 1e9, dt, min(threads, len(jobs)), desc


# What each decode kernel computes in (the bench line's dtype).
KERNEL_DTYPE = {
    "decode_qk4": "nvfp4 K codes x nvfp4 q terms (block-scaled MMA), f16 P x exact f16 V MMA, "
                  "fp32 accumulate and softmax",
    "decode_tc": "f16 MMA on exactly dequantised K/V (q rounded to f16), f16 weights, "
                 "fp32 accumulate",
    "decode_simt": "fp32 on CUDA cores",
}


def prefill_oracle_sample(pw):
    """Time the float64 oracle on the prefill chunk's row sample: the first
    64, the last 64 and every 31st query, all heads, each over its causal
    keys (keys and values quantised once per kv-head, rows from the dense
    definition).  Returns (TFLOP/s on the sample, seconds, sampled rows,
    extrapolated seconds for the whole chunk, description)."""
    import oracle
    n = pw.T
    sample = sorted(set(range(min(64, n))) | set(range(max(0, n - 64), n)) | set(range(0, n, 31)))
    q = pw.queries()
    G = pw.group
    kv_len = int(pw.kv_lens[0])
    k, v = pw.kv_rows(0, 0, kv_len)
    oracle.lib()
    t0 = time.perf_counter()
    flops = 0.0
    for h in range(pw.num_kv_heads):
        k_hat = oracle.qdq_rows(np.ascontiguousarray(k[:, h]))
        v_hat = oracle.qdq_rows(np.ascontiguousarray(v[:, h]))
        qs = np.stack([q[i, h * G + g] for i in sample for g in range(G)])
        nvis = [pw.query_position(0, i) + 1 for i in sample for _ in range(G)]
        oracle.attention_dense(k_hat, v_hat, qs, nvis, pw.sm_scale)
        flops += 4.0 * pw.head_dim * sum(nvis)
    dt = time.perf_counter() - t0
    full = 4.0 * pw.head_dim * pw.num_q_heads * sum(pw.query_position(0, i) + 1 for i in range(n))
    desc = (f"{len(sample)} of {n} chunk queries (first 64, last 64, every 31st) x "
            f"{pw.num_q_heads} heads over their causal keys; float64 oracle (dequantised once "
            f"per kv-head, numpy float64 products); measured on the sample, whole chunk "
            f"extrapolated by FLOP")
    return flops / dt / 1e12, dt, len(sample) * pw.num_q_heads, full / (flops / dt), desc


def run_reference(args):
    from nvfp4_quantized_kv_b200 import workload as W
    if int(os.environ.get("RANK", "0")) != 0:
        return
    wl = W.long_context(T=args.T)
    cap = args.ref_ctx
    if cap is None:
        # Size the per-step sample so that all warm-up and timed steps take
        # about REF_BUDGET_S of oracle time: calibrate on 4096 positions.
        probe = oracle_sample(wl, ctx_cap=4096)
        per_step = REF_BUDGET_S / (args.steps + args.warmup)
        cap = int(4096 * per_step / max(probe[1], 1e-6))
        cap = max(256, min(cap, int(wl.kv_lens[0])))
    kv = wl.kv_rows(0, 0, min(cap, int(wl.kv_lens[0])))
    vals = []
    for _ in range(args.warmup):
        oracle_sample(wl, ctx_cap=cap, kv=kv)
    secs = 0.0
    for _ in range(args.steps):
        v, dt, threads, desc = oracle_sample(wl, ctx_cap=cap, kv=kv)
        vals.append(v)
        secs += dt
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--T", type=int, default=1, help="queries per sequence: 1 decode, 6 MTP verify")
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--ref-ctx", type=int, default=None,
                    help="reference arm: cap the sampled context (default: whole sequence 0)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-prefill", action="store_true", help="skip the chunked-prefill line")
    ap.add_argument("--no-spill", action="store_true", help="skip the page spill/restore line")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph replay line (a step captured once, replayed)")
    ap.add_argument("--no-k8v4", action="store_true",
                    help="skip the K8V4-cache decode line (3 x 60k context)")
    ap.add_argument("--no-verify", action="store_true",
                    help="skip the T=6 MTP-verify line (measured on the T=1 pool)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the batch-2, ragged, 3 x 470,001 and T=16 sub-lines")
    ap.add_argument("--ctx", type=str, default=None,
                    help="comma-separated cached lengths replacing 330000,420000,470000 "
                         "(smaller cases for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist
    import nvfp4_quantized_kv_b200 as nv
    from nvfp4_quantized_kv_b200 import workload as W
    from nvfp4_quantized_kv_b200.harness import DeviceWorkload

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: the native arm needs a CUDA GPU (B200); "
                         "--impl reference runs on the host cores")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    ctx = tuple(int(x) for x in args.ctx.split(",")) if args.ctx else (330000, 420000, 470000)
    wl = W.long_context(T=args.T, ctx=ctx)
    dw = DeviceWorkload(wl, dev, fill=None, num_splits=args.num_splits)
    dw.fill_context()
    dw.load_step_inputs()
    S = dw.num_splits or nv.nvkv_default_num_splits()
    stream = torch.cuda.current_stream(dev)

    def step():
        dw.append(stream)
        dw.attend(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    def timed_steps(dw, K):
        """K steps with events around every kernel, on the launching stream;
        returns (ms per step, mean append / decode / combine ms)."""
        wl = dw.wl
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        t_start.record(stream)
        for i in range(K):
            e = ev[i]
            e[0].record(stream)
            nv.nvkv_append(dw.cache, dw.seqs, dw.k_new, dw.v_new, dw.cu_new, wl.batch * wl.T, wl.T,
                           stream)
            e[1].record(stream)
            nv.nvkv_decode_attn(dw.cache, dw.seqs, dw.q, wl.T, wl.num_q_heads, wl.sm_scale, S,
                                dw.workspace, stream)
            e[2].record(stream)
            nv.nvkv_combine(dw.seqs, dw.workspace, wl.T, wl.num_q_heads, wl.num_kv_heads,
                            wl.head_dim, S, dw.out, stream)
            e[3].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        ms = max_over_ranks(t_start.elapsed_time(t_end) / K, dev)
        return (ms, statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
                statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
                statistics.mean(e[2].elapsed_time(e[3]) for e in ev))

    # ---- timed region: K steps, events around every kernel ----
    K = args.steps
    clocks = ClockSampler(local)
    time.sleep(0.3)
    ms, t_append, t_decode, t_combine = timed_steps(dw, K)
    clk = clocks.stop()
    err = dw.err_bits()

    kv_bytes = wl.kv_bytes_per_step()
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    l2_note = (f"inputs larger than L2 ({kv_bytes / 1e9:.2f} GB of KV per step, L2 "
               f"{l2_bytes / 1e6:.0f} MB): no flush needed" if kv_bytes > l2_bytes else
               f"inputs SMALLER than L2 ({kv_bytes / 1e6:.0f} MB of KV, L2 {l2_bytes / 1e6:.0f} MB):"
               f" a profiling size, not a benchmark value")
    value = world * kv_bytes / (ms * 1e-3) / 1e9
    tokens_per_s = world * wl.batch * wl.T / (ms * 1e-3)
    peak, peak_kind = hbm_peak()
    decode_gbs = kv_bytes / (t_decode * 1e-3) / 1e9
    kernel = nv.nvkv_decode_kernel_name(dw.cache, wl.T, wl.num_q_heads)

    # ---- end to end through the public API with host buffers ----
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    h_k = pin(dw.k_new_np.view(np.int16))
    h_v = pin(dw.v_new_np.view(np.int16))
    h_q = pin(dw.q_np.view(np.int16))
    h_out = torch.empty(dw.out.shape, dtype=torch.bfloat16).pin_memory()
    d_k, d_v, d_q = (torch.empty(t.shape, dtype=torch.int16, device=dev) for t in (h_k, h_v, h_q))

    def e2e_step():
        d_k.copy_(h_k, non_blocking=True)
        d_v.copy_(h_v, non_blocking=True)
        d_q.copy_(h_q, non_blocking=True)
        nv.nvkv_append(dw.cache, dw.seqs, d_k.view(torch.bfloat16), d_v.view(torch.bfloat16),
                       dw.cu_new, wl.batch * wl.T, wl.T, stream)
        nv.nvkv_decode_attn(dw.cache, dw.seqs, d_q.view(torch.bfloat16), wl.T, wl.num_q_heads,
                            wl.sm_scale, S, dw.workspace, stream)
        nv.nvkv_combine(dw.seqs, dw.workspace, wl.T, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                        S, dw.out, stream)
        h_out.copy_(dw.out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)
    h2d = h_k.numel() * 2 + h_v.numel() * 2 + h_q.numel() * 2
    d2h = h_out.numel() * 2

    # ---- host KV spill / restore of pool pages through a pinned arena ----
    spill = None
    if not args.no_spill:
        pb = nv.nvkv_page_bytes(wl.num_kv_heads, wl.head_dim)
        n_sp = min(4096, wl.num_pages)
        sp_pages = torch.from_numpy(np.random.default_rng([wl.seed, 17]).choice(
            wl.num_pages, size=n_sp, replace=False).astype(np.int32)).to(dev)
        sp_slots = torch.arange(n_sp, dtype=torch.int32, device=dev)
        arena = torch.empty(n_sp * pb, dtype=torch.uint8).pin_memory()
        for _ in range(3):  # spill then restore the same pairs: the pool is unchanged
            nv.nvkv_pages_spill(dw.cache, sp_pages, sp_slots, arena, dw.err, stream)
            nv.nvkv_pages_restore(dw.cache, sp_pages, sp_slots, arena, dw.err, stream)
        se = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        reps = 5
        torch.cuda.synchronize(dev)
        se[0].record(stream)
        for _ in range(reps):
            nv.nvkv_pages_spill(dw.cache, sp_pages, sp_slots, arena, dw.err, stream)
        se[1].record(stream)
        for _ in range(reps):
            nv.nvkv_pages_restore(dw.cache, sp_pages, sp_slots, arena, dw.err, stream)
        se[2].record(stream)
        torch.cuda.synchronize(dev)
        spill_ms = se[0].elapsed_time(se[1]) / reps
        restore_ms = se[1].elapsed_time(se[2]) / reps
        spill = {"pages": n_sp, "bytes": n_sp * pb, "arena": "pinned host",
                 "spill_ms": spill_ms, "spill_gbs": n_sp * pb / (spill_ms * 1e-3) / 1e9,
                 "restore_ms": restore_ms,
                 "restore_gbs": n_sp * pb / (restore_ms * 1e-3) / 1e9,
                 "device_errors": dw.err_bits()}
        del arena

    # ---- MTP verify (T=6) on the same cached context ----
    verify = None
    if args.T == 1 and not args.no_verify:
        wl6 = W.long_context(T=6, ctx=ctx)
        dw6 = DeviceWorkload(wl6, dev, fill=None, num_splits=args.num_splits, cache_from=dw)
        dw6.load_step_inputs()
        for _ in range(args.warmup):
            dw6.append(stream)
            dw6.attend(stream)
        K6 = max(1, min(K, 500))
        ms6, _, d6, _ = timed_steps(dw6, K6)
        kv6 = wl6.kv_bytes_per_step()
        verify = {"workload": wl6.name, "T": 6, "steps": K6, "ms_per_step": ms6,
                  "kernel": nv.nvkv_decode_kernel_name(dw6.cache, 6, wl6.num_q_heads),
                  "value": world * kv6 / (ms6 * 1e-3) / 1e9, "unit": "GB/s",
                  "decode_attn_ms": d6, "decode_attn_gbs": kv6 / (d6 * 1e-3) / 1e9,
                  "tokens_per_s": world * wl6.batch * wl6.T / (ms6 * 1e-3),
                  "device_errors": dw6.err_bits()}
        del dw6

    # ---- the other decode workloads: batch-2 MTP verify (pools rotated so
    # that a step never finds its KV in L2), the 64-sequence ragged batch,
    # 3 x 470,001 tokens (the metric string's "3x~470k"), and a T=16 verify
    # window on the long pool ----
    def config_line(name, make, copies=1, cache_from=None, K_sub=100):
        try:
            dws = []
            for _ in range(copies):
                w = make()
                d = DeviceWorkload(w, dev, fill=None, num_splits=args.num_splits,
                                   cache_from=cache_from)
                if cache_from is None:
                    d.fill_context()
                d.load_step_inputs()
                dws.append(d)
            w = dws[0].wl
            for i in range(3 * copies):
                dws[i % copies].step(stream)
            Sw = dws[0].num_splits or nv.nvkv_default_num_splits()
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_sub)]
            torch.cuda.synchronize(dev)
            for i in range(K_sub):
                d, e = dws[i % copies], ev[i]
                e[0].record(stream)
                d.append(stream)
                e[1].record(stream)
                nv.nvkv_decode_attn(d.cache, d.seqs, d.q, w.T, w.num_q_heads, w.sm_scale, Sw,
                                    d.workspace, stream)
                e[2].record(stream)
                nv.nvkv_combine(d.seqs, d.workspace, w.T, w.num_q_heads, w.num_kv_heads,
                                w.head_dim, Sw, d.out, stream)
                e[3].record(stream)
            torch.cuda.synchronize(dev)
            kvb = w.kv_bytes_per_step()
            t_dec = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
            t_step = statistics.mean(e[0].elapsed_time(e[3]) for e in ev)
            line = {"workload": w.name, "kernel": nv.nvkv_decode_kernel_name(
                        dws[0].cache, w.T, w.num_q_heads), "T": w.T, "batch": w.batch,
                    "kv_bytes_per_step": kvb, "steps": K_sub, "step_ms": t_step,
                    "step_gbs": kvb / (t_step * 1e-3) / 1e9, "decode_attn_ms": t_dec,
                    "decode_attn_gbs": kvb / (t_dec * 1e-3) / 1e9,
                    "frac": kvb / (t_dec * 1e-3) / 1e9 / peak,
                    "tokens_per_s": w.batch * w.T / (t_step * 1e-3),
                    "l2": (f"{copies} pool copies rotated ({copies * kvb / 1e6:.0f} MB, L2 "
                           f"{l2_bytes / 1e6:.0f} MB)" if copies > 1 else
                           f"KV {kvb / 1e6:.0f} MB per step, L2 {l2_bytes / 1e6:.0f} MB"),
                    "device_errors": max(d.err_bits() for d in dws)}
            del dws
            torch.cuda.empty_cache()
            return line
        except Exception as exc:  # a failure here must not cost the headline line
            return {"workload": name, "error": repr(exc)[:300]}

    configs = None
    if not args.no_configs:
        configs = {}
        if args.T == 1:
            configs["verify_T16"] = config_line(
                "verify_T16", lambda: W.long_context(T=16, ctx=ctx), cache_from=dw, K_sub=50)
        b2 = W.batch2_verify()
        n_copies = max(1, -(-2 * l2_bytes // b2.kv_bytes_per_step()) + 1)
        configs["batch2_T4"] = config_line("batch2_T4", W.batch2_verify, copies=n_copies)
        configs["ragged64"] = config_line("ragged64", W.ragged_batch)

    # ---- chunked prefill (65536 cached + 2048 new tokens), tensor-core kernel ----
    prefill = None
    rope = None
    if not args.no_configs:
        del dw
        torch.cuda.empty_cache()
        configs["long_3x470001"] = config_line(
            "long_3x470001", lambda: W.long_context(T=1, ctx=(470000, 470000, 470000)), K_sub=50)
    else:
        del dw
        torch.cuda.empty_cache()
    if not args.no_prefill:
        pw = W.chunked_prefill()
        # the key-split call with the automatic split count (5 on 148 SMs:
        # 384 tile CTAs fill 2.59 of 3 waves, 1920 fifth-length ones 12.97 of 13)
        pdw = DeviceWorkload(pw, dev, fill=None, prefill_splits=0)
        pdw.fill_context()
        pdw.load_step_inputs()
        pdw.append(stream)
        for _ in range(3):
            pdw.attend(stream)
        pe0 = torch.cuda.Event(enable_timing=True)
        pe1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        pe0.record(stream)
        reps = 10
        for _ in range(reps):
            pdw.attend(stream)
        pe1.record(stream)
        torch.cuda.synchronize(dev)
        p_ms = pe0.elapsed_time(pe1) / reps
        pairs = sum(int(pw.ctx[0]) + i + 1 for i in range(pw.T))  # causal (query, key) pairs
        flops = 4.0 * pw.head_dim * pw.num_q_heads * pairs
        tf_peak, tf_kind = bf16_peak()
        prefill = {"workload": pw.name, "kernel": "prefill_tc",
                   "num_splits": nv.nvkv_prefill_num_splits(pdw.cache, pw.batch, pw.T,
                                                            pw.num_q_heads),
                   "ms": p_ms, "tflops": flops / (p_ms * 1e-3) / 1e12,
                   "flop_per_call": flops, "bound": "tensor", "peak_tflops": tf_peak,
                   "peak_kind": tf_kind, "frac": flops / (p_ms * 1e-3) / 1e12 / tf_peak,
                   "frac_datasheet": flops / (p_ms * 1e-3) / 1e12 / DATASHEET_BF16_TFLOPS,
                   "device_errors": pdw.err_bits()}
        # ---- fused RoPE + quantise-append of the same 2048-row chunk ----
        # (after the prefill timing: it rewrites the chunk's K rotated, then
        # the plain append writes it back unrotated)
        try:
            r = pw.head_dim
            rows = pw.batch * pw.T
            cs = torch.empty((int(pw.kv_lens.max()), r // 2, 2), dtype=torch.float32, device=dev)
            nv.nvkv_rope_table(cs, r, ROPE_BASE, ROPE_SCALE, stream)

            def rope_once():
                nv.nvkv_append_rope(pdw.cache, pdw.seqs, pdw.k_new, pdw.v_new, pdw.cu_new, rows,
                                    pw.T, cs, r, stream)

            def plain_once():
                nv.nvkv_append(pdw.cache, pdw.seqs, pdw.k_new, pdw.v_new, pdw.cu_new, rows, pw.T,
                               stream)

            for _ in range(3):
                rope_once()
                plain_once()
            re_ = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            torch.cuda.synchronize(dev)
            re_[0].record(stream)
            for _ in range(10):
                rope_once()
            re_[1].record(stream)
            for _ in range(10):
                plain_once()
            re_[2].record(stream)
            torch.cuda.synchronize(dev)
            t_rope = re_[0].elapsed_time(re_[1]) / 10
            t_plain = re_[1].elapsed_time(re_[2]) / 10
            # algorithmic bytes: bf16 K and V in, NVFP4 K and V out
            io = rows * pw.num_kv_heads * pw.head_dim * (2 * 2 + 2 * 0.5625)
            rope = {"rows": rows, "rotary_dim": r, "base": ROPE_BASE, "scale": ROPE_SCALE,
                    "ms": t_rope, "gbs": io / (t_rope * 1e-3) / 1e9, "plain_append_ms": t_plain,
                    "plain_append_gbs": io / (t_plain * 1e-3) / 1e9,
                    "device_errors": pdw.err_bits()}
            del cs
        except Exception as exc:  # a failure here must not cost the headline line
            rope = {"error": repr(exc)[:300]}
        del pdw

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, threads, desc = oracle_sample(wl)
        cpu = {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}
        if prefill is not None and "error" not in prefill:
            try:
                tf, pdt, nrows, full_s, pdesc = prefill_oracle_sample(W.chunked_prefill())
                prefill["cpu_baseline"] = {
                    "value": tf, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                    "sample": pdesc, "rows": nrows, "seconds": pdt,
                    "extrapolated_chunk_seconds": full_s}
            except Exception as exc:
                prefill["cpu_baseline"] = {"error": repr(exc)[:300]}

    # ---- decode step captured in a CUDA Graph and replayed (the serving mode
    # of the pages' engine), on its own 3 x 60k context, last so that nothing
    # measured above can depend on it ----
    graph = None
    if not args.no_graph:
        try:
            gw = W.long_context(T=1, ctx=(60000, 60000, 60000))
            gdw = DeviceWorkload(gw, dev, fill=None, num_splits=args.num_splits)
            gdw.fill_context()
            gdw.load_step_inputs()
            for _ in range(3):
                gdw.step()
            torch.cuda.synchronize(dev)
            direct_out = gdw.out.clone()
            cg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(cg):
                gdw.step()
            cg.replay()
            torch.cuda.synchronize(dev)
            same = bool(torch.equal(gdw.out, direct_out))
            reps = 200
            ge = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            cur = torch.cuda.current_stream(dev)
            ge[0].record(cur)
            for _ in range(reps):
                gdw.step()
            ge[1].record(cur)
            for _ in range(reps):
                cg.replay()
            ge[2].record(cur)
            torch.cuda.synchronize(dev)
            d_ms = ge[0].elapsed_time(ge[1]) / reps
            r_ms = ge[1].elapsed_time(ge[2]) / reps
            kvb = gw.kv_bytes_per_step()
            graph = {"workload": gw.name, "direct_ms": d_ms, "replay_ms": r_ms,
                     "direct_gbs": kvb / (d_ms * 1e-3) / 1e9, "replay_gbs": kvb / (r_ms * 1e-3) / 1e9,
                     "replay_equals_direct": same, "device_errors": gdw.err_bits()}
            del cg, gdw
        except Exception as exc:  # a failure here must not cost the lines above
            graph = {"error": repr(exc)[:300]}

    # ---- the same decode step over a K8V4 cache (E4M3 K rows, NVFP4 V), on
    # its own 3 x 60k context ----
    k8 = None
    if not args.no_k8v4:
        try:
            kw = W.long_context(T=1, ctx=(60000, 60000, 60000))
            kdw = DeviceWorkload(kw, dev, fill=None, num_splits=args.num_splits,
                                 kv_format="k8v4")
            kdw.fill_context()
            kdw.load_step_inputs()
            for _ in range(3):
                kdw.step(stream)
            reps = 50
            ke = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            torch.cuda.synchronize(dev)
            ke[0].record(stream)
            for _ in range(reps):
                kdw.step(stream)
            ke[1].record(stream)
            for _ in range(reps):
                kdw.attend(stream)
            ke[2].record(stream)
            torch.cuda.synchronize(dev)
            step_ms = ke[0].elapsed_time(ke[1]) / reps
            attend_ms = ke[1].elapsed_time(ke[2]) / reps
            # K 1 byte per element + an fp32 scale per row, V 4.5 bits per element
            kvb = sum(int(c) + 1 for c in kw.ctx) * kw.num_kv_heads * (
                kw.head_dim + 4 + kw.head_dim * 9 // 16)
            k8 = {"workload": kw.name + "_k8v4",
                  "kernel": nv.nvkv_decode_kernel_name(kdw.cache, kw.T, kw.num_q_heads),
                  "kv_bytes_per_step": kvb, "step_ms": step_ms,
                  "step_gbs": kvb / (step_ms * 1e-3) / 1e9, "attend_ms": attend_ms,
                  "attend_gbs": kvb / (attend_ms * 1e-3) / 1e9,
                  "attend_frac": kvb / (attend_ms * 1e-3) / 1e9 / peak,
                  "l2": f"KV {kvb / 1e6:.0f} MB per step, L2 {l2_bytes / 1e6:.0f} MB",
                  "device_errors": kdw.err_bits()}
            del kdw
        except Exception as exc:  # a failure here must not cost the lines above
            k8 = {"error": repr(exc)[:300]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": KERNEL_DTYPE.get(kernel, kernel),
            "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "context": list(wl.ctx),
                       "T": wl.T, "q_heads": wl.num_q_heads, "kv_heads": wl.num_kv_heads,
                       "head_dim": wl.head_dim, "page_tokens": 16, "num_splits": S,
                       "kv_bytes_per_step": kv_bytes,
                       "l2": l2_note,
                       "parallelism": f"replicas{world}" if world > 1 else "single-gpu"},
            "hbm_frac": value / world / peak,
            "hbm_frac_datasheet": value / world / DATASHEET_HBM_GBS,
            "decode_tokens_per_s": tokens_per_s,
            "kernel_ms": {"append": t_append, "decode_attn": t_decode, "combine": t_combine},
            "roofline": {"bound": "hbm", "achieved": decode_gbs, "peak": peak, "unit": "GB/s",
                         "frac": decode_gbs / peak, "traffic": decode_traffic(kv_bytes, kernel),
                         "kernel": kernel, "peak_kind": peak_kind},
            "e2e": {"value": world * kv_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": 3 * K,
            "clocks": clk,
            "device_errors": err,
            "verify_T6": verify,
            "configs": configs,
            "spill": spill,
            "prefill": prefill,
            "rope_append": rope,
            "cuda_graph": graph,
            "k8v4_decode": k8,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

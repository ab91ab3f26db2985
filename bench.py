#!/usr/bin/env python3
"""Benchmark of one MLA decode step (append, absorb, split attention, combine,
output projection) on DeepSeek-V2 attention shapes: B = 64 sequences,
n_h = 128, ctx = 8192, bf16 latent cache [64, 8192, 576].

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is the whole step's algorithmic HBM
traffic (latent cache read once plus the weights) per second, summed over all
ranks (weak scaling: each rank runs its own batch); `ms_per_step` is the max
over ranks.  `roofline` is the attention call timed on its own stream with
CUDA events inside the timed region.  `e2e` repeats the step through the same
C ABI from pinned host buffers, the per-step host->device and device->host
copies inside the timed region.  `cpu_baseline` times the CPU oracle on a
bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "v2_b64_ctx8k"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--num-parts", type=int, default=0)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the batch size (small cases for profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-query-proj", action="store_true",
                    help="skip the separate timing of the query projection")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the separate timing of attention over an FP8 cache")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the separate timings of the other workloads (V2-Lite, ragged paged, 128K)")
    ap.add_argument("--attn-samples", type=int, default=200,
                    help="attention calls timed one by one for the median and p10/p90")
    ap.add_argument("--only-config", default=None,
                    help="run only the step and attention timing of this workload (any in workloads.WORKLOADS, "
                         "paged and ragged ones included) and print its object; for profiling")
    ap.add_argument("--fused", action="store_true",
                    help="finish the step with mla_combine_out_proj instead of mla_combine_splits + mla_out_proj")
    ap.add_argument("--launch-check", action="store_true",
                    help="only start the ranks, join the process group (gloo without a GPU) and "
                         "report the ranks seen; no GPU work")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1400.0, "fallback"


def measured_traffic(workload_name):
    """DRAM bytes per attention launch from the committed ncu record
    (profiles/attn_pair_traffic.json), scaled there to this workload; None
    when the record is for another workload or the kernel source has changed
    since the capture (a stale counter is not reported)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "attn_pair_traffic.json")) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "head_latent_attention_09_b200", "csrc", "tc_attn_pair.cu")
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except Exception:
        return None
    if workload_name != WORKLOAD or rec.get("kernel_source_sha256") != sha:
        return None
    return float(rec["traffic_per_bench_launch"])


def smallh_traffic(workload_name):
    """DRAM bytes of one 16/32-head attention launch on this workload, from the
    committed ncu record (profiles/attn_smallh_traffic.json); None when the
    kernel source has changed since the capture or the workload is not in it."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "attn_smallh_traffic.json")) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "head_latent_attention_09_b200", "csrc", "tc_attn_smallh.cu")
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except Exception:
        return None
    w = rec.get("workloads", {}).get(workload_name)
    if w is None or rec.get("kernel_source_sha256") != sha:
        return None
    return float(w["traffic_per_launch"])


def algorithmic_bytes(wl, ctx_sum, with_wo=False):
    """Bytes one step must move at least: the latent cache once (sum ctx * D *
    2) plus every weight once (W_DKV, W_KR, W_UK, W_UV [, W_O])."""
    esz = 2 if wl.dtype == "bf16" else 4
    w = (wl.d_c + wl.d_r) * wl.d_model + 2 * wl.n_h * wl.d_h * wl.d_c
    if with_wo:
        w += wl.d_model * wl.n_h * wl.d_h
    return ctx_sum * wl.D * esz + w * esz


def query_proj_bytes(wl, B):
    """Bytes mla_query_proj must move at least: its weights once (W^DQ, W^UQ,
    W^QR, or W^Q, W^QR without query compression), the hidden states read,
    c^Q written and read back by the two up-projections, q^C and q^R written."""
    esz = 2 if wl.dtype == "bf16" else 4
    nq = wl.n_h * (wl.d_h + wl.d_r)
    if wl.d_cq:
        w = wl.d_cq * wl.d_model + nq * wl.d_cq
        act = B * wl.d_model + 3 * B * wl.d_cq + B * nq
    else:
        w = nq * wl.d_model
        act = B * wl.d_model + B * nq
    return (w + act) * esz


def algorithmic_flops(wl, ctx_sum):
    attn = 2 * wl.n_h * ctx_sum * (wl.D + wl.d_c)
    gemms = 2 * wl.B * (wl.n_h * wl.d_h * wl.d_c * 2 + wl.d_model * wl.D)
    return attn, gemms


class ClockSampler:
    """SM clock and throttle-reason samples taken DURING the timed region.

    A thread polls NVML (read-only queries) every millisecond between start()
    and stop(), so that even a timed region of a few milliseconds gets samples
    (an `nvidia-smi -lms` loop needs longer than that to print its first line).
    Without NVML the record says so instead of holding numbers."""

    REASONS = (("hw_slowdown", 0x8), ("sw_power_cap", 0x4), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.thread = None
        self.stop_flag = False
        self.handle = None
        self.err = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            props = torch.cuda.get_device_properties(torch_device)
            bus = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                        props.pci_device_id)
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception as e:  # noqa: BLE001 - any NVML failure just disables sampling
            self.err = f"nvml: {e}"
            self.handle = None

    def _poll(self):
        nv = self.nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while True:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = int(get_reasons(self.handle))
                self.samples.append((sm, mx, rs))
            except Exception as e:  # noqa: BLE001
                self.err = f"nvml poll: {e}"
                return
            if self.stop_flag:
                return
            time.sleep(0.001)

    def start(self):
        if self.handle is None:
            return
        import threading
        self.stop_flag = False
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()
        while not self.samples and self.thread.is_alive():
            time.sleep(0.0005)

    def stop(self):
        if self.thread is None:
            return {"samples": 0, "error": self.err or "no sampler"}
        self.stop_flag = True
        self.thread.join(timeout=5)
        if not self.samples:
            return {"samples": 0, "error": self.err or "no samples"}
        sm = [x[0] for x in self.samples]
        mx = [x[1] for x in self.samples]
        reasons = sorted({n for _, _, r in self.samples for n, bit in self.REASONS if r & bit})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "sm_min_mhz": float(min(sm)), "reasons": reasons, "samples": len(sm),
                "source": "nvml"}


# ----------------------------------------------------------------------------
# multi-rank plumbing (one process per GPU; ranks share nothing on the data path)
# ----------------------------------------------------------------------------

def rank_seed(rank: int) -> int:
    """Seed of a rank's synthetic batch: every rank decodes its own sequences."""
    return 1000 + rank


def reduce_max_over_ranks(values, world, device):
    """Element-wise max over all ranks: the slowest rank sets each time."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_gbs(bytes_per_rank_step, world, ms_per_step):
    """Whole-job throughput: the bytes all ranks moved in one step over the
    (max over ranks) step time."""
    return bytes_per_rank_step * world / (ms_per_step * 1e-3) / 1e9


# ----------------------------------------------------------------------------
# CPU oracle timing (the baseline; also the --impl reference arm)
# ----------------------------------------------------------------------------

def cpu_oracle_sample(wl, n_heads, budget_s=20.0):
    """Time the oracle's explicit-form decode step (per-head keys and values,
    textbook softmax) for one sequence of the workload, over `n_heads` heads,
    repeating up to ~budget_s.  Returns (GB/s of latent cache scanned, sample
    description, threads)."""
    from oracle import mla_oracle as O
    from workloads import draw_weights, queries, random_cache
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    ctx = int(wl.ctx[0]) if wl.ctx else 8192
    w = draw_weights(wl)
    rows = random_cache(wl.with_(B=1), ctx)[0].astype(np.float64)
    qn, qr = queries(wl)
    heads = list(range(n_heads))
    reps, t0 = 0, time.perf_counter()
    while True:
        O.mla_decode_explicit(qn[0], qr[0], ctx - 1, rows, w["w_uk"], w["w_uv"], n_h=wl.n_h,
                              d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=wl.rope_base, heads=heads)
        reps += 1
        el = time.perf_counter() - t0
        if el > budget_s or reps >= 50:
            break
    # algorithmic bytes of the sample: the sequence's latent rows once per
    # pass, scaled to the fraction of heads processed (per-head work).
    per_rep = ctx * wl.D * 2 * (n_heads / wl.n_h)
    gbs = per_rep * reps / el / 1e9
    desc = (f"explicit fp64 oracle, 1 sequence x ctx {ctx} x {n_heads}/{wl.n_h} heads, "
            f"{reps} reps in {el:.1f}s, GB/s scaled by head fraction")
    return gbs, desc, threads, el / reps


def cpu_oracle_workload(wl, budget_s=15.0):
    """The oracle's explicit-form decode step, every head, over the workload's
    sequences in order (each sequence's rows the same seeded draw, cut to its
    length) until all are done or budget_s has passed.  Returns a dict: GB/s
    of latent cache scanned, how much of the workload ran, and the step time
    that rate implies for the whole workload."""
    from oracle import mla_oracle as O
    from workloads import ctx_lengths, draw_weights, queries, random_cache
    ctx = ctx_lengths(wl)
    w = draw_weights(wl)
    qn, qr = queries(wl)
    rows = random_cache(wl.with_(B=1, ctx=(int(ctx.max()),)) if wl.ctx else wl.with_(B=1),
                        int(ctx.max()))[0].astype(np.float64)
    done_tok, done_seq, t0 = 0, 0, time.perf_counter()
    for b in range(wl.B):
        n = int(ctx[b])
        if n > 0:
            O.mla_decode_explicit(qn[b], qr[b], n - 1, rows[:n], w["w_uk"], w["w_uv"], n_h=wl.n_h, d_h=wl.d_h,
                                  d_c=wl.d_c, d_r=wl.d_r, base=wl.rope_base)
            done_tok += n
        done_seq += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    total = int(ctx.sum())
    return {"workload": wl.name, "sequences": f"{done_seq}/{wl.B}", "full": done_seq == wl.B,
            "tokens": done_tok, "seconds": el,
            "value": done_tok * wl.D * (2 if wl.dtype == "bf16" else 4) / el / 1e9 if el > 0 else None,
            "unit": "GB/s", "us_per_step": el / max(done_tok, 1) * total * 1e6,
            "kind": "oracle (explicit fp64, every head)",
            "note": "whole workload" if done_seq == wl.B else "sequences in order until the time budget; us_per_step extrapolated by tokens"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from workloads import WORKLOADS
    wl = WORKLOADS[args.workload]
    n_heads = 16
    vals = []
    for i in range(args.warmup + args.steps):
        gbs, desc, threads, t = cpu_oracle_sample(wl, n_heads, budget_s=0.0)
        if i >= args.warmup:
            vals.append(t)
    t = float(np.mean(vals))
    per_step = wl.ctx[0] * wl.D * 2 * n_heads / wl.n_h
    value = per_step / t / 1e9
    line = {
        "metric": "MLA decode: HBM GB/s (% of peak) and us/step at B=64, n_h=128, ctx 8K",
        "impl": "reference", "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "n_h": wl.n_h, "ctx": wl.ctx[0],
                   "sample_per_step": f"1 sequence x {n_heads} heads (explicit fp64 oracle)"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"1 sequence x ctx {wl.ctx[0]} x {n_heads}/{wl.n_h} heads per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

FP8_WORKLOAD = "v2lite_b4_ctx128k"


def fp8_cache_bytes(tokens, D, groups):
    """Bytes an FP8 cache holds for `tokens` rows: D one-byte codes and
    `groups` float32 scales per row."""
    return tokens * (D + 4 * groups)


def measure_fp8(M, dev, steps, seed):
    """Attention over the same latent cache stored in bf16 and in FP8 (E4M3
    codes + one float32 scale per token and 128-channel group), on the
    V2-Lite 128K workload (16 heads, 4 x 131072 tokens: 604 MB in bf16,
    312 MB in FP8, both larger than L2).  The FP8 cache is quantised from the
    bf16 one by the library.  Returns the mean CUDA-event time of each
    attention call (split plan included) and the bytes each one must read."""
    import torch
    from workloads import WORKLOADS
    wl = WORKLOADS[FP8_WORKLOAD]
    B, H, D, d = wl.B, wl.n_h, wl.D, wl.d_model
    ctx = np.asarray(wl.ctx, dtype=np.int64)
    cap = int(ctx.max())
    cfg = M.mla_config(n_h=H, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, d_model=d, page_size=0,
                       rope_base=wl.rope_base, dtype=M.MLA_BF16)
    handle = M.mla_create(cfg)
    try:
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        bf = torch.bfloat16

        def randn(*shape, std=1.0):
            return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(bf)

        w_dkv = randn(wl.d_c, d, std=d ** -0.5)
        w_kr = randn(wl.d_r, d, std=d ** -0.5)
        cache = torch.empty((B, cap, D), dtype=bf, device=dev)
        chunk = 4096
        for b in range(B):
            for t0 in range(0, int(ctx[b]), chunk):
                t1 = min(int(ctx[b]), t0 + chunk)
                sp = torch.tensor([t0], dtype=torch.int32, device=dev)
                M.mla_cache_append(handle, randn(t1 - t0, d), 1, t1 - t0, sp, w_dkv, w_kr,
                                   cache.data_ptr() + 2 * b * cap * D, cap)
        G = M.mla_fp8_scale_groups(handle)
        codes = torch.empty((B, cap, D), dtype=torch.uint8, device=dev)
        scales = torch.empty((B, cap, G), dtype=torch.float32, device=dev)
        M.mla_quantize_rows_fp8(handle, cache, B * cap, codes, scales)
        q_abs = randn(B, H, D, std=0.5)
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).to(dev)
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        stream = torch.cuda.current_stream()
        sh = stream.cuda_stream

        def timed(call):
            for _ in range(3):
                call()
            torch.cuda.synchronize()
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
            for e in ev:
                e[0].record(stream)
                call()
                e[1].record(stream)
            torch.cuda.synchronize()
            return float(np.mean([e[0].elapsed_time(e[1]) for e in ev])) * 1e3

        us_bf16 = timed(lambda: M.mla_decode_attn(handle, q_abs, cache, cap, None, 0, ctx_d, B, P,
                                                  ws, ws_bytes, sh))
        us_fp8 = timed(lambda: M.mla_decode_attn_fp8(handle, q_abs, codes, scales, cap, None, 0,
                                                     ctx_d, B, P, ws, ws_bytes, sh))
        st = M.mla_get_device_status(handle, sh)
        if st != M.MLA_OK:
            raise M.MlaError(st, "device status after the FP8 timing")
    finally:
        M.mla_destroy(handle)
    tokens = int(ctx.sum())
    return {"workload": FP8_WORKLOAD, "tokens": tokens, "bf16_us": us_bf16, "fp8_us": us_fp8,
            "bf16_bytes": tokens * D * 2, "fp8_bytes": fp8_cache_bytes(tokens, D, G)}


EXTRA_WORKLOADS = ("v2lite_b32_ctx4k", "v2lite_paged_ragged_b128", "v2lite_b4_ctx128k")


def measure_workload(M, wl, dev, steps, seed, hbm_peak, n_samples=100):
    """The decode step (append, absorb, attention, combine, output projection)
    and the attention call alone on another workload's shapes, with its own
    cache filled through mla_cache_append from random hidden states.  A cache
    smaller than twice L2 is kept in two copies used alternately, so that
    every step reads its cache from HBM.  Returns times (µs), the algorithmic
    bytes and the roofline fraction of the attention call."""
    import torch
    from workloads import block_table, ctx_lengths
    B, H, D, d = wl.B, wl.n_h, wl.D, wl.d_model
    ctx = ctx_lengths(wl)
    cfg = M.mla_config(n_h=H, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, d_model=d, page_size=wl.page_size,
                       rope_base=wl.rope_base, dtype=M.MLA_BF16)
    handle = M.mla_create(cfg)
    try:
        M.mla_set_strict(handle, 1)
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        bf = torch.bfloat16

        def randn(*shape, std=1.0):
            return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(bf)

        w_dkv = randn(wl.d_c, d, std=d ** -0.5)
        w_kr = randn(wl.d_r, d, std=d ** -0.5)
        w_uk = randn(H * wl.d_h, wl.d_c, std=wl.d_c ** -0.5)
        w_uv = randn(H * wl.d_h, wl.d_c, std=wl.d_c ** -0.5)
        tokens = int(ctx.sum())
        cache_bytes = tokens * D * 2
        props = torch.cuda.get_device_properties(dev)
        l2 = int(getattr(props, "L2_cache_size", 126 << 20) or (126 << 20))
        copies = 2 if cache_bytes < 2 * l2 else 1
        if wl.page_size:
            table_np, pool = block_table(wl, ctx)
            table = torch.from_numpy(table_np).to(dev)
            max_blk, cap = table_np.shape[1], pool
            caches = [torch.empty((pool, wl.page_size, D), dtype=bf, device=dev) for _ in range(copies)]
        else:
            table, max_blk = None, 0
            cap = int(ctx.max())
            caches = [torch.empty((B, cap, D), dtype=bf, device=dev) for _ in range(copies)]
        chunk = 4096
        for c in caches:
            for b in range(B):
                n = int(ctx[b]) - 1
                for t0 in range(0, n, chunk):
                    t1 = min(n, t0 + chunk)
                    sp = torch.tensor([t0], dtype=torch.int32, device=dev)
                    if wl.page_size:
                        M.mla_cache_append(handle, randn(t1 - t0, d), 1, t1 - t0, sp, w_dkv, w_kr, c, cap,
                                           table.data_ptr() + 4 * b * max_blk, max_blk)
                    else:
                        M.mla_cache_append(handle, randn(t1 - t0, d), 1, t1 - t0, sp, w_dkv, w_kr,
                                           c.data_ptr() + 2 * b * cap * D, cap)
        h_new = randn(B, 1, d)
        q_nope = randn(B, H, wl.d_h)
        q_rope = randn(B, H, wl.d_r)
        pos = torch.from_numpy((ctx - 1).astype(np.int32)).to(dev)
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).to(dev)
        q_abs = torch.empty((B, H, D), dtype=bf, device=dev)
        ctx_lat = torch.empty((B, H, wl.d_c), dtype=bf, device=dev)
        o = torch.empty((B, H, wl.d_h), dtype=bf, device=dev)
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        stream = torch.cuda.current_stream()
        sh = stream.cuda_stream

        def step(i):
            c = caches[i % copies]
            M.mla_cache_append(handle, h_new, B, 1, pos, w_dkv, w_kr, c, cap, table, max_blk, sh)
            M.mla_absorb_q(handle, q_nope, q_rope, pos, w_uk, q_abs, B, sh)
            M.mla_decode_attn(handle, q_abs, c, cap, table, max_blk, ctx_d, B, P, ws, ws_bytes, sh)
            M.mla_combine_splits(handle, ws, ws_bytes, B, P, ctx_lat, None, sh)
            M.mla_out_proj(handle, ctx_lat, w_uv, None, o, None, B, sh)

        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
        step_us = t0.elapsed_time(t1) * 1e3 / steps
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_samples)]
        for i, e in enumerate(ev):
            c = caches[i % copies]
            e[0].record(stream)
            M.mla_decode_attn(handle, q_abs, c, cap, table, max_blk, ctx_d, B, P, ws, ws_bytes, sh)
            e[1].record(stream)
        torch.cuda.synchronize()
        st = M.mla_get_device_status(handle, sh)
        if st != M.MLA_OK:
            raise M.MlaError(st, f"device status after the {wl.name} timing")
        t = np.array([e[0].elapsed_time(e[1]) * 1e3 for e in ev])
    finally:
        M.mla_destroy(handle)
    med = float(np.median(t))
    gbs = cache_bytes / (med * 1e-6) / 1e9
    traffic = smallh_traffic(wl.name) if H in (16, 32) else None
    w_bytes = ((wl.d_c + wl.d_r) * d + 2 * H * wl.d_h * wl.d_c) * 2
    return {"B": B, "n_h": H, "tokens": tokens, "page_size": wl.page_size, "cache_bytes": cache_bytes,
            "cache_copies": copies, "num_parts": P, "us_per_step": step_us,
            "step_gbs": (cache_bytes + w_bytes) / (step_us * 1e-6) / 1e9,
            "attn_median_us": med, "attn_p10_us": float(np.percentile(t, 10)),
            "attn_p90_us": float(np.percentile(t, 90)), "attn_gbs": gbs, "attn_frac": gbs / hbm_peak,
            "tokens_scanned_per_s": tokens / (med * 1e-6), "attn_us_at_70pct_of_8TBps": cache_bytes / 5.6e6,
            "bound": "hbm",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "traffic": traffic, "kernel": "mla_decode_attn (plan + attention)"}}


def run_only_config(args):
    """One workload's decode step and attention calls (measure_workload), on
    one GPU; prints its object.  Lets a profiler capture the attention kernel
    of any workload, paged and ragged ones included."""
    import torch

    import head_latent_attention_09_b200 as M
    from head_latent_attention_09_b200 import build as _build
    from workloads import WORKLOADS
    torch.cuda.set_device(0)
    _build.build()
    M.load()
    r = measure_workload(M, WORKLOADS[args.only_config], torch.device("cuda", 0), args.steps, rank_seed(0) + 29,
                         peaks()[0], n_samples=max(1, min(args.attn_samples, 100)))
    print(json.dumps({"workload": args.only_config, **r}), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    import head_latent_attention_09_b200 as M
    from head_latent_attention_09_b200 import build as _build
    from workloads import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {world} rank(s) were started")
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    M.load()

    wl = WORKLOADS[args.workload]
    if args.batch:
        wl = wl.with_(B=args.batch, ctx=(wl.ctx[0],) * args.batch)
    B, H, D, d = wl.B, wl.n_h, wl.D, wl.d_model
    ctx = np.asarray(wl.ctx, dtype=np.int64)
    cfg = M.mla_config(n_h=H, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, d_model=d,
                       page_size=wl.page_size, rope_base=wl.rope_base, dtype=M.MLA_BF16)
    handle = M.mla_create(cfg)
    g = torch.Generator(device=dev)
    g.manual_seed(rank_seed(rank))
    bf = torch.bfloat16

    def randn(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(bf)

    w_dkv = randn(wl.d_c, d, std=d ** -0.5)
    w_kr = randn(wl.d_r, d, std=d ** -0.5)
    w_uk = randn(H * wl.d_h, wl.d_c, std=wl.d_c ** -0.5)
    w_uv = randn(H * wl.d_h, wl.d_c, std=wl.d_c ** -0.5)
    cap = int(ctx.max())
    cache = torch.empty((B, cap, D), dtype=bf, device=dev)
    # Fill positions 0 .. ctx-2 through the library's own append kernel.
    chunk = 4096
    for b in range(B):
        for t0 in range(0, int(ctx[b]) - 1, chunk):
            t1 = min(int(ctx[b]) - 1, t0 + chunk)
            hb = randn(t1 - t0, d)
            sp = torch.tensor([t0], dtype=torch.int32, device=dev)
            M.mla_cache_append(handle, hb, 1, t1 - t0, sp, w_dkv, w_kr,
                               cache.data_ptr() + 2 * b * cap * D, cap)
    h_new = randn(B, 1, d)
    q_nope = randn(B, H, wl.d_h)
    q_rope = randn(B, H, wl.d_r)
    pos = torch.from_numpy((ctx - 1).astype(np.int32)).to(dev)
    ctx_d = torch.from_numpy(ctx.astype(np.int32)).to(dev)
    q_abs = torch.empty((B, H, D), dtype=bf, device=dev)
    ctx_lat = torch.empty((B, H, wl.d_c), dtype=bf, device=dev)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    o = torch.empty((B, H, wl.d_h), dtype=bf, device=dev)
    P = args.num_parts or M.mla_default_num_parts(handle)
    ws_bytes = M.mla_decode_workspace_size(handle, B, P)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def finish(o_out, lse_out):
        # merge of the split partials and the output projection: two calls
        # (the faster in the step, measured), or (--fused) mla_combine_out_proj
        if args.fused:
            M.mla_combine_out_proj(handle, ws, ws_bytes, B, P, w_uv, None, o_out, None, None, lse_out, sh)
        else:
            M.mla_combine_splits(handle, ws, ws_bytes, B, P, ctx_lat, lse_out, sh)
            M.mla_out_proj(handle, ctx_lat, w_uv, None, o_out, None, B, sh)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        M.mla_cache_append(handle, h_new, B, 1, pos, w_dkv, w_kr, cache, cap, None, 0, sh)
        if ev is not None:
            ev[1].record(stream)
        M.mla_absorb_q(handle, q_nope, q_rope, pos, w_uk, q_abs, B, sh)
        if ev is not None:
            ev[2].record(stream)
        M.mla_decode_attn(handle, q_abs, cache, cap, None, 0, ctx_d, B, P, ws, ws_bytes, sh)
        if ev is not None:
            ev[3].record(stream)
        finish(o, lse)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st = M.mla_get_device_status(handle, sh)
    if st != M.MLA_OK:
        raise M.MlaError(st, "device status after warm-up")

    # ---- timed region: K steps.  Events bracket only the attention call (the
    # roofline kernel); events between the other calls would stop the next
    # kernel from starting while the previous one finishes.
    def timed_step(ev):
        M.mla_cache_append(handle, h_new, B, 1, pos, w_dkv, w_kr, cache, cap, None, 0, sh)
        M.mla_absorb_q(handle, q_nope, q_rope, pos, w_uk, q_abs, B, sh)
        ev[0].record(stream)
        M.mla_decode_attn(handle, q_abs, cache, cap, None, 0, ctx_d, B, P, ws, ws_bytes, sh)
        ev[1].record(stream)
        finish(o, lse)

    clocks = ClockSampler(dev)
    clocks.start()
    attn_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        timed_step(attn_ev[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end) / args.steps
    attn_ms = float(np.mean([ev[0].elapsed_time(ev[1]) for ev in attn_ev]))
    st = M.mla_get_device_status(handle, sh)
    if st != M.MLA_OK:
        raise M.MlaError(st, "device status after timing")

    # ---- per-call breakdown (a separate pass after the timed region: events
    # between every call, so no call overlaps its neighbours here)
    call_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for i in range(args.steps):
        step(call_ev[i])
    torch.cuda.synchronize()
    names = ["cache_append", "absorb_q", "decode_attn",
             "combine_out_proj" if args.fused else "combine_splits + out_proj"]
    per_call = {n: float(np.mean([ev[j].elapsed_time(ev[j + 1]) for ev in call_ev])) * 1e3
                for j, n in enumerate(names)}
    # the two calls each on its own, and the fused call (same workspace)
    two_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        two_ev[i][0].record(stream)
        M.mla_combine_splits(handle, ws, ws_bytes, B, P, ctx_lat, lse, sh)
        two_ev[i][1].record(stream)
        M.mla_out_proj(handle, ctx_lat, w_uv, None, o, None, B, sh)
        two_ev[i][2].record(stream)
        M.mla_combine_out_proj(handle, ws, ws_bytes, B, P, w_uv, None, o, None, None, lse, sh)
        two_ev[i][3].record(stream)
    torch.cuda.synchronize()
    per_call["combine_splits"] = float(np.mean([e[0].elapsed_time(e[1]) for e in two_ev])) * 1e3
    per_call["out_proj"] = float(np.mean([e[1].elapsed_time(e[2]) for e in two_ev])) * 1e3
    per_call["combine_out_proj (fused, not in the step)" if not args.fused else "combine_out_proj (fused)"] = \
        float(np.mean([e[2].elapsed_time(e[3]) for e in two_ev])) * 1e3

    # ---- the attention call alone, timed one call at a time (the latent
    # cache is larger than L2, so every call reads it from HBM): median and
    # spread of the roofline kernel's time.
    n_s = max(args.attn_samples, 1)
    s_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_s)]
    for i in range(n_s):
        s_ev[i][0].record(stream)
        M.mla_decode_attn(handle, q_abs, cache, cap, None, 0, ctx_d, B, P, ws, ws_bytes, sh)
        s_ev[i][1].record(stream)
    torch.cuda.synchronize()
    attn_samples_us = np.array([e[0].elapsed_time(e[1]) * 1e3 for e in s_ev])
    st = M.mla_get_device_status(handle, sh)
    if st != M.MLA_OK:
        raise M.MlaError(st, "device status after the attention samples")

    # ---- the query projection from the hidden state (upstream of the step):
    # its weights fit in L2, so a buffer larger than L2 is written before every
    # call and the events bracket the call alone.
    qproj = None
    if not args.no_query_proj:
        if wl.d_cq:
            w_dq = randn(wl.d_cq, d, std=d ** -0.5)
            w_uq = randn(H * wl.d_h, wl.d_cq, std=wl.d_cq ** -0.5)
            w_qr = randn(H * wl.d_r, wl.d_cq, std=wl.d_cq ** -0.5)
            c_q = torch.empty((B, wl.d_cq), dtype=bf, device=dev)
        else:
            w_dq, c_q = None, None
            w_uq = randn(H * wl.d_h, d, std=d ** -0.5)
            w_qr = randn(H * wl.d_r, d, std=d ** -0.5)
        qn_out = torch.empty_like(q_nope)
        qr_out = torch.empty_like(q_rope)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        q_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for i in range(3 + args.steps):
            flush.fill_(i & 0xFF)
            if i >= 3:
                q_ev[i - 3][0].record(stream)
            M.mla_query_proj(handle, h_new, B, w_dq, wl.d_cq or 0, w_uq, w_qr, c_q, qn_out, qr_out, sh)
            if i >= 3:
                q_ev[i - 3][1].record(stream)
        torch.cuda.synchronize()
        st = M.mla_get_device_status(handle, sh)
        if st != M.MLA_OK:
            raise M.MlaError(st, "device status after the query projection")
        q_us = float(np.mean([ev[0].elapsed_time(ev[1]) for ev in q_ev])) * 1e3
        del flush
        qproj = {"us": q_us, "bytes": query_proj_bytes(wl, B)}

    # ---- end to end: host buffers in pinned memory, copies inside the timed region
    hp = {k: v.cpu().pin_memory() for k, v in
          (("h_new", h_new), ("q_nope", q_nope), ("q_rope", q_rope), ("pos", pos), ("ctx", ctx_d))}
    o_host = torch.empty(o.shape, dtype=bf).pin_memory()
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in hp.items()}
    h2d = sum(v.numel() * v.element_size() for v in hp.values())
    d2h = o_host.numel() * o_host.element_size()

    def e2e_step():
        for k in hp:
            dev_in[k].copy_(hp[k], non_blocking=True)
        M.mla_cache_append(handle, dev_in["h_new"], B, 1, dev_in["pos"], w_dkv, w_kr, cache, cap,
                           None, 0, sh)
        M.mla_absorb_q(handle, dev_in["q_nope"], dev_in["q_rope"], dev_in["pos"], w_uk, q_abs, B, sh)
        M.mla_decode_attn(handle, q_abs, cache, cap, None, 0, dev_in["ctx"], B, P, ws, ws_bytes, sh)
        finish(o, lse)
        o_host.copy_(o, non_blocking=True)

    for _ in range(3):
        e2e_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_serial_ms = e0.elapsed_time(e1) / args.steps

    # The same steps with the transfers overlapped: every step still copies its
    # own inputs from pinned host memory and reads its result back, but the
    # host-to-device copies run on one stream and the device-to-host reads on
    # another, into double buffers, so step i's copies overlap the compute of
    # steps i-1 and i+1.
    def e2e_pipelined_ms():
        copy_s = torch.cuda.Stream(device=dev)
        d2h_s = torch.cuda.Stream(device=dev)
        ins = [{k: torch.empty_like(v, device=dev) for k, v in hp.items()} for _ in range(2)]
        outs = [torch.empty_like(o) for _ in range(2)]
        o_hosts = [torch.empty(o.shape, dtype=bf).pin_memory() for _ in range(2)]
        in_ready = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]         # step using ins[k], outs[k] computed
        out_free = [torch.cuda.Event() for _ in range(2)]     # device-to-host read of outs[k] done
        for k in range(2):
            done[k].record(stream)
            out_free[k].record(d2h_s)

        def one(i):
            k = i & 1
            copy_s.wait_event(done[k])
            with torch.cuda.stream(copy_s):
                for name in hp:
                    ins[k][name].copy_(hp[name], non_blocking=True)
            in_ready[k].record(copy_s)
            stream.wait_event(in_ready[k])
            stream.wait_event(out_free[k])
            d = ins[k]
            # no event between the five calls, so that each kernel's set-up
            # still overlaps the previous one's tail
            M.mla_cache_append(handle, d["h_new"], B, 1, d["pos"], w_dkv, w_kr, cache, cap, None, 0, sh)
            M.mla_absorb_q(handle, d["q_nope"], d["q_rope"], d["pos"], w_uk, q_abs, B, sh)
            M.mla_decode_attn(handle, q_abs, cache, cap, None, 0, d["ctx"], B, P, ws, ws_bytes, sh)
            finish(outs[k], lse)
            done[k].record(stream)
            d2h_s.wait_event(done[k])
            with torch.cuda.stream(d2h_s):
                o_hosts[k].copy_(outs[k], non_blocking=True)
            out_free[k].record(d2h_s)

        for i in range(3):
            one(i)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(copy_s)
        for i in range(args.steps):
            one(i)
        stream.wait_stream(copy_s)
        stream.wait_stream(d2h_s)
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / args.steps

    if world > 1:
        dist.barrier()
    e2e_mode = "pipelined: inputs and results double-buffered, copies on their own streams"
    try:
        e2e_ms = e2e_pipelined_ms()
    except Exception as exc:  # keep the serial figure rather than lose the line
        e2e_ms = e2e_serial_ms
        e2e_mode = f"serial (pipelined run failed: {type(exc).__name__}: {exc})"
    st = M.mla_get_device_status(handle, sh)
    if st != M.MLA_OK:
        raise M.MlaError(st, "device status after the end-to-end runs")

    # ---- attention over an FP8 cache (a separate workload, rank 0 only)
    fp8 = None
    if not args.no_fp8 and rank == 0:
        fp8 = measure_fp8(M, dev, args.steps, rank_seed(rank) + 17)

    # ---- the other workloads (rank 0 only): V2-Lite, ragged paged, 128K
    configs = None
    if not args.no_configs and rank == 0 and not args.batch:
        hbm_peak_, _, _ = peaks()
        configs = {}
        for name in EXTRA_WORKLOADS:
            configs[name] = measure_workload(M, WORKLOADS[name], dev, args.steps, rank_seed(rank) + 29,
                                             hbm_peak_, n_samples=min(n_s, 100))

    # ---- reduce over ranks: max time
    ms, attn_ms, e2e_ms, e2e_serial_ms = reduce_max_over_ranks([ms, attn_ms, e2e_ms, e2e_serial_ms],
                                                               world, dev)
    if world > 1:
        dist.barrier()
    M.mla_destroy(handle)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    ctx_sum = int(ctx.sum())
    step_bytes = algorithmic_bytes(wl, ctx_sum)
    attn_bytes = ctx_sum * D * 2
    hbm_peak, tf_peak, peak_kind = peaks()
    value = whole_job_gbs(step_bytes, world, ms)
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9
    attn_flops, gemm_flops = algorithmic_flops(wl, ctx_sum)
    cpu = None
    if not args.no_cpu_baseline:
        gbs, desc, threads, _ = cpu_oracle_sample(wl, 16, budget_s=15.0)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc}
        if not args.batch:
            cpu["configs"] = {name: cpu_oracle_workload(WORKLOADS[name], budget_s=45.0)
                              for name in ("tiny_fp32", "v2lite_b32_ctx4k", "v2lite_paged_ragged_b128")}
    line = {
        "metric": "MLA decode: HBM GB/s (% of peak) and us/step at B=64, n_h=128, ctx 8K",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "us_per_step": ms * 1e3,
        "pct_of_peak": 100.0 * value / world / hbm_peak,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "n_h": H, "d_h": wl.d_h, "d_c": wl.d_c,
                   "d_r": wl.d_r, "d_model": d, "ctx": int(ctx[0]), "num_parts": P,
                   "cache_bytes": attn_bytes,
                   "l2": "inputs larger than L2 (latent cache %.0f MB per rank)" % (attn_bytes / 1e6),
                   "parallelism": f"dp{world} (independent batches, no collective)"},
        "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": attn_gbs / hbm_peak,
                     "traffic": measured_traffic(wl.name) if not args.batch else None,
                     "peak_kind": peak_kind, "kernel": "mla_decode_attn (plan + attention)",
                     "attn_us": attn_ms * 1e3,
                     "frac_of_8TBps": attn_gbs / 8000.0,
                     "tensor_tflops": attn_flops / (attn_ms * 1e-3) / 1e12},
        "e2e": {"value": whole_job_gbs(step_bytes, world, e2e_ms), "unit": "GB/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": e2e_mode, "serial_ms_per_step": e2e_serial_ms,
                "serial_value": whole_job_gbs(step_bytes, world, e2e_serial_ms)},
        "steps_per_s": world * 1e3 / ms,
        "tokens_scanned_per_s": world * ctx_sum / (ms * 1e-3),
        "attention_samples": {
            "n": int(attn_samples_us.size), "median_us": float(np.median(attn_samples_us)),
            "p10_us": float(np.percentile(attn_samples_us, 10)),
            "p90_us": float(np.percentile(attn_samples_us, 90)),
            "median_gbs": attn_bytes / (float(np.median(attn_samples_us)) * 1e-6) / 1e9,
            "median_frac": attn_bytes / (float(np.median(attn_samples_us)) * 1e-6) / 1e9 / hbm_peak,
            "tokens_scanned_per_s": ctx_sum / (float(np.median(attn_samples_us)) * 1e-6),
            "note": "mla_decode_attn alone, one call per event pair, after the timed region"},
        "gpu_launches": (5 if args.fused else 6) * args.steps,
        "step_calls": ("mla_cache_append, mla_absorb_q, mla_decode_attn (plan + attention), " +
                       ("mla_combine_out_proj" if args.fused else "mla_combine_splits, mla_out_proj")),
        "per_call_us": per_call,
        "per_call_note": "separate pass after the timed region, events between all calls",
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    if fp8 is not None:
        fp8_gbs = fp8["fp8_bytes"] / (fp8["fp8_us"] * 1e-6) / 1e9
        bf16_gbs = fp8["bf16_bytes"] / (fp8["bf16_us"] * 1e-6) / 1e9
        line["fp8_kv"] = {
            "workload": fp8["workload"], "tokens": fp8["tokens"],
            "fp8_attn_us": fp8["fp8_us"], "bf16_attn_us": fp8["bf16_us"],
            "speedup": fp8["bf16_us"] / fp8["fp8_us"],
            "fp8_algorithmic_bytes": fp8["fp8_bytes"], "fp8_achieved_gbs": fp8_gbs,
            "fp8_frac": fp8_gbs / hbm_peak, "bf16_achieved_gbs": bf16_gbs,
            "bf16_frac": bf16_gbs / hbm_peak, "bound": "hbm",
            "note": "mla_decode_attn_fp8 vs mla_decode_attn on the same cache; not part of the step"}
    if configs is not None:
        line["configs"] = configs
    # the step's GEMMs against both of their rooflines: tensor pipe (bf16,
    # sustained peak) and HBM (their weights and activations once)
    esz = 2
    gemm_work = {
        "cache_append": (2.0 * B * D * d, (D * d + B * d + B * D) * esz),
        "absorb_q": (2.0 * B * H * wl.d_h * wl.d_c, (H * wl.d_h * wl.d_c + B * H * wl.d_h + B * H * D) * esz),
        "out_proj": (2.0 * B * H * wl.d_h * wl.d_c, (H * wl.d_h * wl.d_c + B * H * wl.d_c + B * H * wl.d_h) * esz),
    }
    line["gemms"] = {}
    for name, (fl, by) in gemm_work.items():
        us = per_call[name]
        line["gemms"][name] = {
            "us_per_call": us, "gflop": fl / 1e9, "tflops": fl / (us * 1e-6) / 1e12,
            "tensor_frac": fl / (us * 1e-6) / 1e12 / tf_peak, "algorithmic_bytes": by,
            "gbs": by / (us * 1e-6) / 1e9, "hbm_frac": by / (us * 1e-6) / 1e9 / hbm_peak}
    line["gemms"]["note"] = ("per call, events between calls; tensor_frac against the bf16 sustained peak "
                             "(TFLOP/s), hbm_frac against the HBM peak")
    if qproj is not None:
        gbs = qproj["bytes"] / (qproj["us"] * 1e-6) / 1e9
        line["query_proj"] = {
            "us": qproj["us"], "algorithmic_bytes": qproj["bytes"], "achieved_gbs": gbs,
            "frac": gbs / hbm_peak, "bound": "hbm",
            "note": "mla_query_proj alone, L2 flushed before each call; not part of the step"}
    print(json.dumps(line), flush=True)


def rank_launch_command(args_gpus: int, argv, port: int):
    """The command that runs this script as `args_gpus` ranks on one node, one
    process per GPU (torch.distributed.run, rendezvous on 127.0.0.1), with the
    same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={args_gpus}", "--master-addr", "127.0.0.1",
            "--master-port", str(port), os.path.abspath(__file__), *argv]


def _free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_check(args):
    """Join the process group the ranks were started with and report the
    ranks seen (rank 0 prints one JSON line)."""
    import datetime
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    backend = "nccl" if torch.cuda.is_available() and torch.cuda.device_count() >= world else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    ranks = [None] * world
    dist.all_gather_object(ranks, rank)
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"launch_check": True, "world": world, "ranks": sorted(ranks),
                          "backend": backend}), flush=True)


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # Started as a plain process: start the ranks ourselves, one per GPU.
        import subprocess
        cmd = rank_launch_command(args.gpus, sys.argv[1:], _free_port())
        sys.exit(subprocess.call(cmd))
    if args.launch_check:
        launch_check(args)
    elif args.only_config:
        run_only_config(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

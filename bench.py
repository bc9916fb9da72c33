#!/usr/bin/env python
"""Benchmark of the routed mixed-precision KV cache on B200.

One step = one decode step of the 1.3B-like decode workload (batch 64, 16 heads,
head_dim 128, 8192 cached tokens, w = 512): roll each sequence back to 8191 tokens,
quantize-on-write the step's new token of every (sequence, head) (Eq. 4), then routed
decode attention (Eq. 2: scheduler, split-K kernel, log-sum-exp combine) for the query at
t = 8191. `value` = attended KV tokens per second (keys actually read; skip heads read
none, local heads w + 1), timed over K back-to-back steps with nothing recorded between
launches. A separate pass records CUDA events around the split-K kernel of each step for
the kernel's roofline. The same line carries the HBM rate of the routed bytes, the other
workloads (long-context decode; ragged and 160M-like prefill + write: TFLOP/s and GB/s;
grouped-query decode), an end-to-end figure through host buffers and the CPU oracle as a
baseline (one thread and all host cores).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the full workload on its own GPU (independent replicas, no
collective on the data path; weak scaling); rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "decode attended-KV tokens/s & HBM GB/s (% of ~8 TB/s); prefill TFLOP/s"
UNIT = "attended-KV tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples of one GPU while it runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(device_index)
        self.ident = ident

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        t0 = time.time()
        while self.proc and time.time() - t0 < 5 and os.path.getsize(self.path) == 0:
            time.sleep(0.05)

    def mark(self):
        return time.time()

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t_begin: float, t_end: float):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
                except Exception:
                    continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        inside = [r for r in rows if t_begin - 1 <= r[0] <= t_end + 1] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# ------------------------------------------------------------------ workload setup
def paged_pool_pages(wl, page_bytes, dev):
    """Pages a paged cache of the workload needs: each (sequence, head) stream's record
    bytes (widths from the seeded draws) rounded up to whole pages."""
    from mixed_precision_kv_write_b200 import synth
    n = 0
    for s in range(wl.batch):
        per = (synth.widths(wl, s, dev).to(torch.int64) * wl.head_dim // 4).sum(0)
        n += int(((per + page_bytes - 1) // page_bytes).sum())
    return n


def decode_setup(wl, dev, group=1, page_bytes=0):
    """Cache holding L - 1 tokens per sequence; the step's token, query and modes; the
    exact keys and routed bytes one step reads. With group > 1 the cache holds wl.heads KV
    heads shared by groups of `group` query heads (grouped-query attention); with
    page_bytes > 0 the records live in a page pool sized for the workload's widths."""
    from mixed_precision_kv_write_b200 import kvq, synth
    B, H, D, L, w = wl.batch, wl.heads, wl.head_dim, wl.seqlens[0], wl.w
    HQ = H * group
    pool = paged_pool_pages(wl, page_bytes, dev) + B * H if page_bytes else 0
    cache = kvq.KVQCache(B, H, D, [L + 4] * B, device=dev, query_group=group, page_bytes=page_bytes,
                         pool_pages=pool)
    q, modes = synth.decode_queries(synth.scaled(wl, heads=HQ) if group > 1 else wl, dev)
    k_step = torch.empty((B, H, D), dtype=torch.float16, device=dev)
    v_step = torch.empty_like(k_step)
    b_step = torch.empty((B, H), dtype=torch.uint8, device=dev)
    keys = rec_bytes = side_bytes = unique_bytes = 0
    idx = torch.arange(L, device=dev)
    kv_of = torch.arange(HQ, device=dev) // group
    for s in range(B):
        ks, vs, bs = synth.kv_sequence(wl, s, dev)
        one = synth.cu_seqlens([L - 1 if i == s else 0 for i in range(B)], dev)
        kvq.kvq_write(ks[:-1].contiguous(), vs[:-1].contiguous(), bs[:-1].contiguous(), one, cache)
        k_step[s], v_step[s], b_step[s] = ks[-1], vs[-1], bs[-1]
        m = modes[s].to(torch.int64)                                   # [HQ]
        lo = torch.where(m == 1, torch.clamp(torch.tensor(L - 1 - w, device=dev), min=0),
                         torch.zeros_like(m))
        read = (idx[:, None] >= lo[None, :]) & (m[None, :] != 0)       # [L, HQ]
        bf = bs.to(torch.int64)[:, kv_of]                              # [L, HQ]
        keys += int(read.sum())
        rec_bytes += int(((bf * D // 4) * read).sum())
        side_bytes += int((16 * (bf < 16) * read).sum())
        bk = bs.to(torch.int64)
        unique_bytes += int(((bk * D // 4 + 16 * (bk < 16)) * read.view(L, H, group).any(-1)).sum())
        del ks, vs, bs
    torch.cuda.synchronize(dev)
    cache.check()
    return dict(cache=cache, q=q, modes=modes, k_step=k_step, v_step=v_step, b_step=b_step,
                cu_one=synth.cu_seqlens([1] * B, dev),
                roll=torch.full((B,), L - 1, dtype=torch.int32, device=dev),
                out=torch.empty((B, HQ, D), dtype=torch.float32, device=dev),
                keys=keys, rec_bytes=rec_bytes, side_bytes=side_bytes, unique_bytes=unique_bytes,
                q_bytes=B * HQ * D * 2, out_bytes=B * HQ * D * 4)


def decode_step(st, w, events=None):
    """One step through kvq_decode_step: roll each sequence back to L - 1 tokens, append the
    step's token at its width, decode. `events` (before, after) are recorded around the
    split-K kernel only, so the other kernels of the step stay back to back in the stream."""
    from mixed_precision_kv_write_b200 import kvq
    if events is not None:
        kvq.kvq_set_profile_events(*events)
    kvq.decode_step(st["q"], st["k_step"], st["v_step"], st["b_step"], st["cu_one"], st["cache"],
                    st["modes"], w, positions=st["roll"], out=st["out"])
    if events is not None:
        kvq.kvq_set_profile_events(None, None)


LAUNCHES_PER_DECODE_STEP = 3   # plan (roll-back + append + schedule), split-K, combine


def decode_kernel_times(st, w, steps, stream):
    """Mean duration of the split-K kernel over `steps` decode steps (events recorded
    around that kernel by the library's profiling hook). A pass of its own: the events
    between launches stop the programmatic overlap of neighbouring kernels, so the
    headline loop records none."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        decode_step(st, w, ev[i])
    stream.synchronize()
    return statistics.mean(a.elapsed_time(b) * 1e-3 for a, b in ev)


def decode_roofline(st, k_avg, pk, pk_kind, profile_summary):
    kernel_bytes = st["rec_bytes"] + st["side_bytes"] + st["q_bytes"]
    achieved = kernel_bytes / k_avg / 1e9
    hbm_peak = float(pk["hbm_gbs"])
    return {"kernel": "decode_splitk_kernel<128>", "bound": "hbm", "achieved": achieved,
            "peak": hbm_peak, "peak_kind": pk_kind, "unit": "GB/s", "frac": achieved / hbm_peak,
            "traffic": _profiled_traffic(profile_summary, "kvq_decode.cu") if profile_summary else None,
            "algorithmic_bytes_per_launch": kernel_bytes, "avg_launch_s": k_avg}


def decode_workload_measure(name, dev, pk, pk_kind, steps=20, warm=5, group=1, profile_summary=None,
                            page_bytes=0):
    """A decode workload other than the headline: its steps timed back to back (no events
    between launches), then a pass with events around the split-K kernel."""
    from mixed_precision_kv_write_b200 import synth
    wl = synth.WORKLOADS[name]
    if group > 1:
        wl = synth.scaled(wl, heads=wl.heads // group)
    st = decode_setup(wl, dev, group, page_bytes)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warm):
        decode_step(st, wl.w)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        decode_step(st, wl.w)
    e1.record(stream)
    stream.synchronize()
    t_step = e0.elapsed_time(e1) * 1e-3 / steps
    k_avg = decode_kernel_times(st, wl.w, steps, stream)
    st["cache"].check()
    routed = st["rec_bytes"] + st["side_bytes"]
    res = {"value": st["keys"] / t_step, "unit": UNIT, "ms_per_step": t_step * 1e3,
           "attended_keys_per_step": st["keys"], "routed_bytes_per_step": routed,
           "hbm_gbs": routed / t_step / 1e9, "hbm_frac_of_8tbs": routed / t_step / 1e9 / NOMINAL_HBM_GBS,
           "roofline": decode_roofline(st, k_avg, pk, pk_kind, profile_summary)}
    if group > 1:
        res["unique_kv_bytes_per_step"] = st["unique_bytes"]
        res["unique_kv_gbs"] = st["unique_bytes"] / t_step / 1e9
    if page_bytes:
        c = st["cache"]
        res["pages"] = {"page_bytes": page_bytes, "pool_pages": c.pool_pages,
                        "pool_bytes": c.pool_pages * page_bytes,
                        "contiguous_worst_case_bytes": wl.batch * wl.heads * (wl.seqlens[0] + 4) * 4 * wl.head_dim}
    del st
    torch.cuda.empty_cache()
    return res


def prefill_measure(name, dev, pk, pk_kind, reps=5, warm=2, route=False, profiles=(None, None)):
    """A prefill + quantize-on-write workload: kvq_write of every token, then routed
    causal attention of every query. L2 is flushed (256 MB memset) before each rep; the
    write (scan + quantize kernels) and the attention kernel are timed with events the
    library records around them."""
    from mixed_precision_kv_write_b200 import kvq, synth
    wl = synth.WORKLOADS[name]
    H, D = wl.heads, wl.head_dim
    k, v, bits = synth.kv_tokens(wl, dev)
    q, modes = synth.prefill_queries(wl, dev)
    cu = synth.cu_seqlens(wl.seqlens, dev)
    cache = kvq.KVQCache(wl.batch, H, D, list(wl.seqlens), device=dev)
    out = torch.empty((wl.n_tok, H, D), dtype=torch.float32, device=dev)
    # exact query-key pairs
    pairs = 0
    cul = synth.cu_seqlens(wl.seqlens).tolist()
    for s in range(wl.batch):
        L = wl.seqlens[s]
        t = torch.arange(L, device=dev)[:, None]
        m = modes[cul[s]:cul[s] + L].to(torch.int64)
        n = torch.where(m == 2, t + 1, torch.where(m == 1, torch.clamp(t, max=wl.w) + 1, 0))
        pairs += int(n.sum())
    bf = bits.to(torch.int64)
    write_bytes = wl.n_tok * H * D * 2 * 2 + int((bf * D // 4).sum()) + wl.n_tok * H * (16 + 4)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    tw, tp = [], []
    for r in range(warm + reps):
        flush.fill_(r & 255)
        cache.reset()
        if r >= warm:
            torch.cuda.nvtx.range_push("prefill_timed")
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        kvq.kvq_set_profile_events(e[0], e[1])
        kvq.kvq_write(k, v, bits, cu, cache)
        kvq.kvq_set_profile_events(e[2], e[3])
        kvq.routed_attn_prefill(q, cache, modes, wl.w, cu, out=out)
        kvq.kvq_set_profile_events(None, None)
        if r >= warm:
            torch.cuda.nvtx.range_pop()
        stream.synchronize()
        if r >= warm:
            tw.append(e[0].elapsed_time(e[1]) * 1e-3)
            tp.append(e[2].elapsed_time(e[3]) * 1e-3)
    cache.check()
    flops = 4.0 * D * pairs
    t_p, t_w = statistics.median(tp), statistics.median(tw)
    bf16 = float(pk["bf16_tflops"])
    hbm_peak = float(pk["hbm_gbs"])
    res = {"workload": wl.note + f"; bits p={wl.bits_p}, modes p={wl.modes_p}",
           "tflops": flops / t_p / 1e12, "seconds": t_p, "pairs": pairs, "flops": flops,
           "roofline": {"kernel": f"prefill_tc_kernel<{D}>", "bound": "tensor", "achieved": flops / t_p / 1e12,
                        "peak": bf16, "peak_kind": pk_kind + " bf16 dense (burst)", "unit": "TFLOP/s",
                        "frac": flops / t_p / 1e12 / bf16,
                        "traffic": _profiled_traffic(profiles[0], "kvq_prefill_tc.cu") if profiles[0] else None},
           "quantize": {"gbs": write_bytes / t_w / 1e9, "bytes": write_bytes, "seconds": t_w,
                        "frac_of_hbm": write_bytes / t_w / 1e9 / hbm_peak,
                        # DRAM bytes of the quantize kernel (the scan kernel's are not included)
                        "traffic": _profiled_traffic(profiles[1], "kvq_write.cu") if profiles[1] else None}}
    if route:
        # router hard argmax on the same (token, head) rows: 3 + 4 fp32 logits in, 2 bytes out
        za, zb = synth.router_logits(wl, dev)
        route_bytes = wl.n_tok * H * (7 * 4 + 2)
        tr = []
        for r in range(warm + reps):
            flush.fill_(r & 255)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            e[0].record(stream)
            kvq.route_argmax(za, zb)
            e[1].record(stream)
            stream.synchronize()
            if r >= warm:
                tr.append(e[0].elapsed_time(e[1]) * 1e-3)
        t_r = statistics.median(tr)
        res["route"] = {"rows": wl.n_tok * H, "bytes": route_bytes, "seconds": t_r,
                        "gbs": route_bytes / t_r / 1e9, "frac_of_hbm": route_bytes / t_r / 1e9 / hbm_peak,
                        "note": "router hard argmax (kvq_route_argmax), L2 flushed before each rep"}
    del cache, k, v, q, out, flush
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ CPU oracle timing
def _oracle_decode_jobs(wl, n_seq):
    """Host copies of the non-skip decode queries of the first n_seq sequences: one job
    per (sequence, head) with its query, mode, position and the head's fp16 K/V/widths."""
    from mixed_precision_kv_write_b200 import synth
    q, modes = synth.decode_queries(wl, "cpu")
    L = wl.seqlens[0]
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    jobs = []
    for s in range(min(n_seq, wl.batch)):
        ks, vs, bs = synth.kv_sequence(wl, s, gen_dev)
        ks, vs, bs = ks.cpu(), vs.cpu(), bs.cpu()
        for h in range(wl.heads):
            m = int(modes[s, h])
            if m == 0:
                continue
            jobs.append((q[s, h][None].numpy(), m, L, ks[:, h].contiguous().numpy(),
                         vs[:, h].contiguous().numpy(), bs[:, h].contiguous().numpy()))
    return jobs


def _oracle_run(jobs, w, threads):
    """Run the oracle on `jobs` with `threads` host threads (the oracle is C behind ctypes,
    which releases the GIL during the call). Returns (keys, seconds)."""
    import concurrent.futures as cf
    import oracle

    def one(j):
        qv, m, L, kh, vh, bh = j
        oracle.routed_attention_head(qv, [L - 1], [m], w, kh, vh, bh)
        return L if m == 2 else min(L, w + 1)

    t0 = time.perf_counter()
    if threads == 1:
        keys = sum(one(j) for j in jobs)
    else:
        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            keys = sum(ex.map(one, jobs))
    return keys, time.perf_counter() - t0


def oracle_baseline(wl, budget_s=12.0, max_seq=32):
    """The CPU oracle on decode queries of the workload, on one host thread and on all
    host cores. The one-thread sample is the first n1 non-skip queries, sized to about
    half the budget; the all-core sample is every non-skip query of the first sequences
    (at most max_seq, to bound the host memory the K/V copies take)."""
    cores = os.cpu_count() or 1
    probe = _oracle_decode_jobs(wl, 1)
    _, tp = _oracle_run(probe[:3], wl.w, 1)
    per_job = tp / 3
    n1 = max(1, int(0.5 * budget_s / per_job))
    per_seq = max(1, len(probe))
    n_seq = min(wl.batch, max_seq, max(2, -(-max(n1, cores * n1) // per_seq)))
    jobs = _oracle_decode_jobs(wl, n_seq)
    n1 = min(n1, len(jobs))
    k1, t1 = _oracle_run(jobs[:n1], wl.w, 1)
    kn, tn = _oracle_run(jobs, wl.w, cores)
    return {"single": (k1 / t1, k1, t1, n1), "all": (kn / tn, kn, tn, len(jobs)), "cores": cores,
            "n_seq": n_seq}


# ------------------------------------------------------------------ arms
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = False
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
        pg = True
    else:
        torch.cuda.set_device(local)
    return world, rank, local, pg


def max_over_ranks(x: float, pg: bool, dev) -> float:
    if not pg:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, dev):
    if pg:
        if dev.type == "cuda":
            torch.distributed.barrier(device_ids=[dev.index])
        else:
            torch.distributed.barrier()
    if dev.type == "cuda":
        torch.cuda.synchronize(dev)


def weak_scaling_value(units_per_rank: float, elapsed: float, pg: bool, dev, world: int):
    """Every rank processes the same units (one replica of the workload each): the job's
    throughput is all ranks' units over the slowest rank's time. Returns (value, max time)."""
    elapsed_max = max_over_ranks(elapsed, pg, dev)
    return units_per_rank * world / elapsed_max, elapsed_max


def run_ours(args):
    from mixed_precision_kv_write_b200 import build as kbuild, synth
    kbuild.build()
    import oracle
    oracle.build()
    world, rank, local, pg = dist_setup()
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS["decode_1p3b"]
    if args.decode_batch != wl.batch:     # smaller case for profiler captures
        wl = synth.scaled(wl, seqlens=(wl.seqlens[0],) * args.decode_batch)
    pk, pk_kind = peaks()

    st = decode_setup(wl, dev)
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        decode_step(st, wl.w)
    # headline: K steps back to back, nothing recorded between their launches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg, dev)
    t_begin = time.time()
    torch.cuda.nvtx.range_push("decode_timed")
    e0.record(stream)
    for _ in range(args.steps):
        decode_step(st, wl.w)
    e1.record(stream)
    torch.cuda.nvtx.range_pop()
    barrier(pg, dev)
    t_end = time.time()
    sampler.stop()
    st["cache"].check()
    elapsed = e0.elapsed_time(e1) * 1e-3
    clocks = sampler.summary(t_begin, t_end)
    # the split-K kernel alone, in a pass of its own (events around it in every step)
    k_avg = decode_kernel_times(st, wl.w, args.steps, stream)

    keys = st["keys"]
    routed = st["rec_bytes"] + st["side_bytes"]
    value, elapsed_max = weak_scaling_value(keys * args.steps, elapsed, pg, dev, world)
    ms_step = elapsed_max / args.steps * 1e3

    # End to end through host buffers: every step copies its inputs from pinned host memory
    # (H2D) and reads its output back (D2H), inside the timed region. The copies run on a
    # second stream with two buffer sets, so step i+1's inputs and step i's output move
    # while the next step computes; the cache steps stay in order on the compute stream.
    names = ("k_step", "v_step", "b_step", "q", "modes")
    host = {n: st[n].cpu().pin_memory() for n in names}
    out_h = [torch.empty(st["out"].shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    bufs = []
    for _ in range(2):
        b = {n: torch.empty_like(st[n]) for n in names}
        b["out"] = torch.empty_like(st["out"])
        bufs.append(b)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h[0].numel() * 4
    copy = torch.cuda.Stream(dev)

    def e2e_run(n_steps, f0=None, f1=None):
        landed = [torch.cuda.Event() for _ in range(2)]     # inputs of the buffer set copied
        done = [torch.cuda.Event() for _ in range(2)]       # step that used the set finished
        readback = [torch.cuda.Event() for _ in range(2)]   # its output copied to the host

        def h2d_copy(i):
            b = bufs[i % 2]
            with torch.cuda.stream(copy):
                if i >= 2:
                    copy.wait_event(done[i % 2])
                for n in names:
                    b[n].copy_(host[n], non_blocking=True)
                landed[i % 2].record(copy)

        if f0 is not None:
            f0.record(copy)
        h2d_copy(0)
        for i in range(n_steps):
            if i + 1 < n_steps:
                h2d_copy(i + 1)
            b = bufs[i % 2]
            stream.wait_event(landed[i % 2])
            if i >= 2:
                stream.wait_event(readback[i % 2])
            sti = dict(st)
            sti.update(b)
            decode_step(sti, wl.w)
            done[i % 2].record(stream)
            with torch.cuda.stream(copy):
                copy.wait_event(done[i % 2])
                out_h[i % 2].copy_(b["out"], non_blocking=True)
                readback[i % 2].record(copy)
        if f1 is not None:
            f1.record(copy)

    e2e_run(max(3, args.warmup))
    barrier(pg, dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, f0, f1)
    barrier(pg, dev)
    copy.synchronize()
    e2e_value, _ = weak_scaling_value(keys * args.steps, f0.elapsed_time(f1) * 1e-3, pg, dev, world)
    full = args.decode_batch == synth.WORKLOADS["decode_1p3b"].batch
    roof = decode_roofline(st, k_avg, pk, pk_kind, "decode_splitk_decode_1p3b.md" if full else None)
    del st, bufs, host
    torch.cuda.empty_cache()

    extra = {}
    if not args.no_prefill:
        extra["prefill"] = prefill_measure("ragged_prefill", dev, pk, pk_kind, route=True,
                                           profiles=("prefill_tc_ragged_prefill.md", "write_quant_ragged_prefill.md"))
        extra["prefill_160m"] = prefill_measure("prefill_160m", dev, pk, pk_kind,
                                                profiles=("prefill_tc_prefill_160m.md", "write_quant_prefill_160m.md"))
        extra["decode_long"] = decode_workload_measure("decode_long", dev, pk, pk_kind)
        gq = decode_workload_measure("decode_1p3b", dev, pk, pk_kind, group=4)
        gq["workload"] = ("decode_1p3b with grouped-query attention: 16 query heads in groups of 4 over "
                          "4 KV heads, batch 64, context 8192, w=512")
        extra["gqa_decode"] = gq
        extra["decode_long"]["workload"] = synth.WORKLOADS["decode_long"].note
        pg_line = decode_workload_measure("decode_1p3b", dev, pk, pk_kind, page_bytes=65536)
        pg_line["workload"] = ("decode_1p3b on a paged cache: 64 KiB pages from a pool sized for the seeded "
                               "widths, pages handed out in a scrambled order")
        extra["paged_decode"] = pg_line
    barrier(pg, dev)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) fp16 K/V/Q, i.i.d. widths and modes)",
        "config": {
            "workload": "decode_1p3b: batch 64, H=16, head_dim 128, cached context 8192, w=512, "
                        "bits p(2/4/8/16)=.25/.45/.2/.1, modes p(skip/local/full)=.15/.45/.4",
            "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
            "context": wl.seqlens[0], "w": wl.w,
            "step": "kvq_decode_step: roll back to 8191 tokens, append the step token (Eq. 4), routed decode",
            "l2": "no flush: each step reads %.0f MB of routed cache bytes > 126 MB L2" % (routed / 1e6),
            "parallelism": f"{world} independent replica(s), no data-path collective",
            "storage": "packed u2/u4/u8 codes + fp16, fp32 side table"},
        "attended_keys_per_step": keys,
        "routed_bytes_per_step": routed,
        "hbm_gbs": routed / (elapsed_max / args.steps) / 1e9,
        "hbm_frac_of_8tbs": routed / (elapsed_max / args.steps) / 1e9 / NOMINAL_HBM_GBS,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clocks,
        "gpu_launches": LAUNCHES_PER_DECODE_STEP * args.steps,
    }
    line.update(extra)
    if rank == 0 and not args.no_cpu_baseline:
        ob = oracle_baseline(wl, budget_s=args.cpu_budget)
        v1, k1, t1, n1 = ob["single"]
        vn, kn, tn, nn = ob["all"]
        line["cpu_baseline"] = {
            "value": vn, "unit": UNIT, "cores": ob["cores"], "kind": "oracle",
            "sample": (f"oracle decode (C, fp64 softmax) of all {nn} non-skip (sequence, head) queries of "
                       f"the first {ob['n_seq']} sequences of {wl.name} on {ob['cores']} host threads: "
                       f"{kn} keys in {tn:.2f} s"),
            "single_thread": {"value": v1, "unit": UNIT, "cores": 1,
                              "sample": f"first {n1} non-skip queries: {k1} keys in {t1:.2f} s"},
            "host_cores": os.cpu_count()}
    if pg:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args):
    """The reference arm is the CPU oracle (no other implementation of this path exists):
    each step decodes a bounded sample of the same workload's queries, one query per host
    core in parallel."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from mixed_precision_kv_write_b200 import synth
    oracle.build()
    wl = synth.WORKLOADS["decode_1p3b"]
    cores = os.cpu_count() or 1
    jobs = _oracle_decode_jobs(wl, 4)
    per_step = max(1, min(cores, len(jobs)))

    def step(i):
        sel = [jobs[(i * per_step + j) % len(jobs)] for j in range(per_step)]
        return _oracle_run(sel, wl.w, per_step)

    for i in range(args.warmup):
        step(i)
    keys, secs = 0, 0.0
    for i in range(args.steps):
        k, s = step(args.warmup + i)
        keys += k
        secs += s
    v = keys / secs
    desc = (f"oracle decode (C, fp64 softmax) of {per_step} non-skip (sequence, head) queries per step, "
            f"one per host thread, cycling through the first 4 sequences of decode_1p3b")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "decode_1p3b (sampled: " + desc + ")"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": per_step, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _src_hash(name):
    """Hash of a kernel source with its comments and blank lines removed, so that an edit
    of comments alone does not orphan the profile of an unchanged kernel."""
    import hashlib
    import re
    with open(os.path.join(ROOT, "mixed_precision_kv_write_b200", "csrc", name)) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def _profiled_traffic(summary, source):
    """DRAM bytes per launch from an ncu summary in profiles/, if the summary's
    `<!-- traffic: bytes=N source=HASH -->` line matches the current kernel source."""
    import re
    p = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(p):
        return None
    m = re.search(r"<!-- traffic: bytes=(\d+) source=([0-9a-f]+) -->", open(p).read())
    if not m or m.group(2) != _src_hash(source):
        return None
    return int(m.group(1))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--decode-batch", type=int, default=64,
                    help="sequences of the decode workload (64; smaller only for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

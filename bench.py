#!/usr/bin/env python
"""Benchmark of the SR-SWA / DASH block-sparse decode step on B200.

    python bench.py [--gpus N --steps K --warmup W] [--workload long_decode|batched_decode|
                    tiny_decode|ragged_paged_decode] [--impl uocr|reference]

Default workload: long-context decode, batch 16, context 131072 (4096 blocks
of 32 tokens), 12 independent layer caches (126 GiB resident in HBM).  One
step = the decode of every sequence through all 12 layers = 12 calls of
``uocr_sparse_decode`` (scan -> top-k -> split-K attention -> combine).
Metric: decode queries/s per layer (= 16 * 12 / step time) and achieved HBM
bandwidth on the algorithmic bytes (256 B of indexer key per causal token +
512 tokens x 10 heads x 128 dims x 2 B x (K and V) per query).

The default run (long_decode on one GPU) also measures the other workloads, each on its own
after the headline's caches are freed, into a ``configs`` record: tiny, batched and ragged
paged decode (queries/s, HBM fractions of the call and of the scan kernel) and the chunked
prefill (queries/s, the scoring GEMM's tensor-core fraction, the attention stage's and the
whole call's HBM fractions), each with the clocks of its own timed region.

Prints ONE JSON line on rank 0.  Under torchrun each rank runs its own shard
of sequences (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402
from block_sparse_long_uocr_b200 import dist as udist  # noqa: E402

METRIC = "sparse-attn decode queries/s per layer @128K ctx; achieved HBM GB/s vs peak"
UNIT = "queries/s per layer"
KV_BYTES_PER_QUERY = 16 * 32 * 10 * 128 * 2 * 2      # 512 gathered tokens x 10 heads x 128 x bf16 x (K,V)
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic of the dominant kernel from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), per launch of the default workload, and the hash of the
# kernel source it was taken on.  Reported as null once the source has changed.
NCU_TRAFFIC = {
    # ncu --set full on long_decode batch 4 (1 layer), one launch: 134,299,392 B read +
    # 3,379,200 B written (the write-back of the bench's L2 flush), scaled x4 to 16 queries.
    "long_decode": {"bytes": 4 * (134299392 + 3379200), "src": "aea494e8d3b8c4ea"},
    # launch list of chunked_prefill with dram__bytes_read.sum / dram__bytes_write.sum and
    # --cache-control none, averaged over the scoring GEMM's 6 launches: 17,209,301 B read (the
    # indexer keys and queries) + 299,392 B written (the scores stay in L2 for the selection).
    "chunked_prefill": {"bytes": 17209301 + 299392, "src": "a9e518c6742ddbc3"},
}


SCAN_SOURCES = ("index_scan.cu", "scan_core.cuh")   # the scan kernel and its page loop
GEMM_SOURCES = ("prefill_index_gemm.cu", "tcgen05.cuh")   # the scoring GEMM and its tcgen05 helpers


def kernel_source_hash(*names: str) -> str:
    h = hashlib.sha256()
    for name in names:
        h.update(open(os.path.join(ROOT, "block_sparse_long_uocr_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            return json.load(open(path)), "measured"
        except Exception:
            pass
    return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock and throttle reasons.

    start() launches the sampler and waits for its first sample; mark() brackets the
    timed region; stop() waits for one sample after the region and ends the sampler.
    The summary keeps the samples taken inside the region, or, when the region is
    shorter than the sampling period, the one just before and the one just after it.
    """
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        import threading
        self.gpu = gpu_index
        self.proc = None
        self.samples = []          # (time, line)
        self.lock = threading.Lock()
        self.t0 = self.t1 = None
        self.raw_error = None

    def _reader(self):
        for line in self.proc.stdout:
            if line.strip():
                with self.lock:
                    self.samples.append((time.perf_counter(), line.strip()))

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.gpu)],
                                         stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except Exception as e:
            self.raw_error = repr(e)
            return self
        threading.Thread(target=self._reader, daemon=True).start()
        deadline = time.perf_counter() + 10
        while time.perf_counter() < deadline and not self.samples and self.proc.poll() is None:
            time.sleep(0.02)
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self.proc is None:
            return
        deadline = time.perf_counter() + 2
        while time.perf_counter() < deadline and self.proc.poll() is None:
            with self.lock:
                if self.samples and self.samples[-1][0] > (self.t1 or 0):
                    break
            time.sleep(0.02)
        self.proc.terminate()
        try:
            _, err = self.proc.communicate(timeout=5)
            if not self.samples and err:
                self.raw_error = err.strip()[:200]
        except Exception:
            self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with self.lock:
            samples = list(self.samples)
        inside = [l for t, l in samples if self.t0 is not None and self.t0 <= t <= (self.t1 or t)]
        where = "inside the timed region"
        if not inside:
            before = [l for t, l in samples if self.t0 is not None and t < self.t0][-1:]
            after = [l for t, l in samples if self.t1 is not None and t > self.t1][:1]
            inside = before + after
            where = "bracketing the timed region (shorter than the 100 ms sampling period)"
        for l in inside:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0, "error": self.raw_error}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "where": where}


def physical_gpu(local_rank: int) -> str:
    """nvidia-smi id of this process's GPU (honours CUDA_VISIBLE_DEVICES indices or UUIDs)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# --------------------------------------------------------------------------- workloads
def build_workload(name: str, device, seed: int, batch=None, layers=None):
    if name == "long_decode":
        return workloads.long_decode(device=device, seed=seed, B=batch or 16, n_layers=layers or 12)
    if name == "batched_decode":
        return workloads.batched_decode(device=device, seed=seed)
    if name == "tiny_decode":
        return workloads.tiny_decode(device=device, seed=seed)
    if name == "ragged_paged_decode":
        return workloads.ragged_paged_decode(device=device, seed=seed)
    if name == "chunked_prefill":
        return workloads.chunked_prefill(device=device, seed=seed)
    raise SystemExit(f"unknown workload {name}")


def algorithmic_bytes(case) -> tuple[int, int]:
    """(bytes per decode call over all queries, indexer-scan bytes of those queries)."""
    lens = case.seq_lens.cpu().tolist()
    scan = sum(256 * L for L in lens)
    return scan + KV_BYTES_PER_QUERY * len(lens), scan


# --------------------------------------------------------------------------- our arm
def run_uocr(args):
    rank, local_rank, world = udist.env_rank_world()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    import block_sparse_long_uocr_b200 as uocr

    case = build_workload(args.workload, dev, udist.shard_seed(args.seed, rank), args.batch, args.layers)
    n_layers = len(case.layers)
    B, H, mb = case.n_q, case.q.shape[1], case.max_blocks
    bytes_call, scan_bytes_call = algorithmic_bytes(case)
    ws = uocr.alloc_workspace(B, H, mb, dev)
    outs = [torch.empty_like(case.q) for _ in range(n_layers)]
    sels = [torch.empty((B, 16), dtype=torch.int32, device=dev) for _ in range(n_layers)]
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = bytes_call * n_layers < 4 * l2
    flush_l2 = L2Flush(l2, dev) if flush else None

    def step(st=None):
        for l in range(n_layers):
            q, qi = case.q_layers[l]
            kp, vp, ikp = case.layers[l]
            uocr.sparse_decode(q, kp, vp, qi, ikp, case.block_table, case.seq_lens, out=outs[l], sel=sels[l],
                               workspace=ws, stream=st or stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier(device_ids=[local_rank])

    clk = ClockSampler(physical_gpu(local_rank)).start()
    for _ in range(args.warmup):
        if flush:
            flush_l2()
        step()
    timed = TimedSteps(step, flush_l2, stream, args.steps) if flush else None
    if timed is not None:
        timed.warm()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    clk.mark_start()
    if flush:
        # L2 flushed between steps, every step timed between its own events inside one graph
        elapsed_ms = timed.run()
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        elapsed_ms = e0.elapsed_time(e1)
    clk.mark_end()
    clk.stop()
    barrier()
    torch.cuda.synchronize()
    max_ms = udist.max_over_ranks(elapsed_ms, dev)
    ms_per_step = max_ms / args.steps
    queries_per_step = B * n_layers
    # queries/s per layer: each layer call decodes B queries; a step makes n_layers calls
    value = world * queries_per_step * args.steps / (max_ms / 1e3)

    # ---- each step on its own, n_rep launches captured in one CUDA graph and replayed, so the
    #      device time excludes host launch gaps (the scan is the dominant kernel of the roofline)
    scores = torch.empty((B, mb), dtype=torch.float32, device=dev)
    n_rep = max(3, min(args.steps * n_layers, 48))

    def graph_time(fn):
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for r in range(n_layers):           # warm (module load, attributes) outside the capture
                fn(r % n_layers, side)
        side.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for r in range(n_rep):
                if flush:
                    flush_l2()
                fn(r % n_layers, side)
        flush_g = None
        if flush:
            flush_g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(flush_g, stream=side):
                for r in range(n_rep):
                    flush_l2()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        if flush_g is not None:                 # subtract the flushes captured between launches
            flush_g.replay()
            torch.cuda.synchronize()
            e0.record(stream)
            flush_g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            ms -= e0.elapsed_time(e1)
        return ms / n_rep

    scan_ms = graph_time(lambda l, st: uocr.index_score(case.q_layers[l][1], case.layers[l][2], case.block_table,
                                                        case.seq_lens, scores=scores, stream=st))
    topk_ms = graph_time(lambda l, st: uocr.block_topk(scores, case.seq_lens, sel=sels[l], stream=st))
    attn_ms = graph_time(lambda l, st: uocr.sparse_attn(case.q_layers[l][0], case.layers[l][0], case.layers[l][1],
                                                        case.block_table, case.seq_lens, sels[l], out=outs[l],
                                                        stream=st))
    decode_ms = graph_time(lambda l, st: uocr.sparse_decode(case.q_layers[l][0], case.layers[l][0],
                                                            case.layers[l][1], case.q_layers[l][1],
                                                            case.layers[l][2], case.block_table, case.seq_lens,
                                                            out=outs[l], sel=sels[l], workspace=ws, stream=st))
    comparators = None
    if args.workload == "long_decode" and not args.no_comparators:
        # the baselines the pages quote per decode step: full causal attention, and R-SWA read as a
        # reference prefix of 80 % of the context plus the 128-token window (the pages' 7.0x / 5.6x
        # ratios imply R-SWA reads 5.6 / 7.0 = 0.8 of what full attention reads)
        dws = torch.empty(uocr.dense_workspace_bytes(B, H, mb), dtype=torch.uint8, device=dev)
        ref_blocks = int(0.8 * mb)
        full_ms = graph_time(lambda l, st: uocr.dense_decode(case.q_layers[l][0], case.layers[l][0], case.layers[l][1],
                                                             case.block_table, case.seq_lens, out=outs[l],
                                                             workspace=dws, stream=st))
        rswa_ms = graph_time(lambda l, st: uocr.dense_decode(case.q_layers[l][0], case.layers[l][0], case.layers[l][1],
                                                             case.block_table, case.seq_lens, ref_blocks=ref_blocks,
                                                             out=outs[l], workspace=dws, stream=st))
        comparators = {"full_attention_us": round(1e3 * full_ms, 2), "rswa_us": round(1e3 * rswa_ms, 2),
                       "sparse_decode_us": round(1e3 * decode_ms, 2),
                       "speedup_vs_full": round(full_ms / decode_ms, 2), "speedup_vs_rswa": round(rswa_ms / decode_ms, 2),
                       "pages_claim": {"vs_full": 7.0, "vs_rswa": 5.6},
                       "rswa_reading": f"reference prefix {ref_blocks} of {mb} blocks + 4-block window",
                       "full_gbs": round(B * 5120 * int(case.seq_lens[0]) / (full_ms / 1e3) / 1e9, 1)}
        # the next-step variants on the same inputs: block-summary scoring (mean-key summaries,
        # one 256-byte vector per page) and selection under a page-aware candidate mask
        summ = [uocr.block_summary_mean(case.layers[l][2]) for l in range(n_layers)]
        summary_ms = graph_time(lambda l, st: uocr.sparse_decode_summary(
            case.q_layers[l][0], case.layers[l][0], case.layers[l][1], case.q_layers[l][1], summ[l],
            case.block_table, case.seq_lens, out=outs[l], sel=sels[l], workspace=ws, stream=st))
        words = (mb + 31) // 32
        mask = torch.randint(-2 ** 31, 2 ** 31 - 1, (B, words), dtype=torch.int32, device=dev,
                             generator=torch.Generator(device=dev).manual_seed(1))
        masked_topk_ms = graph_time(lambda l, st: uocr.block_topk_masked(scores, case.seq_lens, mask, sel=sels[l],
                                                                         stream=st))
        # the step before the scan (row f2): page2d rotation of one new token per sequence and its
        # append to the caches, here into a separate small cache (one page per sequence) so that the
        # workload's caches stay as they are
        g = torch.Generator(device=dev).manual_seed(3)
        rq = torch.randn((B, H, 128), generator=g, device=dev).to(torch.bfloat16)
        rqi = torch.randn((B, 128), generator=g, device=dev).to(torch.bfloat16)
        rk, rv = torch.randn_like(rq.float()).to(torch.bfloat16), torch.randn_like(rq.float()).to(torch.bfloat16)
        rki = torch.randn_like(rqi.float()).to(torch.bfloat16)
        rpos = case.seq_lens - 1
        rpage = rpos // 4096
        rbt = torch.arange(B, dtype=torch.int32, device=dev).view(B, 1)
        rsl = torch.full((B,), 32, dtype=torch.int32, device=dev)
        rkc = torch.zeros((B, H, 32, 128), dtype=torch.bfloat16, device=dev)
        rvc, rkic = torch.zeros_like(rkc), torch.zeros((B, 32, 128), dtype=torch.bfloat16, device=dev)
        rope_ms = graph_time(lambda l, st: uocr.rope_append(rq, rqi, rk, rv, rki, rpos, rpage, rbt, rsl, rkc, rvc,
                                                            rkic, stream=st))
        del rq, rqi, rk, rv, rki, rkc, rvc, rkic
        summary_bytes = B * (256 * mb + KV_BYTES_PER_QUERY)     # one 256-byte summary per causal block
        comparators["variants"] = {
            "summary_decode_us": round(1e3 * summary_ms, 2),
            "summary_decode_gbs": round(summary_bytes / (summary_ms / 1e3) / 1e9, 1),
            "summary_speedup_vs_token_scan": round(decode_ms / summary_ms, 2),
            "masked_topk_us": round(1e3 * masked_topk_ms, 2), "topk_us": round(1e3 * topk_ms, 2),
            "rope_append_us": round(1e3 * rope_ms, 2), "rope_append_tokens": B}
        del summ
        for o in outs:
            o.zero_()
    read_cal = read_calibration(dev, stream)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    scan_gbs = scan_bytes_call / (scan_ms / 1e3) / 1e9
    read_cal["scan_frac_of_read"] = round(scan_gbs / read_cal["gbs"], 4)
    step_gbs = bytes_call * n_layers / (ms_per_step / 1e3) / 1e9
    tr = NCU_TRAFFIC.get(args.workload) if (args.workload != "long_decode" or B == 16) else None
    traffic = tr["bytes"] if tr and tr.get("src") == kernel_source_hash(*SCAN_SOURCES) else None

    # ---- end to end through the public API: pinned host inputs in, results out, every step
    e2e = run_e2e(args, uocr, case, ws, outs, sels, stream, world, dev)

    clocks = clk.summary()
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": case.name, "batch_per_gpu": B, "context": int(case.seq_lens.max().item()),
                   "layers": n_layers, "heads": H, "head_dim": 128, "block": 32, "local_blocks": 4,
                   "remote_blocks": 12, "max_blocks": mb,
                   "l2": L2_FLUSH_NOTE if flush else "inputs larger than L2 (no flush)", "launch": STEPS_IN_ONE_GRAPH,
                   "launch": STEPS_IN_ONE_GRAPH if flush else "stream launches queued ahead",
                   "parallelism": f"dp{world} (independent sequence shards)"},
        "roofline": {"bound": "hbm", "kernel": "index_scan_kernel", "achieved": round(scan_gbs, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(scan_gbs / peak, 4), "traffic": traffic,
                     "peak_kind": f"{peak_kind} hbm copy", "bytes_per_launch": scan_bytes_call,
                     "avg_launch_ms": round(scan_ms, 5), "frac_of_8tbs": round(scan_gbs / NOMINAL_HBM_GBS, 4)},
        "step_roofline": {"bound": "hbm", "achieved": round(step_gbs, 1), "peak": peak, "unit": "GB/s",
                          "frac": round(step_gbs / peak, 4), "frac_of_8tbs": round(step_gbs / NOMINAL_HBM_GBS, 4),
                          "bytes_per_step": bytes_call * n_layers},
        "breakdown_us": {"index_scan": round(1e3 * scan_ms, 2), "block_topk": round(1e3 * topk_ms, 2),
                         "sparse_attn": round(1e3 * attn_ms, 2), "decode_call_graph": round(1e3 * decode_ms, 2),
                         "decode_call_eager": round(1e3 * ms_per_step / n_layers, 2),
                         "note": "device time per launch from CUDA-graph replays of each entry point alone; "
                                 "the decode call chains the three with programmatic dependent launch"},
        "comparators": comparators,
        "hbm_read_calibration": read_cal,
        "e2e": e2e,
        "gpu_launches": args.steps * n_layers * 3,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(case, budget_s=args.cpu_budget)
    if world == 1 and args.workload == "long_decode" and not args.no_configs:
        # the other workloads, each measured on its own after the headline's caches are freed
        del case, ws, outs, sels, scores, timed, flush_l2, step
        import gc
        gc.collect()
        torch.cuda.empty_cache()
        cfg_steps = max(5, min(args.steps, 50))
        result["configs"] = {
            "tiny_decode": decode_config_record("tiny_decode", args, uocr, dev, cfg_steps),
            "batched_decode": decode_config_record("batched_decode", args, uocr, dev, cfg_steps),
            "ragged_paged_decode": decode_config_record("ragged_paged_decode", args, uocr, dev, cfg_steps),
            "chunked_prefill": prefill_config_record(args, uocr, dev, cfg_steps),
            "note": "each workload measured alone after the headline (its own warm-up, timed calls and clocks); "
                    "value = queries of one call / device time of one call",
        }
        result["gpu_launches"] += sum(v["gpu_launches"] for k, v in result["configs"].items() if k != "note")
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def read_calibration(dev, stream, gib: int = 4, reps: int = 5):
    """Read-only HBM stream for context beside the copy peak: torch.sum over `gib` GiB of bf16
    (the scan is a pure read stream, which can run above a copy's read + write rate)."""
    x = torch.ones(gib * (1 << 30) // 2, dtype=torch.bfloat16, device=dev)
    for _ in range(2):
        x.sum()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        x.sum()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    gbs = x.numel() * 2 / (ms / 1e3) / 1e9
    del x
    torch.cuda.empty_cache()
    return {"kind": f"torch.sum over {gib} GiB bf16", "gbs": round(gbs, 1), "ms": round(ms, 4)}


L2_FLUSH_NOTE = "flushed between steps (2 x L2 written, then 2 x L2 of another buffer read)"


class L2Flush:
    """Evicts a step's data from L2 between timed steps: writes a buffer of twice the L2 size, then
    reads another of the same size.  The write is the flush; the read pass then evicts the flush's
    own dirty lines (written back here, outside the timed region), so that the next step starts with
    none of its inputs in L2 and no foreign write-back in its DRAM traffic."""

    def __init__(self, l2_bytes, dev):
        self.w = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(2 * l2_bytes // 4, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.acc)


STEPS_IN_ONE_GRAPH = ("all timed steps in one CUDA graph, each step timed between its own event-record "
                      "nodes (no host launch inside a step)")


class TimedSteps:
    """`steps` steps of fn(stream), each after an L2 flush when one is given, captured in one CUDA
    graph with an event-record node right before and right after every step.  A replay runs them
    back to back on the device; each step is timed between its own two events, so neither a flush
    nor a host-side launch falls inside a step's time.  `run()` replays once to warm up, then once
    timed, and returns the sum of the steps' device ms."""

    def __init__(self, fn, flush_l2, stream, steps):
        self.ev = [(torch.cuda.Event(enable_timing=True, external=True),
                    torch.cuda.Event(enable_timing=True, external=True)) for _ in range(steps)]
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn(side)
        side.synchronize()
        self.g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g, stream=side):
            for e0, e1 in self.ev:
                if flush_l2 is not None:
                    flush_l2()
                e0.record(side)
                fn(side)
                e1.record(side)
        torch.cuda.synchronize()

    def warm(self):
        self.g.replay()
        torch.cuda.synchronize()

    def run(self):
        self.g.replay()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in self.ev)


def graph_time_fn(fn, stream, n_rep, flush_l2=None):
    """Device ms per call of fn(stream) from n_rep calls captured in one CUDA graph
    (minus the captured L2 flushes between them, when an L2Flush is given)."""
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        fn(side)
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(n_rep):
            if flush_l2 is not None:
                flush_l2()
            fn(side)
    fg = None
    if flush_l2 is not None:
        fg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(fg, stream=side):
            for _ in range(n_rep):
                flush_l2()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if fg is not None:
        fg.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        fg.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms -= e0.elapsed_time(e1)
    return ms / n_rep


def run_prefill(args):
    """Chunked prefill: one uocr_sparse_prefill call of 2048 queries over a 65536-token sequence per step."""
    rank, local_rank, world = udist.env_rank_world()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import block_sparse_long_uocr_b200 as uocr

    result = prefill_measure(args, uocr, dev, rank, local_rank, world, args.steps, extras=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def prefill_measure(args, uocr, dev, rank, local_rank, world, steps, extras):
    """The chunked-prefill measurement: `steps` timed calls (L2 flushed before each), the per-kernel
    breakdown, the rooflines; with `extras` also the end-to-end leg and the oracle baseline."""
    case = workloads.chunked_prefill(device=dev, seed=udist.shard_seed(args.seed, rank))
    n_q, H, mb = case.n_q, case.q.shape[1], case.max_blocks
    ws = uocr.alloc_prefill_workspace(n_q, H, mb, dev)
    out = torch.empty_like(case.q)
    sel = torch.empty((n_q, 16), dtype=torch.int32, device=dev)
    scores = ws[: n_q * mb * 4].view(torch.float32).view(n_q, mb)
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_l2 = L2Flush(l2, dev)

    def step(st=None):
        uocr.sparse_prefill(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                            case.seq_lens, 0, case.q_pos, out=out, sel=sel, workspace=ws, stream=st or stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier(device_ids=[local_rank])

    clk = ClockSampler(physical_gpu(local_rank)).start()
    for _ in range(args.warmup):
        flush_l2()
        step()
    timed = TimedSteps(step, flush_l2, stream, steps)
    timed.warm()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clk.mark_start()
    elapsed_ms = timed.run()
    clk.mark_end()
    clk.stop()
    barrier()
    max_ms = udist.max_over_ranks(elapsed_ms, dev)
    ms_per_step = max_ms / steps
    value = world * n_q * steps / (max_ms / 1e3)

    n_rep = 10
    gemm_ms = graph_time_fn(lambda st: uocr.prefill_index_score(case.idx_q, case.idx_k_pool, case.block_table,
                                                                case.seq_lens, 0, case.q_pos, scores=scores,
                                                                stream=st), stream, n_rep, flush_l2)
    topk_ms = graph_time_fn(lambda st: uocr.block_topk(scores, case.seq_lens, case.q_seq, case.q_pos, sel=sel,
                                                       stream=st), stream, n_rep, flush_l2)
    attn_ms = graph_time_fn(lambda st: uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table,
                                                        case.seq_lens, sel, case.q_seq, case.q_pos, out=out,
                                                        stream=st), stream, n_rep, flush_l2)
    seq_ws = torch.empty(max(uocr.sparse_attn_seq_workspace_bytes(n_q, H, mb), 1), dtype=torch.uint8, device=dev)
    out_seq = torch.empty_like(out)
    attn_seq_ms = graph_time_fn(lambda st: uocr.sparse_attn_seq(case.q, case.k_pool, case.v_pool, case.block_table,
                                                                case.seq_lens, 0, case.q_pos, sel, out=out_seq,
                                                                workspace=seq_ws, stream=st), stream, n_rep, flush_l2)
    call_ms = graph_time_fn(lambda st: step(st), stream, n_rep, flush_l2)
    pos = case.q_pos.cpu().long()
    idx_flops = float(((pos + 1) * 128 * 2).sum())                 # causal q_idx . k_idx products
    attn_flops = float(n_q * H * 16 * 32 * 128 * 4)                 # QK and PV over 512 tokens
    peaks, peak_kind = measured_peaks()
    tc_peak = float(peaks.get("bf16_tflops", 1590.0))
    tc_sust = float(peaks.get("bf16_tflops_sustained", 1400.0))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    gemm_tflops = idx_flops / (gemm_ms / 1e3) / 1e12
    tr = NCU_TRAFFIC.get("chunked_prefill")
    gemm_traffic = tr["bytes"] if tr and tr.get("src") == kernel_source_hash(*GEMM_SOURCES) else None
    kv_union = case.num_pages * H * 32 * 128 * 2 * 2               # every page is selected by some query
    n_sel_blocks = int(torch.unique(sel[sel >= 0]).numel())
    attn_bytes = n_sel_blocks * H * 32 * 128 * 2 * 2 + 2 * n_q * H * 128 * 2   # selected K/V tiles once, q, out
    attn_gbs = attn_bytes / (attn_seq_ms / 1e3) / 1e9
    step_bytes = kv_union + case.num_pages * 32 * 128 * 2 + 2 * n_q * mb * 4 + 2 * n_q * H * 128 * 2
    result = {
        "metric": "chunked-prefill queries/s per layer; tensor-core TFLOP/s of the scoring GEMM vs peak",
        "value": round(value, 1), "unit": "queries/s per layer", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": case.name, "queries": n_q, "context": int(case.seq_lens[0]), "heads": H,
                   "max_blocks": mb, "l2": L2_FLUSH_NOTE, "launch": STEPS_IN_ONE_GRAPH,
                   "parallelism": f"dp{world}"},
        "roofline": {"bound": "tensor", "kernel": "prefill_index_gemm_kernel", "achieved": round(gemm_tflops, 1),
                     "peak": tc_peak, "unit": "TFLOP/s", "frac": round(gemm_tflops / tc_peak, 4), "traffic": gemm_traffic,
                     "peak_kind": f"{peak_kind} bf16 burst", "frac_of_sustained": round(gemm_tflops / tc_sust, 4),
                     "flops_per_launch": idx_flops, "avg_launch_ms": round(gemm_ms, 5)},
        "step_roofline": {"bound": "hbm", "achieved": round(step_bytes / (call_ms / 1e3) / 1e9, 1),
                          "peak": hbm_peak, "unit": "GB/s",
                          "frac": round(step_bytes / (call_ms / 1e3) / 1e9 / hbm_peak, 4),
                          "bytes_per_step": step_bytes, "flops_per_step": idx_flops + attn_flops},
        "attn_roofline": {"bound": "hbm", "entry": "uocr_sparse_attn_seq: classification, tcgen05 local-window "
                          "kernel, inversion, block kernel, merge (5 kernels)", "achieved": round(attn_gbs, 1),
                          "peak": hbm_peak, "unit": "GB/s", "frac": round(attn_gbs / hbm_peak, 4),
                          "bytes_per_launch": attn_bytes, "avg_launch_ms": round(attn_seq_ms, 5),
                          "selected_blocks": n_sel_blocks},
        "breakdown_us": {"prefill_index_gemm": round(1e3 * gemm_ms, 2), "block_topk": round(1e3 * topk_ms, 2),
                         "sparse_attn_seq": round(1e3 * attn_seq_ms, 2),
                         "sparse_attn_query_centric": round(1e3 * attn_ms, 2),
                         "prefill_call_graph": round(1e3 * call_ms, 2)},
        "gpu_launches": steps * PREFILL_LAUNCHES,
        "clocks": clk.summary(),
    }
    if extras:
        result["e2e"] = run_prefill_e2e(args, uocr, case, ws, out, sel, stream, world, dev)
        if rank == 0 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(case, args.cpu_budget)
    return result


# kernels of one uocr_sparse_prefill call: scoring GEMM, selection, classification, local-window
# attention (tcgen05), inversion, block attention, merge
PREFILL_LAUNCHES = 7


def decode_config_record(name, args, uocr, dev, steps):
    """One decode workload measured on its own for the `configs` record of the default run:
    `steps` timed decode calls (all captured in one CUDA graph, each timed between its own event
    nodes, L2 flushed before each when the call's bytes would otherwise stay in L2), the scan
    kernel and the whole call from CUDA-graph replays, the HBM fractions on the algorithmic bytes,
    and the clocks of its timed region."""
    case = build_workload(name, dev, args.seed)
    B, H, mb = case.n_q, case.q.shape[1], case.max_blocks
    bytes_call, scan_bytes = algorithmic_bytes(case)
    ws = uocr.alloc_workspace(B, H, mb, dev)
    out = torch.empty_like(case.q)
    sel = torch.empty((B, 16), dtype=torch.int32, device=dev)
    scores = torch.empty((B, mb), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = bytes_call < 4 * l2
    flush_l2 = L2Flush(l2, dev) if flush else None

    def call(st=None):
        uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                           case.seq_lens, out=out, sel=sel, workspace=ws, stream=st or stream)

    for _ in range(max(3, args.warmup)):
        if flush:
            flush_l2()
        call()
    timed = TimedSteps(call, flush_l2, stream, steps)
    timed.warm()
    clk = ClockSampler(physical_gpu(torch.cuda.current_device())).start()
    clk.mark_start()
    call_ms = timed.run() / steps
    clk.mark_end()
    clk.stop()
    n_rep = 20
    scan_ms = graph_time_fn(lambda st: uocr.index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens,
                                                        scores=scores, stream=st), stream, n_rep, flush_l2)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    gbs = bytes_call / (call_ms / 1e3) / 1e9
    scan_gbs = scan_bytes / (scan_ms / 1e3) / 1e9
    tr = NCU_TRAFFIC.get(name)
    traffic = tr["bytes"] if tr and tr.get("src") == kernel_source_hash(*SCAN_SOURCES) else None
    rec = {"workload": case.name, "queries_per_call": B,
           "value": round(B / (call_ms / 1e3), 1), "unit": "queries/s per layer",
           "ms_per_call": round(call_ms, 5), "steps": steps,
           "l2": L2_FLUSH_NOTE if flush else "inputs larger than L2 (no flush)", "launch": STEPS_IN_ONE_GRAPH,
           "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                        "frac": round(gbs / peak, 4), "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                        "bytes_per_call": bytes_call, "peak_kind": f"{peak_kind} hbm copy"},
           "scan": {"kernel": "index_scan_kernel", "achieved": round(scan_gbs, 1), "frac": round(scan_gbs / peak, 4),
                    "bytes_per_launch": scan_bytes, "avg_launch_ms": round(scan_ms, 5), "traffic": traffic},
           "gpu_launches": steps * 3, "clocks": clk.summary()}
    del case, ws, out, sel, scores, timed, flush_l2
    torch.cuda.empty_cache()
    return rec


def prefill_config_record(args, uocr, dev, steps):
    """The chunked-prefill workload for the `configs` record of the default run."""
    full = prefill_measure(args, uocr, dev, 0, torch.cuda.current_device(), 1, steps, extras=False)
    r = full["roofline"]
    rec = {"workload": full["config"]["workload"], "queries_per_call": full["config"]["queries"],
           "value": full["value"], "unit": full["unit"], "ms_per_call": full["ms_per_step"], "steps": steps,
           "l2": full["config"]["l2"],
           "gemm": {"kernel": r["kernel"], "bound": "tensor", "achieved": r["achieved"], "unit": "TFLOP/s",
                    "peak": r["peak"], "frac": r["frac"], "frac_of_sustained": r["frac_of_sustained"],
                    "flops_per_launch": r["flops_per_launch"], "avg_launch_ms": r["avg_launch_ms"],
                    "traffic": r["traffic"]},
           "attention_stage": full["attn_roofline"],
           "roofline": full["step_roofline"],
           "breakdown_us": full["breakdown_us"], "gpu_launches": full["gpu_launches"], "clocks": full["clocks"]}
    torch.cuda.empty_cache()
    return rec


def _serial_e2e(args, inputs, results, run_step, stream, dev):
    """Time `steps` end-to-end steps on one stream: copy every input from pinned host memory (one
    transfer), run `run_step`, copy every result back to pinned host memory (one transfer), step
    after step.  Returns device ms."""
    h_in, h_in_views = _packed(inputs, "cpu", pin=True)
    for hv, t in zip(h_in_views, inputs):
        hv.copy_(t.cpu())
    d_in, d_in_views = _packed(inputs, dev)
    d_out, d_out_views = _packed(results, dev)
    h_out, _ = _packed(results, "cpu", pin=True)

    def step():
        d_in.copy_(h_in, non_blocking=True)
        run_step(d_in_views, d_out_views)
        h_out.copy_(d_out, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(max(1, args.steps)):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def _e2e(args, inputs, results, run_step, stream, dev, units_per_step, world):
    """Both ways of running end-to-end steps, each with every step's copies inside the timed
    region: serial (one stream) and pipelined (copies of neighbouring steps overlap the compute).
    Pipelining hides the copies of long steps; a step of a few microseconds is bound by the host
    issuing three streams' work, where the serial loop is faster.  The faster mode is the reported
    value; the other is kept beside it."""
    steps = max(1, args.steps)
    res = {}
    for mode, fn in (("serial", _serial_e2e), ("pipelined", _pipelined_e2e)):
        ms = udist.max_over_ranks(fn(args, inputs, results, run_step, stream, dev), dev)
        res[mode] = {"value": round(world * units_per_step * steps / (ms / 1e3), 1), "ms_per_step": round(ms / steps, 4)}
    best = max(res, key=lambda m: res[m]["value"])
    other = "serial" if best == "pipelined" else "pipelined"
    return {"value": res[best]["value"], "unit": UNIT,
            "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in inputs),
            "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in results),
            "ms_per_step": res[best]["ms_per_step"], "copies_per_step": 2, "mode": best, other: res[other]}


def _pipelined_e2e(args, inputs, results, run_step, stream, dev):
    """Time `steps` end-to-end steps: step k copies every input from pinned host memory (one
    transfer), runs `run_step` on the device copy and copies every result back to pinned host
    memory (one transfer).  Device inputs and results are double-buffered and the two copies run
    on their own streams, so step k + 1's inputs travel while step k computes and step k's results
    travel while step k + 1 computes, as in a serving loop; every copy of every step is inside the
    timed region (from the first input copy to the last result copy).  Returns device ms."""
    h_in, h_in_views = _packed(inputs, "cpu", pin=True)
    for hv, t in zip(h_in_views, inputs):
        hv.copy_(t.cpu())
    d_in = [_packed(inputs, dev) for _ in range(2)]
    d_out = [_packed(results, dev) for _ in range(2)]
    h_out = [_packed(results, "cpu", pin=True)[0] for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in", "comp", "out")}
    k = [0]

    def step():
        b, reuse = k[0] % 2, k[0] >= 2
        with torch.cuda.stream(h2d):
            if reuse:
                h2d.wait_event(ev["comp"][b])          # step k - 2 has read this input buffer
            d_in[b][0].copy_(h_in, non_blocking=True)
            ev["in"][b].record(h2d)
        stream.wait_event(ev["in"][b])
        if reuse:
            stream.wait_event(ev["out"][b])            # step k - 2's results have left this buffer
        run_step(d_in[b][1], d_out[b][1])
        ev["comp"][b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev["comp"][b])
            h_out[b].copy_(d_out[b][0], non_blocking=True)
            ev["out"][b].record(d2h)
        k[0] += 1

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(1, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    for _ in range(steps):
        step()
    e1.record(d2h)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def run_prefill_e2e(args, uocr, case, ws, out, sel, stream, world, dev):
    """Same metric through sparse_prefill, end to end: every step copies the chunk's queries,
    indexer queries and positions from pinned host memory in one transfer, runs the call, and
    copies the output and the selection back in one transfer, inside the timed region (serial or
    pipelined across steps, see _e2e).  The caches stay resident (the sequence's state; the
    chunk's own keys are already appended)."""
    inputs = [case.q, case.idx_q, case.q_pos]
    results = [out, sel]

    def run_step(din, dout):
        d_q, d_qi, d_pos = din
        uocr.sparse_prefill(d_q, case.k_pool, case.v_pool, d_qi, case.idx_k_pool, case.block_table, case.seq_lens,
                            0, d_pos, out=dout[0], sel=dout[1], workspace=ws, stream=stream)

    return _e2e(args, inputs, results, run_step, stream, dev, case.n_q, world)


def _packed(tensors, device, pin=False):
    """One uint8 buffer holding `tensors` at 256-byte aligned offsets, and typed views into it."""
    offs, off = [], 0
    for t in tensors:
        offs.append(off)
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.empty(max(off, 1), dtype=torch.uint8, device=device)
    if pin:
        buf = buf.pin_memory()
    views = [buf[o: o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(tensors, offs)]
    return buf, views


def run_e2e(args, uocr, case, ws, outs, sels, stream, world, dev):
    """Same metric through sparse_decode, end to end: every step copies its inputs (the block table,
    the lengths and every layer's query and indexer query) from pinned host memory in one transfer,
    runs the 12 layer calls, and copies every layer's output and selection back in one transfer,
    all inside the timed region (serial or pipelined across steps, see _e2e).  The KV / indexer
    caches stay resident (the decode state)."""
    n_layers = len(case.layers)
    inputs = [case.block_table, case.seq_lens] + [case.q_layers[l][0] for l in range(n_layers)] + \
             [case.q_layers[l][1] for l in range(n_layers)]
    results = list(outs) + list(sels)

    def run_step(din, dout):
        d_bt, d_sl = din[0], din[1]
        for l in range(n_layers):
            kp, vp, ikp = case.layers[l]
            uocr.sparse_decode(din[2 + l], kp, vp, din[2 + n_layers + l], ikp, d_bt, d_sl, out=dout[l],
                               sel=dout[n_layers + l], workspace=ws, stream=stream)

    return _e2e(args, inputs, results, run_step, stream, dev, case.n_q * n_layers, world)


# --------------------------------------------------------------------------- oracle timing
def _gather_for_oracle(case, layer, queries):
    """Host copies of what the oracle reads for `queries`: their queries and, once per
    sequence, that sequence's indexer pages (a small pool with its own block table)."""
    import numpy as np
    q, qi = case.q_layers[layer]
    ikp = case.layers[layer][2]
    mb = case.max_blocks
    seqs = sorted({int(case.q_seq[i]) for i in queries})
    need = {b: max(int(case.q_pos[i]) // 32 + 1 for i in queries if int(case.q_seq[i]) == b) for b in seqs}
    pages, rows, where, off = [], [], {}, 0
    for b in seqs:
        nb = need[b]
        pages.append(case.block_table[b, :nb].long())
        row = np.full(mb, -1, np.int32)
        row[:nb] = np.arange(off, off + nb)
        where[b] = len(rows)
        rows.append(row)
        off += nb
    mini_idx = ikp[torch.cat(pages)].cpu()
    qs = np.array([where[int(case.q_seq[i])] for i in queries], np.int32)
    pos = np.array([int(case.q_pos[i]) for i in queries], np.int32)
    return q[list(queries)].cpu(), qi[list(queries)].cpu(), mini_idx, np.stack(rows), qs, pos


def _gather_kv(case, layer, queries, sel):
    import numpy as np
    kp, vp, _ = case.layers[layer]
    rows, pages = [], []
    off = 0
    for n, i in enumerate(queries):
        b = int(case.q_seq[i])
        row = np.full(case.max_blocks, -1, np.int32)
        for j in sel[n]:
            if j >= 0:
                row[j] = off
                pages.append(int(case.block_table[b, j]))
                off += 1
        rows.append(row)
    pidx = torch.tensor(pages, dtype=torch.long, device=kp.device)
    return kp[pidx].cpu(), vp[pidx].cpu(), np.stack(rows)


class OracleInputs:
    """Host copies of what the oracle reads for `queries` of one layer: their queries, the
    sequences' indexer pages, and (after a first selection) the selected K/V pages."""

    def __init__(self, case, layer, queries):
        import oracle
        self.n = len(queries)
        self.q, self.qi, self.mini_idx, self.bt, self.qs, self.qp = _gather_for_oracle(case, layer, queries)
        H = self.q.shape[1]
        dummy = torch.zeros((1, H, 32, 128), dtype=torch.bfloat16)
        r = oracle.run(self.q, self.qi, dummy, dummy, self.mini_idx, self.bt, self.qs, self.qp, want_out=False,
                       want_scores=False)
        self.sel = r["sel"]
        self.kp, self.vp, self.bt2 = _gather_kv(case, layer, queries, self.sel)
        self.dummy = dummy

    def time(self, threads=0):
        """Seconds of oracle work (scores + selection, then attention over the selection)."""
        import numpy as np
        import oracle
        t0 = time.perf_counter()
        r = oracle.run(self.q, self.qi, self.dummy, self.dummy, self.mini_idx, self.bt, self.qs, self.qp,
                       want_out=False, want_scores=False, threads=threads)
        t1 = time.perf_counter()
        own_row = np.arange(self.n, dtype=np.int32)     # bt2 has one row per query
        r2 = oracle.run(self.q, self.qi, self.kp, self.vp, self.mini_idx[:1], self.bt2, own_row, self.qp,
                        sel_in=r["sel"], threads=threads)
        t2 = time.perf_counter()
        return t2 - t0, r["threads"], r2


def oracle_time_queries(case, layer, queries, threads=0):
    """Seconds of oracle work (scores + selection, then attention) for `queries` of one layer."""
    return OracleInputs(case, layer, queries).time(threads)


def cpu_baseline(case, budget_s: float = 10.0, max_layers: int = 2):
    """The oracle as it stands, on this host's cores, on a bounded sample of the same workload:
    whole layers of queries (the inputs of up to `max_layers` layers read back once), timed pass
    after pass until about budget_s seconds of oracle time."""
    n_layers = min(len(case.layers), max_layers)
    inputs = [OracleInputs(case, l, list(range(case.n_q))) for l in range(n_layers)]
    done, secs, threads, calls = 0, 0.0, 1, 0
    while secs < budget_s and calls < 1000:
        t, threads, _ = inputs[calls % n_layers].time()
        secs += t
        done += case.n_q
        calls += 1
    # the same oracle on one thread, on a few queries of the first layer (about 2 s)
    one, n1 = 0.0, 0
    while one < 2.0 and n1 < case.n_q:
        k = min(max(1, n1), case.n_q - n1)
        t, _, _ = oracle_time_queries(case, 0, list(range(n1, n1 + k)), threads=1)
        one += t
        n1 += k
    return {"value": round(done / secs, 2), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} queries ({calls} passes over {n_layers} layer(s) of {case.n_q} queries) of "
                      f"{case.name}, fp64, {secs:.1f} s of oracle time (host reads excluded)",
            "host_cpus": os.cpu_count(),
            "value_1_thread": round(n1 / one, 2), "sample_1_thread": f"{n1} queries, {one:.1f} s"}


# --------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle as the reference arm: same metric / unit / workload, on host cores."""
    rank, local_rank, world = udist.env_rank_world()
    if rank != 0:
        return
    dev = torch.device("cuda", local_rank) if torch.cuda.is_available() else torch.device("cpu")
    if dev.type == "cuda":
        torch.cuda.set_device(dev)
    name = args.workload
    if name == "long_decode":
        case = workloads.long_decode(device=dev, seed=args.seed, n_layers=1)
    else:
        case = build_workload(name, dev, args.seed)
    queries = list(range(min(case.n_q, 128)))     # a bounded sample per step
    for _ in range(args.warmup):
        oracle_time_queries(case, 0, queries[:1])
    secs, threads = [], 1
    for _ in range(args.steps):
        t, threads, _ = oracle_time_queries(case, 0, queries)
        secs.append(t)
    total = sum(secs)
    value = len(queries) * args.steps / total
    full_name = "long_decode_b16_ctx131072_layers12" if name == "long_decode" else case.name
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 2),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": full_name, "sample_per_step": f"{len(queries)} queries of one layer"},
           "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": threads, "kind": "oracle",
                            "sample": f"{len(queries)} queries x {args.steps} steps of {case.name}"},
           "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="uocr", choices=["uocr", "reference"])
    ap.add_argument("--workload", default="long_decode",
                    choices=["long_decode", "batched_decode", "tiny_decode", "ragged_paged_decode",
                             "chunked_prefill"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None, help="long_decode only: sequences (default 16)")
    ap.add_argument("--layers", type=int, default=None, help="long_decode only: layer caches (default 12)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-comparators", action="store_true", help="skip the full-attention / R-SWA timings")
    ap.add_argument("--no-configs", action="store_true",
                    help="long_decode only: skip the per-workload records of the other configs")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "uocr":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "chunked_prefill":
        run_prefill(args)
    else:
        run_uocr(args)


if __name__ == "__main__":
    main()

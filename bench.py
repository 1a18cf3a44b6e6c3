#!/usr/bin/env python3
"""Decode-step benchmark: sparse-attention decode tokens/s at 128K context, batch 8.

One step = one ls_decode_step over a batch of 8 requests at 131,072 tokens each:
fp8 indexer over every cached token (64 heads x 128), per-request top-2048, MLA
attention (128 heads, 576-wide latent KV, bf16) over the selected rows, all inputs
resident in HBM.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own batch of 8 requests (requests are
independent; no collective on the data path); the time is the max over ranks.
--impl reference times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn decode tokens/s at 128K ctx, batch 8; indexer+attn HBM GB/s vs peak"
UNIT = "tokens/s"
BATCH, CTX, TOPK = 8, 131072, 2048
H_I, D_I = 64, 128
INDEX_BYTES_PER_TOKEN = D_I + 4 + 4      # e4m3 key row + fp32 key scale read, fp32 score written
ATTN_ROW_BYTES = 576 * 2
WORKLOAD = "mla_decode_b8_ctx131072_top2048"
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "index_score_tc_mla_decode_b8_ctx131072.md")
CONFIG = {"workload": WORKLOAD, "batch": BATCH, "ctx": CTX, "topk": TOPK, "indexer": "64x128 e4m3",
          "attention": "MLA 128 heads x 576 (V 512) bf16", "page": 64,
          "l2": "flushed before every step: 256 MB written, then a second 256 MB buffer read so the "
                "flush's own dirty lines are written back before the step starts"}


def rank_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def profile_traffic():
    """Per-launch DRAM bytes of the indexer kernel from the committed ncu summary, valid
    only while the kernel source is unchanged since the capture."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    text = open(PROFILE_SUMMARY).read()
    m = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "sparse_attention_decode_ls_b200", "csrc", "index_score.cuh")
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != h.group(1):
        return None
    return float(m.group(1))


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x1: "gpu_idle"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- CPU oracle
def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info()] + [1]))
    except Exception:  # noqa: BLE001
        return 1


def oracle_request_runner(ctx, k, seed=1002):
    """Inputs of one request of the workload (context `ctx`, top-`k`) and a callable that
    runs the CPU oracle's decode step on it."""
    import oracle.ls_oracle as O
    from sparse_attention_decode_ls_b200 import synthetic as syn
    inp = syn.indexer_fp8([ctx], seed=seed)
    q, kv = syn.mla_attention(1, inp.key_pool.shape[0], seed=seed + 1000)
    qb = q.view(torch.int16).numpy().view(np.uint16)
    kvb = kv.view(torch.int16).numpy().view(np.uint16)
    wb = inp.w.view(torch.int16).numpy().view(np.uint16)

    def run():
        O.decode_step(q8=inp.q.numpy(), q_scale=inp.q_scale.numpy(), w_bits=wb, key_pool=inp.key_pool.numpy(),
                      key_scale_pool=inp.key_scale.numpy(), page_table=inp.page_table.numpy(), lens=[ctx], k=k,
                      q_attn_bits=qb, kv_pool_bits=kvb, scale=syn.softmax_scale(576), dv=512)
    return run


def _oracle_runs(run, budget_s, min_runs=1):
    """Call `run` until the next call would pass `budget_s` seconds (at least `min_runs`
    calls); returns the per-call times in seconds."""
    times, t_all = [], time.perf_counter()
    while True:
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
        el = time.perf_counter() - t_all
        if len(times) >= min_runs and el * (len(times) + 1) / len(times) > budget_s:
            return times


def oracle_single_thread(budget_s=6.0, frac=0.125):
    """The CPU oracle restricted to one thread, on one request at `frac` of the workload's
    context and top-k (a bounded sample): tokens/s, counting a run as `frac` tokens."""
    from threadpoolctl import threadpool_limits
    ctx_f = max(64 * 64, int(round(frac * CTX / 64)) * 64)
    f = ctx_f / CTX
    k_f = max(1, int(round(TOPK * f)))
    run = oracle_request_runner(ctx_f, k_f)
    with threadpool_limits(limits=1):
        times = _oracle_runs(run, budget_s)
    return {"value": len(times) * f / sum(times), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{len(times)} request(s) at context {ctx_f} with top-{k_f} ({f:.4f} of a {WORKLOAD} "
                      f"request each), one thread, float64 numpy, {sum(times):.1f} s"}


def cpu_oracle_sample(seconds_budget=15.0):
    """The CPU oracle on whole requests of the workload (indexer over 131,072 tokens,
    top-2048, MLA attention), as many as fit the budget (at least one), on all the host's
    cores; beside it the same oracle on one thread over a smaller sample."""
    run = oracle_request_runner(CTX, TOPK)
    times = _oracle_runs(run, seconds_budget)
    el = sum(times)
    return {"value": len(times) / el, "unit": UNIT, "cores": _oracle_cores(), "kind": "oracle",
            "sample": f"{len(times)} whole request(s) of {WORKLOAD} (one decode token each), float64 numpy, "
                      f"{el:.1f} s",
            "single_thread": oracle_single_thread()}


def run_reference(args):
    """Reference arm: the CPU oracle as it stands.  Each step runs it on ONE request whose
    context (and selection) is a fixed fraction f of the workload's, sized so the whole
    run stays within LS_REF_BUDGET_S seconds; a step counts as f decode tokens, and
    ms_per_step is the measured time of those steps."""
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    budget = float(os.environ.get("LS_REF_BUDGET_S", "150"))
    full = oracle_request_runner(CTX, TOPK)
    t0 = time.perf_counter()
    full()
    t_full = time.perf_counter() - t0
    n = args.warmup + args.steps
    f = min(1.0, 0.85 * budget / max(n * t_full, 1e-9))
    ctx_f = max(64 * 64, int(round(f * CTX / 64)) * 64)
    f = ctx_f / CTX
    k_f = max(1, int(round(TOPK * f)))
    run = full if ctx_f == CTX else oracle_request_runner(ctx_f, k_f)
    times = []
    for i in range(n):
        t0 = time.perf_counter()
        run()
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    value = len(times) * f / sum(times)
    sample = (f"each step: 1 request at context {ctx_f} with top-{k_f} ({f:.4f} of a {WORKLOAD} request, so "
              f"{f:.4f} tokens per step) on the CPU oracle (float64 numpy, all cores); one full request took "
              f"{t_full:.2f} s")
    config = dict(CONFIG, batch=1, reference_step=f"one request at context {ctx_f}, top-{k_f}",
                  tokens_per_step=f)
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
           "impl": "reference",
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": _oracle_cores(), "kind": "oracle",
                            "sample": sample,
                            "single_thread": oracle_single_thread(budget_s=min(10.0, 0.1 * budget))},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args):
    rank, world, local = rank_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from sparse_attention_decode_ls_b200 import binding as B
    from sparse_attention_decode_ls_b200 import workload as W

    wl = W.mla_decode(batch=BATCH, ctx=CTX, k=TOPK, seed=1002 + 7919 * rank, device="cuda")
    stream = torch.cuda.current_stream()
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    flush_sink = torch.empty((), dtype=torch.float32, device="cuda")

    class _Flush:  # evicts L2: write a buffer larger than L2, then read another one
        @staticmethod
        def zero_():
            flush_w.zero_()
            torch.sum(flush_r, dim=0, out=flush_sink)

    flush = _Flush()
    K, Wm = args.steps, args.warmup

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)
        return evs

    for _ in range(Wm):
        flush.zero_()
        wl.step()
    torch.cuda.synchronize()
    B.ls_check_device_status()
    # timed steps: nothing is recorded inside a step, so each kernel after the indexer
    # starts as a programmatic dependent of the one before (an event between two kernels
    # would serialise them)
    step_ev = [new_events(2) for _ in range(K)]
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.zero_()
            step_ev[i][0].record(stream)
            wl.step()
            step_ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = [s[0].elapsed_time(s[1]) for s in step_ev]
    # second timed pass, same steps: the indexer (the roofline kernel) bracketed by events
    idx_ev = [new_events(2) for _ in range(K)]
    arrs = [B.event_array([e[0], e[1], None, None, None, None]) for e in idx_ev]
    with ClockSampler(local) as clk2:
        for i in range(K):
            flush.zero_()
            wl.step(events=arrs[i])
        torch.cuda.synchronize()
    status = B.ls_check_device_status()
    idx_ms = [s[0].elapsed_time(s[1]) for s in idx_ev]
    # stage breakdown (not part of the timed number): every stage boundary recorded
    nb = min(K, 100)
    stage_ev = [new_events(6) for _ in range(nb)]
    for i in range(nb):
        flush.zero_()
        wl.step(events=B.event_array(stage_ev[i]))
    torch.cuda.synchronize()
    topk_ms = [s[1].elapsed_time(s[4]) for s in stage_ev]
    attn_ms = [s[4].elapsed_time(s[5]) for s in stage_ev]
    # the indexer kernel's own duration: launch after launch through ls_index_score (its
    # 143 MB of keys and scales exceed the 126 MB L2, so nothing is reused between launches;
    # inside a flushed step the events also enclose the launch gap before the kernel)
    t = wl.tensors
    scores = torch.empty((BATCH, wl.args.index.max_len), dtype=torch.float32, device="cuda")
    ia = B.index_args(q=t["i_q"], w=t["i_w"], key_pool=t["i_key_pool"], page_table=t["i_page_table"],
                      lens=t["i_lens"], scores=scores, q_scale=t["i_q_scale"], key_scale=t["i_key_scale"])
    lib, ia_ref, st_handle = B.lib(), B.C.byref(ia), stream.cuda_stream
    def run_indexer():  # arguments built once: the host keeps ahead of the GPU
        if lib.ls_index_score(ia_ref, st_handle) != 0:
            raise RuntimeError(lib.ls_get_error_string().decode())
    for _ in range(Wm):
        run_indexer()
    kb = new_events(2)
    torch.cuda.synchronize()
    kb[0].record(stream)
    for _ in range(K):
        run_indexer()
    kb[1].record(stream)
    torch.cuda.synchronize()
    idx_kernel_ms = kb[0].elapsed_time(kb[1]) / K
    total_ms = sum(step_ms)
    if dist:
        t = torch.tensor([total_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / K
    value = world * BATCH / (ms_per_step / 1e3)

    # ---- end to end through the C ABI with host buffers: per-step inputs (queries,
    # head weights, scales, lengths, page tables) go host->device, outputs come back
    t = wl.tensors
    # one packed buffer each way (the workload keeps a step's inputs, and its outputs, in
    # one device buffer): one host->device and one device->host copy per step
    # the attention's queries go on a second copy stream and the step waits for them just
    # before its attention, so their copy overlaps the indexer and the top-k
    host_in = torch.empty_like(t["step_in"], device="cpu").pin_memory()
    host_in.copy_(t["step_in"])
    host_in_attn = torch.empty_like(t["step_in_attn"], device="cpu").pin_memory()
    host_in_attn.copy_(t["step_in_attn"])
    host_out = torch.empty_like(t["step_out"], device="cpu").pin_memory()
    h2d_bytes = (host_in.numel() + host_in_attn.numel()) * host_in.element_size()
    d2h_bytes = host_out.numel() * host_out.element_size()
    copy_stream = torch.cuda.Stream()
    q_ready = torch.cuda.Event()
    in_done = torch.cuda.Event()
    e2e_ev = [new_events(2) for _ in range(K)]
    for i in range(Wm + K):
        flush.zero_()
        if i >= Wm:
            e2e_ev[i - Wm][0].record(stream)
        # the indexer's inputs first, with the host link to themselves (sharing it with the
        # queries' copy made them arrive ~25 us later); the queries follow on the copy
        # stream while the indexer runs (and after the last step, which read them)
        t["step_in"].copy_(host_in, non_blocking=True)
        in_done.record(stream)
        copy_stream.wait_event(in_done)
        with torch.cuda.stream(copy_stream):
            t["step_in_attn"].copy_(host_in_attn, non_blocking=True)
            q_ready.record(copy_stream)
        wl.args.attn_q_ready = q_ready.cuda_event
        wl.step()
        wl.args.attn_q_ready = None
        host_out.copy_(t["step_out"], non_blocking=True)
        if i >= Wm:
            e2e_ev[i - Wm][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(s[0].elapsed_time(s[1]) for s in e2e_ev)
    if dist:
        tt = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = float(tt.item())
    e2e_value = world * BATCH / (e2e_ms / K / 1e3)

    peak, peak_kind = measured_peaks()
    idx_bytes = BATCH * CTX * INDEX_BYTES_PER_TOKEN
    idx_mean_ms = statistics.mean(idx_ms)
    achieved = idx_bytes / (idx_kernel_ms / 1e3) / 1e9
    attn_bytes = BATCH * TOPK * ATTN_ROW_BYTES + BATCH * 128 * (576 + 512) * 2
    combined = (idx_bytes + attn_bytes) / ((idx_kernel_ms + statistics.mean(attn_ms)) / 1e3) / 1e9
    traffic = profile_traffic()
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm,
           "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "e4m3+bf16 (f32 accumulate)", "data": "synthetic",
           "config": dict(CONFIG, parallelism=f"requests sharded, {BATCH} per GPU" if world > 1 else "1 GPU"),
           "roofline": {"bound": "hbm", "kernel": "index_score_tc", "achieved": achieved, "peak": peak,
                        "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                        "algorithmic_bytes_per_launch": idx_bytes,
                        "indexer_ms": idx_kernel_ms, "indexer_ms_in_step": idx_mean_ms,
                        "topk_ms": statistics.mean(topk_ms),
                        "attn_ms": statistics.mean(attn_ms),
                        "indexer_plus_attn_GBps": combined, "indexer_plus_attn_frac": combined / peak,
                        "stage_note": "value from steps with no events inside them; indexer_ms (achieved) "
                                      "from K back-to-back indexer launches between two events; "
                                      "indexer_ms_in_step from a timed pass of the steps with the indexer "
                                      "bracketed by events; topk_ms and attn_ms from a pass with every "
                                      "stage boundary recorded"},
           "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
                   "d2h_bytes_per_step": d2h_bytes},
           "clocks": clk.summary(), "gpu_launches": K * wl.kernels_per_step, "device_status": status}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_oracle_sample(seconds_budget=args.cpu_seconds)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


def host_link_peaks(batch, n_slots=4096, reps=5):
    """The host link's read rate measured in this process, two ways over the same bytes (a
    whole hot buffer's worth of 1,152-byte rows, contiguous in pinned host memory): a plain
    copy-engine host-to-device copy, and the library's miss-gather kernel reading every row
    over the link (SM zero-copy loads, its own launch shape).  Best of `reps`, GB/s."""
    import torch
    from sparse_attention_decode_ls_b200 import binding as B
    stream = torch.cuda.current_stream()
    rows = batch * n_slots
    host = torch.empty((rows // 64, 64, 576), dtype=torch.bfloat16, pin_memory=True)
    host.view(torch.int16).random_(generator=torch.Generator().manual_seed(5))
    dev = torch.empty(host.shape, dtype=torch.bfloat16, device="cuda")
    nbytes = host.numel() * 2

    def best(fn):
        t = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            t.append(e0.elapsed_time(e1))
        return nbytes / (min(t) / 1e3) / 1e9

    ce = best(lambda: dev.copy_(host, non_blocking=True))
    pages = n_slots // 64
    table = torch.arange(rows // 64, dtype=torch.int32, device="cuda").view(batch, pages)
    pos = torch.arange(n_slots, dtype=torch.int32, device="cuda").repeat(batch, 1)
    n = torch.full((batch,), n_slots, dtype=torch.int32, device="cuda")
    hbuf = dev.view(batch, n_slots, 576)
    sm = best(lambda: B.ls_gather_misses(host_kv=host, page_table=table, miss_pos=pos, miss_slot=pos, n_miss=n,
                                         hbuf=hbuf))
    assert torch.equal(hbuf.view(-1).view(torch.int16).cpu(), host.view(-1).view(torch.int16))
    del host, dev
    return {"copy_engine_GBps": ce, "sm_gather_contiguous_GBps": sm, "bytes": nbytes}


def run_hotbuf(args):
    """Optional line (not the headline): the hot-buffer decode step -- indexer, top-k,
    hot-buffer resolve, gather of the misses from pinned host memory over the host link,
    attention -- at batch 36 x 131,072 with a 4,096-slot buffer per request.  The buffer
    state is restored, and L2 evicted, before every step (untimed)."""
    import torch
    from sparse_attention_decode_ls_b200 import binding as B
    from sparse_attention_decode_ls_b200 import workload as W

    batch = args.batch or 36
    wl = W.mla_hotbuf_decode(batch=batch, ctx=CTX, k=TOPK, miss_frac=args.miss, device="cuda")
    stream = torch.cuda.current_stream()
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    sink = torch.empty((), dtype=torch.float32, device="cuda")

    def prep():
        wl.restore_hotbuf()
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=sink)

    for _ in range(args.warmup):
        prep()
        wl.step()
    torch.cuda.synchronize()
    B.ls_check_device_status()
    ev = []
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            prep()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            wl.step()
            e1.record(stream)
            ev.append((e0, e1))
        torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    # stage breakdown (not part of the timed number): indexer, top-k, resolve, miss gather,
    # then the miss pass and the merge (the resident-row pass runs beside the gather)
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(min(args.steps, 20))]
    for evs in stage_ev:
        for e in evs:
            e.record(stream)   # created by torch; the library records them again inside the step
    for evs in stage_ev:
        prep()
        wl.step(events=B.event_array(evs))
    torch.cuda.synchronize()
    status = B.ls_check_device_status()
    names = ("indexer", "topk", "resolve", "gather", "attention")
    stages = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in stage_ev) for i, n in enumerate(names)}
    n_miss = int(wl.tensors["n_miss"].sum().item())
    link_bytes = n_miss * 576 * 2
    peaks = host_link_peaks(batch)
    link_peak = max(peaks["copy_engine_GBps"], peaks["sm_gather_contiguous_GBps"])
    fetch_GBps = link_bytes / (stages["gather"] / 1e3) / 1e9
    step_GBps = link_bytes / (ms / 1e3) / 1e9
    out = {"metric": "hot-buffer sparse-attn decode tokens/s at 128K ctx", "value": batch / (ms / 1e3),
           "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16 (f32 accumulate)",
           "data": "synthetic",
           "config": {"workload": wl.name, "batch": batch, "ctx": CTX, "topk": TOPK, "hot_slots": 4096,
                      "miss_frac": args.miss, "history": "pinned host memory, read over the host link",
                      "l2": "evicted before every step (256 MB written, then 256 MB read)"},
           "gpu_launches": wl.kernels_per_step * args.steps,
           "host_link": {"bytes_per_step": link_bytes, "GBps": step_GBps, "gather_GBps": fetch_GBps,
                         "peak_GBps": link_peak, "peaks_measured": peaks,
                         "fetch_frac": fetch_GBps / link_peak, "step_frac": step_GBps / link_peak,
                         "note": "peak = the faster of a plain pinned host-to-device copy and the miss-gather "
                                 "kernel over contiguous rows, measured in this run; fetch_frac: the step's miss "
                                 "fetch (scattered 1,152-byte rows) over its stage time; step_frac: the misses' "
                                 "bytes over the whole step"},
           "stages_ms": stages,
           "clocks": clk.summary(), "device_status": status}
    print(json.dumps(out), flush=True)
    return 0


def run_tiny(args):
    """Optional line: the tiny fp32 configuration (one request at 8,192 tokens, indexer 8
    heads x 64, top-256, 16 attention heads of 128 over one K and one V head) -- a
    launch-latency-bound step, reported in microseconds."""
    import torch
    from sparse_attention_decode_ls_b200 import binding as B
    from sparse_attention_decode_ls_b200 import workload as W

    wl = W.tiny_f32(device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()
    ev = []
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            wl.step()
            e1.record(stream)
            ev.append((e0, e1))
        torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    # the same step captured once in a CUDA graph and replayed: the launches' host cost
    # leaves the critical path (a decode loop would replay the graph every step)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        wl.step()
    stream.wait_stream(side)
    with torch.cuda.graph(g):
        wl.step()
    for _ in range(args.warmup):
        g.replay()
    gev = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        gev.append((e0, e1))
    torch.cuda.synchronize()
    graph_ms = statistics.median(a.elapsed_time(b) for a, b in gev)
    del g
    status = B.ls_check_device_status()
    out = {"metric": "tiny fp32 decode step latency", "value": ms * 1e3, "unit": "us", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": {"workload": wl.name, "batch": 1, "ctx": 8192, "topk": 256, "indexer": "8x64 f32",
                      "attention": "16 heads x 128, one K and one V head, f32", "statistic": "median",
                      "l2": "not evicted: the whole working set (~2.4 MB) is L2-resident, as it would be"},
           "tokens_per_s": 1 / (ms / 1e3), "graph_replay_us": graph_ms * 1e3,
           "gpu_launches": wl.kernels_per_step * args.steps,
           "clocks": clk.summary(), "device_status": status}
    print(json.dumps(out), flush=True)
    return 0


def run_sweep(args):
    """Optional line: the ragged mixed-batch sweep -- batch 1, 16, 64, 192 and 256, context
    lengths ~U[4096, 16384] per request, top-2048, a 4,096-slot hot buffer per request with
    20% of the selection missing, history in pinned host memory -- per-step latency (the
    TPOT proxy of one layer) and tokens/s against the batch."""
    import gc
    import torch
    from sparse_attention_decode_ls_b200 import binding as B
    from sparse_attention_decode_ls_b200 import synthetic as syn
    from sparse_attention_decode_ls_b200 import workload as W

    batches = [int(x) for x in args.batches.split(",")] if args.batches else [1, 16, 64, 192, 256]
    stream = torch.cuda.current_stream()
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    sink = torch.empty((), dtype=torch.float32, device="cuda")
    rows, statuses = [], []
    peaks = host_link_peaks(64)
    link_peak = max(peaks["copy_engine_GBps"], peaks["sm_gather_contiguous_GBps"])
    with ClockSampler(0) as clk:
        for bsz in batches:
            lens = syn.ragged_lens(bsz, 4096, 16384, seed=1005)
            wl = W.mla_hotbuf_decode(lens=lens, miss_frac=0.2, seed=1005, device="cuda")

            def prep():
                wl.restore_hotbuf()
                flush_w.zero_()
                torch.sum(flush_r, dim=0, out=sink)

            for _ in range(args.warmup):
                prep()
                wl.step()
            torch.cuda.synchronize()
            statuses.append(B.ls_check_device_status())
            ev = []
            for _ in range(args.steps):
                prep()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                wl.step()
                e1.record(stream)
                ev.append((e0, e1))
            torch.cuda.synchronize()
            statuses.append(B.ls_check_device_status())
            ms = statistics.median(a.elapsed_time(b) for a, b in ev)
            # the miss fetch's own time from a pass with the stage boundaries recorded
            stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(5)]
            for evs in stage_ev:
                for e in evs:
                    e.record(stream)
            for evs in stage_ev:
                prep()
                wl.step(events=B.event_array(evs))
            torch.cuda.synchronize()
            gather_ms = statistics.median(e[3].elapsed_time(e[4]) for e in stage_ev)
            n_miss = int(wl.tensors["n_miss"].sum().item())
            link = n_miss * 1152
            rows.append({"batch": bsz, "ms_per_step": ms, "tokens_per_s": bsz / (ms / 1e3),
                         "mean_ctx": sum(lens) / bsz, "link_bytes_per_step": link,
                         "fetch_GBps": link / (gather_ms / 1e3) / 1e9, "step_link_GBps": link / (ms / 1e3) / 1e9,
                         "fetch_frac": link / (gather_ms / 1e3) / 1e9 / link_peak,
                         "step_frac": link / (ms / 1e3) / 1e9 / link_peak,
                         "gpu_launches_per_step": wl.kernels_per_step})
            del wl
            gc.collect()
            torch.cuda.empty_cache()
    out = {"metric": "ragged batch sweep: per-step latency (one layer) and tokens/s vs batch",
           "value": rows[-1]["tokens_per_s"], "unit": UNIT, "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": rows[-1]["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16 (f32 accumulate)", "data": "synthetic",
           "config": {"workload": "ragged_hotbuf_sweep", "batches": batches, "ctx": "U[4096, 16384] per request",
                      "topk": TOPK, "hot_slots": 4096, "miss_frac": 0.2,
                      "history": "pinned host memory, misses read over the host link",
                      "l2": "evicted before every step (256 MB written, then 256 MB read)",
                      "statistic": "median over the timed steps"},
           "sweep": rows, "host_link_peak_GBps": link_peak, "host_link_peaks_measured": peaks,
           "clocks": clk.summary(), "device_status": max(statuses) if statuses else 0}
    print(json.dumps(out), flush=True)
    return 0


def run_c2f(args):
    """Optional line (not the headline): the coarse-to-fine decode step at batch 4 x
    1,048,576 tokens -- block bounds over the summaries, the candidate blocks' exact
    scores, pruning, the survivors' exact scores, top-k, attention -- with the original
    indexer keys in HBM or (``--keys host``) in pinned host memory."""
    import torch
    from sparse_attention_decode_ls_b200 import binding as B
    from sparse_attention_decode_ls_b200 import workload as W

    batch, ctx = args.batch or 4, 1048576
    on_host = args.keys == "host"
    wl = W.c2f_decode(batch=batch, ctx=ctx, k=TOPK, keys_on_host=on_host, device="cuda")
    stream = torch.cuda.current_stream()
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    sink = torch.empty((), dtype=torch.float32, device="cuda")

    def prep():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=sink)

    for _ in range(args.warmup):
        prep()
        wl.step()
    torch.cuda.synchronize()
    B.ls_check_device_status()
    ev = []
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            prep()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            wl.step()
            e1.record(stream)
            ev.append((e0, e1))
        torch.cuda.synchronize()
    status = B.ls_check_device_status()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    full = None
    if not on_host:
        # the full scan on the same data: every key scored, then the top-k -- the selection
        # must be the coarse-to-fine one, and its time is what the pruning saves
        t = wl.tensors
        scores = torch.empty((batch, ctx), dtype=torch.float32, device="cuda")
        idx_full = torch.empty((batch, TOPK), dtype=torch.int32, device="cuda")

        def full_scan():
            B.ls_index_score(q=t["i_q"], w=t["i_w"], key_pool=t["i_key_pool"], page_table=t["i_page_table"],
                             lens=t["i_lens"], scores=scores, q_scale=t["i_q_scale"], key_scale=t["i_key_scale"])
            B.ls_topk_select(scores=scores, lens=t["i_lens"], idx=idx_full)

        for _ in range(args.warmup):
            prep()
            full_scan()
        fev = []
        for _ in range(args.steps):
            prep()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            full_scan()
            e1.record(stream)
            fev.append((e0, e1))
        # the coarse-to-fine part of the step alone, for the same comparison
        cev = []
        for _ in range(args.steps):
            prep()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
            for e in evs:
                e.record(stream)
            wl.step(events=B.event_array(evs))
            cev.append(evs)
        torch.cuda.synchronize()
        fms = statistics.mean(a.elapsed_time(b) for a, b in fev)
        cms = statistics.mean(e[0].elapsed_time(e[4]) for e in cev)
        full = {"indexer_plus_topk_ms": fms, "c2f_indexer_plus_topk_ms": cms, "speedup": fms / cms,
                "same_selection": bool(torch.equal(idx_full, wl.idx))}
        status |= B.ls_check_device_status()
    n_surv = [int(x) for x in wl.tensors["n_survivors"].tolist()]
    n_blocks = -(-ctx // 64)
    nb0 = (TOPK + 63) // 64 + 1
    block_bytes = 64 * 128 + 64 * 4  # e4m3 keys + fp32 token scales
    out = {"metric": "coarse-to-fine sparse-attn decode tokens/s at 1M ctx", "value": batch / (ms / 1e3),
           "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16 (f32 accumulate)",
           "data": "synthetic",
           "config": {"workload": wl.name, "batch": batch, "ctx": ctx, "topk": TOPK,
                      "keys": "pinned host memory (only summaries in HBM)" if on_host else "HBM",
                      "l2": "evicted before every step (256 MB written, then 256 MB read)"},
           "survivors": {"per_request": n_surv, "of_blocks": n_blocks,
                         "fraction": sum(n_surv) / (batch * n_blocks)},
           "full_scan": full,
           "indexer_key_bytes": {"in_hbm": 0 if on_host else batch * ctx * 132,
                                 "over_host_link_per_step": (batch * nb0 + sum(n_surv)) * block_bytes if on_host else 0},
           "gpu_launches": wl.kernels_per_step * args.steps,
           "clocks": clk.summary(), "device_status": status}
    print(json.dumps(out), flush=True)
    return 0


def run_prefill(args):
    """Optional line: the two-buffer layer-streaming prefill -- each layer's indexer keys
    and scales copied from pinned host memory into one of two staging buffers while the
    previous layer's block summaries are built and its hot buffer is seeded -- at batch 4
    x 1,048,576 tokens per layer, 4 layers.  Reported against a plain host-to-device copy
    of the same bytes (the link's rate on this machine)."""
    import torch
    from sparse_attention_decode_ls_b200 import binding as B
    from sparse_attention_decode_ls_b200 import synthetic as syn

    batch, ctx, n_layers, n_slots = args.batch or 4, 1048576, 4, 4096
    lens = [ctx] * batch
    table, n_pool = syn.page_layout(lens, 1021)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1022)
    keys, scales = [], []
    for _ in range(n_layers):  # seeded keys per layer, quantised on the device, then pinned
        k8 = torch.empty((n_pool, 64, 128), dtype=torch.uint8, pin_memory=True)
        sk = torch.empty((n_pool, 64), dtype=torch.float32, pin_memory=True)
        for i in range(0, n_pool, 4096):
            j = min(n_pool, i + 4096)
            x = torch.randn(((j - i) * 64, 128), generator=gen, device="cuda")
            amax = x.abs().amax(dim=1, keepdim=True).clamp_min(1e-12)
            sc = amax / 448.0
            k8[i:j].copy_((x / sc).to(torch.float8_e4m3fn).view(torch.uint8).view(j - i, 64, 128))
            sk[i:j].copy_(sc.view(j - i, 64))
        keys.append(k8)
        scales.append(sk)
    kv = torch.empty((n_pool, 64, 576), dtype=torch.bfloat16, pin_memory=True)  # one history, all layers
    for i in range(0, n_pool, 4096):
        j = min(n_pool, i + 4096)
        kv[i:j].copy_(torch.randn((j - i, 64, 576), generator=gen, device="cuda").to(torch.bfloat16))
    torch.cuda.synchronize()
    dev = "cuda"
    mb = -(-ctx // 64)
    a = B.prefill_args(page_table=table.to(dev), lens=torch.tensor(lens, dtype=torch.int32, device=dev), max_len=ctx,
                       host_keys=keys, host_key_scales=scales,
                       summaries=[torch.empty((batch, mb, 256), dtype=torch.uint8, device=dev) for _ in range(n_layers)],
                       block_scale=[torch.empty((batch, mb), device=dev) for _ in range(n_layers)],
                       host_kv=[kv] * n_layers,
                       hbuf=[torch.empty((batch, n_slots, 576), dtype=torch.bfloat16, device=dev)
                             for _ in range(n_layers)],
                       pos_of_slot=[torch.empty((batch, n_slots), dtype=torch.int32, device=dev) for _ in range(n_layers)],
                       slot_of_pos=[torch.empty((batch, ctx), dtype=torch.int32, device=dev) for _ in range(n_layers)],
                       recent_score=[torch.empty((batch, n_slots), device=dev) for _ in range(n_layers)])
    ws = torch.empty(B.ls_prefill_stream_workspace_size(a), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        ev = []
        for _ in range(n):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            ev.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.mean(x.elapsed_time(y) for x, y in ev)

    for _ in range(args.warmup):
        B.ls_prefill_stream(a, ws)
    torch.cuda.synchronize()
    B.ls_check_device_status()
    with ClockSampler(0) as clk:
        ms = timed(lambda: B.ls_prefill_stream(a, ws), args.steps)
    status = B.ls_check_device_status()
    # the link's own rate: one layer's keys and scales with two plain copies on this stream
    dst_k = torch.empty((n_pool, 64, 128), dtype=torch.uint8, device=dev)
    dst_s = torch.empty((n_pool, 64), dtype=torch.float32, device=dev)
    copy_ms = timed(lambda: (dst_k.copy_(keys[0], non_blocking=True), dst_s.copy_(scales[0], non_blocking=True)), 5)
    layer_bytes = n_pool * 64 * (128 + 4)
    seed_bytes = batch * n_slots * 576 * 2
    out = {"metric": "layer-streaming prefill: indexer-key GB/s over the host link", "value":
           n_layers * layer_bytes / (ms / 1e3) / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "e4m3 (summaries: exact)", "data": "synthetic",
           "config": {"workload": f"prefill_stream_b{batch}_ctx{ctx}_layers{n_layers}", "batch": batch, "ctx": ctx,
                      "layers": n_layers, "hot_slots": n_slots, "step": "one call: every layer streamed, "
                      "summarised and its hot buffer seeded"},
           "per_layer_ms": ms / n_layers, "layer_key_bytes": layer_bytes, "seed_bytes_per_layer": seed_bytes,
           "plain_copy": {"ms_per_layer": copy_ms, "GBps": layer_bytes / (copy_ms / 1e3) / 1e9},
           "frac_of_plain_copy": (copy_ms * n_layers) / ms,
           "clocks": clk.summary(), "device_status": status}
    print(json.dumps(out), flush=True)
    return 0


def run_cp(args):
    """Optional line: one batch of long requests split by context over the ranks
    (context-parallel, strong scaling): batch 4 x 1,048,576 tokens, full indexer scan of
    each rank's shard, candidates and partial outputs all-gathered over NCCL."""
    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from sparse_attention_decode_ls_b200 import binding as B
    from sparse_attention_decode_ls_b200 import cp
    from sparse_attention_decode_ls_b200 import synthetic as syn

    batch, ctx, k = args.batch or 4, 1048576, TOPK
    ranges = cp.shard_ranges([ctx] * batch, world)
    begin = [ranges[b][rank][0] for b in range(batch)]
    end = [ranges[b][rank][1] for b in range(batch)]
    llens = [e - s for s, e in zip(begin, end)]
    table, n_pool = syn.page_layout(llens, 3001 + rank)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(3002 + rank)  # this rank's shard of the history
    k8 = torch.empty((n_pool, 64, 128), dtype=torch.uint8, device="cuda")
    sk = torch.empty((n_pool, 64), dtype=torch.float32, device="cuda")
    kv = torch.empty((n_pool, 64, 576), dtype=torch.bfloat16, device="cuda")
    for i in range(0, n_pool, 4096):
        j = min(n_pool, i + 4096)
        x = torch.randn(((j - i) * 64, 128), generator=gen, device="cuda")
        sc = x.abs().amax(dim=1, keepdim=True).clamp_min(1e-12) / 448.0
        k8[i:j] = (x / sc).to(torch.float8_e4m3fn).view(torch.uint8).view(j - i, 64, 128)
        sk[i:j] = sc.view(j - i, 64)
        kv[i:j] = torch.randn((j - i, 64, 576), generator=gen, device="cuda").to(torch.bfloat16)
    g = torch.Generator().manual_seed(3000)  # the queries: the same on every rank
    q8, qs = syn.quantize_e4m3(torch.randn((batch, 64, 128), generator=g))
    w = (torch.randn((batch, 64), generator=g) * 0.1).to(torch.bfloat16)
    qa = torch.randn((batch, 128, 576), generator=g).to(torch.bfloat16)
    dev = "cuda"
    tdev = table.to(dev)
    ml = max(4, (max(llens) + 3) // 4 * 4)
    ix = B.index_args(q=q8.to(dev), w=w.to(dev), key_pool=k8, page_table=tdev,
                      lens=torch.tensor(llens, dtype=torch.int32, device=dev), q_scale=qs.view(batch, 64).to(dev),
                      key_scale=sk, max_len=ml)
    step = cp.ShardStep(index=ix, k=k, attn=dict(q=qa.to(dev), kv=kv, page_table=tdev, scale=syn.softmax_scale(576)),
                        begin=torch.tensor(begin, dtype=torch.int32, device=dev),
                        end=torch.tensor(end, dtype=torch.int32, device=dev), world=world)
    o = torch.empty((batch, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((batch, 128), device=dev)
    stream = torch.cuda.current_stream()
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        step.step(o, lse)
    torch.cuda.synchronize()
    B.ls_check_device_status()
    if dist:
        dist.barrier()
    ev = []
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            flush_w.zero_()
            torch.sum(flush_r, dim=0, out=sink)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step.step(o, lse)
            e1.record(stream)
            ev.append((e0, e1))
        torch.cuda.synchronize()
    status = B.ls_check_device_status()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    if dist:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    if rank == 0:
        out = {"metric": "context-parallel sparse-attn decode tokens/s at 1M ctx", "value": batch / (ms / 1e3),
               "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
               "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
               "dtype": "e4m3+bf16 (f32 accumulate)", "data": "synthetic",
               "config": {"workload": f"cp_b{batch}_ctx{ctx}", "batch": batch, "ctx": ctx, "topk": k,
                          "parallelism": f"context-parallel over {world} GPU(s)",
                          "exchange_bytes_per_step": world * batch * (k * 8 + 128 * 512 * 4 + 128 * 4),
                          "l2": "evicted before every step (256 MB written, then 256 MB read)"},
               "clocks": clk.summary(), "device_status": status}
        print(json.dumps(out), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batches", default="", help="sweep: comma-separated batch sizes (default 1,16,64,192,256)")
    ap.add_argument("--workload", choices=["mla", "hotbuf", "c2f", "prefill", "cp", "sweep", "tiny"], default="mla",
                    help="mla: the headline step (default); hotbuf: the hot-buffer step; c2f: the "
                         "coarse-to-fine step at 1M context; prefill: layer-streaming prefill (one GPU each); "
                         "cp: 1M-context requests split by context over the ranks; sweep: ragged batch sweep; "
                         "tiny: the fp32 8K-context step")
    ap.add_argument("--keys", choices=["hbm", "host"], default="hbm", help="c2f: where the original keys live")
    ap.add_argument("--batch", type=int, default=0, help="hotbuf: requests (default 36)")
    ap.add_argument("--miss", type=float, default=0.2, help="hotbuf: fraction of the selection that misses")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.workload == "hotbuf":
        return run_hotbuf(args)
    if args.workload == "c2f":
        return run_c2f(args)
    if args.workload == "prefill":
        return run_prefill(args)
    if args.workload == "cp":
        return run_cp(args)
    if args.workload == "sweep":
        return run_sweep(args)
    if args.workload == "tiny":
        return run_tiny(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python3
"""Benchmark of the decode-attention stack (q_rotate, kv_append,
paged_decode_attn, attn_combine for every full-attention layer) on one B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...        # the oracle on the host cores

A step is one decode step of the whole attention stack: for each of the 16
layers, rotate the query (q4_0), append this step's K/V token, run the split-K
decode over the full context and combine the splits.  Inputs are resident in
HBM when the timed region starts; the KV pool (4.83 GB for the default
workload) is larger than L2, so no flush is needed between steps.  Under
torchrun each rank runs an independent replica (weak scaling, no collective
on the data path); the reported time is the max over ranks.

One JSON line is printed by rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn KV GB/s & % HBM peak; attn-stack tokens/s at 262K ctx (1 B200)"
DEFAULT_WORKLOAD = "qwen27b_q4_0_262k"
FALLBACK_HBM_GBS = 6650.0


FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense fp16/bf16 tensor throughput to hold a kernel timed on its own against (burst)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured cuBLAS bf16 GEMM (burst)"
    return FALLBACK_BF16_TFLOPS, "fallback 1.59 PFLOP/s"


def decode_source_hash() -> str:
    """Hash of the decode kernel's code (comments and whitespace removed), the
    key under which profiles/decode_traffic.json records ncu DRAM counters."""
    import re
    h = hashlib.sha256()
    for f in ("kvq_decode.cu", "kvq_internal.cuh", "kvq_append_dev.cuh"):
        text = open(os.path.join(ROOT, "quantized_kv_cache_17_b200", "csrc", f)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_tag: str, workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(f"{kernel_tag}:{workload}")
        if e and e.get("source_hash") == decode_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


class ClockSampler:
    """nvidia-smi samples of this GPU during the timed region."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        return self.summarize(self.lines, self.uuid)

    @staticmethod
    def summarize(lines, uuid: str):
        """Median SM clock, the max clock, and the throttle reasons seen active,
        over the sample lines of this GPU (uuid; empty = every line)."""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9 or (uuid and uuid not in parts[0]):
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
def max_over_ranks(dist, values, device="cpu"):
    """Element-wise max of per-rank timings over all ranks (the values as they
    are with one process).  Every rank must call it, in the same order."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_gbs(world: int, bytes_per_rank_step: float, ms_per_step: float) -> float:
    """Whole-job GB/s when every rank streams the same bytes per step
    (independent replicas) and a step takes ms_per_step (max over ranks)."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_oracle_parallel(fmt: str, groups, threads: int):
    """The oracle (as it stands) over whole (layer, KV head) groups on `threads`
    host threads: every group's token range is cut into chunks, each chunk is
    one oracle partial (the oracle's own split form, ctypes releases the GIL),
    and each group's partials are merged with the oracle's merge.  `groups` is
    a list of ((kc, ks, vc, vs), qp).  Returns (seconds, tokens, bytes)."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    per_tok = oracle.format_bytes_per_token_head(fmt)
    n_chunks = max(1, -(-threads // len(groups)))
    tasks = []
    for gi, (codes, qp) in enumerate(groups):
        T = codes[0].shape[0]
        for c in range(n_chunks):
            t0, t1 = c * T // n_chunks, (c + 1) * T // n_chunks
            if t1 > t0:
                tasks.append((gi, t0, t1))

    def run(task):
        gi, t0, t1 = task
        codes, qp = groups[gi]
        return gi, oracle.attn_partial(fmt, qp, t0, t1, *codes)

    t_start = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(run, tasks))
    merged = {}
    for gi, part in parts:
        merged[gi] = part if gi not in merged else oracle.merge_partials(merged[gi], part)
    for gi, (m, l, o) in merged.items():
        oracle.finish(fmt, l, o)
    dt = time.perf_counter() - t_start
    tokens = sum(c[0].shape[0] for c, _ in groups)
    return dt, tokens, tokens * per_tok


def cpu_append_us(fmt: str, n_kv: int, layers: int, k_rows: np.ndarray, v_rows: np.ndarray, reps: int = 20):
    """The oracle's kv_append of one decode step (one token per KV head and
    layer), single thread, in microseconds per step."""
    import oracle
    t0 = time.perf_counter()
    for _ in range(reps):
        for _l in range(layers):
            oracle.append_rows(fmt, k_rows[:n_kv], v_rows[:n_kv])
    return (time.perf_counter() - t0) / reps * 1e6


def run_reference(args):
    """The oracle on the host cores, each step a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import kvq_inputs
    import oracle
    w = kvq_inputs.workload(args.workload)
    layer, b, g = 0, 0, 0
    T_sample = min(w.seq_lens[-1], 8192)
    k = w.k_rows(layer, b, 0, T_sample)[:, g]
    v = w.v_rows(layer, b, 0, T_sample)[:, g]
    codes = oracle.append_rows(w.fmt, k, v)
    qp = oracle.q_prepare(w.fmt, w.q_row(layer, b)[g * w.group:(g + 1) * w.group])
    per_tok = oracle.format_bytes_per_token_head(w.fmt)
    cores = host_cores()
    groups = [(codes, qp)]
    for _ in range(args.warmup):
        cpu_oracle_parallel(w.fmt, groups, cores)
    times = []
    for _ in range(args.steps):
        times.append(cpu_oracle_parallel(w.fmt, groups, cores)[0])
    dt = sum(times) / len(times)
    gbs = T_sample * per_tok / dt / 1e9
    sample = (f"oracle fp64 attention of one (layer, KV head) group ({w.group} query heads) over the first "
              f"{T_sample} tokens of {w.name} (codes from the oracle's own append), cut into token chunks run "
              f"on {cores} threads ({cpu_model()}) and merged with the oracle's own merge")
    line = {"metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "format": w.fmt, "seq_lens": w.seq_lens, "layers": w.n_layers,
                       "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": 256},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(), "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
OTHER_WORKLOADS = ("qwen27b_int8_32k", "flashnext_k8v4_128k", "ragged4_q4_0", "ragged4_k8v4", "qwen27b_fp8_262k",
                   "qwen27b_nvfp4_262k")


def measure_prefill(T: int, n_tok: int, steps: int, warmup: int, uuid: str):
    """paged_prefill_attn of the last n_tok tokens of a T-token sequence on one
    layer of the 27B q4_0 shape (24 Q / 4 KV heads), timed with CUDA events
    over `steps` calls; useful FLOPs = 4 x 256 per (query row, key) pair in the
    causal range (QK and PV, 2 per multiply-add).  Returns a sub-record."""
    import torch
    import kvq_inputs
    import quantized_kv_cache_17_b200 as kvq
    from kvq_inputs import device as kdev
    w = kvq_inputs.Workload(name=f"prefill_q4_0_{T // 1024}k_{n_tok}", index=4, fmt="q4_0", n_layers=1,
                            n_q_heads=24, n_kv_heads=4, seq_lens=[T], page_order="contiguous", n_outlier=8,
                            outlier_kind="student_t", q_post=1.0 / 16, q_outliers=False)
    dw = kdev.build_pool(w, prefill_last=True)
    qt = kdev.DeviceTable(w.q_table(0), "cuda")
    qp = kvq.q_rotate(kdev.gen_rows_device(w.q_key(0, 0), qt, 0, n_tok))
    out_bf = torch.empty((n_tok, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos0 = T - n_tok
    n_split, wb = kvq.prefill_split(dw.pool.desc, pos0, n_tok)
    ws = torch.empty(max(wb, 16) // 4, dtype=torch.float32, device="cuda")

    def run(ns):
        kvq.paged_prefill_attn(dw.pool, 0, qp, 0, pos0, dw.page_table, out_bf, status=status, n_split=ns,
                               workspace=ws if ns > 1 else None)

    for _ in range(warmup):
        run(n_split)
        run(1)
    torch.cuda.synchronize()
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    stream = torch.cuda.current_stream()
    ev[0].record(stream)
    for _ in range(steps):
        run(n_split)
    ev[1].record(stream)
    ev[2].record(stream)
    for _ in range(steps):
        run(1)
    ev[3].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    assert int(status.item()) == 0, f"kernel status {status.item()} in the prefill"
    us = ev[0].elapsed_time(ev[1]) * 1e3 / steps
    us_one = ev[2].elapsed_time(ev[3]) * 1e3 / steps
    keys = float(np.arange(pos0 + 1, T + 1, dtype=np.float64).sum())
    flops = 4.0 * 256 * w.n_q_heads * keys
    tpk, tsrc = tensor_peak()
    tflops = flops / (us * 1e-6) / 1e12
    rec = {"workload": w.name, "format": "q4_0", "context": T, "chunk_tokens": n_tok, "us_per_layer": round(us, 1),
           "n_split": n_split, "us_per_layer_unsplit": round(us_one, 1),
           "useful_tflops": round(tflops, 2), "tok_s_16_layers": round(n_tok / (16 * us * 1e-6), 1),
           "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": tpk, "unit": "TFLOP/s",
                        "frac": round(tflops / tpk, 4), "peak_source": tsrc},
           "clocks": clocks}
    del dw, qp, out_bf, ws
    torch.cuda.empty_cache()
    return rec


def measure_resident(T: int, steps: int, warmup: int, uuid: str):
    """Host-resident KV: one layer of the 27B q4_0 shape at T tokens kept in a
    pinned host pool, paged into a device cache by kvq_resident_load (the
    zero-copy page-in kernel), timed with CUDA events; beside it the copy engine
    moving the same bytes in one cudaMemcpyAsync (the bus ceiling), the host
    planning time of kvq_resident_map for an all-miss and an all-hit call, and a
    cold layer (page-in of every page, then the decode).  Returns a sub-record."""
    import torch
    import kvq_inputs
    import quantized_kv_cache_17_b200 as kvq
    from kvq_inputs import device as kdev
    w = kvq_inputs.Workload(name=f"resident_q4_0_{T // 1024}k", index=4, fmt="q4_0", n_layers=1, n_q_heads=24,
                            n_kv_heads=4, seq_lens=[T], page_order="permuted", n_outlier=8,
                            outlier_kind="student_t", q_post=1.0 / 16, q_outliers=False)
    dw = kdev.build_pool(w)
    H = kvq.KVPool.allocate(dw.pool.desc, "pinned")
    H.buf.copy_(dw.pool.buf)
    n_pages = dw.pool.desc.n_pages
    dw.pool = None
    torch.cuda.empty_cache()
    C = kvq.KVPool.allocate(kvq.make_desc(1, w.n_kv_heads, w.n_q_heads, n_pages, "q4_0"))
    rc = kvq.ResidentCache(H, C)
    t0 = time.perf_counter()
    cpt, loads = rc.map(0, dw.page_table_host, w.seq_lens)
    map_miss_us = (time.perf_counter() - t0) * 1e6
    t0 = time.perf_counter()
    for _ in range(20):
        rc.map(0, dw.page_table_host, w.seq_lens)
    map_hit_us = (time.perf_counter() - t0) * 1e6 / 20
    nbytes = len(loads) * kvq.pool_layout(C.desc).slot_stride
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    cpt_d = torch.from_numpy(cpt).cuda()
    plan, info = kvq.decode_plan(C.desc, w.seq_lens, cpt.shape[1])
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    qt = kdev.DeviceTable(w.q_table(0), "cuda")
    qp = kvq.q_rotate(kdev.gen_rows_device(w.q_key(0, 0), qt, 0, 1))
    out_bf = torch.empty((1, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(warmup):                        # every kernel of the timed loops runs here first
        rc.load(0, loads)
        kvq.paged_decode_attn_combined(C, 0, qp, cpt_d, plan_d, info, ws, out_bf, status=status)
    torch.cuda.synchronize()
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    ev[0].record(stream)
    for _ in range(steps):
        rc.load(0, loads)
    ev[1].record(stream)
    dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dst.copy_(H.buf[:nbytes], non_blocking=True)
    ev[2].record(stream)
    for _ in range(steps):
        dst.copy_(H.buf[:nbytes], non_blocking=True)
    ev[3].record(stream)
    # cold layer: page every page in, then decode over the cache
    ev[4].record(stream)
    for _ in range(steps):
        rc.load(0, loads)
        kvq.paged_decode_attn_combined(C, 0, qp, cpt_d, plan_d, info, ws, out_bf, status=status)
    ev[5].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    assert int(status.item()) == 0, f"kernel status {status.item()} in the resident decode"
    load_us = ev[0].elapsed_time(ev[1]) * 1e3 / steps
    copy_us = ev[2].elapsed_time(ev[3]) * 1e3 / steps
    cold_us = ev[4].elapsed_time(ev[5]) * 1e3 / steps
    rec = {"workload": w.name, "format": "q4_0", "context": T, "pages": len(loads), "page_bytes": nbytes // len(loads),
           "page_in_us": round(load_us, 1), "page_in_gbs": round(nbytes / load_us / 1e3, 2),
           "copy_engine_gbs": round(nbytes / copy_us / 1e3, 2),
           "page_in_vs_copy_engine": round(copy_us / load_us, 3),
           "cold_layer_us": round(cold_us, 1), "map_all_miss_us": round(map_miss_us, 1),
           "map_all_hit_us": round(map_hit_us, 1), "clocks": clocks}
    del H, C, rc, dst, ws
    torch.cuda.empty_cache()
    return rec


def measure_workload(name: str, layers: int, steps: int, warmup: int, peak: float, uuid: str):
    """One decode step per layer (paged_decode_step, the bench's timed kernel)
    of workload `name` restricted to its first `layers` layers, captured as a
    CUDA graph and timed with CUDA events over `steps` replays, with the SM
    clocks sampled meanwhile.  The pool of `layers` layers is larger than L2
    for every workload, so no flush is needed.  Returns a sub-record."""
    import torch
    import kvq_inputs
    import quantized_kv_cache_17_b200 as kvq
    from kvq_inputs import device as kdev
    w0 = kvq_inputs.workload(name)
    w = kvq_inputs.scaled(w0, w0.seq_lens, n_layers=min(layers, w0.n_layers), name=w0.name)
    L = w.n_layers
    dw = kdev.build_pool(w, extra_slots=0)
    q, k_new, v_new, pos = kdev.step_inputs(w, list(range(L)))
    plan, info = kvq.decode_plan(dw.pool.desc, w.seq_lens, dw.page_table.shape[1], 0)
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    out_bf = torch.empty((L, w.batch, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
    out_f = torch.empty((L, w.batch, w.n_q_heads, 256), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    layout = kvq.pool_layout(dw.pool.desc)
    kv_bytes_layer = sum(w.seq_lens) * w.n_kv_heads * layout.bytes_per_token_head

    def step():
        for l in range(L):
            kvq.paged_decode_step(dw.pool, l, q[l], k_new[l], v_new[l], dw.page_table, plan_d, info, ws, out_bf[l],
                                  out_f[l], status)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"kernel status {status.item()} on {name}"
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            step()
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    n_rep = max(steps, 2)
    for _ in range(n_rep):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    assert int(status.item()) == 0, f"kernel status {status.item()} on {name}"
    us_layer = a.elapsed_time(b) * 1e3 / (n_rep * L)
    gbs = kv_bytes_layer / (us_layer * 1e-6) / 1e9
    del g
    rec = {"workload": name, "format": w.fmt, "seq_lens": w.seq_lens, "layers_timed": L,
           "us_per_layer_step": round(us_layer, 3), "kv_bytes_per_layer": kv_bytes_layer,
           "gbs": round(gbs, 2), "frac": round(gbs / peak, 4), "n_units": info.n_units, "clocks": clocks}
    del dw, q, k_new, v_new, ws, out_bf, out_f
    torch.cuda.empty_cache()
    return rec


# ---------------------------------------------------------------------------
def run_ours(args):
    import torch
    import kvq_inputs
    import quantized_kv_cache_17_b200 as kvq
    from kvq_inputs import device as kdev

    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))

    kvq.lib()   # fails loudly if the library is missing
    w = kvq_inputs.workload(args.workload)
    if args.layers:
        w = kvq_inputs.scaled(w, w.seq_lens, n_layers=args.layers, name=w.name)
    L = w.n_layers
    fmt = w.fmt
    dw = kdev.build_pool(w, extra_slots=0)
    q, k_new, v_new, pos = kdev.step_inputs(w, list(range(L)))
    plan, info = kvq.decode_plan(dw.pool.desc, w.seq_lens, dw.page_table.shape[1], args.n_ctas)
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    q_rot = torch.empty_like(q)
    out_bf = torch.empty((L, w.batch, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
    out_f = torch.empty((L, w.batch, w.n_q_heads, 256), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rot_q, rot_v = kvq.rotated_q(fmt), kvq.rotated_v(fmt)
    use_alu = args.decode == "alu"
    fused = not use_alu and not args.no_fuse
    layout = kvq.pool_layout(dw.pool.desc)
    kv_bytes_layer = sum(w.seq_lens) * w.n_kv_heads * layout.bytes_per_token_head

    def layer_step(l):
        if fused:       # kv_append, q_rotate and the decode with its merge: one launch
            kvq.paged_decode_step(dw.pool, l, q[l], k_new[l], v_new[l], dw.page_table, plan_d, info, ws, out_bf[l],
                                  out_f[l], status)
            return
        qq = q[l]
        if rot_q:       # q_rotate and kv_append in one launch
            kvq.kv_append_q_rotate(dw.pool, l, k_new[l], v_new[l], pos, dw.page_table, qq, q_rot[l], status=status)
            qq = q_rot[l]
        else:
            kvq.kv_append(dw.pool, l, k_new[l], v_new[l], pos, dw.page_table, status=status)
        if fused:
            kvq.paged_decode_attn_combined(dw.pool, l, qq, dw.page_table, plan_d, info, ws, out_bf[l], out_f[l],
                                           status)
        else:
            kvq.paged_decode_attn(dw.pool, l, qq, dw.page_table, plan_d, info, ws, status, cudacore=use_alu)
            kvq.attn_combine(ws, plan_d, info, rot_v, out_bf[l], out_f[l])

    def step():
        for l in range(L):
            layer_step(l)

    def decode_only():
        for l in range(L):
            qq = q_rot[l] if rot_q else q[l]
            if fused:
                kvq.paged_decode_attn_combined(dw.pool, l, qq, dw.page_table, plan_d, info, ws, out_bf[l], out_f[l],
                                               status)
            else:
                kvq.paged_decode_attn(dw.pool, l, qq, dw.page_table, plan_d, info, ws, status, cudacore=use_alu)

    launches_per_layer = 1 if fused else 3      # paged_decode_step, or (kv_append[_q_rotate], decode, combine)

    def barrier():
        if dist is not None:
            dist.barrier()

    # eager warm-up (sets kernel attributes, fills caches of the runtime), then
    # capture one whole step and the decode launches alone as CUDA graphs
    if rot_q:
        kvq.q_rotate(q, q_rot)      # the decode-only graph takes the rotated query
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"kernel status {status.item()}"
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g_step, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g_step, stream=cap):
            step()
        with torch.cuda.graph(g_dec, stream=cap):
            decode_only()
    torch.cuda.current_stream().wait_stream(cap)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize()

    uuid = ""
    try:
        uuid = str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStart()      # an ncu launch list with --profile-from-start off sees only this region
    t_start.record(stream)
    for _ in range(args.steps):
        g_step.replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStop()
    barrier()
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)

    # the decode kernel alone: back-to-back launches of all layers, CUDA events on
    # the launching stream around the replays
    d_start, d_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g_dec.replay()
    torch.cuda.synchronize()
    d_start.record(stream)
    for _ in range(args.steps):
        g_dec.replay()
    d_end.record(stream)
    torch.cuda.synchronize()
    dec_avg_ms = d_start.elapsed_time(d_end) / (args.steps * L)

    # ---- end to end: host buffers, copies inside the timed region ---------------
    q_h = q.cpu().pin_memory()
    k_h = k_new.cpu().pin_memory()
    v_h = v_new.cpu().pin_memory()
    o_h = torch.empty(out_bf.shape, dtype=torch.bfloat16).pin_memory()
    h2d = q_h.numel() * 4 + k_h.numel() * 4 + v_h.numel() * 4
    d2h = o_h.numel() * 2
    # One graph per step: the first layers' inputs are copied in on the compute
    # stream, the others on a side stream that the compute stream waits for
    # only before layer HEAD; the outputs of all layers but the last are
    # copied out while the last layer runs.
    HEAD = min(2, L)
    side = torch.cuda.Stream()
    g_e2e = torch.cuda.CUDAGraph()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g_e2e, stream=cap):
            fork = torch.cuda.Event()
            fork.record(cap)
            side.wait_event(fork)
            with torch.cuda.stream(side):
                q[HEAD:].copy_(q_h[HEAD:], non_blocking=True)
                k_new[HEAD:].copy_(k_h[HEAD:], non_blocking=True)
                v_new[HEAD:].copy_(v_h[HEAD:], non_blocking=True)
                rest_in = torch.cuda.Event()
                rest_in.record(side)
            q[:HEAD].copy_(q_h[:HEAD], non_blocking=True)
            k_new[:HEAD].copy_(k_h[:HEAD], non_blocking=True)
            v_new[:HEAD].copy_(v_h[:HEAD], non_blocking=True)
            for l in range(L):
                if l == HEAD:
                    cap.wait_event(rest_in)
                layer_step(l)
                if l == L - 2:
                    before_last = torch.cuda.Event()
                    before_last.record(cap)
                    side.wait_event(before_last)
                    with torch.cuda.stream(side):
                        o_h[:L - 1].copy_(out_bf[:L - 1], non_blocking=True)
            o_h[L - 1:].copy_(out_bf[L - 1:], non_blocking=True)
            cap.wait_stream(side)
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(args.warmup):
        g_e2e.replay()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    for s in range(args.steps):
        g_e2e.replay()
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    assert torch.equal(o_h, out_bf.cpu()), "end-to-end output differs from the device result"
    e2e_ms = e_start.elapsed_time(e_end)
    assert int(status.item()) == 0, f"kernel status {status.item()}"
    del g_step, g_dec, g_e2e

    elapsed_ms, e2e_ms, dec_avg_ms = max_over_ranks(dist, [elapsed_ms, e2e_ms, dec_avg_ms], "cuda")

    ms_per_step = elapsed_ms / args.steps
    kv_bytes_step = kv_bytes_layer * L
    value = weak_scaling_gbs(world, kv_bytes_step, ms_per_step)
    e2e_value = weak_scaling_gbs(world, kv_bytes_step, e2e_ms / args.steps)
    tok_s = world * w.batch / (ms_per_step * 1e-3)
    peak, peak_kind = peaks()
    if fused:
        # the timed region runs the decode step kernel alone, once per layer:
        # its average launch is the region's time over its launches
        launch_ms = ms_per_step / L
        kernel_tag = "decode_step_fused"
    else:
        # several kernels per layer: the decode is timed on its own graph
        launch_ms = dec_avg_ms
        kernel_tag = "decode_alu" if use_alu else "decode_mma"
    achieved = kv_bytes_layer / (launch_ms * 1e-3) / 1e9
    traffic = ncu_traffic(kernel_tag, w.name)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        from tests import kvq_layout
        b = len(w.seq_lens) - 1
        cores = host_cores()
        n_groups = min(args.cpu_groups, L * w.n_kv_heads)
        groups = []
        for idx in range(n_groups):
            lay, g = L - 1 - idx // w.n_kv_heads, idx % w.n_kv_heads          # last layers first
            codes = kvq_layout.gather_sequence(fmt, dw.pool.buf, layout, lay, g, dw.page_table_host[b], w.seq_lens[b])
            groups.append((codes, oracle.q_prepare(fmt, q[lay, b, g * w.group:(g + 1) * w.group].cpu().numpy())))
        dt_all, tok_all, bytes_all = cpu_oracle_parallel(fmt, groups, cores)
        dt_one, tok_one, bytes_one = cpu_oracle_parallel(fmt, groups[:2], 1)
        kv_step_seq = w.seq_lens[b] * w.n_kv_heads * L * layout.bytes_per_token_head
        app_us = cpu_append_us(fmt, w.n_kv_heads, L, k_new[0, b].cpu().numpy(), v_new[0, b].cpu().numpy())
        cpu = {"value": round(bytes_all / dt_all / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "cpu_model": cpu_model(),
               "single_core_gbs": round(bytes_one / dt_one / 1e9, 4),
               "ms_per_step_all_cores": round(kv_step_seq / (bytes_all / dt_all) * 1e3, 1),
               "ms_per_step_single_core": round(kv_step_seq / (bytes_one / dt_one) * 1e3, 1),
               "append_us_per_step": round(app_us, 1),
               "sample": f"oracle fp64 attention of {n_groups} (layer, KV head) groups ({w.group} query heads each) "
                         f"over {w.seq_lens[b]} tokens of {w.name}, codes read back from the GPU pool, cut into "
                         f"token chunks on {cores} threads ({dt_all:.1f} s) and merged with the oracle's merge; "
                         f"single core: two groups ({dt_one:.1f} s); the ms per 16-layer step figures extrapolate "
                         f"these rates to all {L * w.n_kv_heads} groups of sequence {b}; append: the oracle's "
                         f"encode of one token per KV head and layer, single thread"}

    others = None
    prefill = None
    resident = None
    if rank == 0 and world == 1 and not args.no_others and args.workload == DEFAULT_WORKLOAD and not use_alu \
            and not args.layers:
        del dw, q, k_new, v_new, ws, out_bf, out_f, q_rot
        torch.cuda.empty_cache()
        others = [measure_workload(n, args.other_layers, args.steps, args.warmup, peak, uuid) for n in OTHER_WORKLOADS]
        prefill = measure_prefill(32768, 512, max(2, args.steps // 4), args.warmup, uuid)
        resident = measure_resident(131072, max(2, args.steps // 4), args.warmup, uuid)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32 (codes u4/i8, fp16 scales, fp16 tensor-core "
                "operands with hi/lo split)" if not use_alu else "f32",
                "data": "synthetic (seeded counter-based generator; shapes and value distributions of the pages' "
                        "workloads)",
                "config": {"workload": w.name, "format": fmt, "seq_lens": w.seq_lens, "layers": L,
                           "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": 256, "page_tokens": 256,
                           "decode_kernel": kernel_tag, "n_units": info.n_units, "chunk_tokens": info.chunk_tokens,
                           "kv_bytes_per_step": kv_bytes_step,
                           "l2": "no flush: the 16-layer KV pool read per step is larger than L2",
                           "parallelism": f"replicas x{world}"},
                "attn_stack_tok_s": round(tok_s, 2),
                "us_per_layer_step": round(ms_per_step * 1e3 / L, 3),
                "us_decode_per_layer": round(dec_avg_ms * 1e3, 3),
                "pct_of_8tbs_spec": round(100 * value / world / 8000.0, 2),
                "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                             "frac": round(achieved / peak, 4), "traffic": traffic,
                             "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                             if peak_kind == "measured" else "fallback 6.65 TB/s",
                             "bytes_per_launch": kv_bytes_layer,
                             "us_per_launch": round(launch_ms * 1e3, 3),
                             "kernel": kernel_tag},
                "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / args.steps, 4)},
                "gpu_launches": args.steps * L * launches_per_layer,
                "launch": "CUDA graph of the 16-layer step",
                "clocks": clocks,
                "cpu_baseline": cpu,
                "other_workloads": others,
                "prefill": prefill,
                "resident": resident}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--decode", default="mma", choices=["mma", "alu"])
    ap.add_argument("--n-ctas", type=int, default=0)
    ap.add_argument("--no-fuse", action="store_true", help="separate attn_combine launch")
    ap.add_argument("--layers", type=int, default=0, help="use only this many layers (profiling captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-groups", type=int, default=16, help="(layer, KV head) groups in the CPU baseline")
    ap.add_argument("--no-others", action="store_true", help="skip the sub-records of the other workloads")
    ap.add_argument("--other-layers", type=int, default=4, help="layers timed per other workload")
    ap.add_argument("--only", choices=["prefill", "resident"],
                    help="run one sub-record alone (profiling captures) and print it")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        return run_sub_record(args)
    return run_ours(args)


def run_sub_record(args):
    """One sub-record of the default run, alone, on GPU 0."""
    import torch
    import quantized_kv_cache_17_b200 as kvq
    kvq.lib()
    uuid = ""
    try:
        uuid = str(torch.cuda.get_device_properties(0).uuid)
    except Exception:
        pass
    if args.only == "prefill":
        rec = measure_prefill(32768, 512, args.steps, args.warmup, uuid)
    else:
        rec = measure_resident(131072, args.steps, args.warmup, uuid)
    print(json.dumps({args.only: rec}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

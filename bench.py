"""HiKVP knowledge-graph attention benchmark (one JSON line on rank 0).

A step = one atlaskv_attend call over one batch of B queries: the whole hot
path (query sums, three levels of scoring + top-K, host-leaf staging when the
leaves live in host memory, knowledge + causal-sequence attention, merge).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

Default workload: the 100x100x100 tree (M = 1e6 keys per KV head, H = 32,
H_kv = 8, D = 128, B = 64 queries of N = 64 tokens, T = 1024, K = 16/16/64),
fully HBM resident.  Inputs are larger than the 126 MB L2 and L2 is also
flushed (256 MB write) before every timed step.  Under torchrun every rank runs
an independent replica on its own GPU (weak scaling, no data-path collective).

Per workload: the headline steps are timed clean (no library instrumentation);
a second pass of as many steps records the library's per-stage CUDA events
(each kernel timed on its own stream), from which the per-kernel rooflines
come; one more call reads the descent's refinement counters.  On one GPU the
line also carries `per_config`, the same measurement for the other four
benchmark shapes (the tiny one replayed as a CUDA graph).  --only skips it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HiKVP KG-attention queries/s (M=1e6..1.25e8); achieved HBM & host-link GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fanout", default=None, help="override the tree fan-outs, e.g. 100,100,100 (smaller cases)")
    ap.add_argument("--batch", type=int, default=None, help="override the number of queries B")
    ap.add_argument("--only", action="store_true", help="time the --config workload only (no per_config block)")
    ap.add_argument("--descent", default="auto", choices=["auto", "fused", "parent_major"],
                    help="how the descent runs (the results are the same)")
    ap.add_argument("--leaf-cache", type=int, default=0,
                    help="host-resident leaves: an HBM cache of this many staged leaf blocks across steps "
                         "(every step repeats the same batch, so this measures the all-hit case)")
    return ap.parse_args()


def workload_shape(args):
    import dataclasses
    from hierarchical_kv_pruning_b200 import synth
    sh = synth.shape(args.config)
    if args.fanout:
        fo = tuple(int(x) for x in args.fanout.split(","))
        sh = dataclasses.replace(sh, fanout=fo, name="%s@%s" % (sh.name, "x".join(map(str, fo))))
    if args.batch:
        sh = dataclasses.replace(sh, batch=args.batch, name="%s@B%d" % (sh.name, args.batch))
    return sh


def config_of(sh, world):
    """The workload description both arms print."""
    return {"workload": sh.name, "M": sh.n_leaves, "fanout": list(sh.fanout), "K": list(sh.keep),
            "B": sh.batch, "N": sh.n_tokens, "T": sh.seq_len, "H": sh.n_heads, "H_kv": sh.n_kv_heads,
            "D": sh.head_dim, "leaves": "pinned host" if sh.leaf_on_host else "HBM",
            "l2": "inputs larger than L2 and 256 MB flush before each timed step",
            "parallelism": "replicas x%d" % world}


def splits_attention(sh):
    """bf16, D = 128 with host-resident leaves: the sequence part is its own
    launch beside the descent and the staging, and the knowledge part merges
    with it (tensor-core attention)."""
    import torch
    return sh.dtype == torch.bfloat16 and sh.head_dim == 128 and sh.leaf_on_host


def uses_parent_major(sh, descent="auto"):
    """The descent the library runs (ATLASKV_DESCENT_AUTO: parent-major from
    B * H >= 1024 traversals)."""
    if descent != "auto":
        return descent == "parent_major"
    return sh.batch * sh.n_heads >= 1024


def kernels_per_step(sh, descent="auto", leaf_cache=False):
    """Kernels one atlaskv_attend call launches.  The fused descent is one
    launch; the parent-major one is the token sums, then per level a scoring,
    a selection and a refinement launch, and per level below the roots a scan
    and a fill.  Leaves in HBM: the descent, then the attention (one launch).
    Host-resident leaves: per query chunk (four chunks when B >= 8, else one)
    the descent up to the level above the leaves, a de-duplication and a
    staging copy of the leaf-key blocks (and, with the mids on the host, of the
    mid blocks before level 1), the leaf level, a de-duplication and a staging
    copy of the value rows, and the knowledge part; plus one sequence-part
    launch for the whole batch (bf16, D = 128).  A leaf-block cache adds its
    map and commit launches per chunk."""
    pm = uses_parent_major(sh, descent)

    def levels(first, last):
        if not pm:
            return 1
        n = 0
        for lvl in range(first, last + 1):
            n += 3 + (1 if lvl == 0 else 2)
        return n

    if not sh.leaf_on_host:
        return levels(0, 2) + 1
    chunks = 4 if sh.batch >= 8 else 1
    if sh.mid_on_host:
        per = levels(0, 0) + 2 + levels(1, 1) + 2 + levels(2, 2) + 2 + 1
    else:
        per = levels(0, 1) + 2 + levels(2, 2) + 2 + 1
    if leaf_cache:
        per += 2
    return chunks * per + (1 if splits_attention(sh) else 0)


def max_over_ranks(x, world, device):
    """The largest value of x over all ranks (x itself on one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, batch, total_ms, steps):
    """Queries per second of all ranks together: every rank processes `batch`
    queries per step and the slowest rank's time counts."""
    return world * batch / (total_ms / steps * 1e-3)


def attend_kernel_name(sh):
    import torch
    if sh.dtype == torch.float32:
        return "attend_f32_kernel"
    return "attend_tc_kernel"


# Source files of each profiled stage (the descent is a chain of kernels).
KERNEL_SOURCES = {"attend_tc_kernel": ["attend_tc.cuh"], "attend_f32_kernel": ["attend.cuh"], "descent": ["descend.cuh", "descend_pm.cuh"],
                  "stage_blocks_kernel": ["staging.cuh"]}


def sources_digest(kernel):
    """sha256 over the stage's source files, concatenated in order."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "hierarchical_kv_pruning_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch (read + write; for the descent, per call: the sum
    over its kernels) from the committed ncu summary of this stage on this
    workload, if its sources still hash to the ones profiled; otherwise None."""
    summ = os.path.join(ROOT, "profiles", "%s__%s.md" % (kernel, workload))
    if not (os.path.exists(summ) and kernel in KERNEL_SOURCES):
        return None
    fields = {}
    with open(summ) as f:
        for line in f:
            if line.startswith("- ") and ": " in line:
                k, v = line[2:].split(": ", 1)
                fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_sha256") != sources_digest(kernel) or "dram_bytes_per_launch" not in fields:
        return None
    return int(fields["dram_bytes_per_launch"])


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons polled through NVML every
    millisecond while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def _reasons(self):
        nv = self._nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(fn(self._h))

    def sample(self):
        """One reading now (also called by the timing loop after every step:
        the polling thread can be starved of the interpreter lock)."""
        if self._thread is None:
            return
        try:
            self.samples.append((float(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)),
                                 self._reasons()))
        except Exception:
            pass

    def _poll(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.001)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = sorted(n for n, bit in self.REASONS.items() if mask & bit)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "source": "NVML: 1 ms polling thread during the timed steps plus one reading "
                "as each step completes"}


# ---------------------------------------------------------------------------
# Algorithmic bytes (the minimum each kernel must move; unique rows counted
# over the batch from the kept sets, dense tensors once).

def algorithmic_bytes(sh, res, w):
    import torch
    e = 4 if sh.dtype == torch.float32 else 2
    B, N, H, D, T, Hkv = sh.batch, sh.n_tokens, sh.n_heads, sh.head_dim, sh.seq_len, sh.n_kv_heads
    bR, bI, bL = sh.fanout
    K_R, K_I, K_L = sh.keep
    G = sh.group
    hkv = (torch.arange(H, device=res["kept_root"].device) // G)

    def unique_rows(kept, rows_per_head):
        key = hkv[None, :, None].long() * rows_per_head + kept.long()
        return int(torch.unique(key).numel())

    u_root = unique_rows(res["kept_root"], bR)
    u_mid = unique_rows(res["kept_mid"], bR * bI)
    u_leaf = unique_rows(res["kept_leaf"], sh.n_leaves)
    mid_cand_rows = u_root * bI          # children of every kept root, once per batch
    leaf_cand_rows = u_mid * bL          # children of every kept mid
    table = 4 * (mid_cand_rows + leaf_cand_rows) if w.root_child is not None else 0
    descend = (e * B * N * H * D + e * D * (Hkv * bR + mid_cand_rows + leaf_cand_rows) + table
               + 4 * B * H * (K_R + K_I + K_L))
    # the attention's bytes, split by part: the sequence part reads q_seq and
    # the sequence K/V; the knowledge part reads q_kg, the kept ids and the
    # kept leaves' K/V rows and writes out and the LSE
    attend_seq = e * (B * N * H * D + 2 * B * T * Hkv * D)
    attend_leaf = e * 2 * B * N * H * D + 4 * B * N * H + 4 * B * H * K_L + 2 * e * D * u_leaf
    vis = sum(T - N + n + 1 for n in range(N))
    attend_flops = 4 * B * H * D * (vis + N * K_L)
    staging = e * D * (leaf_cand_rows + u_leaf) if sh.leaf_on_host else 0
    return {"descend": descend, "attend": attend_seq + attend_leaf, "attend_seq": attend_seq,
            "attend_leaf": attend_leaf, "attend_flops": attend_flops, "staging": staging,
            "u_root": u_root, "u_mid": u_mid, "u_leaf": u_leaf}


def oracle_cpu_baseline(w, sh, target_s):
    """Time the oracle (as it stands) on a bounded sample of whole queries."""
    import numpy as np
    import torch
    import oracle

    def storage(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    tree = oracle.Tree(storage(w.root_keys), storage(w.mid_keys), storage(w.leaf_keys), storage(w.leaf_values),
                       sh.fanout, None if w.root_child is None else w.root_child.cpu().numpy(),
                       None if w.mid_child is None else w.mid_child.cpu().numpy())
    q_kg, q_seq, k_seq, v_seq = (storage(w.q_kg), storage(w.q_seq), storage(w.k_seq), storage(w.v_seq))
    done, spent = 0, 0.0
    while done < sh.batch and spent < target_s:
        trav = [(done, h) for h in range(sh.n_heads)]
        t0 = time.perf_counter()
        oracle.hikvp(tree, q_kg, q_seq, k_seq, v_seq, sh.keep, trav)
        spent += time.perf_counter() - t0
        done += 1
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": done / spent, "unit": "queries/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d queries (all %d heads each) of %s, %.1f s" % (done, sh.batch, sh.n_heads, sh.name,
                                                                              spent)}


def pinned_h2d_gbs(torch):
    src = torch.empty(1 << 30, dtype=torch.uint8).pin_memory()
    dst = torch.empty(1 << 30, dtype=torch.uint8, device="cuda")
    best = 0.0
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        b.synchronize()
        best = max(best, (1 << 30) / (a.elapsed_time(b) * 1e-3) / 1e9)
    del src, dst
    return best


def host_memory_ok(sh):
    """Enough free host memory to pin a host-leaf shape's leaf keys and values."""
    if not sh.leaf_on_host:
        return True
    free_host = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_AVPHYS_PAGES")
    return free_host >= 2 * sh.n_leaves * sh.n_kv_heads * sh.head_dim * 2 + (8 << 30)


def roofline_of(sh, alg, st, ms_per_step, peaks, peak_src, link_gbs, descent="auto"):
    """Rooflines from the algorithmic bytes and the per-launch stage times
    (CUDA events on each kernel's own stream, averaged over the stage pass).
    Leaves in HBM: the headline is the whole step against HBM (descent and
    attention bytes over the step time), `dominant` the stage with the largest
    time.  Host-resident leaves: the headline is the staging against the host
    link (the streams overlap).  `kernels` lists each stage; `step` is the
    whole step against HBM (and, with host leaves, the staged bytes against
    the host link)."""
    import torch
    hbm = peaks["hbm_gbs"]
    kernels = {}

    def entry(name, nbytes, ms, kernel):
        if not ms or ms <= 0:
            return
        ach = nbytes / (ms * 1e-3) / 1e9
        kernels[name] = {"kernel": kernel, "ms": round(ms, 5), "algorithmic_bytes": nbytes, "achieved": ach,
                         "unit": "GB/s", "frac": ach / hbm, "bound": "hbm"}

    entry("descend", alg["descend"], st["descend"],
          "descent (parent-major chain: token sums; per level score, select, refine; scan and fill)"
          if uses_parent_major(sh, descent) else "descent (descend_kernel)")
    if splits_attention(sh):
        entry("attend_seq", alg["attend_seq"], st["attend_seq"], "attend_tc_kernel (sequence part)")
        entry("attend_leaf", alg["attend_leaf"], st["attend_leaf"], "attend_tc_kernel (knowledge part + merge)")
    else:
        entry("attend", alg["attend"], st["attend"], attend_kernel_name(sh))
    if sh.leaf_on_host:
        ach = alg["staging"] / (st["staging"] * 1e-3) / 1e9 if st["staging"] > 0 else 0.0
        kernels["staging"] = {"kernel": "stage_blocks_kernel + stage_value_rows_kernel",
                              "ms": round(st["staging"], 5), "algorithmic_bytes": alg["staging"], "achieved": ach,
                              "unit": "GB/s", "frac": ach / link_gbs, "bound": "host_link",
                              "peak": link_gbs, "peak_source": "pinned cudaMemcpyAsync H2D measured in this run"}
    step_bytes = alg["descend"] + alg["attend"]
    step = {"algorithmic_bytes": step_bytes, "ms": ms_per_step,
            "achieved": step_bytes / (ms_per_step * 1e-3) / 1e9, "unit": "GB/s", "peak": hbm}
    step["frac"] = step["achieved"] / hbm
    if sh.leaf_on_host:
        # the two streams overlap: the step is bound by the host link
        link_ach = alg["staging"] / (ms_per_step * 1e-3) / 1e9
        step["host_link"] = {"algorithmic_bytes": alg["staging"], "achieved": link_ach, "peak": link_gbs,
                             "frac": link_ach / link_gbs}
        top = dict(kernels["staging"])
        top["bound"] = "host_link"
        top["traffic"] = None   # host-link bytes are not DRAM counters
    else:
        # the headline is the whole step against HBM (its stages run one after
        # the other); the stage with the largest time is kept as `dominant`
        name = max(kernels, key=lambda k: kernels[k]["ms"])
        dom = dict(kernels[name])
        dom["peak"] = hbm
        dom["traffic"] = profiled_traffic(dom["kernel"].split(" ")[0], sh.name)
        parts = [profiled_traffic(kernels[k]["kernel"].split(" ")[0], sh.name) for k in kernels]
        top = {"kernel": "whole step (descent + attention)", "bound": "hbm", "achieved": step["achieved"],
               "peak": hbm, "unit": "GB/s", "frac": step["frac"], "algorithmic_bytes": step_bytes,
               "ms": ms_per_step, "traffic": sum(parts) if parts and None not in parts else None,
               "dominant": dom}
        top["peak_source"] = peak_src + " (burst)"
    attend_ms = st["attend"]
    tflops = alg["attend_flops"] / (attend_ms * 1e-3) / 1e12 if attend_ms > 0 else None
    top.update({"kernels": kernels, "step": step, "stage_ms": {k: round(v, 5) for k, v in st.items()},
                "attend_flops": alg["attend_flops"], "attend_tflops": tflops,
                "attend_tensor_frac": (tflops / peaks["bf16_tflops"]
                                       if tflops and sh.dtype == torch.bfloat16 and sh.head_dim == 128 else None)})
    return top


def measure(sh, seed, args, world, rank, local, cpu_seconds, use_graph=False):
    """Benchmark one workload: returns the fields of its JSON entry."""
    import torch

    from hierarchical_kv_pruning_b200 import synth
    from hierarchical_kv_pruning_b200.binding import STAGE_NAMES, HikvpTree

    dev = torch.device("cuda", local)
    w = synth.make_workload(sh, "cuda", seed)
    stream = torch.cuda.current_stream()
    tree = HikvpTree.from_workload(w)
    tree.set_descent({"auto": 0, "fused": 1, "parent_major": 2}[args.descent])
    if args.leaf_cache and sh.leaf_on_host:
        tree.set_leaf_cache(args.leaf_cache)
    K = sh.keep
    out = torch.empty_like(w.q_kg)
    lse = torch.empty((sh.batch, sh.n_tokens, sh.n_heads), dtype=torch.float32, device=dev)
    kept = tuple(torch.empty((sh.batch, sh.n_heads, k), dtype=torch.int32, device=dev) for k in K)
    nbytes = tree.workspace_size(K, sh.batch, sh.n_tokens, sh.n_heads, sh.seq_len)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    flush = synth.flush_buffer(dev)

    def step():
        return tree.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, K, out=out, lse=lse, kept=kept, workspace=ws)

    for _ in range(args.warmup):
        step()
    tree.sync_status()
    run = step
    graph = None
    if use_graph:
        # a launch-latency-bound step: capture it once and replay the graph
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            step()
        stream.wait_stream(cap)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap, capture_error_mode="thread_local"):
            step()
        torch.cuda.synchronize()
        run = graph.replay
        for _ in range(args.warmup):
            run()

    def timed(fn, n, label_flush):
        ms = []
        for _ in range(n):
            flush.fill_(label_flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ms.append(a.elapsed_time(b))
        return ms

    # ---- timed region: clean steps (no library instrumentation), L2 flushed before each ----
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms = []
        for _ in range(args.steps):
            step_ms.extend(timed(run, 1, 1.0))
            clk.sample()
        torch.cuda.synchronize()
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(world, sh.batch, total_ms, args.steps)
    tree.sync_status()

    # ---- stage pass: the same steps with the library's stage events on ----
    tree.set_profiling(times=True, counters=False)
    stage = [0.0] * len(STAGE_NAMES)
    n_stage = max(3, args.steps)
    for _ in range(n_stage):
        flush.fill_(3.0)
        step()
        for i, v in enumerate(tree.stage_times()):
            stage[i] += v
    # ---- one call with the descent counters ----
    tree.set_profiling(times=False, counters=True)
    step()
    refine = tree.refine_stats()
    tree.set_profiling(times=False, counters=False)
    tree.sync_status()
    st = {n: v / n_stage for n, v in zip(STAGE_NAMES, stage)}

    # ---- end to end: pinned host inputs in, result out, through the public API ----
    host = {k: getattr(w, k).cpu().pin_memory() for k in ("q_kg", "q_seq", "k_seq", "v_seq")}
    dbuf = {k: torch.empty_like(getattr(w, k)) for k in host}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size() + lse_host.numel() * 4

    def e2e_step():
        for k in host:
            dbuf[k].copy_(host[k], non_blocking=True)
        tree.attend(dbuf["q_kg"], dbuf["q_seq"], dbuf["k_seq"], dbuf["v_seq"], K, out=out, lse=lse, kept=kept,
                    workspace=ws)
        out_host.copy_(out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ms = timed(e2e_step, max(3, args.steps // 2), 2.0)
    e2e_total = max_over_ranks(sum(e2e_ms), world, dev)
    e2e_value = whole_job_rate(world, sh.batch, e2e_total, len(e2e_ms))

    res = {"kept_root": kept[0], "kept_mid": kept[1], "kept_leaf": kept[2]}
    alg = algorithmic_bytes(sh, res, w)
    peaks, peak_src = measured_peaks()
    link = pinned_h2d_gbs(torch) if sh.leaf_on_host else None
    roof = roofline_of(sh, alg, st, ms_per_step, peaks, peak_src, link, args.descent)
    roof["exact_refinement"] = refine
    entry = {"value": value, "unit": "queries/s", "ms_per_step": ms_per_step,
             "us_per_query": 1e3 * ms_per_step / sh.batch,
             "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
             "gpu_launches": kernels_per_step(sh, args.descent, bool(args.leaf_cache) and sh.leaf_on_host) * args.steps, "roofline": roof, "clocks": clk.summary(),
             "config": config_of(sh, world), "cuda_graph": use_graph,
             "dtype": "f32" if sh.dtype == torch.float32 else "bf16"}
    if args.leaf_cache and sh.leaf_on_host:
        entry["leaf_cache"] = dict(tree.leaf_cache_stats(), blocks=args.leaf_cache,
                                   note="cumulative over warm-up, timed and profiling steps; every step "
                                        "repeats the same batch, so blocks hit after the first; the staging "
                                        "roofline still counts every staged block as host-link bytes")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        entry["cpu_baseline"] = oracle_cpu_baseline(w, sh, cpu_seconds)
    if graph is not None:
        del graph
    tree.close()
    del w, out, lse, kept, ws, flush, host, dbuf, out_host, lse_host
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


def run_ours(args):
    import torch
    import torch.distributed as dist

    from hierarchical_kv_pruning_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    sh = workload_shape(args)
    head = measure(sh, 1000 + args.config + 100 * rank, args, world, rank, local, args.cpu_seconds,
                   use_graph=(args.config == 0))
    line = {
        "metric": METRIC, "value": head["value"], "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": head["dtype"],
        "data": "synthetic (seeded hierarchical-Gaussian tree and queries)",
        "config": head["config"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
        "roofline": head["roofline"], "clocks": head["clocks"],
    }
    if "cpu_baseline" in head:
        line["cpu_baseline"] = head["cpu_baseline"]
    if "leaf_cache" in head:
        line["leaf_cache"] = head["leaf_cache"]
    # every other benchmark shape, one GPU only (the host-leaf shape needs
    # about 130 GB of pinned host memory per process)
    if world == 1 and not args.only and not (args.fanout or args.batch):
        per = {}
        for c in (0, 1, 2, 3, 4):
            if c == args.config:
                continue
            csh = synth.shape(c)
            if not host_memory_ok(csh):
                per[csh.name] = {"skipped": "not enough free host memory to pin the leaves"}
                continue
            per[csh.name] = measure(csh, 1000 + c, args, 1, rank, local, args.cpu_seconds / 2, use_graph=(c == 0))
        line["per_config"] = per
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args):
    """The oracle (test infrastructure, as it stands) on the host cores: each
    step is a bounded sample of whole queries of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    from hierarchical_kv_pruning_b200 import synth
    sh = workload_shape(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = synth.make_workload(sh, dev, 1000 + args.config)
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_cpu_baseline(w, sh, per_step)
    vals = []
    samples = []
    for _ in range(args.steps):
        r = oracle_cpu_baseline(w, sh, per_step)
        vals.append(r["value"])
        samples.append(r["sample"])
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * sh.batch / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded hierarchical-Gaussian tree and queries)",
        "config": config_of(sh, 1),
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "cpu_baseline": {"value": value, "unit": "queries/s", "kind": "oracle",
                         "cores": int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)),
                         "sample": samples[-1]},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

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


def kernels_per_step(sh):
    """Kernels one atlaskv_attend call launches: per level (root or children
    scoring, selection, exact pass) x 3 and the attention.  With host-resident
    leaves add two de-duplications and two staging copies, and the call runs
    all of them once per query chunk (four chunks when B >= 8, else one)."""
    if not sh.leaf_on_host:
        return 3 * 3 + 1
    return (3 * 3 + 1 + 4) * (4 if sh.batch >= 8 else 1)


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
    return "attend_tc_kernel" if sh.head_dim == 128 else "attend_bf16_kernel"


KERNEL_SOURCES = {"attend_tc_kernel": "attend_tc.cuh", "attend_bf16_kernel": "attend.cuh",
                  "attend_f32_kernel": "attend.cuh"}


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch (read + write) from the committed ncu summary of
    this kernel on this workload, if the kernel source still hashes to the one
    profiled; otherwise None."""
    import hashlib
    summ = os.path.join(ROOT, "profiles", "%s__%s.md" % (kernel, workload))
    src = os.path.join(ROOT, "hierarchical_kv_pruning_b200", "csrc", KERNEL_SOURCES.get(kernel, ""))
    if not (os.path.exists(summ) and os.path.isfile(src)):
        return None
    fields = {}
    with open(summ) as f:
        for line in f:
            if line.startswith("- ") and ": " in line:
                k, v = line[2:].split(": ", 1)
                fields[k.strip()] = v.strip().strip("`")
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    if fields.get("source_sha256") != digest or "dram_bytes_per_launch" not in fields:
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
    attend = (e * (3 * B * N * H * D + 2 * B * T * Hkv * D) + 4 * B * N * H + 4 * B * H * K_L
              + 2 * e * D * u_leaf)
    vis = sum(T - N + n + 1 for n in range(N))
    attend_flops = 4 * B * H * D * (vis + N * K_L)
    staging = e * D * (leaf_cand_rows + u_leaf) if sh.leaf_on_host else 0
    return {"descend": descend, "attend": attend, "attend_flops": attend_flops, "staging": staging,
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


def run_ours(args):
    import torch
    import torch.distributed as dist

    from hierarchical_kv_pruning_b200 import synth
    from hierarchical_kv_pruning_b200.binding import HikvpTree

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    sh = workload_shape(args)
    w = synth.make_workload(sh, "cuda", 1000 + args.config + 100 * rank)
    stream = torch.cuda.current_stream()
    tree = HikvpTree.from_workload(w)
    K = sh.keep
    dev = torch.device("cuda", local)
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

    # ---- timed region: per-step CUDA events, L2 flushed before each step ----
    tree.set_profiling(True)
    stage = [0.0, 0.0, 0.0]
    step_ms = []
    launches = 0
    n_launch = kernels_per_step(sh)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step()
            b.record(stream)
            b.synchronize()
            clk.sample()
            step_ms.append(a.elapsed_time(b))
            st = tree.stage_times()
            for i in range(3):
                stage[i] += st[i]
            launches += n_launch
        refine = tree.refine_stats()
        torch.cuda.synchronize()
    tree.set_profiling(False)
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(world, sh.batch, total_ms, args.steps)
    tree.sync_status()

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
    e2e_ms = []
    for _ in range(max(3, args.steps // 2)):
        flush.fill_(2.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        b.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_total = max_over_ranks(sum(e2e_ms), world, dev)
    e2e_value = whole_job_rate(world, sh.batch, e2e_total, len(e2e_ms))

    # ---- roofline of the dominant kernel ----
    res = {"kept_root": kept[0], "kept_mid": kept[1], "kept_leaf": kept[2]}
    alg = algorithmic_bytes(sh, res, w)
    peaks, peak_src = measured_peaks()
    st_ms = [s / args.steps for s in stage]
    names = ["descend", "staging", "attend"]
    # The dominant kernel: with leaves in HBM, the attention kernel is the
    # largest single kernel of a step (the descent stage is nine shorter
    # launches); with host-resident leaves the stages overlap on two streams
    # and the path is bound by the host link.
    if sh.leaf_on_host:
        link = pinned_h2d_gbs(torch)
        achieved = alg["staging"] / (st_ms[1] * 1e-3) / 1e9
        roof = {"bound": "host_link", "achieved": achieved, "peak": link, "unit": "GB/s", "frac": achieved / link,
                "traffic": None, "kernel": "stage_leaf_blocks_kernel + stage_value_rows_kernel",
                "peak_source": "pinned cudaMemcpyAsync H2D measured in this run"}
    else:
        kname = attend_kernel_name(sh)
        t_hbm = alg["attend"] / (peaks["hbm_gbs"] * 1e9)
        t_tc = alg["attend_flops"] / (peaks["bf16_tflops"] * 1e12)
        if sh.dtype == torch.bfloat16 and t_tc > t_hbm:
            achieved = alg["attend_flops"] / (st_ms[2] * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops"]}
        else:
            achieved = alg["attend"] / (st_ms[2] * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"]}
        roof.update({"traffic": profiled_traffic(kname, sh.name), "kernel": kname,
                     "peak_source": peak_src + " (burst)"})
    desc_gbs = alg["descend"] / (st_ms[0] * 1e-3) / 1e9 if st_ms[0] > 0 else None
    roof["descent"] = {"ms": round(st_ms[0], 4), "algorithmic_bytes": alg["descend"], "achieved": desc_gbs,
                       "unit": "GB/s", "frac_of_hbm": desc_gbs / peaks["hbm_gbs"] if desc_gbs else None,
                       "kernels": "root_kernel, score_kernel x2, select_kernel x3, exact_kernel x3"}
    roof["stage_ms"] = {n: round(v, 4) for n, v in zip(names, st_ms)}
    roof["algorithmic_bytes"] = {k: alg[k] for k in ("descend", "attend", "staging")}
    roof["attend_flops"] = alg["attend_flops"]
    roof["attend_tflops"] = alg["attend_flops"] / (st_ms[2] * 1e-3) / 1e12 if st_ms[2] > 0 else None
    # the attention's tensor-pipe share: achieved dense bf16 rate / measured burst peak
    roof["attend_tensor_frac"] = (roof["attend_tflops"] / peaks["bf16_tflops"]
                                  if roof["attend_tflops"] and sh.dtype == torch.bfloat16 else None)
    roof["exact_refinement_last_step"] = refine

    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if sh.dtype == torch.float32 else "bf16",
        "data": "synthetic (seeded hierarchical-Gaussian tree and queries)",
        "config": config_of(sh, world),
        "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "roofline": roof,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_cpu_baseline(w, sh, args.cpu_seconds)
    tree.close()
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
        "warmup": args.warmup, "ms_per_step": 1e3 / value, "higher_is_better": True, "scaling": "weak",
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

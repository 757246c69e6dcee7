"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Under torchrun every rank runs an independent replica; the only collectives
are the barrier and the max-over-ranks reduction of the timed totals, from
which the whole-job rate is formed.  These run here with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, totals, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        m = bench.max_over_ranks(totals[rank], world, "cpu")
        rate = bench.whole_job_rate(world, 64, m, 20)
        out.put((rank, m, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world = 2
    totals = [12.5, 17.25]          # ms over 20 steps on each rank
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, totals, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate in res:
        assert m == max(totals)                               # every rank sees the slowest rank's time
        assert rate == pytest.approx(world * 64 / (max(totals) / 20 * 1e-3))


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(1, 64, 10.0, 10) == pytest.approx(64 / 1e-3)


def test_kernels_per_step_and_config():
    import dataclasses

    from hierarchical_kv_pruning_b200 import synth
    dev = synth.shape(2)
    host = synth.shape(4)
    # leaves in HBM, B H >= 512: parent-major descent (token sums; 3 levels of
    # score, select, refine; scan and fill below the roots) and one attention
    assert bench.uses_parent_major(dev) and bench.kernels_per_step(dev) == 1 + 3 * 3 + 2 * 2 + 1
    assert bench.kernels_per_step(dev, "fused") == 2
    # host leaves: per query chunk (four) levels 0-1, leaf-block staging (2),
    # level 2, value staging (2), knowledge part; plus one sequence part
    per = (1 + 3 + 3 + 2) + 2 + (3 + 2) + 2 + 1
    assert host.batch >= 8 and bench.kernels_per_step(host) == 4 * per + 1
    assert bench.kernels_per_step(dataclasses.replace(host, batch=7), "fused") == 7 + 1
    mids = dataclasses.replace(host, mid_on_host=True)
    assert bench.kernels_per_step(mids, "fused") == 4 * 10 + 1
    # fp32, one query, and 16 queries of 32 heads: the fused descent and one attention launch
    assert not bench.uses_parent_major(synth.shape(0)) and bench.kernels_per_step(synth.shape(0)) == 2
    assert not bench.uses_parent_major(synth.shape(1)) and bench.kernels_per_step(synth.shape(1)) == 2
    c = bench.config_of(dev, 4)
    assert c["workload"] == dev.name and c["parallelism"] == "replicas x4"
    assert c["B"] == dev.batch and c["K"] == list(dev.keep)


def test_algorithmic_bytes_worked_example():
    # B = 1, N = 2, H = 2 heads on H_kv = 1, D = 4, bf16 (2 bytes), fan-outs
    # (3, 2, 2), K = (2, 2, 2), T = 3.  Kept sets of the two heads overlap, so
    # the unique rows of the batch are roots {0,1,2}, mids {0,1,3}, leaves
    # {0,5,7}: 3 each.  By hand:
    #   descent: q_kg 2*1*2*2*4 = 32; key rows read (roots 1*3, mid candidates
    #            3*2, leaf candidates 3*2) * 4 * 2 = 120; kept ids
    #            4*1*2*(2+2+2) = 48; total 200 (plus 4 B per child-table
    #            entry read, 4*(6+6) = 48, when the tree has tables)
    #   attention: q_kg, q_seq, out 3*1*2*2*4*2 = 96; k_seq, v_seq
    #            2*1*3*1*4*2 = 48; lse 4*1*2*2 = 16; leaf ids 4*1*2*2 = 16;
    #            leaf K and V rows 2*2*4*3 = 48; total 224
    #   flops: 4 * B*H*D * (visible sequence keys 2 + 3, plus N*K_L = 4) = 288
    import dataclasses
    import types

    import torch

    from hierarchical_kv_pruning_b200 import synth
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=4, fanout=(3, 2, 2),
                      keep=(2, 2, 2), batch=1, n_tokens=2, seq_len=3)
    res = {"kept_root": torch.tensor([[[0, 1], [1, 2]]]),
           "kept_mid": torch.tensor([[[0, 1], [1, 3]]]),
           "kept_leaf": torch.tensor([[[0, 5], [5, 7]]])}
    a = bench.algorithmic_bytes(sh, res, types.SimpleNamespace(root_child=None))
    assert (a["u_root"], a["u_mid"], a["u_leaf"]) == (3, 3, 3)
    assert a["descend"] == 200 and a["attend"] == 224 and a["attend_flops"] == 288 and a["staging"] == 0
    a = bench.algorithmic_bytes(sh, res, types.SimpleNamespace(root_child=torch.zeros(1)))
    assert a["descend"] == 200 + 48
    # host-resident leaves: the staged bytes are the leaf-key blocks of the
    # unique kept mids (6 rows) and the unique kept leaves' value rows (3)
    host = dataclasses.replace(sh, leaf_on_host=True)
    a = bench.algorithmic_bytes(host, res, types.SimpleNamespace(root_child=None))
    assert a["staging"] == 2 * 4 * (6 + 3)


def test_profiled_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    # The bench line's `traffic` comes from a committed summary only while the
    # kernel's source still hashes to the one that was captured.
    import hashlib
    csrc = tmp_path / "hierarchical_kv_pruning_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "attend_tc.cuh"
    src.write_bytes(b"// kernel v1\n")
    digest = hashlib.sha256(b"// kernel v1\n").hexdigest()
    (tmp_path / "profiles" / "attend_tc_kernel__w.md").write_text(
        "# summary\n\n- kernel: `attend_tc_kernel`\n- source_sha256: `%s`\n  (note)\n"
        "- dram_bytes_per_launch: 12345\n" % digest)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("attend_tc_kernel", "w") == 12345
    assert bench.profiled_traffic("attend_tc_kernel", "other") is None     # no summary for that workload
    src.write_bytes(b"// kernel v2\n")
    assert bench.profiled_traffic("attend_tc_kernel", "w") is None         # source changed since the capture
    # the descent is a chain of kernels from two files: the digest covers both, in order
    (csrc / "descend.cuh").write_bytes(b"a")
    (csrc / "descend_pm.cuh").write_bytes(b"b")
    (tmp_path / "profiles" / "descent__w.md").write_text(
        "- source_sha256: `%s`\n- dram_bytes_per_launch: 7\n" % hashlib.sha256(b"ab").hexdigest())
    assert bench.profiled_traffic("descent", "w") == 7
    (csrc / "descend_pm.cuh").write_bytes(b"c")
    assert bench.profiled_traffic("descent", "w") is None


def test_peaks_fall_back_when_unmeasured(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, source = bench.measured_peaks()
    assert source == "fallback" and peaks["hbm_gbs"] == 6650.0 and peaks["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}')
    peaks, source = bench.measured_peaks()
    assert source == "measured" and peaks["hbm_gbs"] == 6000.0


def test_clock_summary_decodes_throttle_reasons():
    # NVML clock-event bits: 0x4 software power cap, 0x8 hardware slowdown,
    # 0x20 software thermal, 0x40 hardware thermal; others (0x1 idle) ignored.
    c = bench.ClockSampler(0)
    c.max_mhz = 1965.0
    c.samples = [(1965.0, 0x0), (1320.0, 0x4), (1900.0, 0x1)]
    s = c.summary()
    assert s["sm_mhz"] == 1900.0 and s["samples"] == 3 and s["reasons"] == ["sw_power_cap"]
    c.samples.append((900.0, 0x8 | 0x40 | 0x20))
    assert bench.ClockSampler.summary(c)["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap",
                                                        "sw_thermal_slowdown"]
    assert bench.ClockSampler(0).summary()["samples"] == 0


def test_reference_arm_contract():
    # `--impl reference` times the oracle on the host cores: rank 0 prints one
    # JSON line with the contract's keys, any other rank exits without work.
    import json
    import subprocess
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "0", "--steps", "2",
           "--warmup", "1", "--cpu-seconds", "0.5"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "e2e", "cpu_baseline"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "tiny_fp32_10x10x10"
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=dict(env, RANK="1"), cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_headline_roofline_is_the_whole_step():
    # leaves in HBM: frac = (descent + attention bytes) / step time / peak;
    # the slowest stage is reported beside it, not instead of it
    from hierarchical_kv_pruning_b200 import synth
    sh = synth.shape(2)
    alg = {"descend": 200e6, "attend": 400e6, "attend_seq": 300e6, "attend_leaf": 100e6, "attend_flops": 7e10,
           "staging": 0}
    st = {"descend": 0.25, "staging": 0.0, "attend": 0.15, "attend_seq": 0.0, "attend_leaf": 0.15}
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}
    top = bench.roofline_of(sh, alg, st, 0.4, peaks, "measured", 50.0)
    assert top["frac"] == pytest.approx(600e6 / 0.4e-3 / 1e9 / 6000.0)
    assert top["kernel"].startswith("whole step") and top["bound"] == "hbm"
    assert top["dominant"]["kernel"].startswith("descent")
    assert top["dominant"]["frac"] == pytest.approx(200e6 / 0.25e-3 / 1e9 / 6000.0)
    assert set(top["kernels"]) == {"descend", "attend"}

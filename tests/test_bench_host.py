"""Host logic of bench.py without a GPU: max-over-ranks timing across two gloo
ranks (the path of a multi-GPU run, where every rank is an independent
replica), clock-sample parsing and the profile/traffic bookkeeping."""
import json
import os
import pathlib
import socket
import sys

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, local, w = bench.dist_setup(n_gpus=0)  # gloo
    assert (r, local, w) == (rank, rank, world)
    bench.barrier(w)
    mx = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    bench.barrier(w)
    results[rank] = mx
    import torch.distributed as dist

    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(results) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_clock_summary_parsing():
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1965, 1965, 300.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1335, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1350, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 120, 1965, 90.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage",
    ]
    s = cs.summary()
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert s["sm_mhz"] == 1350  # idle sample (120 MHz) excluded, median of the rest
    assert s["samples"] == 4


def test_profiled_traffic_requires_matching_source(tmp_path, monkeypatch):
    import synth

    w = synth.WORKLOADS["global_s9_g64"]
    f = tmp_path / "summary.txt"
    f.write_text(f"tokens: {w.n_q // 3}\nsource_sha256_16: {bench.kernel_source_hash()}\n"
                 "dram_bytes_per_launch: 1000\n")
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(f))
    assert bench.profiled_traffic(w) == 3000.0
    assert bench.profiled_traffic(synth.WORKLOADS["frame_s8_g37"]) is None
    f.write_text("tokens: 10\nsource_sha256_16: 0000\ndram_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic(w) is None


@pytest.mark.parametrize("name", ["global_s2_g16", "frame_s8_g37", "descriptor_s200_g37_kd4",
                                  "omega_frame_s32_g32", "omega_global_s32_g32", "frame_s8_g37_f32",
                                  "global_s9_g64_affine8"])
def test_oracle_leg_runs_on_a_small_sample(name):
    import synth

    w = synth.ALL_WORKLOADS[name]
    if w.n_q > 50000:
        pytest.skip("large setup; covered by the reference arm")
    tf, dt, rows = bench.OracleLeg(w).run(8)
    assert tf > 0 and dt > 0 and rows >= 8


def test_secondary_workloads_are_known_and_exclude_nothing_of_the_pages_shapes():
    import synth

    assert all(n in synth.ALL_WORKLOADS for n in bench.SECONDARY)
    # every configuration of the pages' shapes is either the headline or secondary
    assert set(synth.WORKLOADS) <= set(bench.SECONDARY) | {bench.DEFAULT_WORKLOAD}


def test_attention_kernel_names():
    import synth

    assert bench.attention_kernel_name(synth.ALL_WORKLOADS["global_s9_g64"]) == "attn_fwd_kernel"
    assert "precise" in bench.attention_kernel_name(synth.ALL_WORKLOADS["global_s9_g64_affine8"])
    assert "fp32" in bench.attention_kernel_name(synth.ALL_WORKLOADS["global_s9_g64_f32"])


_REFERENCE_ARM_CHILD = r"""
import json, sys
sys.path.insert(0, sys.argv[1])
import bench
rc = bench.main(["--impl", "reference", "--workload", "global_s2_g16", "--steps", "1", "--warmup", "0",
                 "--reference-budget-s", "2"])
maps = open("/proc/self/maps").read()
print(json.dumps({"rc": rc, "lib_mapped": "libvggt_attn" in maps,
                  "package_imported": "feed_forward_view_b200" in sys.modules}))
"""


def test_reference_arm_never_loads_the_product_library():
    # The oracle arm's process must hold neither the package nor its shared
    # library: it times the oracle alone.
    import subprocess

    root = str(pathlib.Path(__file__).resolve().parents[1])
    res = subprocess.run([sys.executable, "-c", _REFERENCE_ARM_CHILD, root], capture_output=True, text=True,
                         timeout=600, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    arm, probe = json.loads(lines[0]), json.loads(lines[-1])
    assert arm["impl"] == "reference" and arm["value"] > 0
    assert probe == {"rc": 0, "lib_mapped": False, "package_imported": False}

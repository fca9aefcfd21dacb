"""Host-side checks of bench.py: the replica aggregation and the max-over-ranks timing on two
gloo ranks (CPU), and the JSON line of the CPU reference arm."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_whole_job_aggregate():
    # two replicas of 10 units each, slowest rank 2 s -> 10 units/s for the job
    assert bench.whole_job(10.0, [1.0, 2.0], 2) == pytest.approx(10.0)
    assert bench.whole_job(5.0, [0.5], 1) == pytest.approx(10.0)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.dist_init(world, "gloo")
    bench.barrier(world)
    m = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
    out[rank] = m
    torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == pytest.approx(2.5)


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", "strided_merged_n3072_l64"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0


def test_reference_arm_loads_no_cuda_library():
    """The reference arm is the oracle alone: running it maps liboracle.so but never the CUDA
    library (its FLOP count comes from the canonical tile table)."""
    code = ("import sys, runpy; sys.argv = ['bench.py', '--impl', 'reference', '--steps', '1', "
            "'--warmup', '0', '--workload', 'strided_n256_l16_fp32']\n"
            "try:\n    runpy.run_path('bench.py', run_name='__main__')\nexcept SystemExit:\n    pass\n"
            "maps = open('/proc/self/maps').read()\n"
            "print('LIBST' if 'libst_attn' in maps else 'NOLIBST', 'ORACLE' if 'liboracle' in maps else 'NOORACLE')")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().splitlines()[-1] == "NOLIBST ORACLE"


def test_canonical_tile_table_matches_the_library_census():
    import block_sparse_factorized_b200 as bsf
    from workloads import WORKLOADS
    assert set(bench.CANONICAL_TILES) == set(WORKLOADS)
    for name, w in WORKLOADS.items():
        info = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).info()
        assert bench.CANONICAL_TILES[name] == info["exec_tiles"], name
        assert bench.canonical_flops(w) == bench.step_flops(w, info)[0], name


def test_reference_arm_nonzero_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_headline_flop_and_byte_counts():
    """The metric's FLOP count at the headline workload: 10,368 active 128 x 128 tile pairs (4 x 96
    same-block + 4 x 1,200 summary per batch element, x 2), 4 d FLOPs per score entry in the
    forward and 2.5 times that in the backward; the algorithmic bytes count each tensor once
    (a summary head reads n / l * c key rows)."""
    import block_sparse_factorized_b200 as bsf
    from workloads import WORKLOADS
    w = WORKLOADS["fixed_n12288_l128_c32"]
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c)
    flops, bwd_flops, useful = bench.step_flops(w, lay.info())
    pairs = 2 * (4 * 96 + 4 * 1200)
    assert pairs == 10368
    assert flops == pairs * 128 * 128 * 4 * 64 * 3.5
    assert bwd_flops == pairs * 128 * 128 * 4 * 64 * 2.5
    assert useful == 78673920 * 2 * 4 * 64 * 3.5  # allowed (i, j) pairs only
    fwd_b, bwd_b = bench.step_bytes(w, lay)
    rows, row = 2 * 8 * 12288, 128
    used = 2 * (4 * 12288 + 4 * 96 * 32)  # K/V rows read: 4 full heads + 4 summary heads
    assert fwd_b == 2 * rows * row + 2 * used * row + rows * 4
    assert bwd_b == fwd_b + rows * row + rows * 4 + 3 * rows * row


def test_cpu_baseline_covers_whole_slabs():
    """The CPU baseline runs the oracle on whole (batch, head) slabs, cycling over the workload
    until the time floor is met, and reports throughput over the slabs it covered."""
    from workloads import Workload, STRIDED, ALTERNATING
    w = Workload("s_n512_l16", STRIDED, ALTERNATING, 512, 16, 0, 1, 2)
    cpu = bench.cpu_baseline(w, flops=1e9, min_seconds=0.2)
    assert cpu["kind"] == "oracle" and cpu["unit"] == "TFLOP/s" and cpu["cores"] >= 1
    assert cpu["value"] > 0 and "slabs at full n=512" in cpu["sample"]
    done = int(cpu["sample"].split("oracle fwd+bwd of ")[1].split()[0])
    assert done >= 1


def test_traffic_comes_from_the_committed_table_at_the_current_source_hash(tmp_path):
    """roofline.traffic is read from the ncu table under profiles/ (summed over a workload's
    passes) only while the kernel's sources hash to the recorded value; otherwise it is None."""
    src = bench.kernel_src_hash("bwd_kernel")
    table = tmp_path / "t.md"
    table.write_text("| workload | kernel | pass | source hash | read | write |\n|---|---|---|---|---|---|\n"
                     f"| wl_a | bwd_kernel | 1/2 | {src} | 100 | 20 |\n"
                     f"| wl_a | bwd_kernel | 2/2 | {src} | 7 | 3 |\n"
                     f"| wl_a | fwd_bf16_kernel | 1/1 | {src} | 999 | 999 |\n"
                     "| wl_b | bwd_kernel | 1/1 | 0000000000000000 | 5 | 5 |\n")
    assert bench.recorded_traffic("wl_a", "bwd_kernel", str(table)) == 130
    assert bench.recorded_traffic("wl_b", "bwd_kernel", str(table)) is None   # stale hash
    assert bench.recorded_traffic("wl_c", "bwd_kernel", str(table)) is None   # not captured
    assert bench.recorded_traffic("wl_a", "bwd_kernel", str(tmp_path / "missing.md")) is None

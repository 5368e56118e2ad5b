"""The reference arm of bench.py on the CPU: it times the fp64 oracle on a
bounded sample of the bench workload and prints one JSON line with the
keys the benchmark contract fixes (the same metric, unit and config as the
GPU arm, its own cpu_baseline, and an e2e object with no host transfers)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "1"], env=env, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] >= 3
    assert d["config"]["workload"] == bench.WORKLOAD
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"] and cb["unit"] == d["unit"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_decode_flops_and_roofline_bound():
    # FLOPs per step: 2 * s_q * heads * rows * (512 + 64 + 512); the 256K
    # two-token case sits above the measured ridge (bf16 peak / HBM copy
    # rate) and is reported against the tensor peak, the others against HBM
    sys.path.insert(0, ROOT)
    import bench
    from head_latent_attention_02_b200.workloads import WORKLOADS
    peaks = {"hbm_gbs": 6543.4, "bf16_tflops": 1623.7}
    cases = [("bf16_b16_4k", [4096] * 16, None, 18_253_611_008, "hbm"),
             ("bf16_long_256k", [262144] * 2, None, 292_057_776_128, "tensor"),
             ("redknot_56_8", [24576], [256], 2 * 1088 * (8 * 24576 + 56 * 256), "hbm")]
    for name, rows, ng, flops, bound in cases:
        wl = WORKLOADS[name]
        assert bench.decode_flops(wl, rows, ng) == flops
        cb = (sum(rows) + (sum(ng) if ng else 0)) * 1152
        r = bench.decode_roofline(flops, cb, 0.05, peaks, "measured", None, "k")
        assert r["bound"] == bound
        if bound == "hbm":
            assert r["unit"] == "GB/s" and r["achieved"] == round(cb / 0.05e-3 / 1e9, 1)
        else:
            assert r["unit"] == "TFLOP/s" and r["achieved"] == round(flops / 0.05e-3 / 1e12, 1)
        assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-4


def test_cache_copies_keep_each_decode_out_of_l2():
    sys.path.insert(0, ROOT)
    import bench
    for cache_bytes in (28_311_552, 75_497_472, 604_045_312, 1_340_657_664):
        n = bench.n_cache_copies(cache_bytes)
        assert n >= 3 and (n - 1) * cache_bytes >= 2 * bench.L2_BYTES


def test_gpu_count_must_match_the_launched_ranks():
    # a rank count that disagrees with --gpus is refused before any GPU work
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--steps", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode != 0 and "WORLD_SIZE=1" in res.stderr

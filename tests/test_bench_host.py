"""Host-side pieces of bench.py: the roofline work model pinned to the worked example the pages
print, and the multi-rank helpers run as two gloo ranks on the CPU."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _example():
    return json.load(open(os.path.join(GOLDEN, "roofline_worked_example.json")))


def _digits(x, printed):
    """x rounded the way the page prints `printed` (same number of decimals)."""
    s = repr(printed)
    dec = len(s.split(".")[1]) if "." in s else 0
    return round(x, dec)


def test_step_time_model_reproduces_the_worked_example():
    """'INT8 vs INT4 Quantization, in depth', section 'Worked example: where the lines cross':
    8B parameters on a 2 TB/s, 400 TFLOPS (fp16) / 800 TOPS (int8) GPU."""
    ex = _example()
    P, bw, f16, i8 = ex["params"], ex["hbm_bytes_per_s"], ex["fp16_flops_per_s"], ex["int8_ops_per_s"]
    pr = ex["printed"]
    bits = {"fp16": 16, "w8a8": 8, "w4a16": ex["w4a16_bits_per_weight"]}
    flops = {"fp16": f16, "w8a8": i8, "w4a16": f16}
    assert _digits(P * bits["w4a16"] / 8 / 1e9, pr["w4a16_weight_GB"]) == pr["w4a16_weight_GB"]
    for fmt, ms in pr["floor_ms"].items():
        _, t_mem, _ = bench.step_time_model(P, bits[fmt], bw, flops[fmt], 1)
        assert _digits(t_mem * 1e3, ms) == ms
    # batch-1 tokens/s: the page prints 125 and 250 exactly and 480 for 1 / 2.0625 ms = 484.8
    for fmt, tps in pr["tok_per_s_batch1"].items():
        t, _, _ = bench.step_time_model(P, bits[fmt], bw, flops[fmt], 1)
        assert 1.0 / t == pytest.approx(tps, rel=0.015)
    for fmt, ms in pr["compute_ms_per_batch"].items():
        _, _, t_math = bench.step_time_model(P, bits[fmt], bw, flops[fmt], 1)
        assert _digits(t_math * 1e3, ms) == ms
    for fmt, b in pr["compute_bound_from_batch"].items():
        assert int(bench.crossover_batch(P, bits[fmt], bw, flops[fmt])) == b
    # the W4A16 and W8A8 step-time curves cross where both are compute-bound at equal time
    t4 = lambda B: bench.step_time_model(P, bits["w4a16"], bw, f16, B)[0]
    t8 = lambda B: bench.step_time_model(P, bits["w8a8"], bw, i8, B)[0]
    cross = next(B for B in range(1, 1000) if t4(B) >= t8(B))
    assert cross == pr["curves_cross_near_batch"]
    for fmt, ms in pr["step_ms_at_batch_256"].items():
        t, _, _ = bench.step_time_model(P, bits[fmt], bw, flops[fmt], 256)
        assert _digits(t * 1e3, ms) == ms


def test_decode_traffic_record_applies_only_to_its_sources(tmp_path, monkeypatch):
    """The ncu traffic record behind `roofline.traffic`: scaled to a launch's algorithmic bytes
    while its source hash matches the decode kernel's sources, null (stale) once they differ."""
    rec = json.load(open(bench.TRAFFIC_FILE))
    assert {"sources_sha", "dram_bytes", "algorithmic_bytes", "capture"} <= set(rec)
    assert 1.0 <= rec["dram_bytes"] / rec["algorithmic_bytes"] < 1.1   # each unit record read once
    path = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    path.write_text(json.dumps(dict(rec, sources_sha=bench.decode_sources_sha())))
    b, info = bench.decode_traffic(3 * rec["algorithmic_bytes"])
    assert b == pytest.approx(3 * rec["dram_bytes"])
    assert info["ratio_to_algorithmic"] == pytest.approx(rec["dram_bytes"] / rec["algorithmic_bytes"])
    path.write_text(json.dumps(dict(rec, sources_sha="0" * 16)))
    b, info = bench.decode_traffic(1e8)
    assert b is None and info["stale"]


def test_algorithmic_bytes_match_the_format():
    """0.515625 byte/weight for g128 with an FP16 scale; + 0.5/128 with INT4 zero-points."""
    K, N = 4096, 4096
    sym = bench.algorithmic_bytes(1, K, N, group=128, sym=1, act_bytes=0, out_bytes=0)
    asym = bench.algorithmic_bytes(1, K, N, group=128, sym=0, act_bytes=0, out_bytes=0)
    assert sym / (K * N) == 0.515625
    assert asym / (K * N) == 0.515625 + 0.5 / 128
    assert bench.algorithmic_bytes(3, K, N, sym=1) - sym == 2 * 3 * K + 2 * 3 * N
    assert bench.gemm_flops(2, 3, 5) == 60


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    r, w, lr = bench.dist_env()
    mx = bench.max_over_ranks(1.5 + 10.0 * r, w)
    out[rank] = (r, w, lr, bench.replica_seed(1234, r), mx)
    dist.barrier()
    dist.destroy_process_group()


def test_rank_helpers_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank, (r, w, lr, seed, mx) in res.items():
        assert (r, w, lr) == (rank, world, rank)
        assert mx == 11.5                       # the slower rank's time on every rank
    assert res[0][3] != res[1][3]               # each rank draws its own replica
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the FP64 oracle on the host cores and prints one JSON
    line with the keys the harness reads (no GPU needed)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                         cwd=root, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]

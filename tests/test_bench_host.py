"""Host-side pieces of bench.py (no GPU): the algorithmic byte count the
roofline uses, the clock-record summary and the recorded-traffic lookup."""
import bench
import synth


def test_algorithmic_bytes_of_the_1m_scoring_launch():
    w = synth.workload("1m")
    nblk = [w.L // synth.POOL] * w.B
    # 4 x (262,144 blocks x 256 B key + 8 KiB query + 128 B weights); the
    # score writes are overhead outside the algorithmic bytes
    assert bench.score_algorithmic_bytes(nblk, w.B) == 268_468_736
    assert bench.score_write_bytes(nblk) == 4 * 262144 * 4
    # INT8 cache: 128 B of codes + 4 B scale per block; 4 KiB of query codes
    # + 128 B of weights per row
    assert bench.score_algorithmic_bytes(nblk, w.B, "int8") == 4 * 262144 * 132 + 4 * (4096 + 128)


def test_algorithmic_bytes_of_the_1m_decode_step():
    # per query: keys 67,108,864 + latent 2048 x 1 KiB + q_idx 8,192 + w 128
    # + q 65,536 + out 65,536 = 69,345,408 B
    assert bench.step_algorithmic_bytes(4, 1 << 20, 64) == 4 * 69_345_408
    # a partial tail adds its rows; a short row attends to every token
    assert bench.step_algorithmic_bytes(1, 4 * 1000 + 3, 16) == (
        1000 * 256 + 8192 + 128 + (4 * 512 + 3) * 1024 + 2 * 16 * 1024)
    assert bench.step_algorithmic_bytes(1, 1536, 64) == 384 * 256 + 8320 + 1536 * 1024 + 2 * 65536


def test_prefill_flops_count_the_causal_blocks():
    # query t sees (pos0 + t + 1) // 4 complete blocks; 2 x 32 x 128 flop per block
    assert bench.score_algorithmic_flops_prefill(8, 4) == 2 * 32 * 128 * (2 + 2 + 2 + 3)
    # attention: 4 H D flop per attended token (every token while n <= 2051)
    assert bench.attention_flops_prefill(8, 4, 64) == 4 * 64 * 512 * (9 + 10 + 11 + 12)
    assert bench.attention_flops_prefill(2048 * 4, 1, 16) == 4 * 16 * 512 * (2048 + 1)


def test_stratified_prefill_subset():
    sub = bench.stratified_prefill_queries(4096)
    assert len(sub) == 256 and len(set(sub)) == 256 and sub == sorted(sub)
    assert {0, 1, 2, 3, 4095} <= set(sub) and {t % 4 for t in sub} == {0, 1, 2, 3}
    assert {7, 8, 511, 512, 1023, 1024} <= set(sub)  # edges of 8-query scoring groups
    assert bench.stratified_prefill_queries(10) == list(range(10))


def _sampler(lines):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples = [bench.ClockSampler._parse_smi(l) for l in lines]
    s.source = "nvidia-smi"
    return s


def test_clock_summary_reports_median_and_active_reasons():
    ok = "0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    capped = "0, 1800, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active"
    summ = _sampler([ok, capped, ok]).summary()
    assert summ["sm_mhz"] == 1965.0 and summ["sm_max_mhz"] == 1965.0
    assert summ["reasons"] == ["sw_power_cap"]
    assert summ["samples"] == 3 and summ["sm_mhz_min"] == 1800.0
    hot = "0, 1500, 1965, 999.0, 0x40, Not Active, Active, Not Active, Not Active"
    assert "hw_thermal_slowdown" in _sampler([hot]).summary()["reasons"]
    assert bench.ClockSampler._parse_smi("garbage") is None


def test_recorded_traffic_matches_only_the_current_kernel_source():
    t = bench.recorded_traffic("decode_1m")
    alg = bench.score_algorithmic_bytes([262144] * 4, 4)
    assert t is None or alg <= t < 1.05 * alg  # recorded for this source, no re-reads
    assert bench.recorded_traffic("no such workload") is None


def test_reference_arm_line_on_cpu():
    """`bench.py --impl reference` (the oracle, timed on host cores) prints one
    JSON line with the contract's keys; ranks other than 0 print nothing."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
           "--warmup", "1"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, RANK="0"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "queries/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "queries/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    # the same config dict as this library's decode line on that workload
    import bench
    import synth
    w = synth.workload("tiny")
    assert d["config"] == bench.decode_config(w, w.B, w.L, w.heads, 1)
    assert d["metric"] == bench.METRIC
    r1 = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300,
                        env=dict(os.environ, RANK="1"))
    assert r1.returncode == 0 and not r1.stdout.strip()

"""Host-side arithmetic of bench.py, on the CPU: the algorithmic work per launch,
the roofline fraction, the ncu traffic table lookup and the clock log parsing.

These numbers end up in the bench line (roofline.achieved, frac, traffic,
clocks), so each is checked against a value worked out by hand here.
"""

import os

import pytest

import bench


def test_la_prefill_work_per_head_token():
    # One head-token at C=128, d'=16, dv=64, D=273:
    # 2*128*16 + 2*128*64 + 2*128 + 4*273*64 + 4*273 = 4096 + 16384 + 256 + 69888 + 1092.
    flops, byts = bench.la_prefill_work(1, 1, 1, 16, 64, 128)
    assert flops == 91_716
    # q, k, v, y in bf16 (2*16 + 2*64 values) plus one fp32 state (273*64 + 273).
    assert byts == 320 + 70_980
    # The 360M-shaped launch: B=8, H=16, N=2048.
    flops, byts = bench.la_prefill_work(8, 16, 2048, 16, 64, 128)
    assert flops == 91_716 * 8 * 16 * 2048 == 24_042_799_104
    assert byts == 8 * 16 * 2048 * 320 + 8 * 16 * 70_980 == 92_971_520


def test_decode_and_swa_work():
    # LA decode reads and writes the fp32 state once: 2*(273*64 + 273)*4 + (2*16 + 2*64)*2.
    assert bench.la_decode_work(1, 1, 16, 64)[1] == 142_280
    # The symmetric layout has 1 + 16 + 136 = 153 rows.
    assert bench.la_decode_work(1, 1, 16, 64, packed=True)[1] == 2 * (153 * 64 + 153) * 4 + 320
    # SWA decode: ring read (2*64*64 bf16), new slot written, q, k, v, y.
    assert bench.swa_decode_work(1, 1, 64, 64)[1] == 2 * 64 * 64 * 2 + 2 * 64 * 2 + 4 * 64 * 2 == 17_152
    # SWA prefill at one head-token: 4*w*d flops.
    assert bench.swa_prefill_work(1, 1, 1, 64, 64)[0] == 16_384


def test_roofline_fraction_takes_the_slower_bound():
    peaks = dict(bf16_tflops=1000.0, hbm_gbs=5000.0)
    # 1 TFLOP in 2 ms: the tensor bound is 1 ms -> 0.5; 1 GB is 0.2 ms.
    assert bench._frac(1e12, 1e9, 2.0, peaks) == pytest.approx(0.5)
    # 1 GFLOP and 10 GB in 4 ms: the HBM bound is 2 ms -> 0.5.
    assert bench._frac(1e9, 10e9, 4.0, peaks) == pytest.approx(0.5)


def test_whole_job_rate_uses_the_slowest_rank():
    # 2 ranks x 100 units x 10 steps over 0.5 s.
    assert bench.whole_job_rate(2, 100, 10, 500.0) == pytest.approx(4000.0)


def _fake_tree(tmp_path, text):
    csrc = tmp_path / "linear_attention_sequence_causal_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in {n for names in bench.KERNEL_SOURCES.values() for n in names}:
        (csrc / name).write_text(f"// {name}\n")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.md").write_text(text)
    return csrc


def test_traffic_row_counts_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = _fake_tree(tmp_path, "")
    h = bench.kernel_source_hash("la_prefill")
    assert len(h) == 12
    table = ("| kernel | source hash | bytes per bench launch | capture |\n|---|---|---|---|\n"
             f"| la_prefill | {h} | 8.153e7 | fake |\n| swa_prefill | 000000000000 | 1.0e8 | fake |\n")
    (tmp_path / "profiles" / "dram_traffic.md").write_text(table)
    assert bench.measured_traffic("la_prefill") == pytest.approx(8.153e7)
    assert bench.measured_traffic("swa_prefill") is None          # hash of other sources
    # Any edit to one of the kernel's sources retires the row.
    (csrc / "la_prefill_tc.cu").write_text("// changed\n")
    assert bench.kernel_source_hash("la_prefill") != h
    assert bench.measured_traffic("la_prefill") is None


def test_clock_log_parsing(tmp_path):
    log = tmp_path / "clocks.csv"
    log.write_text(
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "0, 1950, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active\n"
        "0, 1965, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "garbage line\n")

    class Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s = bench.ClockSampler(0)
    s.proc, s.path, s.out = Done(), str(log), open(os.devnull, "w")
    got = s.stop()
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1965.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]
    assert not log.exists()

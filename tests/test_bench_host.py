"""Host-side helpers of bench.py, on CPU: the FC1/FC2 launch rule it mirrors from
moe_expert_ffn (one launch when FC1 has at most 2 work items per SM), the committed DRAM
traffic record and its source digest, and the peak figures."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from skew_aware_token_b200 import native as N  # noqa: E402
from skew_aware_token_b200.synth import WORKLOADS, Workload  # noqa: E402


@pytest.mark.parametrize("name,one", [("tiny", True), ("olmoe_a1", False), ("qwen3_a1.5", False),
                                      ("sweep_all4_p0_b128", False), ("dsv3_a1", False)])
def test_one_launch_rule_at_148_sms(name, one):
    # FC1 items = (T k / 128) (f / 128): tiny 32, OLMoE 2048, Qwen3 3072, sweep 6144,
    # DeepSeek-V3 16384; the threshold is 2 x 148 = 296
    assert bench.ffn_one_launch(WORKLOADS[name], 0, 148) is one


def test_one_launch_rule_boundary_and_flags():
    wl = Workload("edge", T=296 * 128 // 8, d=256, E=8, k=8, f=128, beta=128, P=1, s=0)
    assert wl.T * wl.k // 128 * (wl.f // 128) == 2 * 148
    assert bench.ffn_one_launch(wl, 0, 148)            # at the threshold: one launch
    assert not bench.ffn_one_launch(wl, 0, 147)        # over the threshold: two
    for flag in (N.MOE_FFN_WRITE_O, N.MOE_FFN_STRICT_SLOTS, N.MOE_FFN_SM_PAIR,
                 N.MOE_FFN_GATHER_X, N.MOE_FFN_TWO_LAUNCHES):
        assert not bench.ffn_one_launch(wl, flag, 148), flag
    assert bench.ffn_one_launch(WORKLOADS["dsv3_a1"], N.MOE_FFN_ONE_LAUNCH, 148)


def test_traffic_record_follows_the_ffn_source():
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for name, r in rec.items():
        if r["ffn_source_sha1"] == bench.ffn_source_digest():
            assert bench.measured_traffic(name) == r["bytes_per_step"]
        else:
            assert bench.measured_traffic(name) is None
    assert bench.measured_traffic("no_such_workload") is None


def test_traffic_record_is_dropped_when_the_source_changes(monkeypatch):
    monkeypatch.setattr(bench, "ffn_source_digest", lambda: "0" * 40)
    assert all(bench.measured_traffic(n) is None for n in WORKLOADS)


def test_peaks_come_from_the_measured_file_when_present():
    peaks, src = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert src == "of measured"
        assert peaks["bf16_tflops_sustained"] <= peaks["bf16_tflops"]
    else:
        assert src == "of fallback" and peaks == bench.FALLBACK_PEAKS


def test_traffic_record_only_for_the_captured_configuration():
    for name in WORKLOADS:
        assert bench.measured_traffic(name, default_ffn=False) is None


def test_peak_follows_the_timed_region_length():
    peaks = {"bf16_tflops": 1612.8, "bf16_tflops_sustained": 1367.4}
    assert bench.pick_peak(peaks, 0.3) == (1612.8, "burst")
    assert bench.pick_peak(peaks, bench.SUSTAINED_AFTER_S) == (1367.4, "sustained")


def test_roofline_fraction_is_algorithmic_flops_over_time():
    wl = WORKLOADS["dsv3_a1"]
    peaks = {"bf16_tflops": 1612.8, "bf16_tflops_sustained": 1367.4}
    rl = bench.roofline(wl, 12.0, 0.24, peaks, "of measured")
    achieved = 6 * wl.T * wl.k * wl.d * wl.f / 12e-3 / 1e12
    assert rl["achieved"] == round(achieved, 2)
    assert rl["frac"] == round(achieved / 1612.8, 4) and rl["peak"] == 1612.8
    assert rl["frac_of_sustained"] == round(achieved / 1367.4, 4)


def test_launch_count_per_step():
    wl = WORKLOADS["dsv3_a1"]  # 131072 pairs: the dispatch's count and prefix kernels run
    assert bench.gpu_launches_per_step(wl, 0, 148) == 10
    assert bench.gpu_launches_per_step(wl, N.MOE_FFN_WRITE_O, 148) == 11
    assert bench.gpu_launches_per_step(wl, N.MOE_FFN_GATHER_X, 148) == 9
    # 512 pairs (one dispatch chunk), one FFN launch
    assert bench.gpu_launches_per_step(WORKLOADS["tiny"], 0, 148) == 7


def test_oracle_sample_fits_its_memory_bound():
    wl = WORKLOADS["dsv3_a1"]
    logits = bench.synth.make_logits(wl).numpy()
    n = bench.sample_size(wl, logits, max_bytes=4e9)
    experts = bench.sample_experts(wl, logits, n)
    assert 1 <= n < wl.T
    assert len(experts) * 3 * wl.d * wl.f * 4 <= 4e9
    # the next doubling would not fit
    assert len(bench.sample_experts(wl, logits, 2 * n)) * 3 * wl.d * wl.f * 4 > 4e9


def test_layer_runs_large_y_with_o_rows(monkeypatch):
    """A fused-combine call of a layer whose y exceeds the threshold runs FC2 with O rows and
    the ordered combine; explicit choices win; the O buffer exists whenever it is used."""
    from skew_aware_token_b200 import layer as L
    wl = WORKLOADS["tiny"]
    y_bytes = wl.T * wl.d * 4
    monkeypatch.setattr(L, "O_ROWS_MIN_Y_BYTES", y_bytes)
    big = L.MoeLayer(wl, "cpu")
    assert big.o_rows and big.o is not None
    assert big.ffn_mode(0) == N.MOE_FFN_WRITE_O
    assert big.ffn_mode(N.MOE_FFN_STRICT_SLOTS) == N.MOE_FFN_STRICT_SLOTS | N.MOE_FFN_WRITE_O
    assert big.ffn_mode(N.MOE_FFN_ONE_LAUNCH) == N.MOE_FFN_ONE_LAUNCH  # fused by design
    monkeypatch.setattr(L, "O_ROWS_MIN_Y_BYTES", y_bytes + 1)
    small = L.MoeLayer(wl, "cpu")
    assert not small.o_rows and small.o is None and small.ffn_mode(0) == 0
    assert L.MoeLayer(wl, "cpu", o_rows=True).o_rows
    assert not L.MoeLayer(wl, "cpu", o_rows=False, write_o=True).o_rows


def test_o_rows_threshold_splits_the_workloads():
    """O rows on every benchmark layer (32 MiB of y and more), fused on the 256-token one."""
    from skew_aware_token_b200 import layer as L
    for name, wl in WORKLOADS.items():
        big = wl.T * wl.d * 4 >= L.O_ROWS_MIN_Y_BYTES
        assert big == (name != "tiny"), name

"""The host-side arithmetic of bench.py (CPU only): the algorithmic bytes that
the roofline divides by, the clock record that decides whether a run is
rejected, and the gate that withholds recorded DRAM traffic once the kernel
sources change.

Byte counts follow the per-step accounting of the path: attention reads Q, K
and V once and writes O once, plus cu_seqlens and the CLS rows; pack reads
the mask and the kept rows and writes the kept rows and cu_seqlens; the fused
launch reads the mask and the kept dense rows and writes the packed rows, O,
the CLS rows and cu_seqlens.  Each expected value below is counted from the
workload's lengths, not from the workload's own T or row_bytes helpers."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synthetic  # noqa: E402


@pytest.mark.parametrize("make", [lambda: synthetic.serving(4, 0.5), lambda: synthetic.deit_b_pruned80(),
                                  lambda: synthetic.serving(1, 0.0)])
def test_algorithmic_bytes_from_the_lengths(make):
    w = make()
    T = int(np.sum(w.lengths))
    e = 2                                     # f16 / bf16 elements
    head_row = 64 * e                         # one (token, head) row
    dense_row = 3 * w.H * head_row            # one fused q/k/v token row
    assert bench.attn_bytes(w) == 4 * T * w.H * head_row + 4 * (w.B + 1) + w.B * w.H * head_row
    assert bench.pack_bytes(w) == w.B * w.L_full + 2 * T * dense_row + 4 * (w.B + 1)
    out_and_cls = T * w.H * head_row + w.B * w.H * head_row
    assert bench.fused_bytes(w) == (w.B * w.L_full + 2 * T * dense_row + out_and_cls + 4 * (w.B + 1))
    assert bench.fused_bytes(w, packed_written=False) == (w.B * w.L_full + T * dense_row + out_and_cls
                                                         + 4 * (w.B + 1))


def test_deit_b_attention_bytes_match_the_scope_estimate():
    """DeiT-B at 80% pruning, B=32: about 7.67 MB of q/k/v/o at E[L] = 39
    (1,248 tokens), scaling with the drawn T."""
    w = synthetic.deit_b_pruned80()
    T = int(np.sum(w.lengths))
    assert abs(bench.attn_bytes(w) - 7.67e6 * T / 1248) < 0.01 * 7.67e6


def test_us_per_call_counts_every_rank():
    # 12 calls per step, 10 steps, 2 ranks, 24 ms slowest rank -> 100 us per call
    assert bench.us_per_call(24.0, steps=10, calls_per_step=12, world=2) == pytest.approx(100.0)


class _FinishedProcess:
    """Stands in for the nvidia-smi child: already done, nothing to stop."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with(lines, t0=100.0, t1=101.0):
    s = bench.ClockSampler("0")
    s.proc = _FinishedProcess()
    s.lines = [(ts, line) for ts, line in lines]
    s.t0, s.t1 = t0, t1
    return s


def _row(mhz, hw="Not Active", thermal="Not Active", sw_thermal="Not Active", power="Not Active"):
    return f"0, {mhz}, 1965, 600.0, 0x0, {hw}, {thermal}, {sw_thermal}, {power}"


def test_clock_record_inside_the_timed_region():
    lines = [(99.0, _row(900)), (100.2, _row(1965)), (100.5, _row(1950)), (100.8, _row(1965)),
             (103.0, _row(800, hw="Active"))]
    rec = _sampler_with(lines).stop()
    assert rec["samples"] == 3                      # only the samples inside [t0, t1 + 0.1]
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == []


def test_clock_record_names_active_throttle_reasons():
    lines = [(100.1, _row(1500, power="Active")), (100.4, _row(1400, hw="Active")),
             (100.7, _row(1300, sw_thermal="Active"))]
    rec = _sampler_with(lines).stop()
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
    assert rec["sm_mhz"] == 1400.0


def test_clock_record_falls_back_to_the_nearest_sample():
    # a timed region shorter than the sampling period holds no sample
    lines = [(99.0, _row(1000)), (101.3, _row(1965))]
    rec = _sampler_with(lines, t0=100.0, t1=100.01).stop()
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1000.0


def test_recorded_traffic_is_withheld_when_sources_change(monkeypatch):
    """The committed record is reported while the fused kernel's sources hash
    to the recorded value, and withheld (None) once they do not, or when the
    record is missing."""
    recorded = None
    with open(bench.TRAFFIC_RECORD) as f:
        for line in f:
            if line.startswith("dram_bytes_per_launch_mean:"):
                recorded = int(line.split(":", 1)[1])
    assert recorded is not None and bench.recorded_traffic() == recorded
    monkeypatch.setattr(bench, "fused_source_hash", lambda: "0" * 64)
    assert bench.recorded_traffic() is None
    monkeypatch.undo()
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", os.path.join(ROOT, "profiles", "no_such_record.txt"))
    assert not os.path.exists(bench.TRAFFIC_RECORD)
    assert bench.recorded_traffic() is None


def test_committed_traffic_record_matches_the_current_kernel():
    """The committed DRAM record belongs to the fused kernel as it stands."""
    assert bench.recorded_traffic() is not None


def test_a_failing_extra_measurement_is_reported_not_raised(capsys):
    """The JSON line must survive a failure in one of the optional measurements."""
    def boom():
        raise RuntimeError("comparator unavailable")
    assert bench.optional(lambda: {"x": 1}) == {"x": 1}
    rec = bench.optional(boom)
    assert rec == {"error": "RuntimeError: comparator unavailable"}
    assert "comparator unavailable" in capsys.readouterr().err


def test_sdpa_backend_is_named():
    """The padded baseline names the SDPA backend torch picks for its call."""
    import torch
    from torch.nn.attention import SDPBackend
    q = torch.randn(2, 3, 5, 64)
    mask = torch.ones(2, 1, 1, 5, dtype=torch.bool)
    name = bench.sdpa_backend(q, q, q, mask)
    assert name in SDPBackend.__members__ or name.startswith("unknown")

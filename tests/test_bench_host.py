"""bench.py host logic that needs no GPU: the algorithmic bytes per unit behind
every roofline, the dominant-kernel roofline arithmetic, the digest gate on
the recorded ncu traffic, and the parsing of the nvidia-smi clock record."""
import os

import pytest

import bench


def test_algorithmic_bytes_per_chunk():
    # bf16 tiles of one (batch, head, 128-token chunk): q, k 128x96x2; v, o, dO
    # 128x192x2; a 128x4; a bf16 96x192 state 36,864; q.dq and k.dk 128x4 each
    q = k = 128 * 96 * 2
    v = o = dO = 128 * 192 * 2
    a = 128 * 4
    h = 96 * 192 * 2
    assert bench.CHUNK_BYTES["chunk_fwd_fused_kernel"] == q + k + v + o + a == 147_968
    assert bench.CHUNK_BYTES["chunk_state_fwd_kernel"] == k + v + a + h == 111_104
    assert bench.CHUNK_BYTES["chunk_state_rev_kernel"] == q + dO + a + h == 111_104
    # dq/dk: q, k, v, dO, h, D, a in; dq, dk, q.dq, k.dk out
    assert bench.CHUNK_BYTES["bwd_dqdk_kernel"] == q + k + v + dO + 2 * h + a + q + k + 2 * a == 271_872
    # dv: q, k, dO, D, a in; dv out
    assert bench.CHUNK_BYTES["bwd_dv_kernel"] == q + k + dO + h + a + v == 184_832
    assert bench.CHUNK_BYTES["da_finish_kernel"] == 3 * a


def test_roofline_takes_the_dominant_kernel():
    peaks = {"hbm_gbs": 6539.5}
    units = 8 * 16 * 16
    summary = [("chunk_fwd_fused_kernel", 3, 3 * 0.108), ("bwd_dqdk_kernel", 3, 3 * 0.155),
               ("bwd_dv_kernel", 3, 3 * 0.092)]
    roof, shares = bench.kernel_roofline(summary, peaks, "measured", units, 8, 16)
    assert roof["kernel"] == "bwd_dqdk_kernel"
    by = bench.CHUNK_BYTES["bwd_dqdk_kernel"] * units
    assert roof["bytes_per_launch"] == by
    assert roof["achieved"] == pytest.approx(by / 155e-6 / 1e9, rel=1e-3)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6539.5, rel=1e-3)
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert sum(shares.values()) == pytest.approx(1.0, abs=1e-3)
    # the fused forward also writes the final state of every head
    roof_f, _ = bench.kernel_roofline(summary[:1], peaks, "measured", units, 8, 16)
    assert roof_f["bytes_per_launch"] == bench.CHUNK_BYTES["chunk_fwd_fused_kernel"] * units + 73_728 * 8 * 16


def test_recorded_traffic_only_for_the_profiled_sources(monkeypatch):
    path = os.path.join(bench.ROOT, "profiles", "dram_traffic.md")
    rows = [ln for ln in open(path) if ln.startswith("| bwd_dqdk_kernel |")]
    assert rows, "the dominant kernel has a recorded traffic row"
    cells = [c.strip() for c in rows[0].strip().strip("|").split("|")]
    read, write, total = (int(cells[i].replace(",", "")) for i in (2, 3, 4))
    assert read + write == total
    # the row counts only while the kernel's sources hash to the recorded digest
    monkeypatch.setattr(bench, "kernel_digest", lambda name: cells[1])
    assert bench.recorded_traffic("bwd_dqdk_kernel") == total
    monkeypatch.setattr(bench, "kernel_digest", lambda name: "0" * 12)
    assert bench.recorded_traffic("bwd_dqdk_kernel") is None
    assert bench.recorded_traffic("no_such_kernel") is None


def test_kernel_digest_follows_the_sources():
    d = bench.kernel_digest("bwd_dqdk_kernel")
    assert len(d) == 12 and all(ch in "0123456789abcdef" for ch in d)
    assert bench.kernel_digest("no_such_kernel") is None


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_record_parsing(tmp_path):
    rec = tmp_path / "clocks.csv"
    rec.write_text("\n".join([
        "0, 1965, 1965, 812.3, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 640.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]) + "\n")
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.path = str(rec)
    out = s.stop()
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(rec)


def test_clock_record_flags_slowdowns(tmp_path):
    rec = tmp_path / "clocks.csv"
    rec.write_text("0, 1200, 1965, 700.0, 0x08, Active, Not Active, Active, Not Active\n")
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.path = str(rec)
    out = s.stop()
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert out["sm_mhz"] == 1200.0

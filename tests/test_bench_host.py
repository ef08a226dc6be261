"""bench.py host logic that needs no GPU: the algorithmic bytes per unit behind
every roofline, the dominant-kernel roofline arithmetic, the digest gate on
the recorded ncu traffic, and the parsing of the nvidia-smi clock record."""
import os

import pytest

import bench


def test_method_and_design_bytes_per_chunk():
    # bf16 tiles of one (batch, head, 128-token chunk): q, k 128x96x2; v, o, dO
    # 128x192x2; a 128x4; one bf16 plane of a 96x192 state 36,864; q.dq and
    # k.dk 128x4 each
    q = k = dq = dk = 128 * 96 * 2
    v = o = dO = dv = 128 * 192 * 2
    a = da = 128 * 4
    h = 96 * 192 * 2
    M, D = bench.METHOD_BYTES, bench.DESIGN_BYTES
    assert M["chunk_fwd_fused_kernel"] == q + k + v + o + a == 147_968
    assert M["chunk_state_fwd_kernel"] == k + v + a and D["chunk_state_fwd_kernel"] == 2 * h
    assert M["chunk_state_rev_kernel"] == q + dO + a and D["chunk_state_rev_kernel"] == 2 * h
    # dq/dk: q, k, v, dO, a in; dq, dk out (+ h and D as hi, lo planes; q.dq, k.dk)
    assert M["bwd_dqdk_kernel"] == q + k + v + dO + a + dq + dk == 197_120
    assert D["bwd_dqdk_kernel"] == 4 * h + 2 * a
    # the reverse sweep with dv: q, k, dO, a in; dv out (+ D_c as hi, lo planes)
    assert M["chunk_rev_fused_kernel"] == q + k + dO + a + dv == 147_968
    assert D["chunk_rev_fused_kernel"] == 2 * h
    assert M["da_finish_kernel"] == da
    # the step: forward and backward inputs and outputs, 3,084 B per token-head
    assert bench.STEP_BYTES == (q + k + v + a + o) + (q + k + v + dO + a + dq + dk + dv + da)
    assert bench.STEP_BYTES == 3084 * 128


def test_algorithmic_flops_per_chunk():
    mm = lambda m, n, kk: 2 * m * n * kk  # noqa: E731
    F = bench.CHUNK_FLOPS
    assert F["chunk_fwd_fused_kernel"] == 18_874_368
    assert F["chunk_state_fwd_kernel"] == F["chunk_state_rev_kernel"] == mm(96, 192, 128)
    assert F["bwd_dqdk_kernel"] == mm(128, 128, 192) + 2 * mm(128, 96, 192) + 2 * mm(128, 96, 128)
    # reverse sweep with dv: scores^T, K D, P~ dO (dv) and the state update Q~^T dO
    assert F["chunk_rev_fused_kernel"] == (mm(128, 128, 96) + mm(128, 192, 128) + mm(128, 192, 96)
                                           + F["chunk_state_rev_kernel"])
    # forward 18.9 MF and backward 45.6 MF per chunk-head: 132 GF at B8 H16 T2048
    assert bench.STEP_FLOPS * 8 * 16 * 16 == pytest.approx(132.07e9, rel=1e-4)


def test_roofline_takes_the_dominant_kernel():
    peaks = {"hbm_gbs": 6539.5, "bf16_tflops": 1624.7, "bf16_tflops_sustained": 1376.7}
    units = 8 * 16 * 16
    summary = [("chunk_fwd_fused_kernel", 3, 3 * 0.108), ("bwd_dqdk_kernel", 3, 3 * 0.155),
               ("bwd_dv_kernel", 3, 3 * 0.092)]
    roof, shares = bench.kernel_roofline(summary, peaks, "measured", units, 8, 16)
    assert roof["kernel"] == "bwd_dqdk_kernel"
    by = bench.METHOD_BYTES["bwd_dqdk_kernel"] * units
    assert roof["bytes_per_launch"] == by
    assert roof["design_bytes_per_launch"] == bench.DESIGN_BYTES["bwd_dqdk_kernel"] * units
    assert roof["achieved"] == pytest.approx(by / 155e-6 / 1e9, rel=1e-3)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6539.5, rel=1e-3)
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    fl = bench.CHUNK_FLOPS["bwd_dqdk_kernel"] * units
    assert roof["tensor"]["achieved"] == pytest.approx(fl / 155e-6 / 1e12, rel=1e-3)
    assert roof["tensor"]["frac"] == pytest.approx(roof["tensor"]["achieved"] / 1376.7, rel=1e-3)
    assert sum(shares.values()) == pytest.approx(1.0, abs=1e-3)
    # the fused forward also writes the final state of every head
    roof_f, _ = bench.kernel_roofline(summary[:1], peaks, "measured", units, 8, 16)
    assert roof_f["bytes_per_launch"] == bench.METHOD_BYTES["chunk_fwd_fused_kernel"] * units + 73_728 * 8 * 16


def test_step_roofline():
    peaks = {"hbm_gbs": 6539.5, "bf16_tflops": 1624.7, "bf16_tflops_sustained": 1376.7}
    r = bench.step_roofline(0.4568e-3, 8 * 16 * 16, 8, 16, peaks, "measured")
    # 808.5 MB of inputs and outputs + 9.4 MB of final state per step
    assert r["hbm"]["bytes_per_step"] == 3084 * 262_144 + 73_728 * 128
    assert r["hbm"]["frac"] == pytest.approx(817.9e6 / 0.4568e-3 / 6539.5e9, rel=1e-3)
    assert r["tensor"]["frac"] == pytest.approx(132.07e9 / 0.4568e-3 / 1376.7e12, rel=1e-3)


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


def test_digest_ignores_comments_only():
    src = 'int a = 1; // one\n/* block\n comment */ const char* s = "//x";\n\nint b = 2;\n'
    same = 'int a = 1;\n const char* s = "//x";\nint b = 2; // two\n'
    assert bench.strip_comments(src) == bench.strip_comments(same)
    assert bench.strip_comments(src) != bench.strip_comments(src.replace("b = 2", "b = 3"))
    assert '"//x"' in bench.strip_comments(src)


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


def test_per_kernel_rooflines():
    peaks = dict(bench.FALLBACK_PEAKS)
    units = 8 * 16 * 16
    summary = [("chunk_fwd_fused_kernel", 10, 1.0), ("bwd_dqdk_kernel", 10, 1.5), ("unmodelled_kernel", 3, 0.1)]
    r = bench.kernel_rooflines(summary, peaks, units, 8, 16)
    assert set(r) == {"chunk_fwd_fused_kernel", "bwd_dqdk_kernel"}
    e = r["bwd_dqdk_kernel"]
    assert e["mean_launch_us"] == 150.0
    mb = bench.METHOD_BYTES["bwd_dqdk_kernel"] * units
    assert e["frac"] == pytest.approx(mb / 150e-6 / 1e9 / peaks["hbm_gbs"], abs=1e-4)
    assert e["frac_incl_design_bytes"] > e["frac"] and 0 < e["tensor_frac"] < 1

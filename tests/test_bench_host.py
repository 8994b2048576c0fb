"""Host-side pieces of bench.py that need no GPU: the clock record taken during
the timed region, the throttle check on it, and the traffic figure read from a
profile summary only while its kernel sources are unchanged."""
import os

import bench


class _FakeSmi:
    """Stands in for the nvidia-smi sampling process: returns canned CSV rows."""

    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def kill(self):
        pass

    def communicate(self, timeout=None):
        return self.out, ""


def _stop(out):
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi(out)
    return s.stop()


def test_clock_record_uses_loaded_samples():
    out = "\n".join([
        "0, 345, 1965, 120.5, 0x1, Not Active, Active, Not Active, Not Active",   # idle: ignored
        "0, 1950, 1965, 870.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 905.2, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1935, 1965, 998.9, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, n/a, 1965, 900, 0x0, Not Active, Not Active, Not Active, Not Active",  # unparsable: skipped
    ])
    c = _stop(out)
    assert c == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert not bench.any_rank_throttled(c, 1, "cpu")


def test_clock_record_flags_thermal_slowdown_and_idle_only_runs():
    hot = "0, 1500, 1965, 700, 0x40, Not Active, Active, Not Active, Not Active\n"
    c = _stop(hot)
    assert c["reasons"] == ["hw_thermal_slowdown"] and bench.any_rank_throttled(c, 1, "cpu")
    idle = "0, 345, 1965, 90, 0x0, Not Active, Not Active, Not Active, Not Active\n"
    assert _stop(idle)["samples"] == 1  # no loaded sample: every row counts
    assert _stop("") is None
    s = bench.ClockSampler(0)
    assert s.stop() is None  # never started (no nvidia-smi)


def test_traffic_only_from_a_summary_of_the_current_sources(tmp_path, monkeypatch):
    kernel = "fa_fwd_kernel"
    prof = tmp_path / "profiles"
    prof.mkdir()
    csrc = tmp_path / "exact_tiled_attention_36_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES[kernel]:
        (csrc / name).write_text(f"// {name}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.csrc_digest(kernel)
    (prof / f"{kernel}.txt").write_text(
        f"# header line: ignored\nkernel: {kernel}\ncsrc_sha256_16: {digest}\ndram_bytes_per_launch: 406866432\n")
    assert bench.profiled_traffic(kernel) == 406866432.0
    # any edit of the kernel's sources invalidates the figure
    first = bench.KERNEL_SOURCES[kernel][0]
    (csrc / first).write_text("// changed\n")
    assert bench.csrc_digest(kernel) != digest and bench.profiled_traffic(kernel) is None
    os.remove(prof / f"{kernel}.txt")
    assert bench.profiled_traffic(kernel) is None

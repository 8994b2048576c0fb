"""The per-device cache behind the library's device state (error word address,
kernel attributes, SM count): compiled with g++ and driven with fake device
indices, so it runs without a GPU."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "exact_tiled_attention_36_b200", "csrc")


def test_per_device_cache(tmp_path):
    exe = tmp_path / "per_device_check"
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC,
                           os.path.join(HERE, "per_device_check.cpp"), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"


def test_library_keys_device_state_per_device():
    """Every per-process cache of device state in the host code goes through PerDevice."""
    src = open(os.path.join(CSRC, "fa_api.cu")).read()
    # the one call_once left is the driver's tensor-map encoder, which is process-wide
    assert src.count("std::call_once") == 1 and "cuTensorMapEncodeTiled" in src
    for needle in ("static bool attr_ok", "static int launch_regs", "static int counts["):
        assert needle not in src, needle
    assert src.count("fa::PerDevice<") >= 3
    noalloc = open(os.path.join(CSRC, "fa_noalloc.cu")).read()
    assert "fa::PerDevice<void*>" in noalloc

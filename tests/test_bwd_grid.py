"""The backward's choice of grid order (key tile fastest or heaviest first), a host rule
in csrc/bwd_grid.h: compiled with g++ and checked on the shapes it was measured on, so it
runs without a GPU."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "exact_tiled_attention_36_b200", "csrc")


def test_bwd_grid_order_rule(tmp_path):
    exe = tmp_path / "bwd_grid_check"
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", CSRC, os.path.join(HERE, "bwd_grid_check.cpp"),
                           "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"


def test_library_takes_the_rule_from_the_header():
    src = open(os.path.join(CSRC, "fa_api.cu")).read()
    assert '#include "bwd_grid.h"' in src
    assert src.count("fa::bwd_key_tile_fastest(") == 1

"""The window tiling plan (host code, csrc/plan.cpp) checked on the CPU: a small
C++ checker is compiled against plan.cpp and run on the workload shapes, the
edge shapes of the GPU tests and seeded random geometries. Every window must be
covered exactly once by in-bounds, non-wrapping TMA boxes at 8-row aligned tile
offsets."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from sparse_window_attention_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_window_attention_b200", "csrc")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("plan") / "plan_check")
    cuda_inc = "/usr/local/cuda/include"
    subprocess.run([gxx, "-std=c++17", "-O2", "-I", cuda_inc, "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "native", "plan_check.cpp"), os.path.join(CSRC, "plan.cpp"),
                    "-o", exe], check=True)
    return exe


def run(exe, geos):
    text = "".join(" ".join(str(x) for x in g) + "\n" for g in geos)
    out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout.split("\n")
    return out[: len(geos)]


def test_workload_shapes_every_shift(checker):
    geos = []
    for name, wl in synth.WORKLOADS.items():
        for sh in synth.SHIFT_CYCLES[name]:
            geos.append((*wl.grid, *wl.window, *sh))
    for g, r in zip(geos, run(checker, geos)):
        assert r.startswith("ok"), (g, r)


def test_edge_shapes(checker):
    geos = [
        (4, 8, 12, 2, 4, 4, 1, 2, 3),        # wraps in t, y and x: eight window types
        (1, 4, 80, 1, 1, 40, 0, 1, 17),      # single-row boxes
        (5, 7, 9, 5, 7, 9, 2, 3, 4),         # window = grid, odd extents, all axes shifted
        (5, 24, 32, 5, 6, 8, 2, 3, 4),       # full-T windows with a temporal shift
        (1, 64, 256, 1, 64, 64, 0, 5, 33),   # 4096-token windows
        (21, 60, 104, 21, 15, 26, 3, 7, 13), # video windows, every axis wrapping
        (1, 128, 144, 1, 4, 4, 0, 2, 2),     # 1152 small windows
    ]
    for g, r in zip(geos, run(checker, geos)):
        assert r.startswith("ok"), (g, r)


def test_random_geometries(checker):
    rng = np.random.default_rng(2024)
    geos = []
    while len(geos) < 300:
        w = [int(rng.integers(1, 9)), int(rng.integers(1, 17)), int(rng.integers(1, 33))]
        n = [int(rng.integers(1, 4)), int(rng.integers(1, 5)), int(rng.integers(1, 5))]
        grid = [a * b for a, b in zip(w, n)]
        if grid[0] * grid[1] * grid[2] > 40000:
            continue
        shift = [int(rng.integers(0, g)) for g in grid]
        geos.append((*grid, *w, *shift))
    res = run(checker, geos)
    supported = 0
    for g, r in zip(geos, res):
        assert r.startswith("ok") or r == "unsupported", (g, r)
        supported += r.startswith("ok")
    assert supported >= 290  # the plan's limits are only reached by unusual shapes

"""The fused pre-pass's index arithmetic (csrc/pool_route_fused.cu) checked on the
CPU: the real box planner and the per-box run and cell builders are compiled
into tests/native/fused_check.cu with nvcc and run on the workload shapes, the
GPU tests' shapes and seeded random geometries."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from sparse_window_attention_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    nvcc = shutil.which("nvcc") or ("/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else None)
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("fused") / "fused_check")
    subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                    os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "native", "fused_check.cu"), "-o", exe],
                   check=True)
    return exe


def run(exe, geos):
    text = "".join(" ".join(str(x) for x in g) + "\n" for g in geos)
    return subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout.split("\n")[: len(geos)]


def _geo(wl, shift):
    return (*wl.grid, *wl.window, *shift, *wl.pool, wl.d, 0 if wl.dtype == "bf16" else 1)


def test_workload_and_test_shapes(checker):
    from tests.test_gpu_parity import FUSED

    geos = []
    for name, wl in synth.WORKLOADS.items():
        if all(p > 0 for p in wl.pool) and wl.routed_k > 0:
            geos += [_geo(wl, sh) for sh in synth.SHIFT_CYCLES[name]]
    geos += [_geo(wl, wl.shift) for wl in FUSED]
    for g, r in zip(geos, run(checker, geos)):
        assert r.startswith("ok"), (g, r)


def test_random_geometries(checker):
    rng = np.random.default_rng(77)
    geos = []
    while len(geos) < 200:
        pool = [int(rng.integers(1, 5)), int(rng.integers(1, 7)), int(rng.integers(1, 9))]
        grid = [p * int(rng.integers(1, 6)) for p in pool]
        win = []
        for g in grid:
            divs = [x for x in range(1, g + 1) if g % x == 0]
            win.append(int(rng.choice(divs)))
        if grid[0] * grid[1] * grid[2] > 60000 or all(g == w for g, w in zip(grid, win)):
            continue
        shift = [int(rng.integers(0, g)) for g in grid]
        geos.append((*grid, *win, *shift, *pool, 128, int(rng.integers(0, 2))))
    res = run(checker, geos)
    ok = 0
    for g, r in zip(geos, res):
        assert r.startswith("ok") or r == "unsupported", (g, r)
        ok += r.startswith("ok")
    assert ok >= 150

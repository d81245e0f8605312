"""The megakernel's smem stage arena, simulated on the host.

The producer's allocation (StageAlloc) and its rule for when a new stage may
be written (stage_blocked) are host/device code in the library's shared
header; tests/arena_sim.cpp drives them with mixed stage sizes (tensor-core
stages of 16..128 token rows and stream stages of 1..64 KB) and an in-order
consumer, and checks every reservation against the stages still in flight.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "event_driven_persistent_b200", "csrc")


@pytest.fixture(scope="module")
def sim(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path_factory.mktemp("arena") / "arena_sim")
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, os.path.join(HERE, "arena_sim.cpp"), "-o", exe],
                   check=True)
    return exe


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_no_stage_overwrites_one_in_flight(sim, seed):
    r = subprocess.run([sim, str(seed), "200000", "0"], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout


def test_oldest_stage_rule_alone_is_caught(sim):
    """Checking only the oldest in-flight stage lets a wrapped allocation
    overwrite newer stages; the simulation must see it."""
    bad = 0
    for seed in range(1, 6):
        r = subprocess.run([sim, str(seed), "200000", "1"], capture_output=True, text=True)
        bad += r.returncode == 2
    assert bad > 0

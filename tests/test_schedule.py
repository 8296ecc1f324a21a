"""The forward's and backward's work schedules, checked on the host (CPU).

tests/host/sched_check.cu includes the very functions the kernels use to
pick their tiles (fwd_sched.cuh, bwd_sched.cuh, host-callable), walks every
work item of 2916 problems, at every head-group size from one head to all
of them, and compares the tiles visited with the visibility rule written row
by row.  The group sizes the launches choose must lie in that range.  The problems cover ragged and unequal
query and key counts, all masks, random block masks with empty rows and
columns, and per-sequence lengths.  It also checks the order the
deterministic backward adds dQ in.  Planted mistakes in copies of the
headers must make it fail."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_65_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

pytestmark = pytest.mark.skipif(not os.path.exists(NVCC), reason="needs nvcc")


def _build(out_dir, include_dir=CSRC):
    exe = os.path.join(out_dir, "sched_check")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2",
                    "-I", os.path.join(ROOT, "include"), "-I", include_dir,
                    os.path.join(ROOT, "tests", "host", "sched_check.cu"), "-o", exe], check=True)
    return exe


def test_schedules_visit_exactly_the_needed_tiles(tmp_path):
    r = subprocess.run([_build(str(tmp_path))], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")


MUTANTS = [
    ("fwd_causal_bound", "fwd_sched.cuh", "return min(qt * BM + BM - 1, it.Lq - 1) + it.off;",
     "return min(qt * BM + BM - 2, it.Lq - 1) + it.off;"),
    ("bwd_add_rank", "bwd_sched.cuh", "  return (uint32_t)j;", "  return (uint32_t)(j > 0 ? j - 1 : 0);"),
    ("bwd_item_map", "bwd_sched.cuh", "  it.j = r / gsize;", "  it.j = r % gsize;"),
    ("fwd_single_tile_items", "fwd_sched.cuh", "  it.q0 = p.tiles_per_item * c;", "  it.q0 = 2 * c;"),
]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_check_catches_planted_schedule_mistake(mutant, tmp_path):
    name, header, old, new = mutant
    inc = tmp_path / "inc"
    inc.mkdir()
    for f in os.listdir(CSRC):
        if f.endswith((".cuh", ".h")):
            shutil.copy(os.path.join(CSRC, f), inc / f)
    src = (inc / header).read_text()
    assert src.count(old) == 1, f"anchor of {name} not found exactly once"
    (inc / header).write_text(src.replace(old, new))
    r = subprocess.run([_build(str(tmp_path), str(inc))], capture_output=True, text=True, timeout=300)
    assert r.returncode == 1 and "MISMATCH" in r.stdout, f"{name} not caught: {r.stdout}"

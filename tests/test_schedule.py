"""The host's grid choice for the round-robin decode attention (csrc/schedule.h), compiled with
g++ on the CPU. CTA c takes units c, c + grid, ...; with fixed-length splits the grid must share
no factor with the split count S (else CTA c meets only the split indices congruent to c modulo
gcd(grid, S)), as long as that costs the busiest CTA at most one more unit."""
import math
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "memory_bounded_kv_b200", "csrc", "schedule.h")

DRIVER = r"""
#include <cstdio>
#include "schedule.h"
int main() {
    int units, slots, S, fixed;
    while (std::scanf("%d %d %d %d", &units, &slots, &S, &fixed) == 4)
        std::printf("%d\n", kvb::rr_grid(units, slots, S, fixed != 0));
    return 0;
}
"""


@pytest.fixture(scope="module")
def rr_grid(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not found")
    d = tmp_path_factory.mktemp("schedule")
    src, exe = d / "driver.cpp", d / "driver"
    src.write_text(DRIVER)
    subprocess.check_call([gxx, "-std=c++17", "-O1", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])

    def run(cases):
        text = "".join(f"{u} {s} {S} {int(f)}\n" for u, s, S, f in cases)
        out = subprocess.run([str(exe)], input=text, capture_output=True, text=True, check=True).stdout
        return [int(x) for x in out.split()]
    return run


def busiest(units, grid):
    return -(-units // grid)


def test_measured_cases(rr_grid):
    # memento workload, 64 x 8 rows on 296 resident CTAs: splits of 768 (S = 23) keep their grid;
    # splits of 1280 (S = 14) leave 287 CTAs (7 modulo 14) for 285; splits of 512 (S = 34) 296 -> 295
    assert rr_grid([(512 * 23, 296, 23, True), (512 * 14, 296, 14, True), (512 * 34, 296, 34, True)]) == \
        [295, 285, 295]
    # equal splits (split_len 0) and one split keep the plain round robin: the long-context
    # workload's 4 x 8 rows x 64 splits on 293 CTAs of 7 units, the layer's 256 rows on 256 CTAs
    assert rr_grid([(4 * 8 * 64, 296, 64, False), (256, 296, 1, True)]) == [293, 256]


def test_properties_over_a_sweep(rr_grid):
    cases = [(units, slots, S, fixed) for units in (7, 64, 300, 1000, 4096, 7168, 11776)
             for slots in (8, 148, 296) for S in (1, 2, 3, 6, 14, 23, 34) for fixed in (False, True)]
    grids = rr_grid(cases)
    for (units, slots, S, fixed), g in zip(cases, grids):
        per = -(-units // slots)
        plain = -(-units // per)
        assert 1 <= g <= min(units, slots), (units, slots, S, fixed, g)
        if not fixed or S < 2 or per < 4:
            assert g == plain
            continue
        # never more than one extra unit for the busiest CTA
        assert busiest(units, g) <= per + 1, (units, slots, S, g)
        if g != plain:
            assert math.gcd(g, S) == 1 and math.gcd(plain, S) > 1
            # the nearest coprime count below the plain grid
            assert all(math.gcd(x, S) > 1 for x in range(g + 1, plain))

"""Host split-plan rule (csrc/plan_host.h), compiled with g++ into a tiny probe: chunks are
multiples of the granule, cover every row's tokens exactly once, and fit one wave of workers
whenever the rows allow it."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = r'''
#include <cstdio>
#include <cstdlib>
#include <vector>
#include "plan_host.h"
int main(int argc, char** argv) {
    int batch = atoi(argv[1]), s_q = atoi(argv[2]), units = atoi(argv[3]), granule = atoi(argv[4]);
    std::vector<int> lens(batch);
    for (int b = 0; b < batch; ++b) lens[b] = atoi(argv[5 + b]);
    int c = mla::plan_chunk(lens.data(), batch, s_q, units, granule);
    printf("%d %lld\n", c, mla::plan_count(lens.data(), batch, s_q, c));
    return 0;
}
'''


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("plan")
    src = d / "probe.cpp"
    src.write_text(SRC)
    exe = d / "probe"
    subprocess.run([gxx, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "mla_latent_kv_24_b200", "csrc"),
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)

    def run(lens, s_q, units, granule):
        out = subprocess.run([str(exe), str(len(lens)), str(s_q), str(units), str(granule), *map(str, lens)],
                             check=True, capture_output=True, text=True).stdout.split()
        return int(out[0]), int(out[1])
    return run


def _rows(lens, s_q):
    return [int(L) - s_q + j + 1 for L in lens for j in range(s_q)]


@pytest.mark.parametrize("lens,s_q,units", [
    ([131072] * 4, 1, 74), ([4096] * 8, 1, 74), ([64], 1, 74), ([1], 1, 74), ([1, 2, 3], 2, 74),
    (list(range(1024, 1024 + 128 * 200, 200)), 2, 74), ([65536] * 32, 2, 74), ([5000, 7, 130000], 1, 3),
    ([1024 + 997 * i % 31744 for i in range(64)], 2, 74), ([300] * 200, 1, 74),
])
@pytest.mark.parametrize("granule", [32, 128])
def test_plan_rule(probe, lens, s_q, units, granule):
    chunk, count = probe(lens, s_q, units, granule)
    rows = _rows(lens, s_q)
    assert chunk % granule == 0 and chunk >= granule
    assert count == sum(-(-r // chunk) for r in rows)
    # every token of every row lands in exactly one chunk [i*chunk, min(len, (i+1)*chunk))
    for r in rows:
        covered = sum(min(r, (i + 1) * chunk) - i * chunk for i in range(-(-r // chunk)))
        assert covered == r
    if len(rows) <= units:
        assert count <= units, "a plan that fits one wave exists but was not chosen"
        if chunk > granule:   # and no smaller chunk would still fit
            assert sum(-(-r // (chunk - granule)) for r in rows) > units
    else:
        # more rows than workers: three quarters of the even split of all tokens, on the granule
        round_up = lambda c: max(granule, -(-c // granule) * granule)
        even = round_up(-(-sum(rows) // units))
        if even < round_up(max(rows)):
            assert chunk == round_up(even * 3 // 4)

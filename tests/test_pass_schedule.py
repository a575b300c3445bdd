"""The prefill kernels' pass schedule (`PassIter` in jl_prefill_common.cuh),
checked on the CPU pair by pair.

The schedule is the fused form of the pages' inclusion-exclusion merge
(techwalker explainer §四, bittide paper summary §3.2): every causal pair of a
query tile must be scored exactly once, with standard RoPE when it is local
(q - k < w_local) and with remapped RoPE otherwise; the band modes of the
unfused three-call path cover the local pairs only, all in one class.  The
struct is compiled here for the host, straight from the header text (its
`__device__` qualifiers defined away), and its passes are replayed against
the per-pair definition.  The kernels also rely on every remote pass coming
before every local one (one Q variant in shared memory at a time)."""
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "long_context_attention_bifocal_b200", "csrc", "jl_prefill_common.cuh")

K_STD, K_REM = 0, 1
BAND_NONE, BAND_STD, BAND_REM = 0, 1, 2
MASK_NONE, MASK_FAR, MASK_LOCAL = 0, 1, 2
INT_MAX = 2**31 - 1

HARNESS = r"""
#include <climits>
#include <cstdio>
#define __device__
constexpr int kBN = %(kBN)s;
%(body)s
int main() {
  int i, w, band;
  while (std::scanf("%%d %%d %%d", &i, &w, &band) == 3) {
    PassIter it;
    it.begin(i, w, band);
    while (!it.done()) {
      std::printf("%%d %%d %%d ", it.kind(), it.mask(), it.j);
      it.next();
    }
    std::printf("\n");
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def schedule(tmp_path_factory):
    src = open(HDR).read()
    kbn = re.search(r"constexpr int kBN = (\d+);", src).group(1)
    start = src.index("enum : int { kStd = 0, kRem = 1 };")
    end = src.index("};", src.index("struct PassIter {")) + 2
    d = tmp_path_factory.mktemp("passiter")
    (d / "h.cpp").write_text(HARNESS % {"kBN": kbn, "body": src[start:end]})
    exe = d / "h"
    subprocess.run(["g++", "-O1", "-std=c++17", str(d / "h.cpp"), "-o", str(exe)], check=True)

    def run(cases):
        inp = "".join(f"{i} {w} {b}\n" for i, w, b in cases)
        out = subprocess.run([str(exe)], input=inp, capture_output=True, text=True,
                             check=True).stdout.splitlines()
        res = []
        for line in out:
            v = [int(x) for x in line.split()]
            res.append([tuple(v[n:n + 3]) for n in range(0, len(v), 3)])
        return res
    return run, int(kbn)


def coverage(passes, i, w, bn):
    """Per causal pair of query tile i: how many passes score it, and with
    which RoPE class (-1 where none does).  Every pass must score at least one
    pair (a pass that scores none is a wasted tile of work)."""
    q = bn * i + np.arange(bn)[:, None]
    k = np.arange(bn * (i + 1))[None, :]
    count = np.zeros((bn, bn * (i + 1)), np.int32)
    cls = np.full((bn, bn * (i + 1)), -1, np.int32)
    for kind, mask, j in passes:
        kk = k[:, bn * j:bn * (j + 1)]
        dist = q - kk
        cov = dist >= 0
        if mask == MASK_FAR:
            cov &= dist >= w
        elif mask == MASK_LOCAL:
            cov &= dist < w
        assert cov.any(), ("empty pass", i, w, kind, mask, j)
        count[:, bn * j:bn * (j + 1)] += cov
        cls[:, bn * j:bn * (j + 1)][cov] = kind
    causal = (q - k) >= 0
    local = causal & ((q - k) < w)
    return count, cls, causal, local


TILES = (0, 1, 2, 5, 17, 40)
WINDOWS = (0, 1, 5, 127, 128, 129, 255, 256, 300, 2048, 5000, INT_MAX)


def test_every_causal_pair_once_in_its_class(schedule):
    run, bn = schedule
    cases = [(i, w, BAND_NONE) for i in TILES for w in WINDOWS]
    for (i, w, _), passes in zip(cases, run(cases)):
        count, cls, causal, local = coverage(passes, i, w, bn)
        assert (count[causal] == 1).all(), (i, w)
        assert (count[~causal] == 0).all(), (i, w)
        assert (cls[local] == K_STD).all() and (cls[causal & ~local] == K_REM).all(), (i, w)
        kinds = [p[0] for p in passes]
        # all remote passes first: the kind switches at most once, rem -> std
        assert kinds == sorted(kinds, reverse=True), (i, w, kinds)
        # each kv tile at most once per phase
        for kind in (K_STD, K_REM):
            js = [p[2] for p in passes if p[0] == kind]
            assert len(js) == len(set(js)) and js == sorted(js), (i, w)


@pytest.mark.parametrize("band,kind", [(BAND_STD, K_STD), (BAND_REM, K_REM)])
def test_band_modes_cover_the_window_in_one_class(schedule, band, kind):
    run, bn = schedule
    cases = [(i, w, band) for i in TILES for w in WINDOWS]
    for (i, w, _), passes in zip(cases, run(cases)):
        count, cls, causal, local = coverage(passes, i, w, bn)
        assert (count[local] == 1).all(), (i, w, band)
        assert (count[~local] == 0).all(), (i, w, band)
        assert (cls[local] == kind).all(), (i, w, band)


def test_tile_counts_at_the_long_workload(schedule):
    """At w_local = 2048 a query tile deep in a long prompt makes 1 diagonal,
    15 local, 1 boundary (visited twice) and i - 16 far tiles: i + 2 passes."""
    run, bn = schedule
    i = 1023
    (passes,) = run([(i, 2048, BAND_NONE)])
    assert len(passes) == i + 2
    assert sum(1 for p in passes if p[0] == K_REM) == i - 15
    assert sum(1 for p in passes if p[1] != MASK_NONE) == 2

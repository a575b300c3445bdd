"""Every prefill parity case can fail on a wrong bifocal rule (CPU, no GPU).

For each case of the GPU parity tests, on its exact inputs and rows, the oracle
is run under the correct rule and under each near miss that changes the result
for that shape (needles.variants): the group size off by one either way, the
window edge off by one either way, and no remap.  Each near miss must fail the
gate the GPU test applies (max-abs 2e-2 on O, or 1e-2 on the LSE; 5e-2 for the
peaky cases).  So a kernel
with any of these mistakes cannot pass the GPU tests, whatever else it gets
right.  The full-size cases are checked on the needle rows of their first and
last kv heads, a subset of the rows the GPU test compares: failing on a subset
of rows fails the max-abs and LSE gates on the whole set.

The plain full-size cases (the configurations' own inputs, no needles) are not
listed: their near-uniform attention keeps every near miss inside the gates,
which is why each of them has a needle twin.
"""
import numpy as np
import pytest

import needles
import prefill_cases as C
from long_context_attention_bifocal_b200 import workloads as W


@pytest.fixture(scope="module")
def mutants(oracle_mod, tmp_path_factory):
    d = str(tmp_path_factory.mktemp("group_mutants"))
    return {n: needles.build_mutant(oracle_mod, n, d) for n in needles.GROUP_MUTANTS}


def _check_variants(orc, mutants, q, k, v, rows, kw, what, min_variants=1,
                    lse_abs=needles.parity.LSE_ABS):
    A = [W.to_oracle_array(x) for x in (q, k, v)]
    rb, rq, rh = rows
    ref_o, ref_l = orc.bifocal_rows(*A, rb, rq, rh, **kw)
    L = q.shape[1]
    vs = needles.variants(orc, L, kw["w_local"], kw["w_pretrained"])
    assert len(vs) >= min_variants, f"{what}: only {sorted(vs)} apply"
    passed = []
    for name, (mut, vk) in vs.items():
        o2 = orc if mut is None else mutants[mut]
        o, l = o2.bifocal_rows(*A, rb, rq, rh, rope_base=kw["rope_base"], **vk)
        if not needles.gate_fails(o, l, ref_o, ref_l, lse_abs=lse_abs):
            passed.append(name)
    assert not passed, f"{what}: near misses {passed} pass the gates"
    return sorted(vs)


@pytest.mark.parametrize("case", C.SMALL, ids=[C.small_id(c) for c in C.SMALL])
def test_small_case_fails_every_near_miss(oracle_mod, mutants, case):
    orc = oracle_mod.default()
    q, k, v, kw = C.small_inputs(orc, case)
    B, L, Hq = q.shape[0], q.shape[1], q.shape[2]
    bb, qq, hh = np.meshgrid(np.arange(B), np.arange(L), np.arange(Hq), indexing="ij")
    rows = tuple(x.ravel().astype(np.int32) for x in (bb, qq, hh))
    G = orc.group_size(L, kw["w_pretrained"])
    # cases where no near miss changes anything: one token, or a window over
    # every pair with G > 1 (then only G + 1 would, and it cannot: no remote pair)
    trivial = L == 1 or kw["w_local"] >= L
    names = _check_variants(orc, mutants, q, k, v, rows, kw, C.small_id(case),
                            min_variants=0 if trivial else 3)
    if G > 1 and not trivial:
        assert "no_remap" in names


def _full_rows(nd, Hkv, Hq):
    group = Hq // Hkv
    keep = [n for n in nd if n[1] // group in (0, Hkv - 1)]
    return C.needle_rows(keep, 1, 0, Hq)


@pytest.mark.parametrize("name", C.FULL)
def test_full_size_needles_fail_every_near_miss(oracle_mod, mutants, name):
    orc = oracle_mod.default()
    q, k, v, kw, nd = C.needle_inputs(orc, name)
    cfg = W.PREFILL[name]
    rows = _full_rows(nd, cfg["Hkv"], cfg["Hq"])
    names = _check_variants(orc, mutants, q, k, v, rows, kw, name, min_variants=1)
    G = orc.group_size(cfg["L"], cfg["w_pretrained"])
    want = {"G_plus_1"} | ({"no_remap", "G_minus_1", "w_local_minus_1", "w_local_plus_1"}
                           if G > 1 else set())
    assert want <= set(names), (name, names)


@pytest.mark.parametrize("name", sorted(C.PEAKY))
def test_peaky_needles_fail_every_near_miss(oracle_mod, mutants, name):
    orc = oracle_mod.default()
    q, k, v, kw, nd = C.needle_inputs(orc, name, qk_scale=C.PEAKY[name])
    cfg = W.PREFILL[name]
    rows = _full_rows(nd, cfg["Hkv"], cfg["Hq"])
    names = _check_variants(orc, mutants, q, k, v, rows, kw, name, min_variants=5,
                            lse_abs=C.PEAKY_LSE_ABS)
    assert {"no_remap", "G_minus_1", "G_plus_1", "w_local_minus_1",
            "w_local_plus_1"} <= set(names)


def test_plain_full_size_inputs_cannot_tell_the_rules_apart(oracle_mod):
    """Why the needle twins exist: on the 8B/128K configuration's own inputs,
    sampled rows under plain causal RoPE stay within the gates of the bifocal
    result (checked on a few rows of one kv head; needles.py has the reason)."""
    orc = oracle_mod.default()
    q, k, v, kw = C.full_inputs("qwen3_8b_L131072")
    A = [W.to_oracle_array(x) for x in (q, k, v)]
    rq = np.array([4096, 65536, 131071, 100000], np.int32)
    rb = np.zeros_like(rq)
    rh = np.zeros_like(rq)
    ref_o, ref_l = orc.bifocal_rows(*A, rb, rq, rh, **kw)
    o, l = orc.bifocal_rows(*A, rb, rq, rh, w_local=131072,
                            w_pretrained=kw["w_pretrained"], rope_base=kw["rope_base"])
    assert not needles.gate_fails(o, l, ref_o, ref_l)

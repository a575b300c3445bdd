"""Bifocal prefill on the GPU (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import parity
import prefill_cases as C
from long_context_attention_bifocal_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run_prefill(jl, q, k, v, flags=0, **kw):
    out, lse = jl.bifocal_prefill(q.to(DEV), k.to(DEV), v.to(DEV), flags=flags, **kw)
    jl.check_device_status()
    return out, lse


def params(cfg):
    return dict(w_local=cfg["w_local"], w_pretrained=cfg["w_pretrained"],
                rope_base=cfg["rope_base"])


# ----------------------------------------------------------- fp32 tiny ----
def test_tiny_f32_L512_all_rows(jl, oracle_mod):
    cfg = W.PREFILL["tiny_f32_L512"]
    q, k, v = W.prefill_inputs(cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                               dtype="f32", value_scale=cfg["value_scale"], seed=cfg["seed"])
    out, lse = run_prefill(jl, q, k, v, **params(cfg))
    ref_o, ref_l = oracle_mod.default().bifocal_all_rows(
        q.numpy(), k.numpy(), v.numpy(), **params(cfg))
    parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l,
                 max_abs=parity.F32_MAX_ABS, lse_abs=parity.F32_MAX_ABS, what="tiny f32 L512")


def test_tiny_f32_L128_is_plain_rope(jl, oracle_mod):
    """L <= w_pretrained: G = 1, bitwise the non-bifocal kernel, and equal to the
    oracle (itself pinned to library causal RoPE attention)."""
    cfg = W.PREFILL["tiny_f32_L128"]
    q, k, v = W.prefill_inputs(cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                               dtype="f32", value_scale=cfg["value_scale"], seed=cfg["seed"])
    out, lse = run_prefill(jl, q, k, v, **params(cfg))
    out0, lse0 = run_prefill(jl, q, k, v, flags=jl.NO_BIFOCAL, **params(cfg))
    assert torch.equal(out, out0) and torch.equal(lse, lse0)
    ref_o, ref_l = oracle_mod.default().bifocal_all_rows(
        q.numpy(), k.numpy(), v.numpy(), **params(cfg))
    parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l,
                 max_abs=parity.F32_MAX_ABS, lse_abs=parity.F32_MAX_ABS, what="tiny f32 L128")


# ------------------------------------------- bf16, small, every row ----
# The cases (tests/prefill_cases.py) carry needles: keys planted so that a
# group size or window edge off by one, or a missing remap, fails the gates
# (shown on the CPU by test_parity_sensitivity.py).
SMALL = C.SMALL


@pytest.mark.parametrize("case", SMALL, ids=[C.small_id(c) for c in SMALL])
def test_bf16_small_all_rows(jl, oracle_mod, case):
    q, k, v, kw = C.small_inputs(oracle_mod.default(), case)
    out, lse = run_prefill(jl, q, k, v, **kw)
    ref_o, ref_l = oracle_mod.default().bifocal_all_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), **kw)
    parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l,
                 max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS, what=str(case))


@pytest.mark.parametrize("case", SMALL, ids=[C.small_id(c) for c in SMALL])
def test_bf16_small_all_rows_one_tile_kernel(jl, oracle_mod, case, monkeypatch):
    """The same cases on the one-query-tile kernel (the default takes two query
    heads per CTA whenever the group size is even)."""
    monkeypatch.setenv("JL_PREFILL_KERNEL", "one")
    test_bf16_small_all_rows(jl, oracle_mod, case)


@pytest.mark.parametrize("case", SMALL, ids=[C.small_id(c) for c in SMALL])
def test_bf16_small_keys_rotated_once(jl, oracle_mod, case):
    """The same cases with the opt-in mode that rotates the keys once per call
    into a workspace (JL_FLAG_ROTATE_KEYS_ONCE) instead of in the kernel."""
    q, k, v, kw = C.small_inputs(oracle_mod.default(), case)
    out, lse = run_prefill(jl, q, k, v, flags=jl.ROTATE_KEYS_ONCE, **kw)
    ref_o, ref_l = oracle_mod.default().bifocal_all_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), **kw)
    parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l,
                 max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS, what=str(case))


def test_bf16_explicit_softmax_scale(jl, oracle_mod):
    """A softmax scale given by the caller instead of 1/sqrt(D)."""
    q, k, v = W.prefill_inputs(1, 700, 4, 2, 128, dtype="bf16", value_scale=0.5, seed=12)
    kw = dict(w_local=150, w_pretrained=200, rope_base=1e6)
    out, lse = jl.bifocal_prefill(q.to(DEV), k.to(DEV), v.to(DEV), softmax_scale=0.05, **kw)
    jl.check_device_status()
    ref_o, ref_l = oracle_mod.default().bifocal_all_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), scale=0.05, **kw)
    parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l,
                 max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS, what="scale 0.05")


def test_bf16_g1_bitwise_plain(jl):
    """G = 1 takes exactly the non-bifocal path."""
    q, k, v = W.prefill_inputs(1, 777, 4, 2, 128, seed=7)
    kw = dict(w_local=100, w_pretrained=1024, rope_base=1e6)
    a = run_prefill(jl, q, k, v, **kw)
    b = run_prefill(jl, q, k, v, flags=jl.NO_BIFOCAL, **kw)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bf16_bifocal_differs_from_plain_when_g_gt_1(jl):
    """Sanity: with G > 1 and remote pairs, the remap changes the result."""
    q, k, v = W.prefill_inputs(1, 600, 2, 1, 128, value_scale=2.0, seed=8)
    kw = dict(w_local=64, w_pretrained=150, rope_base=1e4)
    a = run_prefill(jl, q, k, v, **kw)
    b = run_prefill(jl, q, k, v, flags=jl.NO_BIFOCAL, **kw)
    assert (a[0].float() - b[0].float()).abs().max().item() > 1e-2


def test_needs_no_workspace_and_repeats_bitwise(jl):
    """The keys are rotated inside the kernel: the call needs no workspace, and
    a workspace handed to it is neither needed nor written; repeated calls give
    identical bits."""
    assert jl.prefill_workspace_size(1, 900, 2, 128) == 0
    q, k, v = W.prefill_inputs(1, 900, 4, 2, 128, seed=9)
    kw = dict(w_local=128, w_pretrained=300, rope_base=1e6)
    a = run_prefill(jl, q, k, v, **kw)
    ws = torch.full((4096,), 7, dtype=torch.uint8, device=DEV)
    b = jl.bifocal_prefill(q.to(DEV), k.to(DEV), v.to(DEV), workspace=ws, **kw)
    jl.check_device_status()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert bool((ws == 7).all())


# ---------------------------------- full sizes, sampled rows per head ----
FULL = C.FULL


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(jl, oracle_mod, name):
    full_size_sampled_rows(jl, oracle_mod, name)


def test_full_size_sampled_rows_one_tile_kernel(jl, oracle_mod, monkeypatch):
    monkeypatch.setenv("JL_PREFILL_KERNEL", "one")
    full_size_sampled_rows(jl, oracle_mod, "qwen3_8b_L131072")


def full_size_sampled_rows(jl, oracle_mod, name):
    """The configuration's own inputs, 512 seeded rows per head plus the rows at
    the window edge, tile and group boundaries and the ends."""
    cfg = W.PREFILL[name]
    B, L, Hq = cfg["B"], cfg["L"], cfg["Hq"]
    q, k, v, kw = C.full_inputs(name)
    out, lse = run_prefill(jl, q, k, v, **kw)
    G = oracle_mod.default().group_size(L, cfg["w_pretrained"])
    rb, rq, rh = W.sample_rows(B, L, Hq, per_head=512, seed=cfg["seed"],
                               extra=C.edge_positions(L, G, cfg["w_local"]))
    ref_o, ref_l = oracle_mod.default().bifocal_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), rb, rq, rh, **kw)
    go, gl = parity.gather_rows(out, lse, rb, rq, rh)
    stats = parity.check(go, gl, ref_o, ref_l, max_abs=parity.BF16_MAX_ABS,
                         mean_abs=parity.BF16_MEAN_ABS, what=name)
    print(name, stats)
    if G == 1:
        out0, lse0 = run_prefill(jl, q, k, v, flags=jl.NO_BIFOCAL, **kw)
        assert torch.equal(out, out0) and torch.equal(lse, lse0)


def needle_case(jl, oracle_mod, name, qk_scale=None, lse_abs=parity.LSE_ABS, flags=0):
    """Full-size inputs with needles: the needle rows (each dominated by one
    key whose score is right only under the bifocal rule) and 16 seeded rows
    per head.  Besides the gates, the output must be far from the same
    kernel's plain-RoPE output (JL_FLAG_NO_BIFOCAL) wherever the two rules
    differ: at least ten times farther than it is from the oracle."""
    orc = oracle_mod.default()
    cfg = W.PREFILL[name]
    B, L, Hq = cfg["B"], cfg["L"], cfg["Hq"]
    q, k, v, kw, nd = C.needle_inputs(orc, name, qk_scale=qk_scale)
    out, lse = run_prefill(jl, q, k, v, flags=flags, **kw)
    rb, rq, rh = C.needle_rows(nd, B, L, Hq, per_head=16, seed=cfg["seed"])
    ref_o, ref_l = orc.bifocal_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), rb, rq, rh, **kw)
    go, gl = parity.gather_rows(out, lse, rb, rq, rh)
    stats = parity.check(go, gl, ref_o, ref_l, max_abs=parity.BF16_MAX_ABS,
                         mean_abs=parity.BF16_MEAN_ABS, lse_abs=lse_abs, what=f"{name} needles")
    n = len(nd)
    row_rel = (np.abs(go[:n] - ref_o[:n]).max(axis=1) /
               np.maximum(np.abs(ref_o[:n]).max(axis=1), 1e-30))
    print(name, "needles", n, stats, "needle-row relative max", float(row_rel.max()))
    assert row_rel.max() <= 0.05, f"{name}: needle-row relative error {row_rel.max():.3e}"
    G = orc.group_size(L, cfg["w_pretrained"])
    if G > 1:
        out0, lse0 = run_prefill(jl, q, k, v, flags=jl.NO_BIFOCAL, **kw)
        po, _ = parity.gather_rows(out0, lse0, rb, rq, rh)
        remote = np.array([x[2] - x[3] >= kw["w_local"] for x in nd])
        err = np.abs(go[:n] - ref_o[:n]).max(axis=1)[remote]
        dist = np.abs(go[:n] - po[:n]).max(axis=1)[remote]
        print(name, "distance to plain RoPE on remote needle rows: min", float(dist.min()),
              "error against the oracle: max", float(err.max()))
        assert dist.min() > 10 * err.max()
    return stats


@pytest.mark.parametrize("name", FULL)
def test_full_size_needles(jl, oracle_mod, name):
    needle_case(jl, oracle_mod, name)


@pytest.mark.parametrize("name", sorted(C.PEAKY))
def test_full_size_peaky(jl, oracle_mod, name):
    """q and k at four times the configurations' scale (scores with a standard
    deviation of ~4: a few dozen keys carry each row) plus needles; the LSE
    gate is prefill_cases.PEAKY_LSE_ABS (the reason is stated there)."""
    needle_case(jl, oracle_mod, name, qk_scale=C.PEAKY[name], lse_abs=C.PEAKY_LSE_ABS)


def test_full_size_needles_keys_rotated_once(jl, oracle_mod):
    """The 8B/128K needle case with the keys rotated once per call."""
    needle_case(jl, oracle_mod, "qwen3_8b_L131072", flags=jl.ROTATE_KEYS_ONCE)


def test_full_size_needles_one_tile_kernel(jl, oracle_mod, monkeypatch):
    monkeypatch.setenv("JL_PREFILL_KERNEL", "one")
    needle_case(jl, oracle_mod, "qwen3_8b_L131072")

"""Bifocal prefill on the GPU (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import parity
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
SMALL = [
    # (B, L, Hq, Hkv, w_pretrained, w_local, value_scale)
    (1, 1000, 4, 2, 300, 200, 0.5),    # G=4, ragged tail, window edge inside a tile
    (2, 640, 2, 1, 200, 37, 0.5),      # G=4, window narrower than a tile
    (1, 513, 2, 2, 100, 0, 0.5),       # every pair remote, G=6
    (1, 700, 2, 1, 100, 5000, 0.5),    # window covers every pair: plain RoPE
    (1, 1, 1, 1, 10, 2, 0.5),          # one token
    (1, 129, 2, 1, 64, 128, 0.5),      # G=3, window of exactly one tile
    (1, 2125, 4, 1, 1024, 256, 0.5),   # GQA 4, G=3
    (1, 1536, 2, 1, 512, 300, 1.0),    # sharper attention (scores 4x larger)
    (2, 700, 8, 2, 256, 100, 0.5),     # B=2, two kv heads of two head pairs (CTA order)
    (1, 600, 6, 2, 200, 64, 0.5),      # GQA 3: odd group, the one-tile kernel
    (2, 400, 3, 3, 128, 50, 0.5),      # multi-head (group 1), B=2
    (1, 4096, 2, 1, 16, 100, 0.5),     # G = 256: 256 keys share each remapped position
]


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}L{c[1]}H{c[2]}x{c[3]}wp{c[4]}wl{c[5]}s{c[6]}" for c in SMALL])
def test_bf16_small_all_rows(jl, oracle_mod, case):
    B, L, Hq, Hkv, wp, wl, sc = case
    q, k, v = W.prefill_inputs(B, L, Hq, Hkv, 128, dtype="bf16", value_scale=sc, seed=L)
    kw = dict(w_local=wl, w_pretrained=wp, rope_base=1e6)
    out, lse = run_prefill(jl, q, k, v, **kw)
    ref_o, ref_l = oracle_mod.default().bifocal_all_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), **kw)
    parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l,
                 max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS, what=str(case))


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}L{c[1]}H{c[2]}x{c[3]}wp{c[4]}wl{c[5]}s{c[6]}" for c in SMALL])
def test_bf16_small_all_rows_one_tile_kernel(jl, oracle_mod, case, monkeypatch):
    """The same cases on the one-query-tile kernel (the default takes two query
    heads per CTA whenever the group size is even)."""
    monkeypatch.setenv("JL_PREFILL_KERNEL", "one")
    test_bf16_small_all_rows(jl, oracle_mod, case)


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


def test_explicit_workspace_matches_library_scratch(jl):
    q, k, v = W.prefill_inputs(1, 900, 4, 2, 128, seed=9)
    kw = dict(w_local=128, w_pretrained=300, rope_base=1e6)
    a = run_prefill(jl, q, k, v, **kw)
    ws = torch.empty(jl.prefill_workspace_size(1, 900, 2, 128), dtype=torch.uint8, device=DEV)
    b = jl.bifocal_prefill(q.to(DEV), k.to(DEV), v.to(DEV), workspace=ws, **kw)
    jl.check_device_status()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ---------------------------------- full sizes, sampled rows per head ----
FULL = ["qwen3_1p7b_L65536", "qwen3_8b_L131072", "qwen3_4b_L16384", "qwen3_4b_L32768",
        "qwen3_4b_L49152", "qwen3_4b_L98304", "qwen3_4b_L131072"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(jl, oracle_mod, name):
    full_size_sampled_rows(jl, oracle_mod, name)


def test_full_size_sampled_rows_one_tile_kernel(jl, oracle_mod, monkeypatch):
    monkeypatch.setenv("JL_PREFILL_KERNEL", "one")
    full_size_sampled_rows(jl, oracle_mod, "qwen3_8b_L131072")


def full_size_sampled_rows(jl, oracle_mod, name):
    cfg = W.PREFILL[name]
    B, L, Hq, Hkv, D = cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"]
    q, k, v = W.prefill_inputs(B, L, Hq, Hkv, D, value_scale=cfg["value_scale"],
                               seed=cfg["seed"])
    kw = params(cfg)
    out, lse = run_prefill(jl, q, k, v, **kw)
    G = oracle_mod.default().group_size(L, cfg["w_pretrained"])
    wl = cfg["w_local"]
    extra = [0, 1, 127, 128, wl - 1, wl, wl + 1, L // 2, L - 2, L - 1]
    extra += [G * m for m in (1, 1000)] + [G * m - 1 for m in (1, 1000)]
    rb, rq, rh = W.sample_rows(B, L, Hq, per_head=512, seed=cfg["seed"], extra=extra)
    ref_o, ref_l = oracle_mod.default().bifocal_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), rb, rq, rh, **kw)
    go, gl = parity.gather_rows(out, lse, rb, rq, rh)
    stats = parity.check(go, gl, ref_o, ref_l, max_abs=parity.BF16_MAX_ABS,
                         mean_abs=parity.BF16_MEAN_ABS, what=name)
    print(name, stats)
    if G == 1:
        out0, lse0 = run_prefill(jl, q, k, v, flags=jl.NO_BIFOCAL, **kw)
        assert torch.equal(out, out0) and torch.equal(lse, lse0)

"""The unfused three-call formulation (A + B - C with the LogSumExp merge) on
the GPU against the fp64 oracle of the per-pair definition, and against the
fused kernel."""
import pytest
import torch

import parity
from long_context_attention_bifocal_b200 import workloads as W
from test_gpu_prefill import SMALL, params

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run_3pass(jl, q, k, v, **kw):
    out, lse = jl.bifocal_prefill_3pass(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
    jl.check_device_status()
    return out, lse


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}L{c[1]}H{c[2]}x{c[3]}wp{c[4]}wl{c[5]}s{c[6]}" for c in SMALL])
def test_3pass_small_all_rows(jl, oracle_mod, case):
    B, L, Hq, Hkv, wp, wl, sc = case
    q, k, v = W.prefill_inputs(B, L, Hq, Hkv, 128, dtype="bf16", value_scale=sc, seed=L)
    kw = dict(w_local=wl, w_pretrained=wp, rope_base=1e6)
    out, lse = run_3pass(jl, q, k, v, **kw)
    ref_o, ref_l = oracle_mod.default().bifocal_all_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), **kw)
    parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l,
                 max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS, what=str(case))


def test_3pass_empty_window_is_call_a(jl):
    """w_local = 0: no window, the result is call A alone, which is the fused
    kernel with every pair remote."""
    q, k, v = W.prefill_inputs(1, 900, 4, 2, 128, seed=12)
    kw = dict(w_local=0, w_pretrained=300, rope_base=1e6)
    a = run_3pass(jl, q, k, v, **kw)
    b = jl.bifocal_prefill(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
    jl.check_device_status()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_3pass_full_size_sampled_rows(jl, oracle_mod):
    name = "qwen3_8b_L131072"
    cfg = W.PREFILL[name]
    B, L, Hq, Hkv, D = cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"]
    q, k, v = W.prefill_inputs(B, L, Hq, Hkv, D, value_scale=cfg["value_scale"],
                               seed=cfg["seed"])
    kw = params(cfg)
    out, lse = run_3pass(jl, q, k, v, **kw)
    wl = cfg["w_local"]
    extra = [0, 1, wl - 1, wl, wl + 1, L - 1]
    rb, rq, rh = W.sample_rows(B, L, Hq, per_head=128, seed=cfg["seed"] + 1, extra=extra)
    ref_o, ref_l = oracle_mod.default().bifocal_rows(
        W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v), rb, rq, rh, **kw)
    go, gl = parity.gather_rows(out, lse, rb, rq, rh)
    stats = parity.check(go, gl, ref_o, ref_l, max_abs=parity.BF16_MAX_ABS,
                         mean_abs=parity.BF16_MEAN_ABS, what=name + " (3 calls)")
    print(name, "3 calls", stats)
    fo, fl = jl.bifocal_prefill(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
    jl.check_device_status()
    d = (fo.float() - out.float()).abs()
    print("fused vs three calls: max", d.max().item(), "mean", d.mean().item(),
          "lse max", (fl - lse).abs().max().item())
    assert d.max().item() < 2 * parity.BF16_MAX_ABS

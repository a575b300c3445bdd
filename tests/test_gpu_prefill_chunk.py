"""Chunked prefill against a cache (queries at positions q_offset + r, keys in
a cache rotated at their original positions) on the GPU against the fp64
oracle of the whole sequence."""
import numpy as np
import pytest
import torch

import parity
from long_context_attention_bifocal_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def unrotated_keys(cache, base):
    """K with R(k) K = cache, in fp64: the cache rotated back by -k theta_i
    (rotate-half pairs).  Handing these to the oracle makes it see exactly the
    cached keys once it applies RoPE itself."""
    x = cache.double().numpy()
    N, D = x.shape[1], x.shape[3]
    half = D // 2
    theta = float(base) ** (-2.0 * np.arange(half) / D)
    ang = -np.arange(N, dtype=np.float64)[:, None] * theta[None, :]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def run_case(jl, oracle_mod, B, p0, Lq, Hq, Hkv, wp, wl, rows_per_head=None, seed=0):
    D, Lt = 128, p0 + Lq
    cap = Lt + 64
    q_all, _, v = W.prefill_inputs(B, Lt, Hq, Hkv, D, value_scale=0.5, seed=seed)
    _, kc, _ = W.decode_inputs(B, Hq, Hkv, D, cap, seed=seed + 1)  # cache ~ N(0,1), rotated
    kc = (kc.float() * 0.5).to(torch.bfloat16)
    vc = torch.zeros((B, cap, Hkv, D), dtype=torch.bfloat16)
    vc[:, :Lt] = v
    kc[:, Lt:] = float("nan")  # slots past the sequence are never read
    vc[:, Lt:] = float("nan")
    q = q_all[:, p0:].contiguous()
    kw = dict(w_local=wl, w_pretrained=wp, rope_base=1e6)
    out, lse = jl.bifocal_prefill_chunk(q.to(DEV), kc.to(DEV), vc.to(DEV), p0, **kw)
    jl.check_device_status()
    if rows_per_head is None:
        rb, rq, rh = np.meshgrid(np.arange(B), np.arange(p0, Lt), np.arange(Hq), indexing="ij")
        rb, rq, rh = rb.ravel(), rq.ravel(), rh.ravel()
    else:
        rb, rq, rh = W.sample_rows(B, Lt, Hq, per_head=rows_per_head, seed=seed)
        keep = rq >= p0
        rb, rq, rh = rb[keep], rq[keep], rh[keep]
    k_raw = unrotated_keys(kc[:, :Lt], 1e6)
    ref_o, ref_l = oracle_mod.default().bifocal_rows(
        q_all.double().numpy(), k_raw, v.double().numpy(), rb, rq, rh, **kw)
    go, gl = parity.gather_rows(out, lse, rb, rq - p0, rh)
    return parity.check(go, gl, ref_o, ref_l, max_abs=parity.BF16_MAX_ABS,
                        mean_abs=parity.BF16_MEAN_ABS, what=f"chunk p0={p0} Lq={Lq}")


CASES = [
    # (B, q_offset, Lq, Hq, Hkv, w_pretrained, w_local)
    (1, 256, 300, 4, 2, 200, 100),    # G=3, window edge inside the chunk's tiles
    (2, 0, 700, 2, 1, 200, 37),       # no prefix: a plain prefill on a cache, G=4
    (1, 1024, 1, 8, 2, 300, 64),      # one new token (the decode shape), G=4
    (1, 512, 130, 4, 4, 1000, 5000),  # window covers every pair: plain RoPE
    (1, 128, 900, 4, 1, 64, 0),       # every pair remote, GQA 4, G=16
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}p{c[1]}L{c[2]}wp{c[5]}wl{c[6]}" for c in CASES])
def test_chunk_all_rows(jl, oracle_mod, case):
    B, p0, Lq, Hq, Hkv, wp, wl = case
    run_case(jl, oracle_mod, B, p0, Lq, Hq, Hkv, wp, wl, seed=p0 + Lq)


def test_chunk_8b_shape_sampled_rows(jl, oracle_mod):
    """8B heads, 32768 tokens of which the last 8192 are the chunk (G=2)."""
    stats = run_case(jl, oracle_mod, 1, 24576, 8192, 32, 8, 16384, 2048, rows_per_head=512,
                     seed=3)
    print("chunk 8B shape", stats)


def test_one_token_chunk_matches_decode(jl):
    """A one-token chunk at position p is the decode of that token over the
    same cache (the same G, from p + 1 keys)."""
    B, Hq, Hkv, D, p0 = 1, 32, 8, 128, 40960
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, p0 + 1, seed=5)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    kw = dict(w_local=2048, w_pretrained=16384, rope_base=1e6)
    a_out, a_lse = jl.bifocal_prefill_chunk(q.view(B, 1, Hq, D), kc, vc, p0, **kw)
    b_out, b_lse = jl.bifocal_decode(q, kc, vc, p0, **kw)
    jl.check_device_status()
    assert (a_out.view(B, Hq, D).float() - b_out.float()).abs().max().item() < 2e-3
    assert (a_lse.view(B, Hq) - b_lse).abs().max().item() < 1e-3

"""The prefill parity cases, shared by the GPU parity tests and the CPU test
that shows each case can fail on a wrong bifocal rule.

Every input here is a seeded draw from the workload generator; the cases with
needles (see needles.py) then overwrite a few keys so that the parity gates
can tell the bifocal rule from its near misses.  The GPU tests hand exactly
these bytes to the CUDA library and to the oracle; the sensitivity test
(test_parity_sensitivity.py) hands them to the oracle under the correct rule and
under each near miss, and checks that every near miss fails the gate its GPU
test applies.
"""
import numpy as np

import needles
from long_context_attention_bifocal_b200 import workloads as W

ROPE_BASE = 1e6

# Small cases, every row compared: (B, L, Hq, Hkv, w_pretrained, w_local, value_scale)
SMALL = [
    (1, 1000, 4, 2, 300, 200, 0.5),    # G=4, ragged tail, window edge inside a tile
    (2, 640, 2, 1, 200, 37, 0.5),      # G=4, window narrower than a tile
    (1, 513, 2, 2, 100, 0, 0.5),       # every pair remote, G=6
    (1, 700, 2, 1, 100, 5000, 0.5),    # window covers every pair: plain RoPE
    (1, 1, 1, 1, 10, 2, 0.5),          # one token
    (1, 129, 2, 1, 64, 128, 0.5),      # G=3, window of exactly one tile
    (1, 2125, 4, 1, 1024, 256, 0.5),   # GQA 4, G=3, window edge on a tile boundary
    (1, 1536, 2, 1, 512, 300, 1.0),    # sharper attention (scores 4x larger)
    (2, 700, 8, 2, 256, 100, 0.5),     # B=2, two kv heads of two head pairs (CTA order)
    (1, 600, 6, 2, 200, 64, 0.5),      # GQA 3: odd group, the one-tile kernel
    (2, 400, 3, 3, 128, 50, 0.5),      # multi-head (group 1), B=2
    (1, 4096, 2, 1, 16, 100, 0.5),     # G = 256: 256 keys share each remapped position
    (1, 1400, 4, 2, 400, 384, 1.0),    # G=4, scale 1.0, window edge on a tile boundary
    (1, 1300, 2, 1, 350, 451, 1.0),    # G=4, scale 1.0, window edge inside a tile
]


def small_id(c):
    return f"B{c[0]}L{c[1]}H{c[2]}x{c[3]}wp{c[4]}wl{c[5]}s{c[6]}"


def small_inputs(orc, case):
    """(q, k, v, kw) for a small case: Gaussian inputs seeded by L, with up to
    eight needles per (batch, kv head)."""
    B, L, Hq, Hkv, wp, wl, sc = case
    q, k, v = W.prefill_inputs(B, L, Hq, Hkv, 128, dtype="bf16", value_scale=sc, seed=L)
    kw = dict(w_local=wl, w_pretrained=wp, rope_base=ROPE_BASE)
    k, _ = needles.planted(orc, q, k, v, seed=L, **kw)
    return q, k, v, kw


# Full-size configurations (sampled rows).
FULL = ["qwen3_1p7b_L65536", "qwen3_8b_L131072", "qwen3_4b_L16384", "qwen3_4b_L32768",
        "qwen3_4b_L49152", "qwen3_4b_L98304", "qwen3_4b_L131072"]

# Peaky variants of two full-size shapes: q and k at 4x the configurations'
# scale (N(0,1) * 2: scores with a standard deviation of about 4, so a few
# dozen keys carry most of each row's weight), v as configured, plus needles.
PEAKY = {"qwen3_8b_L131072": 2.0, "qwen3_4b_L98304": 2.0}
# The LSE gate of the peaky cases.  Their rows' dominant scores are ~16-21 (the
# log-sum-exp ~20), and the tensor-core operands are the rotated q and k in
# bf16, whose 2^-9 relative rounding moves such scores, and so the LSE, by
# ~0.01-0.02 (a B200 measured 0.020-0.021); 1e-2 is the configurations' gate,
# set for their scores of ~0.25.  O stays within the 2e-2 / 2e-3 gates.  Every
# near miss moves the LSE of these rows by 1 to 3 (test_parity_sensitivity.py).
PEAKY_LSE_ABS = 0.05


def cfg_kw(cfg):
    return dict(w_local=cfg["w_local"], w_pretrained=cfg["w_pretrained"],
                rope_base=cfg["rope_base"])


def full_inputs(name):
    """The configuration's own inputs (no needles)."""
    cfg = W.PREFILL[name]
    q, k, v = W.prefill_inputs(cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                               value_scale=cfg["value_scale"], seed=cfg["seed"])
    return q, k, v, cfg_kw(cfg)


def needle_inputs(orc, name, qk_scale=None):
    """(q, k, v, kw, needle list) for a full-size configuration with needles;
    with qk_scale, q and k are drawn at that scale instead (the peaky cases)."""
    cfg = W.PREFILL[name]
    B, L, Hq, Hkv, D = cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"]
    q, k, v = W.prefill_inputs(B, L, Hq, Hkv, D, value_scale=cfg["value_scale"],
                               seed=cfg["seed"])
    if qk_scale is not None:
        q = W.gaussian(q.shape, seed=cfg["seed"], tid=1, scale=qk_scale)
        k = W.gaussian(k.shape, seed=cfg["seed"], tid=2, scale=qk_scale)
    kw = cfg_kw(cfg)
    k, nd = needles.planted(orc, q, k, v, seed=cfg["seed"], **kw)
    return q, k, v, kw, nd


def needle_rows(nd, B, L, Hq, *, per_head=0, seed=0, extra=()):
    """(b, q, h) rows: every needle row, plus `per_head` seeded random rows and
    the `extra` positions for every (b, h)."""
    rb = [n[0] for n in nd]
    rq = [n[2] for n in nd]
    rh = [n[1] for n in nd]
    if per_head or extra:
        b2, q2, h2 = W.sample_rows(B, L, Hq, per_head=per_head, seed=seed, extra=extra)
        rb += list(b2)
        rq += list(q2)
        rh += list(h2)
    return (np.asarray(rb, np.int32), np.asarray(rq, np.int32), np.asarray(rh, np.int32))


def edge_positions(L, G, wl):
    """Rows at the window edge, at tile and group boundaries, and at the ends."""
    x = [0, 1, 127, 128, wl - 1, wl, wl + 1, L // 2, L - 2, L - 1]
    x += [G * m for m in (1, 1000)] + [G * m - 1 for m in (1, 1000)]
    return x

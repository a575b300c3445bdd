"""Inputs on which the parity gates can tell bifocal attention from its near misses.

With the configurations' N(0,1)*0.5 values and D = 128 the scores have a
standard deviation of about 0.25, so attention over tens of thousands of keys is
nearly uniform and a wrong group size, a window edge off by one or a missing
remap moves the outputs by less than the 2e-2 / 1e-2 gates.  A *needle* fixes
that: for a chosen query row (b, h, q) one key k of its kv head is overwritten
with

    K[b, k, h_kv] = c * R(delta) * Q[b, q, h]

where delta is the pair's relative position under the bifocal rule
(q - k for a local pair, f(q) - f(k) = floor(q/G) - floor(k/G) for a remote
one; Jet-Long, techwalker explainer §二, bittide paper summary §3.1-§3.2).
Rotating both sides by their rule's positions then aligns the two vectors
exactly (R(a)^T R(b) = R(b - a)), so the pair's score is c * |Q|^2 * scale,
chosen to carry about 60% of the row's softmax mass.  Under any other rule the
relative angle is off by hundreds or thousands of positions, the high- and
mid-frequency rotation pairs decorrelate, the key's score falls to about half,
and its mass to a fraction of a percent: O moves by about 0.6 * |V_k - O|,
tens of times the gate.

Everything here is test infrastructure: the rotation, the position map and
the group size come from the oracle, and the planted bytes are handed to both
the CUDA library and the oracle.
"""
import numpy as np
import torch

import parity


# The group-size near misses are one-line edits of a copy of the oracle (the
# group size cannot always be moved by one through w_pretrained: at L = 4096 no
# window gives G = 255).
GROUP_MUTANTS = {
    "G_plus_1": ("return g < 1 ? 1 : g;", "return g + 1;"),
    "G_minus_1": ("return g < 1 ? 1 : g;", "return g - 1 < 1 ? 1 : g - 1;"),
}


def build_mutant(oracle_mod, name, workdir):
    """An Oracle built from a copy of oracle/jl_oracle.c with GROUP_MUTANTS[name]."""
    import os
    import subprocess
    before, after = GROUP_MUTANTS[name]
    src_path = os.path.join(os.path.dirname(oracle_mod.__file__), "jl_oracle.c")
    src = open(src_path).read()
    assert src.count(before) == 1, f"mutation site of {name} not found exactly once"
    c_path = os.path.join(workdir, f"{name}.c")
    so_path = os.path.join(workdir, f"lib_{name}.so")
    with open(c_path, "w") as f:
        f.write(src.replace(before, after))
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", c_path, "-o",
                    so_path, "-lm"], check=True)
    return oracle_mod.Oracle(so_path)


def variants(orc, L, w_local, w_pretrained):
    """Plausible mistakes in the bifocal rule.

    Returns {name: (mutant, kwargs)}: the oracle to use (None for the real one,
    else a key of GROUP_MUTANTS) and its w_local / w_pretrained arguments.
    Only the variants that change the result for this shape are listed: the
    group size off by one either way, the window edge off by one either way,
    and no remap at all (every pair at its original positions).
    """
    G = orc.group_size(L, w_pretrained)
    same = dict(w_local=w_local, w_pretrained=w_pretrained)
    out = {}
    has_remote = w_local < L  # some pair (L-1, k) with L-1-k >= w_local
    if G > 1 and has_remote:
        out["no_remap"] = (None, dict(w_local=L, w_pretrained=w_pretrained))
        out["G_minus_1"] = ("G_minus_1", same)
    if has_remote and L >= 2:
        out["G_plus_1"] = ("G_plus_1", same)
    # Moving the edge changes the class of the pairs at one distance: w_local - 1
    # for the narrower window, w_local for the wider one.  At distance 0 (the
    # diagonal) both rules give the same relative angle, so w_local = 0 and 1
    # are the same rule.
    if G > 1:
        if 2 <= w_local <= L:
            out["w_local_minus_1"] = (None, dict(w_local=w_local - 1, w_pretrained=w_pretrained))
        if 1 <= w_local <= L - 1:
            out["w_local_plus_1"] = (None, dict(w_local=w_local + 1, w_pretrained=w_pretrained))
    return out


def choose(B, L, Hq, Hkv, G, w_local, *, per_kv=8, seed=0):
    """Needle rows (b, h, q, k), at most per_kv of them per (b, kv head).

    Kinds, in order: the first remote pair of a row (q - k = w_local), the last
    local pair (q - k = w_local - 1), a remote key at the first and at the last
    position of a remap group, a window edge on a tile boundary (q and k both
    multiples of 128), a far key (k near q / 3), the very first key, and the
    diagonal when every pair is remote.  Key positions are distinct within a
    kv head, and each row (b, h, q) gets one needle; each kind draws its row
    up to 32 times to find an unused one.
    """
    rng = np.random.Generator(np.random.PCG64(seed + 0xD1CE))
    group = Hq // Hkv
    w = w_local

    def first_remote(q):
        return q - w

    def last_local(q):
        return q - (w - 1) if w >= 1 else -1

    def group_first(q):
        return ((q - w) // G) * G if G > 1 else -1

    def group_last(q):
        return ((q - w) // G) * G - 1 if G > 1 else -1

    def tile_edge(q):
        q = (q // 128) * 128
        return q - w if w % 128 == 0 else -1

    def far(q):
        return q // 3 if q // 3 <= q - w else -1

    def first_key(q):
        return 0 if q >= w else -1

    def diagonal(q):
        return q if w == 0 else -1

    kinds = [first_remote, last_local, group_first, group_last, tile_edge, far, first_key,
             diagonal]
    out = []
    for b in range(B):
        for hk in range(Hkv):
            used_k, used_q = set(), set()
            for kind in kinds:
                if len(used_k) >= per_kv:
                    break
                for _ in range(32):
                    q = int(rng.integers(0, L))
                    h = hk * group + int(rng.integers(0, group))
                    if kind is tile_edge:
                        q = (q // 128) * 128
                    k = kind(q)
                    if 0 <= k <= q and k not in used_k and (h, q) not in used_q:
                        used_k.add(k)
                        used_q.add((h, q))
                        out.append((b, h, q, k))
                        break
    return out


def plant(orc, q, k, needles, *, w_local, w_pretrained, rope_base, target_lse,
          scale=None, margin=0.5):
    """Overwrite k (a CPU tensor, modified in place) with the needles' keys.

    target_lse[i] is the row's log-sum-exp without its needle; the needle's
    score is set to target_lse[i] + margin, so that it carries a fixed share of
    the row's softmax mass (e^m / (1 + e^m), about 62% at m = 0.5).
    """
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    G = orc.group_size(L, w_pretrained)
    for i, (b, h, qp, kp) in enumerate(needles):
        qv = q[b, qp, h].double().numpy()
        if qp - kp < w_local:
            delta = qp - kp
        else:
            delta = orc.remap(qp, G) - orc.remap(kp, G)
        want = float(target_lse[i]) + margin
        c = want / (scale * float(qv @ qv))
        kv = c * orc.rope(qv, float(delta), rope_base)
        k[b, kp, h // group] = torch.from_numpy(kv).to(k.dtype)


def planted(orc, q, k, v, *, w_local, w_pretrained, rope_base, per_kv=8, seed=0,
            margin=0.5):
    """(k with needles, needle list) for the inputs q, k, v (CPU tensors)."""
    from long_context_attention_bifocal_b200 import workloads as W
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    G = orc.group_size(L, w_pretrained)
    nd = choose(B, L, Hq, Hkv, G, w_local, per_kv=per_kv, seed=seed)
    if not nd:
        return k, nd
    rb = np.array([n[0] for n in nd], np.int32)
    rh = np.array([n[1] for n in nd], np.int32)
    rq = np.array([n[2] for n in nd], np.int32)
    kw = dict(w_local=w_local, w_pretrained=w_pretrained, rope_base=rope_base)
    _, lse0 = orc.bifocal_rows(W.to_oracle_array(q), W.to_oracle_array(k),
                               W.to_oracle_array(v), rb, rq, rh, **kw)
    k2 = k.clone()
    plant(orc, q, k2, nd, target_lse=lse0, margin=margin, **kw)
    return k2, nd


def gate_fails(out, lse, ref_out, ref_lse, *, max_abs=parity.BF16_MAX_ABS,
               lse_abs=parity.LSE_ABS):
    """True iff (out, lse) would fail the max-abs or the LSE gate against
    (ref_out, ref_lse).  Failing on a subset of a test's rows implies failing
    on the whole set, for both of these gates."""
    return bool(np.abs(out - ref_out).max() > max_abs or np.abs(lse - ref_lse).max() > lse_abs)

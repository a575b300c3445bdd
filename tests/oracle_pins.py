"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with:
  * the worked example printed on the pages (G for L=65536, w=32768),
  * hand-derived closed forms (RoPE of basis vectors; a one-pair D=2 attention
    whose scores are |q||k|cos(angle) written out; Q=0 giving the running mean),
  * library routines on the special cases that reduce to plain attention
    (torch scaled_dot_product_attention on complex-exponential RoPE),
  * brute force with explicit D x D rotation matrices in the relative form
    R(pk - pq) and a materialised L x L mask,
  * the pages' three-call inclusion-exclusion merge built from library softmax
    / logsumexp calls,
  * invariants (rotation composition, remote-distance bound, prefill/decode
    agreement).
tests/test_oracle_pins.py runs them on the oracle; tests/test_oracle_mutants.py
runs them on deliberately broken copies and checks that every copy is caught.
"""
import math
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


# ---------------------------------------------------------------- helpers ----
def complex_rope(x, pos, base):
    """RoPE as complex multiplication: z_i = x_i + j x_{i+D/2} times e^{j pos theta_i}.

    x [..., D]; pos broadcastable to x[..., 0].  Written from the complex-number
    view of rotary embeddings, independently of the oracle's real-pair loop.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    h = D // 2
    freqs = base ** (-np.arange(h, dtype=np.float64) * 2.0 / D)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freqs
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag], axis=-1)


def sdpa_causal(qr, kr, v, scale):
    """Library causal attention on rotated q/k [L,D] (fp64) + logsumexp."""
    qt = torch.from_numpy(qr)[None, None]
    kt = torch.from_numpy(kr)[None, None]
    vt = torch.from_numpy(v)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, is_causal=True, scale=scale)[0, 0].numpy()
    L = qr.shape[0]
    s = torch.from_numpy(qr @ kr.T * scale)
    s = s.masked_fill(~torch.ones(L, L, dtype=torch.bool).tril(), float("-inf"))
    lse = torch.logsumexp(s, dim=-1).numpy()
    return o, lse


def masked_attention(qr, kr, v, allowed, scale):
    """softmax over `allowed` keys with library softmax/logsumexp; rows with no
    allowed key return O=0 and lse=-inf (an empty pass)."""
    s = torch.from_numpy(qr @ kr.T * scale)
    s = s.masked_fill(~torch.from_numpy(allowed), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    p = torch.softmax(s, dim=-1).nan_to_num(0.0)
    return (p @ torch.from_numpy(v)).numpy(), lse.numpy()


def rot_matrix(D, angle_pos, base):
    """Explicit D x D rotate-half RoPE matrix for a (possibly negative) position."""
    h = D // 2
    R = np.zeros((D, D))
    for i in range(h):
        a = angle_pos * base ** (-2.0 * i / D)
        R[i, i], R[i, i + h] = math.cos(a), -math.sin(a)
        R[i + h, i], R[i + h, i + h] = math.sin(a), math.cos(a)
    return R


def ceil_div(a, b):
    return -(-a // b)


def rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def run_rows(orc, q, k, v, **kw):
    """All rows of a single (b=0, heads) problem; q [L,Hq,D] fp64."""
    out, lse = orc.bifocal_all_rows(q[None], k[None], v[None], **kw)
    return out[0], lse[0]


# ------------------------------------------------------------------- pins ----
def pin_group_size_golden(orc):
    path = os.path.join(HERE, "golden", "group_size_example.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert rows, "empty golden file"
    for L, w, G in rows:
        got = orc.group_size(int(L), int(w))
        assert got == int(G), f"G({L},{w})={got}, pages say {G}"


def pin_remap_golden(orc):
    """The pages' merging example: at L = 65536 over a 32768-token window
    adjacent positions share one number, and the numbers fill the pretrained
    range exactly (every number in [0, 32768) used by two positions)."""
    path = os.path.join(HERE, "golden", "remap_example.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert rows and rows[0][0] == "L", "missing header"
    L, w = int(rows[0][1]), int(rows[0][2])
    G = orc.group_size(L, w)
    for x, fx in rows[1:]:
        got = orc.remap(int(x), G)
        assert got == int(fx), f"f({x})={got} at G={G}, pages say {fx}"
    counts = np.bincount([orc.remap(x, G) for x in range(L)])
    assert len(counts) == w and (counts == 2).all()


def pin_group_size_closed_form(orc):
    for L in (1, 2, 127, 128, 129, 512, 32767, 32768, 32769, 49152, 65536,
              98304, 131072, 131073):
        for w in (1, 3, 128, 2048, 32768):
            assert orc.group_size(L, w) == max(1, ceil_div(L, w)), (L, w)
    for x in range(0, 40):
        for G in (1, 2, 3, 4, 5):
            assert orc.remap(x, G) == x // G
    # G is the smallest integer keeping every remapped position inside the window
    for L in (100, 128, 129, 1000, 4097):
        for w in (7, 64, 128, 1024):
            G = orc.group_size(L, w)
            assert (L - 1) // G < w, (L, w, G)
            if G > 1:
                assert (L - 1) // (G - 1) >= w, (L, w, G)


def pin_rope_closed_form(orc):
    # D=4, base=1e4: theta_0 = 1, theta_1 = 1e4^(-1/2) = 0.01 (hand-derived)
    for p in (0.0, 1.0, 2.5, -3.0, 1000.0):
        e0 = orc.rope(np.array([1.0, 0, 0, 0]), p, 1e4)
        assert np.allclose(e0, [math.cos(p), 0, math.sin(p), 0], atol=1e-13), (p, e0)
        e1 = orc.rope(np.array([0, 1.0, 0, 0]), p, 1e4)
        assert np.allclose(e1, [0, math.cos(0.01 * p), 0, math.sin(0.01 * p)],
                           atol=1e-13), (p, e1)
        e2 = orc.rope(np.array([0, 0, 1.0, 0]), p, 1e4)
        assert np.allclose(e2, [-math.sin(p), 0, math.cos(p), 0], atol=1e-13), (p, e2)
    assert abs(orc.theta(1, 4, 1e4) - 0.01) < 1e-15
    assert abs(orc.theta(32, 128, 1e6) - 1e-3) < 1e-15


def pin_rope_complex_form(orc):
    x = rand(128, 3)
    for p in (0, 1, 17, 4095, 131071, 32767.0):
        assert np.allclose(orc.rope(x, p, 1e6), complex_rope(x, p, 1e6), atol=1e-9)
        assert np.allclose(orc.rope(x[:64], p, 1e4), complex_rope(x[:64], p, 1e4),
                           atol=1e-9)


def pin_rope_composition(orc):
    """R(a) R(d) x = R(a + d) x, d of either sign; and R(dk) R(k) K = R(f(k)) K."""
    rng = np.random.Generator(np.random.PCG64(5))
    x = rng.standard_normal(128)
    for _ in range(20):
        a = float(rng.integers(0, 131072))
        d = float(rng.integers(-131072, 131072))
        lhs = orc.rope(orc.rope(x, d, 1e6), a, 1e6)
        rhs = orc.rope(x, a + d, 1e6)
        assert np.allclose(lhs, rhs, atol=1e-9), (a, d)
    for G in (1, 2, 3, 4):
        for kk in (0, 1, 5, 1000, 131071):
            dk = orc.remap(kk, G) - kk
            lhs = orc.rope(orc.rope(x, kk, 1e6), dk, 1e6)
            assert np.allclose(lhs, orc.rope(x, kk // G, 1e6), atol=1e-9), (G, kk)
    # norm preserved
    assert abs(np.linalg.norm(orc.rope(x, 12345.0, 1e6)) - np.linalg.norm(x)) < 1e-12


def pin_remote_bound(orc):
    """Every remote pair has |f(q) - f(k)| <= w_pretrained (bittide §3.1)."""
    for L in (10, 64, 100, 129, 257):
        for w in (3, 7, 16, 64):
            for wl in (0, 1, 4, 16):
                G = orc.group_size(L, w)
                worst = 0
                for qq in range(L):
                    for kk in range(qq + 1):
                        if qq - kk >= wl:
                            worst = max(worst, abs(orc.remap(qq, G) - orc.remap(kk, G)))
                assert worst <= w, (L, w, wl, worst)
    for L, w in ((65536, 32768), (131072, 32768), (98304, 32768), (512, 128)):
        G = orc.group_size(L, w)
        assert orc.remap(L - 1, G) - orc.remap(0, G) <= w - 1


def pin_bruteforce(orc):
    """Oracle == explicit rotation matrices (relative form) + L x L mask."""
    cases = [  # (L, D, Hq, Hkv, w_pretrained, w_local, base)
        (23, 4, 1, 1, 5, 3, 1e4),     # G=5
        (40, 8, 2, 1, 10, 0, 1e4),    # G=4, all remote
        (33, 8, 2, 2, 11, 1, 500.0),  # G=3
        (64, 64, 4, 2, 32, 16, 1e4),  # G=2
        (17, 8, 1, 1, 17, 5, 1e4),    # G=1
        (48, 4, 1, 1, 16, 100, 1e4),  # w_local >= L
    ]
    for (L, D, Hq, Hkv, wp, wl, base) in cases:
        q = rand((L, Hq, D), 11 + L)
        k = rand((L, Hkv, D), 12 + L)
        v = rand((L, Hkv, D), 13 + L)
        scale = 1.0 / math.sqrt(D)
        G = max(1, ceil_div(L, wp))
        qi = np.arange(L)[:, None]
        ki = np.arange(L)[None, :]
        causal = ki <= qi
        local = causal & (qi - ki < wl)
        pq = np.where(local, qi, qi // G)       # effective query position per pair
        pk = np.where(local, ki, ki // G)       # effective key position per pair
        out, lse = run_rows(orc, q, k, v, w_local=wl, w_pretrained=wp,
                            rope_base=base)
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            S = np.full((L, L), -np.inf)
            for a in range(L):
                for b in range(a + 1):
                    # <R(pq)q, R(pk)k> = q^T R(pk - pq) k for rotations
                    S[a, b] = scale * q[a, h] @ rot_matrix(D, pk[a, b] - pq[a, b], base) @ k[b, hk]
            M = S.max(axis=1, keepdims=True)
            P = np.exp(S - M)
            Z = P.sum(axis=1, keepdims=True)
            ref_o = (P / Z) @ v[:, hk]
            ref_lse = (M + np.log(Z))[:, 0]
            assert np.allclose(out[:, h], ref_o, rtol=1e-11, atol=1e-12), (L, D, h)
            assert np.allclose(lse[h], ref_lse, rtol=1e-11, atol=1e-12), (L, D, h)


def pin_g1_is_plain_rope(orc):
    """L <= w_pretrained (G=1) gives plain causal RoPE attention for any w_local;
    so does w_local >= L for any G (bittide §3.1; techwalker Q1)."""
    for (L, D, wp, wl) in ((50, 16, 64, 7), (128, 64, 128, 32), (96, 8, 32, 96),
                           (96, 8, 32, 1000)):
        q, k, v = rand((L, 1, D), 21), rand((L, 1, D), 22), rand((L, 1, D), 23)
        scale = 1.0 / math.sqrt(D)
        pos = np.arange(L)
        ref_o, ref_lse = sdpa_causal(complex_rope(q[:, 0], pos, 1e4),
                                     complex_rope(k[:, 0], pos, 1e4), v[:, 0], scale)
        out, lse = run_rows(orc, q, k, v, w_local=wl, w_pretrained=wp, rope_base=1e4)
        assert np.allclose(out[:, 0], ref_o, atol=1e-12), (L, wp, wl)
        assert np.allclose(lse[0], ref_lse, atol=1e-12), (L, wp, wl)


def pin_all_remote(orc):
    """w_local = 0: every pair remote, i.e. causal attention at positions f(x)."""
    L, D, wp = 70, 16, 20
    G = ceil_div(L, wp)
    q, k, v = rand((L, 1, D), 31), rand((L, 1, D), 32), rand((L, 1, D), 33)
    pos = np.arange(L) // G
    ref_o, ref_lse = sdpa_causal(complex_rope(q[:, 0], pos, 1e4),
                                 complex_rope(k[:, 0], pos, 1e4), v[:, 0], 0.25)
    out, lse = run_rows(orc, q, k, v, w_local=0, w_pretrained=wp, rope_base=1e4)
    assert np.allclose(out[:, 0], ref_o, atol=1e-12)
    assert np.allclose(lse[0], ref_lse, atol=1e-12)


def pin_inclusion_exclusion(orc):
    """The pages' three calls merged with LSE weights equal the per-pair oracle:
    B = full causal at remapped positions, A = local band at original positions,
    C = local band at remapped positions; O = (e^B O_B - e^C O_C + e^A O_A) /
    (e^B - e^C + e^A)  (techwalker §四; bittide §3.2)."""
    for (L, D, wp, wl) in ((90, 16, 30, 10), (64, 8, 16, 1), (50, 8, 10, 60)):
        q, k, v = rand((L, 1, D), 41), rand((L, 1, D), 42), rand((L, 1, D), 43)
        scale = 1.0 / math.sqrt(D)
        G = ceil_div(L, wp)
        pos = np.arange(L)
        qs, ks = complex_rope(q[:, 0], pos, 1e4), complex_rope(k[:, 0], pos, 1e4)
        qr, kr = complex_rope(q[:, 0], pos // G, 1e4), complex_rope(k[:, 0], pos // G, 1e4)
        qi, ki = pos[:, None], pos[None, :]
        causal = ki <= qi
        band = causal & (qi - ki < wl)
        oB, lB = masked_attention(qr, kr, v[:, 0], causal, scale)
        oA, lA = masked_attention(qs, ks, v[:, 0], band, scale)
        oC, lC = masked_attention(qr, kr, v[:, 0], band, scale)
        m = lB[:, None]  # common shift for the exponentials
        wB, wA, wC = np.exp(lB - m[:, 0]), np.exp(lA - m[:, 0]), np.exp(lC - m[:, 0])
        den = wB - wC + wA
        ref_o = (wB[:, None] * oB - wC[:, None] * oC + wA[:, None] * oA) / den[:, None]
        ref_lse = m[:, 0] + np.log(den)
        out, lse = run_rows(orc, q, k, v, w_local=wl, w_pretrained=wp, rope_base=1e4)
        assert np.allclose(out[:, 0], ref_o, atol=1e-10), (L, wl)
        assert np.allclose(lse[0], ref_lse, atol=1e-10), (L, wl)


def pin_one_pair_closed_form(orc):
    """D=2 (one frequency, theta_0 = 1): score = scale*|q||k|cos(dp + a_q - a_k)
    with dp = q - k for local pairs and f(q) - f(k) for remote ones; V_k on the
    unit circle, so O and lse are sums of cosines written out by hand."""
    L, wp, wl, base = 37, 10, 4, 1e4
    G = ceil_div(L, wp)
    rng = np.random.Generator(np.random.PCG64(51))
    aq, ak, psi = rng.uniform(-3, 3, L), rng.uniform(-3, 3, L), rng.uniform(-3, 3, L)
    rq, rk = rng.uniform(0.5, 2.0, L), rng.uniform(0.5, 2.0, L)
    q = np.stack([rq * np.cos(aq), rq * np.sin(aq)], -1)[:, None]
    k = np.stack([rk * np.cos(ak), rk * np.sin(ak)], -1)[:, None]
    v = np.stack([np.cos(psi), np.sin(psi)], -1)[:, None]
    scale = 1.0 / math.sqrt(2)
    out, lse = run_rows(orc, q, k, v, w_local=wl, w_pretrained=wp, rope_base=base)
    for a in range(L):
        num = np.zeros(2)
        den = 0.0
        for b in range(a + 1):
            dp = (a - b) if (a - b) < wl else (a // G - b // G)
            s = scale * rq[a] * rk[b] * math.cos(dp + aq[a] - ak[b])
            w = math.exp(s)
            den += w
            num += w * np.array([math.cos(psi[b]), math.sin(psi[b])])
        assert np.allclose(out[a, 0], num / den, atol=1e-12), a
        assert abs(lse[0, a] - math.log(den)) < 1e-12, a


def pin_zero_query(orc):
    """Q = 0: all scores 0, so O[q] is the mean of V[0..q] and lse = ln(q+1)."""
    L, D = 300, 8
    q = np.zeros((L, 2, D))
    k, v = rand((L, 1, D), 61), rand((L, 1, D), 62)
    out, lse = run_rows(orc, q, k, v, w_local=7, w_pretrained=64, rope_base=1e4)
    csum = np.cumsum(v[:, 0], axis=0) / np.arange(1, L + 1)[:, None]
    for h in range(2):
        assert np.allclose(out[:, h], csum, atol=1e-12)
        assert np.allclose(lse[h], np.log(np.arange(1, L + 1)), atol=1e-12)


def pin_one_hot_values(orc):
    """V[k] = e_k (one-hot rows, D >= L): O[q] is the attention probability
    vector of row q itself, so it must be non-negative, sum to 1, vanish after
    key q (causal), and the first row must attend only to itself."""
    L, D = 12, 16
    v = np.zeros((L, 1, D))
    v[np.arange(L), 0, np.arange(L)] = 1.0
    q, k = rand((L, 2, D), 81, 2.0), rand((L, 1, D), 82, 2.0)
    for wl, wp in ((0, 4), (3, 4), (5, 100), (100, 2)):
        out, _ = run_rows(orc, q, k, v, w_local=wl, w_pretrained=wp, rope_base=1e4)
        for h in range(2):
            probs = out[:, h, :L]
            assert np.all(probs >= 0.0)
            assert np.allclose(probs.sum(axis=1), 1.0, atol=1e-12)
            assert np.all(np.triu(probs, 1) == 0.0)   # no key after the query
            assert np.all(out[:, h, L:] == 0.0)
            assert probs[0, 0] == 1.0


def pin_decode_matches_prefill(orc):
    """Decode over a cache of keys rotated at their original positions, with the
    dq/dk corrections (bittide §3.3), equals the per-pair prefill row L-1."""
    # (33, wp=16): pos + 1 = 33 gives G = 3 where pos alone would give 2
    for (L, D, Hq, Hkv, wp, wl) in ((61, 16, 4, 2, 16, 5), (40, 8, 2, 2, 50, 3),
                                    (100, 32, 2, 1, 25, 0), (77, 8, 1, 1, 10, 200),
                                    (33, 8, 2, 1, 16, 4)):
        q = rand((L, Hq, D), 71)
        k, v = rand((L, Hkv, D), 72), rand((L, Hkv, D), 73)
        cache = np.stack([np.stack([orc.rope(k[kk, h], kk, 1e6) for h in range(Hkv)])
                          for kk in range(L)])
        pos = L - 1
        o_dec, l_dec = orc.bifocal_decode(q[pos][None], cache[None], v[None], pos,
                                          w_local=wl, w_pretrained=wp, rope_base=1e6)
        rows_b = np.zeros(Hq, np.int32)
        rows_q = np.full(Hq, pos, np.int32)
        rows_h = np.arange(Hq, dtype=np.int32)
        o_pre, l_pre = orc.bifocal_rows(q[None], k[None], v[None], rows_b, rows_q,
                                        rows_h, w_local=wl, w_pretrained=wp,
                                        rope_base=1e6)
        assert np.allclose(o_dec[0], o_pre, atol=1e-11), (L, wl)
        assert np.allclose(l_dec[0], l_pre, atol=1e-11), (L, wl)



def pin_batch_independence(orc):
    """Batch elements are separate problems (the method is defined per
    sequence): a B = 3 call equals three B = 1 calls on the slices, for the
    prefill rows and for decode over caches whose capacity exceeds pos + 1.
    The decode slots past pos hold NaN, so reading any of them shows."""
    L, Hq, Hkv, D = 37, 4, 2, 8
    kw = dict(w_local=3, w_pretrained=10, rope_base=1e4)
    q, k, v = rand((3, L, Hq, D), 91), rand((3, L, Hkv, D), 92), rand((3, L, Hkv, D), 93)
    out, lse = orc.bifocal_all_rows(q, k, v, **kw)
    for b in range(3):
        o1, l1 = orc.bifocal_all_rows(q[b:b + 1], k[b:b + 1], v[b:b + 1], **kw)
        assert np.array_equal(out[b], o1[0]) and np.array_equal(lse[b], l1[0]), b
    pos, cap = 29, L + 5
    kc = np.full((3, cap, Hkv, D), np.nan)
    vc = np.full((3, cap, Hkv, D), np.nan)
    kc[:, :pos + 1], vc[:, :pos + 1] = k[:, :pos + 1], v[:, :pos + 1]
    o_dec, l_dec = orc.bifocal_decode(q[:, pos], kc, vc, pos, **kw)
    assert np.isfinite(o_dec).all() and np.isfinite(l_dec).all()
    for b in range(3):
        o1, l1 = orc.bifocal_decode(q[b:b + 1, pos], k[b:b + 1, :pos + 1],
                                    v[b:b + 1, :pos + 1], pos, **kw)
        assert np.array_equal(o_dec[b], o1[0]) and np.array_equal(l_dec[b], l1[0]), b



def _bf16_exact(x):
    """fp64 values that bf16 holds exactly, and their bf16 bit patterns
    (truncation of the fp32 bits; exact because the values are built that way)."""
    bits32 = x.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return bits32.view(np.float32).astype(np.float64), (bits32 >> 16).astype(np.uint16)


def pin_input_dtypes(orc):
    """The same values passed as bf16 bit patterns, fp32 or fp64 give the same
    result (every step is fp64; bf16 is the top half of an fp32 word), for the
    prefill rows and for decode.  Negative values, subnormal-free magnitudes
    from 2^-8 to 2^8."""
    L, Hq, Hkv, D = 29, 2, 1, 8
    rng = np.random.Generator(np.random.PCG64(97))
    def vals(shape):
        return rng.choice([-1.0, 1.0], shape) * np.exp2(rng.uniform(-8, 8, shape))
    (q, qb), (k, kb), (v, vb) = (_bf16_exact(vals(sh)) for sh in
                                 ((1, L, Hq, D), (1, L, Hkv, D), (1, L, Hkv, D)))
    kw = dict(w_local=4, w_pretrained=8, rope_base=1e4)
    o64, l64 = orc.bifocal_all_rows(q, k, v, **kw)
    for args in ((qb, kb, vb), (q.astype(np.float32), k.astype(np.float32), v.astype(np.float32))):
        o, l = orc.bifocal_all_rows(*args, **kw)
        assert np.array_equal(o, o64) and np.array_equal(l, l64), args[0].dtype
    pos = L - 1
    d64 = orc.bifocal_decode(q[:, pos], k, v, pos, **kw)
    for args in ((qb[:, pos], kb, vb),
                 (q[:, pos].astype(np.float32), k.astype(np.float32), v.astype(np.float32))):
        d = orc.bifocal_decode(*args, pos, **kw)
        assert np.array_equal(d[0], d64[0]) and np.array_equal(d[1], d64[1]), args[0].dtype



def pin_explicit_scale(orc):
    """Scores are linear in q (RoPE is a rotation), so an explicit softmax
    scale s equals the default 1/sqrt(D) applied to q * s * sqrt(D)."""
    L, Hq, Hkv, D, s = 33, 2, 1, 8, 0.05
    q, k, v = rand((1, L, Hq, D), 98), rand((1, L, Hkv, D), 99), rand((1, L, Hkv, D), 100)
    kw = dict(w_local=5, w_pretrained=10, rope_base=1e4)
    o1, l1 = orc.bifocal_all_rows(q, k, v, scale=s, **kw)
    o2, l2 = orc.bifocal_all_rows(q * (s * math.sqrt(D)), k, v, **kw)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)
    assert not np.allclose(o1, orc.bifocal_all_rows(q, k, v, **kw)[0], atol=1e-3)


ALL_PINS = [
    pin_group_size_golden, pin_remap_golden, pin_group_size_closed_form, pin_rope_closed_form,
    pin_rope_complex_form, pin_rope_composition, pin_remote_bound,
    pin_bruteforce, pin_g1_is_plain_rope, pin_all_remote,
    pin_inclusion_exclusion, pin_one_pair_closed_form, pin_zero_query,
    pin_one_hot_values, pin_decode_matches_prefill, pin_batch_independence,
    pin_input_dtypes, pin_explicit_scale,
]

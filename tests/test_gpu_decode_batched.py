"""Batched decode with one position per sequence (ragged lengths, a G per
sequence) on the GPU against the fp64 oracle, sequence by sequence."""
import pytest
import torch

import parity
from long_context_attention_bifocal_b200 import workloads as W
from test_gpu_decode import poison_tail

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = [
    # (positions, cap, Hq, Hkv, w_local, w_pretrained)
    ([0, 100, 3000, 40000, 131071], 131100, 32, 8, 2048, 32768),  # G 1,1,1,2,4
    ([5000, 5000, 5000], 6000, 8, 2, 0, 1000),                     # every key remote, G = 6
    ([17, 777, 2100], 2200, 16, 2, 5, 100),                        # GQA 8, G up to 22
    ([129], 200, 4, 4, 64, 32),                                    # B = 1, GQA 1
    ([3000, 77, 1500], 3100, 8, 1, 300, 700),                      # one kv head, GQA 8
    ([8191, 4000], 8192, 8, 2, 100, 16),                           # G = 512 and 251
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{len(c[0])}max{max(c[0])}" for c in CASES])
def test_decode_batched_matches_oracle(jl, oracle_mod, case):
    positions, cap, Hq, Hkv, wl, wp = case
    B, D = len(positions), 128
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, cap, seed=31 + B)
    for b, pos in enumerate(positions):  # NaN after each sequence's last key
        kc[b:b + 1] = poison_tail(kc[b:b + 1], pos)
        vc[b:b + 1] = poison_tail(vc[b:b + 1], pos)
    kw = dict(w_local=wl, w_pretrained=wp, rope_base=1e6)
    out, lse = jl.bifocal_decode_batched(q.to(DEV), kc.to(DEV), vc.to(DEV), positions, **kw)
    jl.check_device_status()
    orc = oracle_mod.default()
    for b, pos in enumerate(positions):
        ref_o, ref_l = orc.bifocal_decode(
            W.to_oracle_array(q[b:b + 1]), W.to_oracle_array(kc[b:b + 1, :pos + 1]),
            W.to_oracle_array(vc[b:b + 1, :pos + 1]), pos, **kw)
        parity.check(parity.to_np(out[b:b + 1]), parity.to_np(lse[b:b + 1]), ref_o, ref_l,
                     max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS,
                     what=f"sequence {b} at pos {pos}")


def test_decode_batched_equal_positions_match_single_call(jl):
    """All sequences at one position: the same result as jl_bifocal_decode
    within rounding (the two plans cut the keys differently)."""
    B, Hq, Hkv, D, pos = 3, 32, 8, 128, 65535
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, pos + 1, seed=41)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    kw = dict(w_local=2048, w_pretrained=32768, rope_base=1e6)
    a = jl.bifocal_decode_batched(q, kc, vc, [pos] * B, **kw)
    b = jl.bifocal_decode(q, kc, vc, pos, **kw)
    jl.check_device_status()
    assert (a[0].float() - b[0].float()).abs().max().item() < 2e-3
    assert (a[1] - b[1]).abs().max().item() < 1e-4


def test_decode_batched_many_sequences_two_waves(jl, oracle_mod):
    """80 short ragged sequences: the plan has more chunks than one wave of
    CTAs (two chunks per sequence at least), so the kernel runs in waves."""
    rng = __import__("numpy").random.Generator(__import__("numpy").random.PCG64(5))
    positions = [int(x) for x in rng.integers(0, 4000, size=80)]
    B, Hq, Hkv, D, cap = len(positions), 8, 2, 128, 4000
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, cap, seed=77)
    for b, pos in enumerate(positions):
        kc[b:b + 1] = poison_tail(kc[b:b + 1], pos)
        vc[b:b + 1] = poison_tail(vc[b:b + 1], pos)
    kw = dict(w_local=512, w_pretrained=1024, rope_base=1e6)
    out, lse = jl.bifocal_decode_batched(q.to(DEV), kc.to(DEV), vc.to(DEV), positions, **kw)
    jl.check_device_status()
    orc = oracle_mod.default()
    for b, pos in enumerate(positions):
        ref_o, ref_l = orc.bifocal_decode(
            W.to_oracle_array(q[b:b + 1]), W.to_oracle_array(kc[b:b + 1, :pos + 1]),
            W.to_oracle_array(vc[b:b + 1, :pos + 1]), pos, **kw)
        parity.check(parity.to_np(out[b:b + 1]), parity.to_np(lse[b:b + 1]), ref_o, ref_l,
                     max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS,
                     what=f"sequence {b} at pos {pos}")

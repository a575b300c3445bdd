"""jl_bifocal_decode_noalloc: the decode entry point that allocates nothing.

Some callers cannot allocate device memory -- an engine whose pool owns every
device byte, or a decode loop that cannot take an allocation's implicit
synchronisation.  This entry point keeps its split partials in a fixed array
compiled into the library instead of a caller workspace.  The GPU test calls it
through the C ABI on five cases, twice each in a row (every call reuses the array
the one before it filled), and compares each result with the fp64 oracle and
with jl_bifocal_decode's.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import parity
from long_context_attention_bifocal_b200 import workloads as W

FAKE = 0x10000


def test_noalloc_rejects_sizes_beyond_its_array():
    """Validation needs no GPU: 64 x 64 heads at 131072 tokens need ~17M floats."""
    import long_context_attention_bifocal_b200 as jl
    lib = jl.load()
    rc = lib.jl_bifocal_decode_noalloc(FAKE, FAKE, FAKE, 131071, 131072, FAKE, FAKE, 64, 64, 8,
                                       128, 2048, 32768, 1e6, 0, None)
    assert rc == 2  # JL_ERR_UNSUPPORTED
    assert b"fixed" in lib.jl_last_error()
    assert lib.jl_bifocal_decode_noalloc(None, FAKE, FAKE, 5, 10, FAKE, FAKE, 1, 8, 2, 128, 16,
                                         64, 1e6, 0, None) == 1  # null pointer


def _noalloc(lib, stream, q, kc, vc, pos, cap, B, Hq, Hkv, wl, wp):
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.bfloat16, device=q.device)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=q.device)
    rc = lib.jl_bifocal_decode_noalloc(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), pos, cap, out.data_ptr(),
        lse.data_ptr(), B, Hq, Hkv, 128, wl, wp, 1e6, 0, stream)
    assert rc == 0, lib.jl_last_error()
    torch.cuda.synchronize()
    return out, lse


# (B, Hq, Hkv, pos, cap, w_local, w_pretrained, seed, qk_scale, gate)
# Head groups of 4, 2 and 3 run the kernel's three instances (four, two and one
# query heads per CTA).  The last case scales q and the cache by 3 (scores with a
# standard deviation of ~9, a few keys carry each row): there a group size off
# by one or a missing remap moves O by ~1 and more, and the gate is 0.1 because
# bf16 operands move scores of ~40 by ~0.05.
CASES = [
    (1, 32, 8, 20000, 20064, 2048, 4096, 31, 1.0, parity.BF16_MAX_ABS),   # G = 5
    (1, 32, 8, 131071, 131072, 2048, 32768, 32, 1.0, parity.BF16_MAX_ABS),  # G = 4
    (1, 16, 8, 4999, 5000, 512, 8192, 33, 1.0, parity.BF16_MAX_ABS),      # G = 1, group 2
    (2, 12, 4, 30000, 30016, 0, 8192, 34, 1.0, parity.BF16_MAX_ABS),      # all remote, group 3
    (1, 8, 2, 39999, 40000, 1000, 16384, 35, 3.0, 0.1),                   # peaked, G = 3
]


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_decode_on_consecutive_calls(oracle_mod):
    """Each case twice in a row through the C ABI: against the fp64 oracle at
    the bf16 gates, and against jl_bifocal_decode (the tensor-core kernel with
    a caller workspace).  The calls follow one another on one stream, so each
    reuses the array the previous one filled."""
    import long_context_attention_bifocal_b200 as jl
    lib = jl.load()
    dev = torch.device("cuda", 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    orc = oracle_mod.default()
    for (B, Hq, Hkv, pos, cap, wl, wp, seed, sc, gate) in CASES:
        q, kc, vc = W.decode_inputs(B, Hq, Hkv, 128, cap, seed=seed)
        if sc != 1.0:
            q, kc = (q.float() * sc).to(torch.bfloat16), (kc.float() * sc).to(torch.bfloat16)
        ref_o, ref_l = orc.bifocal_decode(W.to_oracle_array(q), W.to_oracle_array(kc),
                                          W.to_oracle_array(vc), pos, w_local=wl,
                                          w_pretrained=wp, rope_base=1e6)
        q, kc, vc = q.to(dev), kc.to(dev), vc.to(dev)
        mma_o, mma_l = jl.bifocal_decode(q, kc, vc, pos, w_local=wl, w_pretrained=wp,
                                         rope_base=1e6)
        what = f"noalloc B={B} Hq={Hq} Hkv={Hkv} pos={pos} w_local={wl}"
        for call in range(2):
            out, lse = _noalloc(lib, stream, q, kc, vc, pos, cap, B, Hq, Hkv, wl, wp)
            mean = parity.BF16_MEAN_ABS if gate == parity.BF16_MAX_ABS else None
            lse_gate = parity.LSE_ABS if gate == parity.BF16_MAX_ABS else gate
            parity.check(parity.to_np(out), parity.to_np(lse), ref_o, ref_l, max_abs=gate,
                         mean_abs=mean, lse_abs=lse_gate, what=f"{what} call {call} vs oracle")
            parity.check(parity.to_np(out), parity.to_np(lse), parity.to_np(mma_o),
                         parity.to_np(mma_l), max_abs=gate, mean_abs=mean, lse_abs=lse_gate,
                         what=f"{what} call {call} vs jl_bifocal_decode")

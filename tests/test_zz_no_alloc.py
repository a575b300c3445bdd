"""jl_bifocal_decode_noalloc: the decode entry point that allocates nothing.

Some callers cannot allocate device memory -- an engine whose pool owns every
device byte, or a decode loop that cannot take an allocation's implicit
synchronisation.  This entry point keeps its split partials in a fixed array
compiled into the library instead of a caller workspace.  The GPU test calls it
through the C ABI twice in a row (a second, larger call reuses the array the
first one filled) and compares each result with jl_bifocal_decode's.

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


@pytest.mark.gpu
def test_noalloc_matches_decode_on_two_calls():
    import long_context_attention_bifocal_b200 as jl
    lib = jl.load()
    dev = torch.device("cuda", 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    cases = [  # (B, Hq, Hkv, pos, cap, w_local, w_pretrained, seed)
        (1, 32, 8, 20000, 20064, 2048, 4096, 31),
        (1, 32, 8, 131071, 131072, 2048, 32768, 32),
    ]
    for (B, Hq, Hkv, pos, cap, wl, wp, seed) in cases:
        q, kc, vc = (t.to(dev) for t in W.decode_inputs(B, Hq, Hkv, 128, cap, seed=seed))
        ref_o, ref_l = jl.bifocal_decode(q, kc, vc, pos, w_local=wl, w_pretrained=wp,
                                         rope_base=1e6)
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        rc = lib.jl_bifocal_decode_noalloc(
            q.data_ptr(), kc.data_ptr(), vc.data_ptr(), pos, cap, out.data_ptr(),
            lse.data_ptr(), B, Hq, Hkv, 128, wl, wp, 1e6, 0, stream)
        assert rc == 0, lib.jl_last_error()
        torch.cuda.synchronize()
        parity.check(parity.to_np(out), parity.to_np(lse), parity.to_np(ref_o),
                     parity.to_np(ref_l), max_abs=parity.BF16_MAX_ABS,
                     mean_abs=parity.BF16_MEAN_ABS, what=f"noalloc pos={pos}")

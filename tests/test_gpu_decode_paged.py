"""Batched decode over a paged cache on the GPU: bit for bit the contiguous
batched call over the same keys, and the fp64 oracle sequence by sequence."""
import numpy as np
import pytest
import torch

import parity
from long_context_attention_bifocal_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def page_cache(kc, vc, positions, page_size, *, spare=3, seed=0):
    """Copies contiguous caches [B, cap, Hkv, D] into shuffled pages of a pool.

    Returns (k_pages, v_pages, block_table) on the host.  Sequence b gets
    ceil((pos_b + 1) / page_size) pages drawn without replacement from the pool;
    the pool has `spare` pages nobody owns.  Rows past pos_b, spare pages and
    block-table entries past a sequence's last page are poisoned (NaN, -1): the
    kernel must read none of them."""
    B, _, Hkv, D = kc.shape
    need = [(p + page_size) // page_size for p in positions]
    num_pages = sum(need) + spare
    max_pages = max(need) + 2
    rng = np.random.Generator(np.random.PCG64(seed))
    order = rng.permutation(num_pages)
    kp = torch.full((num_pages, page_size, Hkv, D), float("nan"), dtype=kc.dtype)
    vp = torch.full((num_pages, page_size, Hkv, D), float("nan"), dtype=vc.dtype)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b, pos in enumerate(positions):
        for i in range(need[b]):
            pg = int(order[nxt])
            nxt += 1
            table[b, i] = pg
            lo = i * page_size
            hi = min(lo + page_size, pos + 1)
            kp[pg, :hi - lo] = kc[b, lo:hi]
            vp[pg, :hi - lo] = vc[b, lo:hi]
    return kp, vp, table


CASES = [
    # (positions, page_size, Hq, Hkv, w_local, w_pretrained)
    ([0, 100, 3000, 40000, 70001], 16, 32, 8, 2048, 32768),    # G 1,1,1,2,3; far_end unaligned
    ([5000, 4097, 777], 64, 8, 2, 0, 1000),                    # every key remote
    ([17, 777, 2100], 256, 16, 2, 5, 100),                     # GQA 8, G up to 22
    ([129], 32, 4, 4, 64, 32),                                 # B = 1, GQA 1
    ([15, 16, 31, 32], 16, 8, 8, 3, 8),                        # page edges
]


def _ids(c):
    return f"B{len(c[0])}max{max(c[0])}page{c[1]}"


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_decode_paged_equals_contiguous_and_oracle(jl, oracle_mod, case):
    positions, ps, Hq, Hkv, wl, wp = case
    B, D = len(positions), 128
    cap = max(positions) + 1
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, cap, seed=61 + B)
    kp, vp, table = page_cache(kc, vc, positions, ps, seed=ps)
    kw = dict(w_local=wl, w_pretrained=wp, rope_base=1e6)
    qd = q.to(DEV)
    out_p, lse_p = jl.bifocal_decode_paged(qd, kp.to(DEV), vp.to(DEV), table.to(DEV), positions,
                                           **kw)
    jl.check_device_status()
    out_c, lse_c = jl.bifocal_decode_batched(qd, kc.to(DEV), vc.to(DEV), positions, **kw)
    jl.check_device_status()
    assert torch.equal(out_p, out_c)
    assert torch.equal(lse_p, lse_c)
    orc = oracle_mod.default()
    for b, pos in enumerate(positions):
        ref_o, ref_l = orc.bifocal_decode(
            W.to_oracle_array(q[b:b + 1]), W.to_oracle_array(kc[b:b + 1, :pos + 1]),
            W.to_oracle_array(vc[b:b + 1, :pos + 1]), pos, **kw)
        parity.check(parity.to_np(out_p[b:b + 1]), parity.to_np(lse_p[b:b + 1]), ref_o, ref_l,
                     max_abs=parity.BF16_MAX_ABS, mean_abs=parity.BF16_MEAN_ABS,
                     what=f"sequence {b} at pos {pos}")


def test_decode_paged_no_bifocal_flag(jl):
    positions, ps = [40000, 9000], 128
    B, Hq, Hkv, D = 2, 32, 8, 128
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, max(positions) + 1, seed=71)
    kp, vp, table = page_cache(kc, vc, positions, ps, seed=3)
    kw = dict(w_local=2048, w_pretrained=8192, rope_base=1e6, flags=jl.NO_BIFOCAL)
    out_p, lse_p = jl.bifocal_decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV),
                                           positions, **kw)
    out_c, lse_c = jl.bifocal_decode_batched(q.to(DEV), kc.to(DEV), vc.to(DEV), positions, **kw)
    jl.check_device_status()
    assert torch.equal(out_p, out_c)
    assert torch.equal(lse_p, lse_c)


def test_decode_paged_bad_block_table_entry_is_reported(jl):
    """An entry outside [0, num_pages) is not followed (the kernel reads page
    0 instead) and the call is reported through the device status word; the
    next call is unaffected."""
    positions, ps = [300, 200], 16
    B, Hq, Hkv, D = 2, 8, 2, 128
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, max(positions) + 1, seed=81)
    kp, vp, table = page_cache(kc, vc, positions, ps, seed=5)
    kw = dict(w_local=64, w_pretrained=128, rope_base=1e6)
    bad = table.clone()
    bad[1, 3] = kp.shape[0]  # one past the pool
    qd, kpd, vpd = q.to(DEV), kp.to(DEV), vp.to(DEV)
    jl.bifocal_decode_paged(qd, kpd, vpd, bad.to(DEV), positions, **kw)
    with pytest.raises(jl.JetLongError):
        jl.check_device_status()
    out_p, lse_p = jl.bifocal_decode_paged(qd, kpd, vpd, table.to(DEV), positions, **kw)
    jl.check_device_status()
    out_c, lse_c = jl.bifocal_decode_batched(qd, kc.to(DEV), vc.to(DEV), positions, **kw)
    jl.check_device_status()
    assert torch.equal(out_p, out_c)


def test_decode_paged_full_size_ragged(jl):
    """Eight sequences up to 131072 keys in 256-key pages: bit for bit the
    contiguous batched call (which the oracle pins at these sizes)."""
    positions = [16383, 32767, 49151, 65535, 81919, 98303, 114687, 131071]
    B, Hq, Hkv, D, ps = 8, 32, 8, 128, 256
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    cap = max(positions) + 1
    q = torch.randn((B, Hq, D), generator=g, device=DEV).to(torch.bfloat16)
    kc = torch.randn((B, cap, Hkv, D), generator=g, device=DEV).to(torch.bfloat16)
    vc = torch.randn((B, cap, Hkv, D), generator=g, device=DEV).to(torch.bfloat16)
    need = [(p + ps) // ps for p in positions]
    num_pages = sum(need)
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(9))
    table = torch.full((B, max(need)), -1, dtype=torch.int32)
    kp = torch.empty((num_pages, ps, Hkv, D), dtype=torch.bfloat16, device=DEV)
    vp = torch.empty_like(kp)
    nxt = 0
    for b, pos in enumerate(positions):
        for i in range(need[b]):
            pg = int(perm[nxt])
            nxt += 1
            table[b, i] = pg
            kp[pg] = kc[b, i * ps:(i + 1) * ps]
            vp[pg] = vc[b, i * ps:(i + 1) * ps]
    kw = dict(w_local=2048, w_pretrained=32768, rope_base=1e6)
    out_p, lse_p = jl.bifocal_decode_paged(q, kp, vp, table.to(DEV), positions, **kw)
    out_c, lse_c = jl.bifocal_decode_batched(q, kc, vc, positions, **kw)
    jl.check_device_status()
    assert torch.equal(out_p, out_c)
    assert torch.equal(lse_p, lse_c)

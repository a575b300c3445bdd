"""Seeded synthetic workloads for dynamic bifocal RoPE attention.

This module generates inputs only: Gaussian samples, scaled and rounded to the
storage dtype.  It holds none of the method's arithmetic (no RoPE, no position
map, no group size), so both the CUDA library's tests and the fp64 oracle can
draw the same bytes from it.

The pages evaluate Qwen3-1.7B/4B/8B at up to 128K tokens with a 32768-token
pretrained window (techwalker explainer §五; bittide summary §4).  They give no
head shapes, so the shapes here are the standard Qwen3 attention shapes; the
values are N(0,1) (times 0.5 for the prefill workloads).  No dataset or weight is
involved.

Decode caches hold keys already rotated at their original positions.  A key
rotated by an orthogonal RoPE matrix from an isotropic Gaussian is again an
isotropic Gaussian, so the cache is sampled directly as N(0,1); that has the
same distribution as rotating N(0,1) raw keys and needs no RoPE here.

Generation is chunked along the sequence axis; every chunk has its own
torch CPU generator seeded from (seed, tensor id, batch, chunk), so the bytes
are the same for any thread count and any machine.
"""
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np
import torch

_CHUNK = 4096  # tokens per independently seeded chunk


def _chunk_seed(seed: int, tid: int, b: int, c: int) -> int:
    x = (seed * 0x9E3779B97F4A7C15 + tid * 0xBF58476D1CE4E5B9
         + b * 0x94D049BB133111EB + c * 0x2545F4914F6CDD1D + 0x632BE59BD9B4E019)
    x &= (1 << 64) - 1
    x ^= x >> 31
    return x & ((1 << 63) - 1)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def gaussian(shape, *, seed: int, tid: int, scale: float = 1.0,
             dtype=torch.bfloat16, seq_axis: int = 1) -> torch.Tensor:
    """N(0,1)*scale of `shape`, rounded (RNE) to `dtype`, on the CPU.

    The sequence axis (default 1, i.e. [B, L, ...]) is split into chunks of
    4096; each (batch, chunk) slab is drawn from its own seeded generator.
    """
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=dtype)
    B = shape[0] if seq_axis >= 1 else 1
    S = shape[seq_axis]
    jobs = [(b, c) for b in range(B) for c in range((S + _CHUNK - 1) // _CHUNK)]

    def job(bc):
        b, c = bc
        lo, hi = c * _CHUNK, min(S, (c + 1) * _CHUNK)
        g = torch.Generator().manual_seed(_chunk_seed(seed, tid, b, c))
        sub_shape = list(shape)
        if seq_axis >= 1:
            sub_shape[0] = 1
        sub_shape[seq_axis] = hi - lo
        x = torch.randn(sub_shape, generator=g, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        if seq_axis >= 1:
            out[b:b + 1].narrow(seq_axis, lo, hi - lo).copy_(x)
        else:
            out.narrow(seq_axis, lo, hi - lo).copy_(x)

    if len(jobs) == 1:
        job(jobs[0])
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(job, jobs))
    return out


# ----------------------------------------------------------------------------
# The workloads.  Names say what they are; sizes are stated in full.
# ----------------------------------------------------------------------------
PREFILL = {
    # fp32 tiny case: L=512 with a 128-token pretrained window (G=4), w_local=32.
    "tiny_f32_L512": dict(dtype="f32", B=1, Hq=1, Hkv=1, D=64, L=512,
                          w_pretrained=128, w_local=32, rope_base=1e4,
                          value_scale=1.0, seed=0),
    # the same with L=128 (G=1): must equal plain causal RoPE attention.
    "tiny_f32_L128": dict(dtype="f32", B=1, Hq=1, Hkv=1, D=64, L=128,
                          w_pretrained=128, w_local=32, rope_base=1e4,
                          value_scale=1.0, seed=0),
    # Qwen3-1.7B attention shape at 64K (G=2).
    "qwen3_1p7b_L65536": dict(dtype="bf16", B=1, Hq=16, Hkv=8, D=128, L=65536,
                              w_pretrained=32768, w_local=2048, rope_base=1e6,
                              value_scale=0.5, seed=1),
    # Qwen3-8B attention shape at 128K (G=4).
    "qwen3_8b_L131072": dict(dtype="bf16", B=1, Hq=32, Hkv=8, D=128, L=131072,
                             w_pretrained=32768, w_local=2048, rope_base=1e6,
                             value_scale=0.5, seed=2),
}
# Qwen3-4B attention shape, length sweep (G = 1, 1, 2, 3, 4).
for _i, _L in enumerate((16384, 32768, 49152, 98304, 131072)):
    PREFILL[f"qwen3_4b_L{_L}"] = dict(dtype="bf16", B=1, Hq=32, Hkv=8, D=128, L=_L,
                                      w_pretrained=32768, w_local=2048,
                                      rope_base=1e6, value_scale=0.5, seed=10 + _i)

# Qwen3-8B single-token decode over caches of 8K..128K tokens (pos = n - 1).
DECODE = {
    f"qwen3_8b_decode_n{_n}": dict(dtype="bf16", B=1, Hq=32, Hkv=8, D=128, n=_n,
                                   w_pretrained=32768, w_local=2048,
                                   rope_base=1e6, seed=20 + _i)
    for _i, _n in enumerate((8192, 32768, 65536, 131072))
}


def _torch_dtype(name: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def prefill_inputs(B, L, Hq, Hkv, D, *, dtype="bf16", value_scale=0.5, seed=0):
    """Pre-RoPE q [B,L,Hq,D], k and v [B,L,Hkv,D] on the CPU."""
    td = _torch_dtype(dtype)
    q = gaussian((B, L, Hq, D), seed=seed, tid=1, scale=value_scale, dtype=td)
    k = gaussian((B, L, Hkv, D), seed=seed, tid=2, scale=value_scale, dtype=td)
    v = gaussian((B, L, Hkv, D), seed=seed, tid=3, scale=value_scale, dtype=td)
    return q, k, v


def decode_inputs(B, Hq, Hkv, D, capacity, *, dtype="bf16", seed=0):
    """q_new [B,Hq,D] (pre-RoPE) and caches [B,capacity,Hkv,D], all N(0,1)."""
    td = _torch_dtype(dtype)
    q = gaussian((B, Hq, D), seed=seed, tid=4, dtype=td, seq_axis=1)
    kc = gaussian((B, capacity, Hkv, D), seed=seed, tid=5, dtype=td)
    vc = gaussian((B, capacity, Hkv, D), seed=seed, tid=6, dtype=td)
    return q, kc, vc


def sample_rows(B, L, Hq, *, per_head=512, seed=0, extra=()):
    """(b, q, h) index arrays: `per_head` seeded random rows for every (b, h),
    plus the given extra positions (clipped to [0, L)) for every (b, h)."""
    rng = np.random.Generator(np.random.PCG64(seed + 0x5EED))
    bs, qs, hs = [], [], []
    fixed = sorted({int(x) for x in extra if 0 <= int(x) < L})
    for b in range(B):
        for h in range(Hq):
            n = min(per_head, L)
            rows = rng.choice(L, size=n, replace=False) if n < L else np.arange(L)
            rows = np.unique(np.concatenate([rows, np.array(fixed, dtype=np.int64)]))
            bs.append(np.full(rows.shape, b))
            qs.append(rows)
            hs.append(np.full(rows.shape, h))
    return (np.concatenate(bs).astype(np.int32), np.concatenate(qs).astype(np.int32),
            np.concatenate(hs).astype(np.int32))


def to_oracle_array(t: torch.Tensor) -> np.ndarray:
    """CPU tensor -> numpy in a dtype the oracle takes (bf16 as uint16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.float64:
        return t.numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")

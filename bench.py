"""Benchmark of the bifocal RoPE attention hot path on B200.

One step = one pass of the whole hot path on one GPU:
  * bifocal prefill of a Qwen3-8B-shaped attention layer at L = 131072
    (B=1, Hq=32, Hkv=8, D=128, w_pretrained=32768 -> G=4, w_local=2048,
    rope_base=1e6, bf16 inputs N(0,1)*0.5), and
  * bifocal single-token decode over a 131072-token cache of the same shape
    (pos = 131071, G = 4).
`value` is the prefill's effective TFLOP/s (4*B*Hq*D*L(L+1)/2 FLOPs per call,
one causal QK^T + PV pass) summed over ranks / the slowest rank's time; the
decode's KV-read GB/s is reported beside it.  Inputs (>= 268 MB each) are
larger than the 126 MB L2, so no flush is needed between iterations.

Multi-GPU (--gpus N under torchrun): every rank runs the same independent
problem on its own GPU (weak scaling); there is no data-path collective, only
a barrier and a max-reduction of the timings.

--impl reference times the fp64 CPU oracle (the checker) on a bounded sample
of the same workload, on rank 0 only.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_attention_bifocal_b200 import workloads as W  # noqa: E402

METRIC = "bifocal prefill TFLOP/s & % bf16 peak; decode KV-read GB/s & % HBM"
PAGE_SIZE = 16  # keys per page of the paged-cache decode line
# DRAM bytes (read + write) of one full-size launch of the prefill kernel,
# from ncu (dram__bytes_read.sum + dram__bytes_write.sum, one pass) on B200.
# Must be re-measured (or set to None) whenever that kernel changes.
PREFILL_TRAFFIC_BYTES = 6857217152  # 5.790e9 read + 1.067e9 written, mean of two timed launches
PREFILL_CFG = "qwen3_8b_L131072"
CPU_ROWS_PER_HEAD = 16  # rows per query head in every timed oracle sample
DECODE_CFG = "qwen3_8b_decode_n131072"


def prefill_flops(B, Hq, D, L):
    return 4.0 * B * Hq * D * L * (L + 1) / 2


def rows_flops(D, rows_q):
    return float(sum(4.0 * D * (int(q) + 1) for q in rows_q))


def kv_bytes(B, Hkv, D, n):
    return float(B) * n * Hkv * D * 2 * 2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="jl_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return parse_clock_samples(lines)


def parse_clock_samples(lines):
    """Summarises nvidia-smi lines in ClockSampler.QUERY order (csv, no header,
    no units): median and maximum SM clock, and every throttle reason seen
    active in any sample.  Lines that do not parse are skipped; None if no
    line does."""
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx.append(float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
            "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x, world):
    """Largest x over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed, rank):
    """Seed of rank's independent problem (weak scaling: one problem per GPU)."""
    return seed + 1000 * rank


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


PREFILL_SWEEP = ["qwen3_1p7b_L65536", "qwen3_4b_L16384", "qwen3_4b_L32768", "qwen3_4b_L49152",
                 "qwen3_4b_L98304", "qwen3_4b_L131072"]


def interleaved(stream, fa, fb, reps):
    """Medians (ms) of fa and fb timed alternately with CUDA events on `stream`
    (clock drift and neighbours hit both alike).  The stream first runs a
    ~20 ms wait, so that the host has queued every call before the device
    reaches the first: the events then time the device work alone, not the
    host's launch path (which a short decode call would otherwise wait on)."""
    ea = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    eb = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    with torch.cuda.stream(stream):
        torch.cuda._sleep(40_000_000)
    for i, ((a0, a1), (b0, b1)) in enumerate(zip(ea, eb)):
        a0.record(stream)
        fa(i)
        a1.record(stream)
        b0.record(stream)
        fb(i)
        b1.record(stream)
    torch.cuda.synchronize()
    med = lambda es: sorted(x.elapsed_time(y) for x, y in es)[reps // 2]  # noqa: E731
    return med(ea), med(eb)


def prefill_sweep(jl, dev, stream, world, rank, reps, bf16_sust):
    """Every prefill configuration besides the headline one: the 1.7B shape at
    64K and the 4B shape's length sweep.  Per configuration: median ms per call
    (bifocal and JL_FLAG_NO_BIFOCAL timed alternately), effective TFLOP/s, the
    fraction of the sustained bf16 peak and the overhead of the bifocal rule."""
    res = {}
    for name in PREFILL_SWEEP:
        c = W.PREFILL[name]
        B, L, Hq, Hkv, D = c["B"], c["L"], c["Hq"], c["Hkv"], c["D"]
        kw = dict(w_local=c["w_local"], w_pretrained=c["w_pretrained"], rope_base=c["rope_base"])
        q, k, v = (t.to(dev) for t in W.prefill_inputs(
            B, L, Hq, Hkv, D, value_scale=c["value_scale"], seed=rank_seed(c["seed"], rank)))
        out = torch.empty_like(q)
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
        run = lambda flags: jl.bifocal_prefill(q, k, v, out=out, lse=lse,  # noqa: E731
                                               flags=flags, **kw)
        run(0)
        run(jl.NO_BIFOCAL)
        bif, plain = interleaved(stream, lambda i: run(0), lambda i: run(jl.NO_BIFOCAL), reps)
        bif = max_over_ranks(bif, world)
        plain = max_over_ranks(plain, world)
        fl = prefill_flops(B, Hq, D, L)
        tf = fl / (bif / 1e3) / 1e12
        G = -(-L // c["w_pretrained"])
        res[name] = {"L": L, "Hq": Hq, "Hkv": Hkv, "G": G, "ms_per_call": round(bif, 3),
                     "tflops": round(tf * world, 2), "frac_bf16_sustained": round(tf / bf16_sust, 4),
                     "ms_no_bifocal": round(plain, 3),
                     "overhead_vs_no_bifocal": round(bif / plain - 1.0, 4)}
        del q, k, v, out, lse
    jl.check_device_status()
    return res


def decode_sweep(jl, dev, stream, world, rank, hbm, reps):
    """The decode configuration's cache lengths n = 8192 ... 131072 (pos = n-1).
    Each call reads a different one of several caches in turn, enough of them
    that the others' bytes since its last use exceed three times the L2, so every
    call reads its keys and values from HBM.  Bifocal and JL_FLAG_NO_BIFOCAL
    calls alternate; medians of `reps` calls each."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    res = {}
    for name, c in W.DECODE.items():
        n, B, Hq, Hkv, D = c["n"], c["B"], c["Hq"], c["Hkv"], c["D"]
        pos = n - 1
        kw = dict(w_local=c["w_local"], w_pretrained=c["w_pretrained"], rope_base=c["rope_base"])
        nbytes = kv_bytes(B, Hkv, D, n)
        copies = max(2, int(math.ceil(3 * l2 / nbytes)) + 1)
        q, kc0, vc0 = W.decode_inputs(B, Hq, Hkv, D, n, seed=rank_seed(c["seed"], rank))
        q = q.to(dev)
        caches = []
        for i in range(copies):
            kc, vc = kc0.to(dev), vc0.to(dev)
            if i:
                # distinct bytes per copy (a rotation of the key order), same distribution
                kc, vc = torch.roll(kc, 17 * i, dims=1), torch.roll(vc, 17 * i, dims=1)
            caches.append((kc, vc))
        out = torch.empty_like(q)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(jl.decode_workspace_size(B, Hq, Hkv, D, pos), dtype=torch.uint8,
                         device=dev)

        def call(i, flags):
            kc, vc = caches[i % copies]
            jl.bifocal_decode(q, kc, vc, pos, out=out, lse=lse, workspace=ws, flags=flags, **kw)
        for i in range(2 * copies):
            call(i, 0)
            call(i, jl.NO_BIFOCAL)
        # the two calls of a pair read different caches too
        bif, plain = interleaved(stream, lambda i: call(2 * i, 0),
                                 lambda i: call(2 * i + 1, jl.NO_BIFOCAL), reps)
        bif = max_over_ranks(bif, world)
        plain = max_over_ranks(plain, world)
        gbs = nbytes / (bif / 1e3) / 1e9
        res[name] = {"n": n, "G": -(-n // c["w_pretrained"]), "us_per_call": round(bif * 1e3, 2),
                     "value": round(gbs * world, 1), "unit": "GB/s",
                     "frac_hbm": round(gbs / hbm, 4), "us_no_bifocal": round(plain * 1e3, 2),
                     "overhead_vs_no_bifocal": round(bif / plain - 1.0, 4),
                     "distinct_caches": copies}
        del caches, q, out, lse, ws
    jl.check_device_status()
    return res


def run_cuda(args):
    import long_context_attention_bifocal_b200 as jl

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pc = W.PREFILL[PREFILL_CFG]
    dc = W.DECODE[DECODE_CFG]
    B, L, Hq, Hkv, D = pc["B"], pc["L"], pc["Hq"], pc["Hkv"], pc["D"]
    kwp = dict(w_local=pc["w_local"], w_pretrained=pc["w_pretrained"], rope_base=pc["rope_base"])
    n = dc["n"]
    pos = n - 1
    kwd = dict(w_local=dc["w_local"], w_pretrained=dc["w_pretrained"], rope_base=dc["rope_base"])

    # host inputs (pinned), one independent problem per rank
    q_h, k_h, v_h = W.prefill_inputs(B, L, Hq, Hkv, D, value_scale=pc["value_scale"],
                                     seed=rank_seed(pc["seed"], rank))
    qd_h, kc_h, vc_h = W.decode_inputs(dc["B"], dc["Hq"], dc["Hkv"], dc["D"], n,
                                       seed=rank_seed(dc["seed"], rank))
    host = [t.pin_memory() for t in (q_h, k_h, v_h, qd_h, kc_h, vc_h)]
    q_h, k_h, v_h, qd_h, kc_h, vc_h = host
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    qd, kc, vc = qd_h.to(dev), kc_h.to(dev), vc_h.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    outd = torch.empty_like(qd)
    lsed = torch.empty((dc["B"], dc["Hq"]), dtype=torch.float32, device=dev)
    wsd = torch.empty(jl.decode_workspace_size(dc["B"], dc["Hq"], dc["Hkv"], dc["D"], pos),
                      dtype=torch.uint8, device=dev)
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    outd_h = torch.empty(outd.shape, dtype=outd.dtype, pin_memory=True)
    lsed_h = torch.empty(lsed.shape, dtype=lsed.dtype, pin_memory=True)
    stream = torch.cuda.current_stream(dev)

    def prefill(flags=0):
        jl.bifocal_prefill(q, k, v, out=out, lse=lse, flags=flags, **kwp)

    def decode(flags=0):
        jl.bifocal_decode(qd, kc, vc, pos, out=outd, lse=lsed, workspace=wsd, flags=flags, **kwd)

    # ---------------- warm-up ----------------
    for _ in range(args.warmup):
        prefill()
        decode()
    jl.check_device_status()
    barrier(world)

    # ---------------- timed region (device clock, CUDA events) ----------------
    sampler = ClockSampler(local)
    sampler.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        prefill()
        ev[s][1].record(stream)
        decode()
        ev[s][2].record(stream)
    t1.record(stream)
    barrier(world)
    clocks = sampler.stop()
    jl.check_device_status()
    total_ms = t0.elapsed_time(t1)
    pre_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(args.steps)]
    dec_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(args.steps)]
    total_ms = max_over_ranks(total_ms, world)
    pre_sum = max_over_ranks(sum(pre_ms), world)
    dec_sum = max_over_ranks(sum(dec_ms), world)
    launches = 3 * args.steps  # per step: the prefill kernel, decode + combine

    # ---------------- overhead vs the same kernels without the bifocal rule ----
    def avg_ms(fn, reps):
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        with torch.cuda.stream(stream):
            torch.cuda._sleep(40_000_000)  # the host queues ahead (see interleaved)
        for a, b in es:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return sorted(a.elapsed_time(b) for a, b in es)[reps // 2]

    dec_bif, dec_plain = interleaved(stream, lambda i: decode(0),
                                     lambda i: decode(jl.NO_BIFOCAL), 100)

    # a ragged batch: 8 sequences of one shape at different positions (G 1-4)
    bpos = [16383, 32767, 49151, 65535, 81919, 98303, 114687, 131071]
    bcap = max(bpos) + 1
    gb = torch.Generator(device=dev)
    gb.manual_seed(rank_seed(dc["seed"] + 1, rank))
    qb = torch.randn((len(bpos), dc["Hq"], dc["D"]), generator=gb, device=dev).to(torch.bfloat16)
    kb = torch.randn((len(bpos), bcap, dc["Hkv"], dc["D"]), generator=gb,
                     device=dev).to(torch.bfloat16)
    vb = torch.randn((len(bpos), bcap, dc["Hkv"], dc["D"]), generator=gb,
                     device=dev).to(torch.bfloat16)
    wsb = torch.empty(jl.decode_batched_workspace_size(len(bpos), dc["Hq"], dc["Hkv"], dc["D"]),
                      dtype=torch.uint8, device=dev)
    outb = torch.empty_like(qb)
    lseb = torch.empty((len(bpos), dc["Hq"]), dtype=torch.float32, device=dev)
    dec_batched = avg_ms(lambda: jl.bifocal_decode_batched(qb, kb, vb, bpos, out=outb, lse=lseb,
                                                           workspace=wsb, **kwd), 20)
    batched_bytes = sum(kv_bytes(1, dc["Hkv"], dc["D"], p_ + 1) for p_ in bpos)
    dec_batched = max_over_ranks(dec_batched, world)
    # the same call with the positions on the device (plan made on the GPU)
    bpos_d = torch.tensor(bpos, dtype=torch.int32, device=dev)
    dec_batched_dev = avg_ms(lambda: jl.bifocal_decode_batched(qb, kb, vb, bpos_d, out=outb,
                                                               lse=lseb, workspace=wsb, **kwd), 20)
    dec_batched_dev = max_over_ranks(dec_batched_dev, world)
    # the same batch in a paged cache: 16-key pages of a shared pool, in a
    # seeded random order, one block table row per sequence
    need = [(p_ + PAGE_SIZE) // PAGE_SIZE for p_ in bpos]
    perm = torch.randperm(sum(need), generator=torch.Generator().manual_seed(rank_seed(7, rank)))
    table = torch.full((len(bpos), max(need)), -1, dtype=torch.int32)
    kpg = torch.empty((sum(need), PAGE_SIZE, dc["Hkv"], dc["D"]), dtype=torch.bfloat16, device=dev)
    vpg = torch.empty_like(kpg)
    first = 0
    for b_, p_ in enumerate(bpos):
        pages = perm[first:first + need[b_]]
        first += need[b_]
        table[b_, :need[b_]] = pages.to(torch.int32)
        idx = pages.to(dev)
        kpg[idx] = kb[b_, :need[b_] * PAGE_SIZE].reshape(need[b_], PAGE_SIZE, dc["Hkv"], dc["D"])
        vpg[idx] = vb[b_, :need[b_] * PAGE_SIZE].reshape(need[b_], PAGE_SIZE, dc["Hkv"], dc["D"])
    table = table.to(dev)
    dec_paged = avg_ms(lambda: jl.bifocal_decode_paged(qb, kpg, vpg, table, bpos, out=outb,
                                                       lse=lseb, workspace=wsb, **kwd), 20)
    dec_paged = max_over_ranks(dec_paged, world)
    del kpg, vpg, table
    del qb, kb, vb, wsb, outb, lseb
    pre_plain = avg_ms(lambda: prefill(jl.NO_BIFOCAL), max(1, min(3, args.steps)))
    pre_bif = avg_ms(lambda: prefill(0), max(1, min(3, args.steps)))
    # the opt-in mode: keys rotated once per call into a workspace (512 MiB
    # here) and streamed, instead of rotated per K tile in the kernel
    ws_once = torch.empty(jl.prefill_rotated_keys_bytes(B, L, Hkv, D), dtype=torch.uint8,
                          device=dev)
    pre_once = avg_ms(lambda: jl.bifocal_prefill(q, k, v, out=out, lse=lse, workspace=ws_once,
                                                 flags=jl.ROTATE_KEYS_ONCE, **kwp),
                      max(1, min(3, args.steps)))
    pre_once = max_over_ranks(pre_once, world)
    del ws_once
    # the pages' unfused three-call formulation of the same prefill (A + B - C)
    ws3 = torch.empty(jl.prefill_3pass_workspace_size(B, L, Hq, Hkv, D), dtype=torch.uint8,
                      device=dev)
    out3 = torch.empty_like(out)
    lse3 = torch.empty_like(lse)
    pre_3pass = avg_ms(lambda: jl.bifocal_prefill_3pass(q, k, v, out=out3, lse=lse3,
                                                        workspace=ws3, **kwp),
                       max(1, min(3, args.steps)))
    del ws3, out3, lse3
    # chunked prefill: the last 16384 tokens of the sequence against the
    # decode workload's cache (131072 keys at original positions)
    chunk_lq = 16384
    chunk_off = n - chunk_lq
    qc = q[:, chunk_off:]
    outc = torch.empty_like(qc)
    lsec = torch.empty((B, Hq, chunk_lq), dtype=torch.float32, device=dev)
    pre_chunk = avg_ms(lambda: jl.bifocal_prefill_chunk(qc, kc, vc, chunk_off, out=outc, lse=lsec,
                                                        **kwd),
                       max(1, min(5, args.steps)))
    pre_chunk = max_over_ranks(pre_chunk, world)
    chunk_flops = 4.0 * B * Hq * D * (chunk_lq * chunk_off + chunk_lq * (chunk_lq + 1) / 2)
    del outc, lsec
    # the pages quote the method as a speed ratio over FlashAttention-2 (plain
    # causal attention of the same shape); the installed flash_attn package,
    # when present, gives that baseline on this GPU (context only)
    fa2_local, fa2_dec_local, fa2_why = -1.0, -1.0, None
    try:
        from flash_attn import flash_attn_func, flash_attn_with_kvcache
        fa2 = lambda: flash_attn_func(q, k, v, causal=True)  # noqa: E731
        fa2()
        torch.cuda.synchronize()
        fa2_local = avg_ms(fa2, 3)
        # and its decode over the same cache (one new token per sequence)
        qd4 = qd.view(dc["B"], 1, dc["Hq"], dc["D"])
        lens = torch.full((dc["B"],), n, dtype=torch.int32, device=dev)
        fa2d = lambda: flash_attn_with_kvcache(qd4, kc, vc, cache_seqlens=lens,  # noqa: E731
                                               causal=True)
        fa2d()
        torch.cuda.synchronize()
        fa2_dec_local = avg_ms(fa2d, 50)
    except Exception as exc:  # the package is optional: report why it is missing
        fa2_why = f"unavailable: {type(exc).__name__}: {str(exc)[:80]}"
    fa2_ms = max_over_ranks(fa2_local, world)  # every rank takes part
    fa2_dec_ms = max_over_ranks(fa2_dec_local, world)
    if fa2_ms < 0 or fa2_dec_ms < 0 or fa2_why is not None:
        fa2_ms = fa2_why or "unavailable on some rank"
    jl.check_device_status()

    # ---------------- the other configurations ----------------
    hbm, bf16_burst, bf16_sust, src = peaks()
    sweep_p = prefill_sweep(jl, dev, stream, world, rank, 3, bf16_sust)
    sweep_d = decode_sweep(jl, dev, stream, world, rank, hbm, 50)

    # ---------------- end to end through the public API, host buffers ----------
    # Every step copies its inputs from pinned host memory, runs the prefill
    # and the decode through the Python binding, and copies the outputs back.
    # Two sets of device buffers and two copy streams pipeline the steps the
    # way a serving loop would: step s+1's inputs go up while step s computes,
    # step s's outputs come down while step s+1 computes.  The timed region
    # runs from before the first upload to after the last download.
    h2d_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)
    bufs = [dict(q=q, k=k, v=v, out=out, lse=lse, qd=qd, kc=kc, vc=vc, outd=outd, lsed=lsed)]
    bufs.append({name: torch.empty_like(t) for name, t in bufs[0].items()})
    host_in = dict(q=q_h, k=k_h, v=v_h, qd=qd_h, kc=kc_h, vc=vc_h)
    host_out = dict(out=out_h, lse=lse_h, outd=outd_h, lsed=lsed_h)
    computed = [torch.cuda.Event() for _ in range(2)]   # buffer's inputs consumed
    uploaded = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]  # buffer's outputs read
    e_steps = max(2, args.steps)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)
    d2h_stream.wait_event(e0)

    def upload(step):
        bi = bufs[step % 2]
        with torch.cuda.stream(h2d_stream):
            if step >= 2:
                h2d_stream.wait_event(computed[step % 2])
            for name, t in host_in.items():
                bi[name].copy_(t, non_blocking=True)
            uploaded[step % 2].record(h2d_stream)

    upload(0)
    for st in range(e_steps):
        bi = bufs[st % 2]
        if st + 1 < e_steps:
            upload(st + 1)
        stream.wait_event(uploaded[st % 2])
        if st >= 2:
            stream.wait_event(downloaded[st % 2])
        jl.bifocal_prefill(bi["q"], bi["k"], bi["v"], out=bi["out"], lse=bi["lse"], **kwp)
        jl.bifocal_decode(bi["qd"], bi["kc"], bi["vc"], pos, out=bi["outd"], lse=bi["lsed"],
                          workspace=wsd, **kwd)
        computed[st % 2].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(computed[st % 2])
            for name, t in host_out.items():
                t.copy_(bi[name], non_blocking=True)
            downloaded[st % 2].record(d2h_stream)
    stream.wait_stream(d2h_stream)
    stream.wait_stream(h2d_stream)
    e1.record(stream)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    del bufs[1]
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h, qd_h, kc_h, vc_h))
    d2h = sum(t.numel() * t.element_size() for t in (out_h, lse_h, outd_h, lsed_h))

    flops = prefill_flops(B, Hq, D, L)
    kvb = kv_bytes(dc["B"], dc["Hkv"], dc["D"], n)
    value = flops * args.steps * world / (pre_sum / 1e3) / 1e12
    # decode on its own: median of back-to-back calls (each reads the 512 MiB
    # cache, larger than L2); inside the step it follows the prefill and also
    # pays the write-back of the prefill's output still dirty in L2
    dec_call_ms = max_over_ranks(dec_bif, world)
    dec_gbs = kvb * world / (dec_call_ms / 1e3) / 1e9
    pre_launch_ms = pre_sum / args.steps
    achieved = flops / (pre_launch_ms / 1e3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": "qwen3_8b attention layer: bifocal prefill L=131072 + decode n=131072",
            "prefill": {"B": B, "L": L, "Hq": Hq, "Hkv": Hkv, "D": D, **kwp, "G": 4,
                        "values": "N(0,1)*0.5 bf16, seeded"},
            "decode": {"B": dc["B"], "pos": pos, "Hq": dc["Hq"], "Hkv": dc["Hkv"], "D": dc["D"],
                       **kwd, "G": 4, "values": "N(0,1) bf16, seeded"},
            "l2": "inputs larger than L2 (Q 1 GiB, K/V 256 MiB each, KV cache 512 MiB)",
            "parallelism": f"independent problem per GPU x{world}",
        },
        "decode": {
            "value": round(dec_gbs, 1), "unit": "GB/s",
            "us_per_call": round(dec_call_ms * 1e3, 2),
            "us_per_call_in_step": round(dec_sum / args.steps * 1e3, 2),
            "frac_hbm": round(dec_gbs / world / hbm, 4),
            "overhead_vs_no_bifocal": round(dec_bif / dec_plain - 1.0, 4),
        },
        "decode_batched": {
            "B": len(bpos), "positions": bpos, "inputs": "N(0,1) bf16 on the device, seeded",
            "us_per_call": round(dec_batched * 1e3, 2),
            "value": round(batched_bytes * world / (dec_batched / 1e3) / 1e9, 1),
            "unit": "GB/s",
            "frac_hbm": round(batched_bytes / (dec_batched / 1e3) / 1e9 / hbm, 4),
            "us_per_call_device_positions": round(dec_batched_dev * 1e3, 2),
        },
        "decode_paged": {
            "B": len(bpos), "positions": bpos, "page_size": PAGE_SIZE,
            "pages": "shuffled pool, seeded",
            "us_per_call": round(dec_paged * 1e3, 2),
            "value": round(batched_bytes * world / (dec_paged / 1e3) / 1e9, 1),
            "unit": "GB/s",
            "frac_hbm": round(batched_bytes / (dec_paged / 1e3) / 1e9 / hbm, 4),
        },
        "prefill_unfused_3pass": {
            "ms_per_call": round(pre_3pass, 3),
            "tflops_effective": round(flops / (pre_3pass / 1e3) / 1e12, 2),
            "fused_speedup": round(pre_3pass / pre_bif, 4),
        },
        "pages_comparison": (
            {"flashattention2_causal_ms": round(fa2_ms, 3),
             "fused_bifocal_speedup": round(fa2_ms / pre_bif, 3),
             "unfused_3pass_speedup": round(fa2_ms / pre_3pass, 3),
             "flashattention2_decode_us": round(fa2_dec_ms * 1e3, 2),
             "bifocal_decode_speedup": round(fa2_dec_ms / dec_bif, 3),
             "pages_h100": "prefill: fused 1.28-1.39x, unfused 0.89-0.93x; "
                           "generation: fused 0.96-1.00x FlashAttention-2"}
            if isinstance(fa2_ms, float) else {"flashattention2": fa2_ms}),
        "prefill_chunk": {
            "q_offset": chunk_off, "Lq": chunk_lq, "cache": "the decode workload's",
            "ms_per_call": round(pre_chunk, 3),
            "tflops": round(chunk_flops * world / (pre_chunk / 1e3) / 1e12, 2),
        },
        "prefill_keys_rotated_once": {
            "flag": "JL_FLAG_ROTATE_KEYS_ONCE",
            "workspace_bytes": int(jl.prefill_rotated_keys_bytes(B, L, Hkv, D)),
            "ms_per_call": round(pre_once, 3),
            "tflops": round(flops * world / (pre_once / 1e3) / 1e12, 2),
            "frac_bf16_sustained": round(flops / (pre_once / 1e3) / 1e12 / bf16_sust, 4),
            "speedup_vs_in_kernel_rotation": round(pre_bif / pre_once, 4),
        },
        "prefill_sweep": sweep_p,
        "decode_sweep": sweep_d,
        "prefill": {
            "ms_per_call": round(pre_launch_ms, 3),
            "frac_bf16_sustained": round(achieved / bf16_sust, 4),
            "frac_bf16_burst": round(achieved / bf16_burst, 4),
            "overhead_vs_no_bifocal": round(pre_bif / pre_plain - 1.0, 4),
        },
        "roofline": {
            "bound": "tensor",
            "kernel": "bifocal_prefill_sm100_x2_kernel (keys rotated in the kernel)",
            "achieved": round(achieved, 2),
            "peak": bf16_sust,
            "peak_kind": f"bf16 dense, sustained, {src}",
            "unit": "TFLOP/s",
            "frac": round(achieved / bf16_sust, 4),
            "traffic": PREFILL_TRAFFIC_BYTES,
        },
        "e2e": {
            "value": round(flops * e_steps * world / (e2e_ms / 1e3) / 1e12, 2),
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
            "steps": e_steps,
            "transfers": "pinned host buffers; uploads and downloads on two copy streams, "
                         "overlapped with the neighbouring steps' compute",
        },
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(q_h, k_h, v_h, qd_h, kc_h, vc_h, kwp, kwd, pos,
                                            budget_s=args.cpu_seconds)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def cpu_baseline(q_h, k_h, v_h, qd_h, kc_h, vc_h, kwp, kwd, pos, budget_s=20.0, rows=None):
    """The fp64 oracle, as it stands, on a bounded sample of the same workload:
    a few seeded rows per query head of the prefill (effective TFLOP/s over the
    sampled rows) and the full decode (KV GB/s)."""
    import oracle
    orc = oracle.default()
    B, L, Hq, D = q_h.shape
    qa, ka, va = W.to_oracle_array(q_h), W.to_oracle_array(k_h), W.to_oracle_array(v_h)
    per_head = rows or CPU_ROWS_PER_HEAD
    rb, rq, rh = W.sample_rows(B, L, Hq, per_head=per_head, seed=123)
    t = time.perf_counter()
    orc.bifocal_rows(qa, ka, va, rb, rq, rh, **kwp)
    dt = time.perf_counter() - t
    fl = rows_flops(D, rq)
    t = time.perf_counter()
    orc.bifocal_decode(W.to_oracle_array(qd_h), W.to_oracle_array(kc_h[:, :pos + 1]),
                       W.to_oracle_array(vc_h[:, :pos + 1]), pos, **kwd)
    ddt = time.perf_counter() - t
    kvb = kv_bytes(kc_h.shape[0], kc_h.shape[2], kc_h.shape[3], pos + 1)
    full = prefill_flops(B, Hq, D, L)
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": orc.num_threads(),
            "kind": "oracle",
            "gflops_fp64": round(fl / dt / 1e9, 2),
            "full_prefill_s_extrapolated": round(full / (fl / dt), 1),
            "sample": f"prefill: {per_head} seeded rows per query head ({len(rq)} rows) of the "
                      f"L=131072 workload, {dt:.1f} s; decode: the full n=131072 call, "
                      f"{ddt:.1f} s ({kvb / ddt / 1e9:.3f} GB/s)"}


def run_reference(args):
    """The oracle arm: rank 0 only, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    orc = oracle.default()
    pc = W.PREFILL[PREFILL_CFG]
    B, L, Hq, Hkv, D = pc["B"], pc["L"], pc["Hq"], pc["Hkv"], pc["D"]
    kwp = dict(w_local=pc["w_local"], w_pretrained=pc["w_pretrained"], rope_base=pc["rope_base"])
    q, k, v = W.prefill_inputs(B, L, Hq, Hkv, D, value_scale=pc["value_scale"], seed=pc["seed"])
    qa, ka, va = W.to_oracle_array(q), W.to_oracle_array(k), W.to_oracle_array(v)
    # the same sample size as the in-bench cpu_baseline leg (16 rows per query
    # head), so that the oracle's per-call work on the whole key sequence is
    # spread over as many rows and the two CPU figures measure the same thing
    per_head = CPU_ROWS_PER_HEAD
    times, flops = [], []
    for s in range(args.warmup + args.steps):
        rb, rq, rh = W.sample_rows(B, L, Hq, per_head=per_head, seed=1000 + s)
        t = time.perf_counter()
        orc.bifocal_rows(qa, ka, va, rb, rq, rh, **kwp)
        dt = time.perf_counter() - t
        if s >= args.warmup:
            times.append(dt)
            flops.append(rows_flops(D, rq))
    value = sum(flops) / sum(times) / 1e12
    sample = (f"{per_head} seeded rows per query head ({Hq * per_head} rows) of the L=131072 "
              "prefill per step")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "qwen3_8b attention layer: bifocal prefill L=131072 (row sample)",
                   "parallelism": "CPU oracle, rank 0"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                         "cores": orc.num_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


CASES = {
    # small cases for ncu captures: inputs larger than L2, a few hundred MB on the device
    "prefill_L32768": dict(kind="prefill", B=1, L=32768, Hq=32, Hkv=8, w_pretrained=8192),
    "decode_n131072": dict(kind="decode", n=131072),
}


def run_case(args):
    """One kernel family on a small case (warm-up + steps), for profiling."""
    import long_context_attention_bifocal_b200 as jl
    c = CASES[args.case]
    dev = torch.device("cuda", 0)
    if c["kind"] == "prefill":
        q, k, v = W.prefill_inputs(c["B"], c["L"], c["Hq"], c["Hkv"], 128, seed=5)
        q, k, v = q.to(dev), k.to(dev), v.to(dev)
        kw = dict(w_local=2048, w_pretrained=c["w_pretrained"], rope_base=1e6)
        fn = lambda: jl.bifocal_prefill(q, k, v, **kw)  # noqa: E731
    else:
        n = c["n"]
        qd, kc, vc = W.decode_inputs(1, 32, 8, 128, n, seed=6)
        qd, kc, vc = qd.to(dev), kc.to(dev), vc.to(dev)
        ws = torch.empty(jl.decode_workspace_size(1, 32, 8, 128, n - 1), dtype=torch.uint8,
                         device=dev)
        fn = lambda: jl.bifocal_decode(qd, kc, vc, n - 1, w_local=2048,  # noqa: E731
                                       w_pretrained=32768, rope_base=1e6, workspace=ws)
    for _ in range(args.warmup + args.steps):
        fn()
    jl.check_device_status()
    print(json.dumps({"case": args.case, "launch_groups": args.warmup + args.steps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=sorted(CASES), default=None,
                    help="run one small profiling case instead of the benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "cuda":
        args.warmup = 3
    if args.case:
        run_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()

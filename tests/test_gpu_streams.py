"""Calls on two CUDA streams at once: the results equal those of the same calls
made one after another.  The prefill holds no scratch memory (its keys are
rotated inside the kernels), so two prefills, chunked prefills included, may
overlap with nothing but their own outputs; a decode takes its own workspace."""
import pytest
import torch

from long_context_attention_bifocal_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_prefills_on_two_streams(jl):
    kw = dict(w_local=256, w_pretrained=1024, rope_base=1e6)
    runs = []
    for seed, L in ((11, 3000), (12, 2500)):
        q, k, v = W.prefill_inputs(1, L, 8, 2, 128, seed=seed)
        q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
        ref = jl.bifocal_prefill(q, k, v, **kw)
        runs.append((q, k, v, ref))
    # a chunked prefill over the second sequence's keys as a cache
    q2, k2, v2, _ = runs[1]
    cref = jl.bifocal_prefill_chunk(q2[:, 1024:].contiguous(), k2, v2, 1024, **kw)
    jl.check_device_status()
    streams = [torch.cuda.Stream(DEV) for _ in range(3)]
    outs = []
    torch.cuda.synchronize()
    for (q, k, v, _), st in zip(runs, streams):
        with torch.cuda.stream(st):
            outs.append(jl.bifocal_prefill(q, k, v, stream=st, **kw))
    with torch.cuda.stream(streams[2]):
        cout = jl.bifocal_prefill_chunk(q2[:, 1024:].contiguous(), k2, v2, 1024,
                                        stream=streams[2], **kw)
    torch.cuda.synchronize()
    jl.check_device_status()
    for (_, _, _, (ro, rl)), (o, l) in zip(runs, outs):
        assert torch.equal(o, ro) and torch.equal(l, rl)
    assert torch.equal(cout[0], cref[0]) and torch.equal(cout[1], cref[1])


def test_decode_on_two_streams_with_own_workspaces(jl):
    kw = dict(w_local=2048, w_pretrained=8192, rope_base=1e6)
    runs = []
    for seed, n in ((21, 40000), (22, 17000)):
        q, kc, vc = W.decode_inputs(1, 32, 8, 128, n, seed=seed)
        q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
        ws = torch.empty(jl.decode_workspace_size(1, 32, 8, 128, n - 1), dtype=torch.uint8,
                         device=DEV)
        ref = jl.bifocal_decode(q, kc, vc, n - 1, workspace=ws, **kw)
        runs.append((q, kc, vc, n, ws, ref))
    jl.check_device_status()
    streams = [torch.cuda.Stream(DEV) for _ in runs]
    outs = []
    torch.cuda.synchronize()
    for (q, kc, vc, n, ws, _), st in zip(runs, streams):
        with torch.cuda.stream(st):
            outs.append(jl.bifocal_decode(q, kc, vc, n - 1, workspace=ws, stream=st, **kw))
    torch.cuda.synchronize()
    jl.check_device_status()
    for (*_, (ro, rl)), (o, l) in zip(runs, outs):
        assert torch.equal(o, ro) and torch.equal(l, rl)

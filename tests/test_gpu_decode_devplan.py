"""Batched and paged decode with the positions on the device
(JL_FLAG_DEVICE_POS): the plan made on the device gives bit for bit the result
of the host-planned call, the call can be captured in a CUDA graph and replayed
with new positions, and a position outside the cache is reported."""
import numpy as np
import pytest
import torch

from long_context_attention_bifocal_b200 import workloads as W
from test_gpu_decode import poison_tail
from test_gpu_decode_paged import page_cache

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = [
    # (positions, cap, Hq, Hkv, w_local, w_pretrained)
    ([0, 100, 3000, 40000, 131071], 131100, 32, 8, 2048, 32768),
    ([5000, 5000, 5000], 6000, 8, 2, 0, 1000),
    ([17, 777, 2100], 2200, 16, 2, 5, 100),
    ([129], 200, 4, 4, 64, 32),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{len(c[0])}max{max(c[0])}" for c in CASES])
def test_device_positions_equal_host_positions(jl, case):
    positions, cap, Hq, Hkv, wl, wp = case
    B, D = len(positions), 128
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, cap, seed=91 + B)
    for b, pos in enumerate(positions):
        kc[b:b + 1] = poison_tail(kc[b:b + 1], pos)
        vc[b:b + 1] = poison_tail(vc[b:b + 1], pos)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    kw = dict(w_local=wl, w_pretrained=wp, rope_base=1e6)
    out_h, lse_h = jl.bifocal_decode_batched(q, kc, vc, positions, **kw)
    pos_d = torch.tensor(positions, dtype=torch.int32, device=DEV)
    out_d, lse_d = jl.bifocal_decode_batched(q, kc, vc, pos_d, **kw)
    jl.check_device_status()
    assert torch.equal(out_d, out_h) and torch.equal(lse_d, lse_h)


def test_device_positions_many_sequences(jl):
    rng = np.random.Generator(np.random.PCG64(6))
    positions = [int(x) for x in rng.integers(0, 4000, size=80)]
    B, Hq, Hkv, D, cap = len(positions), 8, 2, 128, 4000
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, cap, seed=78)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    kw = dict(w_local=512, w_pretrained=1024, rope_base=1e6)
    out_h, lse_h = jl.bifocal_decode_batched(q, kc, vc, positions, **kw)
    pos_d = torch.tensor(positions, dtype=torch.int32, device=DEV)
    out_d, lse_d = jl.bifocal_decode_batched(q, kc, vc, pos_d, **kw)
    jl.check_device_status()
    assert torch.equal(out_d, out_h) and torch.equal(lse_d, lse_h)


def test_device_positions_paged(jl):
    positions, ps = [0, 100, 3000, 9999], 16
    B, Hq, Hkv, D = len(positions), 32, 8, 128
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, max(positions) + 1, seed=93)
    kp, vp, table = page_cache(kc, vc, positions, ps, seed=4)
    q, kp, vp, table = q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV)
    kw = dict(w_local=2048, w_pretrained=4096, rope_base=1e6)
    out_h, lse_h = jl.bifocal_decode_paged(q, kp, vp, table, positions, **kw)
    pos_d = torch.tensor(positions, dtype=torch.int32, device=DEV)
    out_d, lse_d = jl.bifocal_decode_paged(q, kp, vp, table, pos_d, **kw)
    jl.check_device_status()
    assert torch.equal(out_d, out_h) and torch.equal(lse_d, lse_h)


def test_graph_capture_and_replay_with_new_positions(jl):
    """Capture one decode step with device positions, then replay the graph
    after writing other positions into the same device array."""
    B, Hq, Hkv, D, cap = 4, 32, 8, 128, 70000
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, cap, seed=94)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    kw = dict(w_local=2048, w_pretrained=16384, rope_base=1e6)
    ws = torch.empty(jl.decode_batched_workspace_size(B, Hq, Hkv, D), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    pos_d = torch.tensor([10, 20000, 40000, 69999], dtype=torch.int32, device=DEV)
    # a first call builds the library's table outside the capture
    jl.bifocal_decode_batched(q, kc, vc, pos_d, out=out, lse=lse, workspace=ws, **kw)
    jl.check_device_status()
    side = torch.cuda.Stream(DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            jl.bifocal_decode_batched(q, kc, vc, pos_d, out=out, lse=lse, workspace=ws,
                                      stream=side, **kw)
    torch.cuda.current_stream(DEV).wait_stream(side)
    for positions in ([5, 6, 7, 8], [69999, 1, 30000, 2048], [100, 20000, 40000, 50000]):
        pos_d.copy_(torch.tensor(positions, dtype=torch.int32))
        graph.replay()
        torch.cuda.synchronize()
        jl.check_device_status()
        ref_o, ref_l = jl.bifocal_decode_batched(q, kc, vc, positions, **kw)
        jl.check_device_status()
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l), positions
    del graph


def test_device_position_out_of_range_is_reported(jl):
    B, Hq, Hkv, D, cap = 3, 8, 2, 128, 1000
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, cap, seed=95)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    kw = dict(w_local=64, w_pretrained=256, rope_base=1e6)
    pos_d = torch.tensor([10, cap, 500], dtype=torch.int32, device=DEV)  # one past the cache
    jl.bifocal_decode_batched(q, kc, vc, pos_d, **kw)
    with pytest.raises(jl.JetLongError):
        jl.check_device_status()
    pos_d = torch.tensor([10, 999, 500], dtype=torch.int32, device=DEV)
    out_d, lse_d = jl.bifocal_decode_batched(q, kc, vc, pos_d, **kw)
    jl.check_device_status()
    out_h, lse_h = jl.bifocal_decode_batched(q, kc, vc, [10, 999, 500], **kw)
    jl.check_device_status()
    assert torch.equal(out_d, out_h)

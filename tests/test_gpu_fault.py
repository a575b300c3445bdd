"""Bounded waits on the GPU: a wait that runs out ends with a status, not a hang.

The test-only flag JL_FLAG_DEBUG_SKIP_ARRIVE makes the decode kernel's TMA
producer withhold its first K/V block, so the consumer warps' wait on it runs
out after about a second.  Nothing faults or traps: the kernel raises the
device status word and returns, the host reads JL_ERR_TIMEOUT through
jl_check_device_status, and the next call works and gives the same result as
before the injected timeout.
"""
import pytest
import torch

from long_context_attention_bifocal_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TIMEOUT = 4  # JL_ERR_TIMEOUT


@pytest.mark.parametrize("pos,w_local", [(3000, 512), (700, 2048)])  # remote + local, local only
def test_decode_wait_timeout_is_reported_and_recovered(jl, pos, w_local):
    B, Hq, Hkv, D = 1, 32, 8, 128
    q, kc, vc = W.decode_inputs(B, Hq, Hkv, D, pos + 1, seed=11)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    kw = dict(w_local=w_local, w_pretrained=1024, rope_base=1e6)

    out0, lse0 = jl.bifocal_decode(q, kc, vc, pos, **kw)
    jl.check_device_status()
    out0, lse0 = out0.clone(), lse0.clone()

    jl.bifocal_decode(q, kc, vc, pos, flags=jl.DEBUG_SKIP_ARRIVE, **kw)
    with pytest.raises(jl.JetLongError) as err:
        jl.check_device_status()
    assert err.value.status == TIMEOUT
    jl.check_device_status()  # the word was cleared

    out1, lse1 = jl.bifocal_decode(q, kc, vc, pos, **kw)
    jl.check_device_status()
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)


def test_debug_flag_rejected_where_it_has_no_meaning(jl):
    q = torch.zeros(1, 256, 4, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(1, 256, 4, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(jl.JetLongError) as err:
        jl.bifocal_prefill(q, k, k, w_local=16, w_pretrained=64, rope_base=1e6,
                           flags=jl.DEBUG_SKIP_ARRIVE)
    assert err.value.status == 1  # JL_ERR_INVALID_ARG: unknown flag for prefill

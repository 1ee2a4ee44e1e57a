"""The decode step from host buffers (DecodeStep.run_host): inputs in with one
copy, the step, the result out with one copy -- eagerly and as one CUDA graph
replay -- gives the same cache bytes and outputs as the step on device
buffers."""
import numpy as np
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W

from helpers import Case, dev64, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fused", [True, False])
def test_host_step_matches_device_step(fused):
    wl = W.workload("llama8b_b8_32k", batch=2)
    case = Case(wl, n_ctx=500)
    A, Ai = dev64(case.A), dev64(case.Ai)
    dev_step = kvq.DecodeStep(case.gpu_cache(), A, Ai, 0.4, wl.n_q_heads, fused=fused)
    host_step = kvq.DecodeStep(case.gpu_cache(), A, Ai, 0.4, wl.n_q_heads, fused=fused)
    as_host = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)  # noqa: E731
    for i in range(5):
        kn, vn = W.make_step_kv(wl, i)
        q = case.q(i)
        dev_step.q.copy_(to_dev(q, "bf16"))
        dev_step.k_new.copy_(to_dev(kn, "bf16"))
        dev_step.v_new.copy_(to_dev(vn, "bf16"))
        want = dev_step.run().clone()
        got = host_step.run_host(as_host(q), as_host(kn), as_host(vn))
        torch.cuda.synchronize()
        assert torch.equal(got, want.cpu()), i
        if i == 1:
            host_step.capture()                  # later steps: one graph replay each
    assert torch.equal(dev_step.cache.pages, host_step.cache.pages)
    assert host_step.cache.seq_len.tolist() == [505, 505]
    assert host_step.h2d_bytes >= (wl.n_q_heads + 2 * wl.n_kv_heads) * 2 * 128 * 2
    assert host_step.d2h_bytes == 2 * wl.n_q_heads * 128 * 4

"""kvq_decode_attn_static: decode for callers that cannot allocate device
memory at call time (an engine plugin with no scratch buffer, a decode loop
that must not call cudaMalloc).  Its split partials live in the library's one
static device array instead of a caller workspace; it runs the same splits of
the same kernel as kvq_decode_attn, so its result must equal that one bit for
bit, call after call.

This file is collected last on purpose: the static array is shared by every
call in the process, so the test also covers reuse after the other tests."""
import numpy as np
import pytest

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W

from helpers import Case, dev64, to_dev

pytestmark = pytest.mark.gpu


def test_static_scratch_decode_matches_workspace_decode():
    case = Case(W.workload("llama8b_b8_32k", batch=2), n_ctx=700)
    cache = case.gpu_cache()
    assert kvq.decode_workspace_bytes(cache, 32, 77) <= kvq.decode_static_scratch_bytes()
    for step in (0, 1):                       # two calls in a row
        q = case.q(step)
        sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), 0.4)
        ref = kvq.decode_attn(cache, sel).cpu().numpy()
        got = kvq.decode_attn_static(cache, sel).cpu().numpy()
        assert np.isfinite(got).all()
        assert np.array_equal(got, ref), (step, float(np.abs(got - ref).max()))


def test_static_scratch_rejects_oversized_request():
    # grow the batch until the partials need more than the static array,
    # whatever split count this device's SM count gives
    k, hq, batch = 77, 256, 1
    while True:
        cache = kvq.new_cache(batch, 32, 512, 2)
        if kvq.decode_workspace_bytes(cache, hq, k) > kvq.decode_static_scratch_bytes():
            break
        batch *= 2
        assert batch <= 1024
    sel = kvq.alloc_selection(cache, hq, k)
    with pytest.raises(kvq.KvqError) as err:
        kvq.decode_attn_static(cache, sel)
    assert err.value.status == -4

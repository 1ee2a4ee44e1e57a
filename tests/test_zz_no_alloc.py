"""kvq_decode_attn_static: decode for callers that cannot allocate device
memory at call time (an engine plugin with no scratch buffer, a decode loop
that must not call cudaMalloc).  Its split partials live in the library's one
static device array instead of a caller workspace; the result must match
kvq_decode_attn's, call after call.

This file is collected last on purpose: the static array is shared by every
call in the process, so the test also covers reuse after the other tests."""
import numpy as np
import pytest

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W

from helpers import Case, dev64, rel_errors, to_dev

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-3
TOL_MEAN = 1e-3


def test_static_scratch_decode_matches_workspace_decode():
    case = Case(W.workload("llama8b_b8_32k", batch=2), n_ctx=700)
    cache = case.gpu_cache()
    assert kvq.decode_workspace_bytes(cache, 32, 77) <= kvq.decode_static_scratch_bytes()
    for step in (0, 1):                       # two calls in a row
        q = case.q(step)
        sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), 0.4)
        ref = kvq.decode_attn(cache, sel).cpu().numpy()
        got = kvq.decode_attn_static(cache, sel).cpu().numpy()
        emax, emean = rel_errors(got, ref)
        assert emax <= TOL_MAX and emean <= TOL_MEAN, (step, emax, emean)
        assert np.isfinite(got).all()


def test_static_scratch_rejects_oversized_request():
    # 16 sequences x 256 query heads x 2 splits of partials need more than 4 MiB
    cache = kvq.new_cache(16, 32, 512, 2)
    k = 77
    assert kvq.decode_workspace_bytes(cache, 256, k) > kvq.decode_static_scratch_bytes()
    sel = kvq.alloc_selection(cache, 256, k)
    with pytest.raises(kvq.KvqError) as err:
        kvq.decode_attn_static(cache, sel)
    assert err.value.status == -4

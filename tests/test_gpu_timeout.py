"""Bounded waits of the tensor-core decode.  Every wait for a staged page has
a limit; a wait that runs out sets KVQ_DEV_TIMEOUT, after which the pair of
warps issues no further copy, lets the copies already in flight land, and
finishes, so the call returns normally (its output is not valid) and the cache,
its counters and the GPU are ready for the next call.  The test makes the wait
run out with a bound of zero polls through the fault-handling hook
kvq_decode_attn_wait_bound: nothing is planted in the kernel and no copy is
lost -- the copies simply have not landed when the wait looks."""
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W

from helpers import Case, dev64, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("protect", [False, True])
def test_wait_give_up_reports_timeout_and_leaves_the_cache_usable(protect):
    wl = W.workload("llama8b_b8_32k", batch=1)
    case = Case(wl, n_ctx=3000)
    tier = dict(n_sink=64, n_recent=256) if protect else {}
    cache = kvq.new_cache(wl.batch, wl.n_kv_heads, case.capacity, wl.bits, **tier)
    kvq.append(cache, to_dev(case.K, "bf16"), to_dev(case.V, "bf16"), dev64(case.A))
    sel = kvq.select_channels(cache, to_dev(case.q(0), "bf16"), dev64(case.Ai), 0.4)
    ref = kvq.decode_attn(cache, sel)
    assert kvq.read_status(cache) == 0

    kvq.decode_attn_wait_bound(cache, sel, 0)
    flags = kvq.read_status(cache)
    assert flags & kvq.KVQ_DEV_TIMEOUT, flags
    # only the flag word is left set: every completion counter is back at zero
    assert int(cache.status[1:].abs().sum()) == 0
    cache.status[0] = 0                       # the caller clears the sticky flag

    again = kvq.decode_attn(cache, sel)
    assert kvq.read_status(cache) == 0
    assert torch.equal(again, ref)
    # a generous bound is the normal call
    out = kvq.decode_attn_wait_bound(cache, sel, 1 << 20)
    assert kvq.read_status(cache) == 0
    assert torch.equal(out, ref)


def test_wait_bound_hook_rejects_shapes_without_staged_pages():
    wl = W.workload("llama8b_b8_32k", batch=1, n_q_heads=8)     # one query head per KV head
    cache = kvq.new_cache(wl.batch, wl.n_kv_heads, 1024, 2)
    sel = kvq.alloc_selection(cache, 8, 77)
    with pytest.raises(kvq.KvqError) as err:
        kvq.decode_attn_wait_bound(cache, sel, 0)
    assert err.value.status == -2

"""GPU parity of the protected BF16 tier (Dual-QK §3.3: the first n_sink and
the most recent n_recent tokens kept in BF16 for keys and values, with the
same query-channel mask; §3.4: one softmax over all tiers).

After a prefill and decode steps -- through kvq_decode_step (one launch for
INT2 with 4 query heads per KV head) or the three calls -- the pages and the
BF16 slots equal the oracle's byte for byte, the selection is the oracle's,
and the outputs are within the decode tolerance of the oracle's attention
over the BF16 tier plus the codes of the other tokens.
"""
import numpy as np
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W
from oracle import oracle as orc

from helpers import Case, check_pages, dev64, rel_errors, to_dev

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-3
TOL_MEAN = 1e-3


def _oracle_slots(case: Case, b: int, h: int, n: int, n_sink: int, n_recent: int) -> np.ndarray:
    wl = case.wl
    Kf = W.as_float(case.K[b, h, :n], wl.dtype)
    Vf = W.as_float(case.V[b, h, :n], wl.dtype)
    slots = orc.new_slots(n_sink, n_recent)
    orc.protect_store(slots, n_sink, n_recent, 0, case.oracle_keys(Kf, h), case.oracle_values(Vf, h), n)
    return slots


def _run(case: Case, n0: int, n_new: int, n_steps: int, n_sink: int, n_recent: int, fused: bool,
         sparsity: float = 0.4, units=None):
    wl = case.wl
    g = wl.group_size
    A, Ai, dl = dev64(case.A), dev64(case.Ai), case.dev_delta()
    cache = kvq.new_cache(wl.batch, wl.n_kv_heads, case.capacity, wl.bits, n_sink=n_sink, n_recent=n_recent,
                          **case.cache_kw())
    if n0:
        kvq.append(cache, to_dev(case.K[:, :, :n0], wl.dtype), to_dev(case.V[:, :, :n0], wl.dtype), A)
    pos = n0
    us = units or [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
    for i in range(n_steps):
        q = case.q(i)
        qd = to_dev(q, wl.dtype)
        kn = to_dev(case.K[:, :, pos:pos + n_new], wl.dtype)
        vn = to_dev(case.V[:, :, pos:pos + n_new], wl.dtype)
        if fused:
            out, sel = kvq.decode_step(cache, qd, kn, vn, A, Ai, sparsity, delta=dl)
        else:
            kvq.append(cache, kn, vn, A)
            sel = kvq.select_channels(cache, qd, Ai, sparsity, delta=dl)
            out = kvq.decode_attn(cache, sel)
        torch.cuda.synchronize()
        pos += n_new
        out = out.cpu().numpy()
        for b, h in us:
            slots = _oracle_slots(case, b, h, pos, n_sink, n_recent)
            want, ref_idx = case.oracle_decode_any(q, b, h, sparsity, pos, slots, n_sink, n_recent)
            got_idx = sel.idx[b, h].cpu().numpy()
            assert np.array_equal(got_idx[:len(ref_idx)] if case.wl.bucket else got_idx, ref_idx)
            emax, emean = rel_errors(out[b, h * g:(h + 1) * g], want)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (i, b, h, emax, emean)
    assert cache.seq_len.tolist() == [pos] * wl.batch
    assert kvq.read_status(cache) == 0
    assert not cache.status[1:].any()
    check_pages(case, cache, units, pos)
    got = cache.slots().cpu().numpy().view(np.uint16)
    for b, h in us:
        want = _oracle_slots(case, b, h, pos, n_sink, n_recent)
        assert np.array_equal(got[b, h], want), (b, h)
    return cache


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("n0,n_new,n_sink,n_recent", [
    (200, 1, 64, 256),      # every token protected
    (319, 1, 64, 256),      # the step that fills both tiers
    (1000, 1, 64, 256),
    (1000, 4, 64, 256),
    (500, 1, 16, 40),       # recent window inside the last coded page
    (700, 2, 64, 0),        # sink only
    (700, 1, 0, 256),       # recent window only
    (126, 3, 128, 128),     # new tokens straddle a page; a sink of a whole page
])
def test_tier_int2_gqa4(n0, n_new, n_sink, n_recent, fused):
    n_steps = 2
    wl = W.workload("llama8b_b8_32k", batch=2)
    case = Case(wl, n_ctx=n0 + n_steps * n_new)
    _run(case, n0, n_new, n_steps, n_sink, n_recent, fused)


@pytest.mark.parametrize("bits,g", [(4, 4), (2, 2), (2, 8), (2, 1)])
def test_tier_other_shapes(bits, g):
    wl = W.workload("llama8b_b8_32k", batch=2, bits=bits, n_q_heads=8 * g)
    case = Case(wl, n_ctx=900 + 2)
    _run(case, 900, 1, 2, 64, 256, fused=True)


@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_tier_sparsities(sparsity):
    wl = W.workload("llama8b_b8_32k", batch=1)
    case = Case(wl, n_ctx=1200 + 1)
    _run(case, 1200, 1, 1, 64, 256, fused=True, sparsity=sparsity)


def test_tier_long_context_sampled_units():
    wl = W.workload("longctx_b1_128k")
    case = Case(wl, n_ctx=6000 + 2)
    _run(case, 6000, 1, 2, 64, 256, fused=True, units=[(0, 0), (0, 7)])

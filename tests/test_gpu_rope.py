"""GPU parity of bucket-relative RoPE (Dual-QK §3.4, App. C.4).

Keys are stored in the frame of their bucket's anchor, K' = (k T_b) A; each
bucket b that holds a token gets its own channel choice from the query moved
into its frame, q'_b = (q T_b) A^{-T}; the decode scores each token with its
bucket's queries and channels under one softmax (pages and the protected
tier alike).

Bars as for the rest of the path: pages, protected slots, channel lists and
the documented qsel / qgsum roundings byte-exact against the oracle; outputs
within 2e-3 max / 1e-3 mean of the oracle's.
"""
import numpy as np
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W
from oracle import oracle as orc

from helpers import Case, check_pages, dev64, expected_qsel_qgsum, rel_errors, to_dev
import test_gpu_protected as tp

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-3
TOL_MEAN = 1e-3
PAGES = dict(rotate_values=True, v_clip=0.92, refine=True)


@pytest.mark.parametrize("w", [128, 384])
@pytest.mark.parametrize("group", [32, 128])
@pytest.mark.parametrize("bits", [2, 4])
def test_append_bit_exact(bits, group, w):
    """Prefill tiles, then decode-sized appends across bucket boundaries."""
    wl = W.workload("llama8b_b8_32k", batch=2, bits=bits, quant_group=group, bucket=w)
    case = Case(wl, n_ctx=770)
    cache = case.gpu_cache(chunks=[765, 1, 4])
    check_pages(case, cache)


@pytest.mark.parametrize("g", [1, 4, 8])
@pytest.mark.parametrize("sparsity", [0.0, 0.4, 0.6])
def test_select_per_bucket(sparsity, g):
    wl = W.workload("llama8b_b8_32k", batch=2, n_q_heads=8 * g, bucket=128, refine=True)
    n = 300                                          # buckets 0, 1, 2 hold tokens; 3.. do not
    case = Case(wl, n_ctx=n, capacity=1024)
    cache = case.gpu_cache()
    k = orc.num_selected(sparsity)
    sel = kvq.alloc_selection(cache, 8 * g, k)
    sel.idx.fill_(-7)
    q = case.q(0)
    kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), sparsity, out=sel, delta=case.dev_delta())
    idx = sel.idx.cpu().numpy()
    qsel = sel.qsel.cpu().numpy()
    qgsum = sel.qgsum.cpu().numpy()
    assert idx.shape == (2, 8, 8, k)
    for b in range(2):
        for h in range(8):
            qf = W.as_float(q[b, h * g:(h + 1) * g], "bf16")
            qpb = orc.bucket_queries(qf, case.Ai[h], case.rope, 3)
            for bk in range(3):
                ref, _ = orc.select(qpb[bk], k, case.delta[h])
                assert np.array_equal(idx[b, h, bk], ref), (b, h, bk)
                rq, rg = expected_qsel_qgsum(qpb[bk], ref)
                assert np.array_equal(qsel[b, h * g:(h + 1) * g, bk], rq)
                assert np.array_equal(qgsum[b, h * g:(h + 1) * g, bk], rg)
            assert (idx[b, h, 3:] == -7).all()           # buckets past the length are not written
    if sparsity > 0:
        assert any(not np.array_equal(idx[0, h, 0], idx[0, h, 1]) for h in range(8))


def _decode_and_compare(case: Case, cache, sparsity, steps=(0, 1), units=None, n=None):
    wl = case.wl
    g = wl.group_size
    n = case.K.shape[2] if n is None else n
    for step in steps:
        q = case.q(step)
        sel = kvq.select_channels(cache, to_dev(q, wl.dtype), dev64(case.Ai), sparsity, delta=case.dev_delta())
        out = kvq.decode_attn(cache, sel).cpu().numpy()
        for b, h in units or [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]:
            ref, ref_idx = case.oracle_decode_any(q, b, h, sparsity, n)
            assert np.array_equal(sel.idx[b, h, :len(ref_idx)].cpu().numpy(), ref_idx)
            emax, emean = rel_errors(out[b, h * g:(h + 1) * g], ref)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (step, b, h, emax, emean)


@pytest.mark.parametrize("group", [32, 128])
@pytest.mark.parametrize("bits,g,w", [(2, 4, 128), (2, 4, 512), (2, 1, 256), (2, 8, 128), (4, 4, 256), (4, 2, 128)])
def test_decode_parity(bits, g, w, group):
    """The tensor-core decode (INT2, 4 heads per KV head) and the CUDA-core
    decode, each running one segment per bucket inside a split."""
    wl = W.workload("llama8b_b8_32k", batch=2, bits=bits, n_q_heads=8 * g, quant_group=group, bucket=w)
    case = Case(wl, n_ctx=1700)
    cache = case.gpu_cache()
    _decode_and_compare(case, cache, 0.4)


def test_one_bucket_equals_no_buckets():
    """Buckets as large as the capacity: anchor 0 (cos 1, sin 0) leaves keys
    and queries as they are; pages and channels are those of the cache
    without buckets, bit for bit, and so are the scores and weights of every
    token.  The outputs agree to float32 summation order only: a bucketed
    decode reads each split's pages as one contiguous range (one segment per
    bucket), an unbucketed one deals the pages round-robin to the pairs, so
    the splits' partial sums are formed in different orders."""
    base = W.workload("llama8b_b8_32k", batch=2)
    outs = []
    for w in (0, 2048):
        case = Case(base.with_(bucket=w), n_ctx=1500, capacity=2048)
        cache = case.gpu_cache()
        q = to_dev(case.q(0), "bf16")
        sel = kvq.select_channels(cache, q, dev64(case.Ai), 0.4)
        out = kvq.decode_attn(cache, sel)
        torch.cuda.synchronize()
        outs.append((cache.all_pages().clone(), sel.idx.reshape(2, 8, -1).clone(), out.clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    emax, _ = rel_errors(outs[0][2].cpu().numpy(), outs[1][2].cpu().numpy())
    assert emax <= 1e-5, emax


@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_decode_sparsity_sweep(sparsity):
    case = Case(W.workload("sweep_b32_16k", batch=3, bucket=256), n_ctx=900)
    cache = case.gpu_cache()
    _decode_and_compare(case, cache, sparsity, steps=(0,))


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("group", [32, 128])
@pytest.mark.parametrize("n0,n_new,n_sink,n_recent,w", [
    (1000, 1, 64, 256, 256),     # recent window across a bucket boundary
    (1000, 4, 64, 256, 128),
    (126, 3, 128, 128, 128),     # new tokens straddle a page and a bucket
    (700, 1, 0, 0, 256),         # no protected tier
    (200, 2, 64, 256, 128),      # every token protected
])
def test_step_with_tier_and_rotation(n0, n_new, n_sink, n_recent, w, group, fused):
    """Decode steps with the pages' whole recipe and buckets (a bucketed step
    runs as the three calls): pages, BF16 slots, per-bucket channel lists,
    outputs."""
    case = Case(W.workload("llama8b_b8_32k", batch=2, quant_group=group, bucket=w, **PAGES), n_ctx=n0 + 3 * n_new)
    tp._run(case, n0, n_new, 3, n_sink, n_recent, fused=fused)


def test_other_shapes_with_tier():
    wl = W.workload("llama8b_b8_32k", batch=2, bits=4, n_q_heads=16, bucket=256, **PAGES)
    case = Case(wl, n_ctx=900 + 2)
    tp._run(case, 900, 1, 2, 64, 256, fused=True)


def test_long_context_sampled_units():
    """The headline shape with the pages' recipe and 2048-token buckets at a
    shortened context (several buckets per split); sampled units."""
    wl = W.workload("longctx_b1_128k", quant_group=128, bucket=2048, **PAGES)
    case = Case(wl, n_ctx=9000 + 2)
    tp._run(case, 9000, 1, 2, 64, 256, fused=True, units=[(0, 0), (0, 7)])


def test_full_size_sampled():
    """Full 128K context (65 buckets of 2048 tokens) in the benchmark's launch
    configuration with the pages' recipe: every unit runs; two are checked."""
    wl = W.workload("longctx_b1_128k", quant_group=128, bucket=2048, **PAGES)
    case = Case(wl)
    cache = case.gpu_cache()
    check_pages(case, cache, units=[(0, 1), (0, 6)])
    _decode_and_compare(case, cache, 0.4, steps=(0,), units=[(0, 1), (0, 6)])

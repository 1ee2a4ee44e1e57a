"""GPU parity of the value rotation with clipped value grids and of the
selection on base queries under a diagonal refinement (Dual-QK §3.3,
App. B.2 and App. C.2).

Values are stored as V Rv, quantized with the grid [0.92 min, 0.92 max]
(keys unclipped); decodes aggregate in the rotated basis and return o Rv^T.
With the refinement D folded into the transforms (key transform A D^{-1},
query transform A^{-T} D) selection uses q' / delta and scores use q'.

Bars as for the plain path: pages, protected slots, channel lists and the
documented qsel / qgsum roundings byte-exact against the oracle; outputs
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
PAGES = dict(rotate_values=True, v_clip=0.92, refine=True)    # the pages' recipe


def _wl(name, **kw):
    base = W.workload(name)
    kw.setdefault("batch", min(2, base.batch))
    return W.workload(name, **PAGES, **kw)


@pytest.mark.parametrize("group", [32, 128])
@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("name,n_ctx", [("single_head_4k", 700), ("llama8b_b8_32k", 300),
                                        ("pipeline_128k_t4", 1000)])
def test_append_bit_exact(name, n_ctx, bits, group):
    """Prefill tiles, then decode-sized appends (the small-append kernel for
    groups of 32): codes and fp16 metadata of the rotated, clipped values."""
    case = Case(_wl(name, bits=bits, quant_group=group), n_ctx=n_ctx)
    cache = case.gpu_cache(chunks=[n_ctx - 5, 1, 4])
    check_pages(case, cache)


def test_clip_alone_and_rotation_alone():
    for kw in (dict(v_clip=0.92), dict(rotate_values=True), dict(refine=True)):
        case = Case(W.workload("llama8b_b8_32k", batch=1, **kw), n_ctx=260)
        cache = case.gpu_cache(chunks=[255, 1, 4])
        check_pages(case, cache)


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_refined_select_bit_exact(sparsity, g):
    wl = W.workload("llama8b_b8_32k", batch=2, n_q_heads=8 * g, refine=True)
    case = Case(wl, n_ctx=128)
    cache = kvq.new_cache(2, 8, 128, 2)
    q = case.q(0)
    sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), sparsity, delta=case.dev_delta())
    k = orc.num_selected(sparsity)
    moved = 0
    for b in range(2):
        for h in range(8):
            qp = case.oracle_qp(q, b, h)
            ref_idx, _ = orc.select(qp, k, case.delta[h])
            got = sel.idx[b, h].cpu().numpy()
            assert np.array_equal(got, ref_idx), (b, h)
            moved += not np.array_equal(got, orc.select(qp, k)[0])
            rq, rg = expected_qsel_qgsum(qp, ref_idx)
            assert np.array_equal(sel.qsel[b, h * g:(h + 1) * g].cpu().numpy(), rq)
            assert np.array_equal(sel.qgsum[b, h * g:(h + 1) * g].cpu().numpy(), rg)
    if 0.0 < sparsity:
        assert moved > 0          # the refinement does change the final queries' order


def _decode_and_compare(case: Case, cache, sparsity, steps=(0, 1), units=None):
    wl = case.wl
    g = wl.group_size
    for step in steps:
        q = case.q(step)
        sel = kvq.select_channels(cache, to_dev(q, wl.dtype), dev64(case.Ai), sparsity, delta=case.dev_delta())
        out = kvq.decode_attn(cache, sel).cpu().numpy()
        for b, h in units or [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]:
            ref, ref_idx, _ = case.oracle_decode(q, b, h, sparsity)
            assert np.array_equal(sel.idx[b, h].cpu().numpy(), ref_idx)
            emax, emean = rel_errors(out[b, h * g:(h + 1) * g], ref)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (step, b, h, emax, emean)


@pytest.mark.parametrize("group", [32, 128])
@pytest.mark.parametrize("bits,g", [(2, 4), (2, 1), (2, 8), (4, 4), (4, 2)])
def test_decode_parity(bits, g, group):
    """The tensor-core decode (INT2, 4 heads per KV head) and the CUDA-core
    decode (other shapes), each rotating its merged output back."""
    wl = W.workload("llama8b_b8_32k", batch=2, bits=bits, n_q_heads=8 * g, quant_group=group, **PAGES)
    case = Case(wl, n_ctx=1500)
    cache = case.gpu_cache()
    _decode_and_compare(case, cache, 0.4)


@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_decode_sparsity_sweep(sparsity):
    case = Case(W.workload("sweep_b32_16k", batch=3, **PAGES), n_ctx=700)
    cache = case.gpu_cache()
    _decode_and_compare(case, cache, sparsity, steps=(0,))


def test_decode_static_matches_workspace_call():
    case = Case(W.workload("llama8b_b8_32k", batch=2, **PAGES), n_ctx=900)
    cache = case.gpu_cache()
    q = case.q(0)
    sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), 0.4, delta=case.dev_delta())
    a = kvq.decode_attn(cache, sel)
    b = kvq.decode_attn_static(cache, sel)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("group", [32, 128])
@pytest.mark.parametrize("n0,n_new,n_sink,n_recent", [
    (1000, 1, 64, 256),
    (1000, 4, 64, 256),
    (126, 3, 128, 128),     # new tokens straddle a page
    (700, 1, 0, 0),         # no protected tier
    (200, 2, 64, 256),      # every token protected
])
def test_step_with_tier(n0, n_new, n_sink, n_recent, group, fused):
    """Decode steps (one launch when fused): pages, BF16 slots of rotated
    values, channel lists and outputs."""
    case = Case(W.workload("llama8b_b8_32k", batch=2, quant_group=group, **PAGES), n_ctx=n0 + 3 * n_new)
    tp._run(case, n0, n_new, 3, n_sink, n_recent, fused=fused)


@pytest.mark.parametrize("bits,g", [(4, 4), (2, 2)])
def test_step_other_shapes(bits, g):
    wl = W.workload("llama8b_b8_32k", batch=2, bits=bits, n_q_heads=8 * g, **PAGES)
    case = Case(wl, n_ctx=900 + 2)
    tp._run(case, 900, 1, 2, 64, 256, fused=True)


def test_step_fused_matches_three_calls():
    """The fused step stores the same bytes and chooses the same channels as
    the three calls; outputs agree within the decode tolerance."""
    wl = W.workload("llama8b_b8_32k", batch=2, **PAGES)
    case = Case(wl, n_ctx=1300)
    A, Ai, dl = dev64(case.A), dev64(case.Ai), case.dev_delta()
    caches = []
    outs = []
    for fused in (True, False):
        cache = kvq.new_cache(2, 8, case.capacity, 2, n_sink=64, n_recent=256, **case.cache_kw())
        kvq.append(cache, to_dev(case.K[:, :, :1296], "bf16"), to_dev(case.V[:, :, :1296], "bf16"), A)
        for i in range(4):
            q = to_dev(case.q(i), "bf16")
            kn = to_dev(case.K[:, :, 1296 + i:1297 + i], "bf16")
            vn = to_dev(case.V[:, :, 1296 + i:1297 + i], "bf16")
            if fused:
                out, sel = kvq.decode_step(cache, q, kn, vn, A, Ai, 0.4, delta=dl)
            else:
                kvq.append(cache, kn, vn, A)
                sel = kvq.select_channels(cache, q, Ai, 0.4, delta=dl)
                out = kvq.decode_attn(cache, sel)
        torch.cuda.synchronize()
        caches.append((cache, sel))
        outs.append(out.cpu().numpy())
    assert torch.equal(caches[0][0].pages, caches[1][0].pages)
    assert torch.equal(caches[0][1].idx, caches[1][1].idx)
    emax, emean = rel_errors(outs[0], outs[1])
    assert emax <= TOL_MAX and emean <= TOL_MEAN


def test_long_context_sampled_units():
    """The headline shape with the pages' recipe (one grid per token, tier,
    rotation, clip, refinement) at a shortened context; sampled units."""
    wl = W.workload("longctx_b1_128k", quant_group=128, **PAGES)
    case = Case(wl, n_ctx=6000 + 2)
    tp._run(case, 6000, 1, 2, 64, 256, fused=True, units=[(0, 0), (0, 7)])


def test_full_size_sampled():
    """Full 128K context in the benchmark's launch configuration with the
    pages' recipe: every unit runs; two are checked against the oracle."""
    wl = W.workload("longctx_b1_128k", quant_group=128, **PAGES)
    case = Case(wl)
    cache = case.gpu_cache()
    check_pages(case, cache, units=[(0, 2), (0, 6)])
    _decode_and_compare(case, cache, 0.4, steps=(0,), units=[(0, 2), (0, 6)])

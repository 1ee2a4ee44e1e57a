"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bars: packed codes, fp16 scale/zero bit patterns, bf16 channel 0 and the
selected channel indices are bit-exact; qsel / qgsum are the documented fp32
roundings, bit-exact; the attention output is within 2e-3 max and 1e-3 mean
relative error (|o - o_ref| / ||o_ref||_inf per output vector) of the oracle
run on the same codes and the same selected channels.
"""
import numpy as np
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W
from oracle import oracle as orc

from helpers import Case, check_pages, dev64, expected_qsel_qgsum, rel_errors, to_dev

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-3
TOL_MEAN = 1e-3


_check_pages = check_pages


def _cases_small():
    return [
        ("single_head_4k", None),
        ("llama8b_b8_32k", 300),
        ("longctx_b1_128k", 257),
        ("sweep_b32_16k", 130),
        ("pipeline_128k_t4", 1000),
    ]


@pytest.mark.parametrize("name,n_ctx", _cases_small())
@pytest.mark.parametrize("bits", [2, 4])
def test_append_bit_exact(name, n_ctx, bits):
    case = Case(W.workload(name, bits=bits), n_ctx=n_ctx)
    cache = case.gpu_cache()
    assert cache.seq_len.cpu().tolist() == [case.K.shape[2]] * case.wl.batch
    assert kvq.read_status(cache) == 0
    _check_pages(case, cache)


@pytest.mark.parametrize("bits", [2, 4])
def test_append_in_chunks_keeps_neighbouring_codes(bits):
    case = Case(W.workload("llama8b_b8_32k", batch=2, bits=bits), n_ctx=291)
    cache = case.gpu_cache(chunks=[7, 1, 130, 1, 3, 16, 133])
    _check_pages(case, cache)


@pytest.mark.parametrize("bits", [2, 4])
def test_append_rounding_edges(bits):
    """Keys whose transformed values sit on or next to fp16 / bf16 rounding
    ties, in the fp16 subnormal range, and groups with a zero range."""
    rng = np.random.default_rng(123)
    edges = np.array([1 + 2.0 ** -11, 1 + 2.0 ** -11 + 2.0 ** -45, 1 + 2.0 ** -11 - 2.0 ** -45,
                      1 + 3 * 2.0 ** -11, 1 + 2.0 ** -8 + 2.0 ** -40, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8,
                      2.0 ** -20, 3 * 2.0 ** -25, 1.0, 2.0 ** -14 * (1 + 2.0 ** -11), 1000.5])
    wl = W.workload("single_head_4k", bits=bits)
    n = 256
    case = Case(wl, n_ctx=n)
    A = np.diag(rng.choice(edges, 128)).reshape(1, 128, 128)
    K = rng.choice([1.0, -1.0, 1.5, 0.75, 2.0, -0.5], size=(1, 1, n, 128)).astype(np.float32)
    K[0, 0, :16, 1:32] = 0.5          # zero-range groups
    V = rng.choice([0.25, -3.0, 1.0 + 2.0 ** -11, 7.5], size=(1, 1, n, 128)).astype(np.float32)
    case.A, case.K, case.V = A, K, V
    cache = case.gpu_cache()
    _check_pages(case, cache)


def test_append_capacity_overflow_sets_flag():
    case = Case(W.workload("llama8b_b8_32k", batch=2), n_ctx=200, capacity=256)
    cache = case.gpu_cache()
    before = cache.pages.clone()
    extra = W.make_kv(case.wl.with_(n_ctx=100))
    kvq.append(cache, to_dev(extra[0], "bf16"), to_dev(extra[1], "bf16"), dev64(case.A))
    assert kvq.read_status(cache) & kvq.KVQ_DEV_CAPACITY
    assert cache.seq_len.cpu().tolist() == [200, 200]
    assert torch.equal(before, cache.pages)
    with pytest.raises(kvq.KvqError):
        kvq.append(cache, to_dev(extra[0][:, :, :1].repeat(300, axis=2), "bf16"),
                   to_dev(extra[1][:, :, :1].repeat(300, axis=2), "bf16"), dev64(case.A))


def _check_selection(case: Case, q: np.ndarray, sel: kvq.Selection, sparsity: float):
    wl = case.wl
    g = wl.group_size
    k = orc.num_selected(sparsity)
    assert sel.k == k
    idx = sel.idx.cpu().numpy()
    qsel = sel.qsel.cpu().numpy()
    qgsum = sel.qgsum.cpu().numpy()
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            qp = case.oracle_qp(q, b, h)
            ref_idx, _ = orc.select(qp, k)
            assert np.array_equal(idx[b, h], ref_idx), (b, h)
            rq, rg = expected_qsel_qgsum(qp, ref_idx)
            assert np.array_equal(qsel[b, h * g:(h + 1) * g], rq), (b, h)
            assert np.array_equal(qgsum[b, h * g:(h + 1) * g], rg), (b, h)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_select_bit_exact(name, sparsity):
    case = Case(W.workload(name), n_ctx=128)
    cache = kvq.new_cache(case.wl.batch, case.wl.n_kv_heads, case.capacity, 2)
    for step in range(2):
        q = case.q(step)
        sel = kvq.select_channels(cache, to_dev(q, case.wl.dtype), dev64(case.Ai), sparsity)
        _check_selection(case, q, sel, sparsity)


def test_select_ties_go_to_lower_channel():
    wl = W.workload("llama8b_b8_32k", batch=2)
    case = Case(wl, n_ctx=128)
    case.Ai = np.broadcast_to(np.eye(128), (wl.n_kv_heads, 128, 128)).copy()
    rng = np.random.default_rng(5)
    q = W.bf16_bits_from_f32(rng.integers(-2, 3, size=(2, 32, 128)).astype(np.float32))
    cache = kvq.new_cache(2, 8, 128, 2)
    for s in (0.2, 0.4, 0.6):
        sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), s)
        _check_selection(case, q, sel, s)


def _decode_and_compare(case: Case, cache, sparsity, steps=(0,), units=None, n=None):
    wl = case.wl
    g = wl.group_size
    errs = []
    for step in steps:
        q = case.q(step)
        sel = kvq.select_channels(cache, to_dev(q, wl.dtype), dev64(case.Ai), sparsity)
        out = kvq.decode_attn(cache, sel).cpu().numpy()
        us = units or [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
        for b, h in us:
            ref, ref_idx, _ = case.oracle_decode(q, b, h, sparsity, n)
            assert np.array_equal(sel.idx[b, h].cpu().numpy(), ref_idx)
            got = out[b, h * g:(h + 1) * g]
            emax, emean = rel_errors(got, ref)
            errs.append((emax, emean))
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (step, b, h, emax, emean)
    return errs


@pytest.mark.parametrize("name,n_ctx", _cases_small())
@pytest.mark.parametrize("bits", [2, 4])
def test_decode_parity(name, n_ctx, bits):
    case = Case(W.workload(name, bits=bits), n_ctx=n_ctx)
    cache = case.gpu_cache()
    _decode_and_compare(case, cache, case.wl.sparsity, steps=(0, 1))


@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_decode_parity_sparsity_sweep(sparsity):
    case = Case(W.workload("sweep_b32_16k", batch=4), n_ctx=700)
    cache = case.gpu_cache()
    _decode_and_compare(case, cache, sparsity)


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_decode_parity_group_sizes(g):
    case = Case(W.workload("llama8b_b8_32k", batch=2, n_q_heads=4 * g, n_kv_heads=4), n_ctx=515)
    cache = case.gpu_cache()
    _decode_and_compare(case, cache, 0.4)


def test_decode_edge_lengths():
    case = Case(W.workload("llama8b_b8_32k", batch=4), n_ctx=300)
    cache = case.gpu_cache()
    q = case.q(0)
    g = case.wl.group_size
    # ragged lengths: the caller owns seq_len; decode must honour it
    lens = [0, 1, 128, 129]
    cache.seq_len.copy_(torch.tensor(lens, dtype=torch.int32))
    sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), 0.4)
    out = kvq.decode_attn(cache, sel).cpu().numpy()
    assert not out[0].any()                                     # empty sequence -> zeros
    for b, n in enumerate(lens[1:], start=1):
        for h in (0, 5):
            ref, _, _ = case.oracle_decode(q, b, h, 0.4, n)
            emax, emean = rel_errors(out[b, h * g:(h + 1) * g], ref)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (b, h, emax)
    # a single token: the output is that token's dequantized value row
    _, Vh = orc.dequant_unit(case.oracle_unit(1, 0), 2, 1)
    np.testing.assert_allclose(out[1, 0], Vh[0], rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("g,n_ctx,qscale", [(4, 1000, 1.0), (1, 777, 1.0), (2, 130, 1.0), (8, 64, 1.0),
                                             (4, 1, 1.0), (4, 3000, 8.0)])
def test_bf16_comparator_matches_plain_attention(g, n_ctx, qscale):
    """The unpruned BF16 comparator against the oracle's plain attention:
    GQA 1/2/4/8, ragged tile tails, a single token, sharp attention."""
    wl = W.workload("llama8b_b8_32k", batch=2, n_q_heads=8 * g)
    case = Case(wl, n_ctx=n_ctx)
    q = W.bf16_bits_from_f32((W.f32_from_bf16_bits(case.q(0)) * qscale).astype(np.float32))
    out = kvq.bf16_decode_attn(to_dev(q, "bf16"), to_dev(case.K, "bf16"), to_dev(case.V, "bf16")).cpu().numpy()
    g = wl.group_size
    for b in range(2):
        for h in range(wl.n_kv_heads):
            ref = orc.attention(W.as_float(q[b, h * g:(h + 1) * g], "bf16"),
                                W.as_float(case.K[b, h], "bf16"), W.as_float(case.V[b, h], "bf16"))
            emax, emean = rel_errors(out[b, h * g:(h + 1) * g], ref)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (b, h, emax)
    empty = kvq.bf16_decode_attn(to_dev(q, "bf16"), to_dev(case.K[:, :, :0], "bf16"),
                                 to_dev(case.V[:, :, :0], "bf16"))
    assert not empty.any()


def test_decode_parity_sharp_attention():
    """Queries scaled x8: most softmax weights are tiny, a few dominate."""
    case = Case(W.workload("llama8b_b8_32k", batch=2), n_ctx=1500)
    cache = case.gpu_cache()
    q = (W.f32_from_bf16_bits(case.q(3)) * 8.0).astype(np.float32)
    qb = W.bf16_bits_from_f32(q)
    sel = kvq.select_channels(cache, to_dev(qb, "bf16"), dev64(case.Ai), 0.4)
    out = kvq.decode_attn(cache, sel).cpu().numpy()
    for b in range(2):
        for h in range(8):
            ref, _, _ = case.oracle_decode(qb, b, h, 0.4)
            emax, emean = rel_errors(out[b, h * 4:(h + 1) * 4], ref)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (b, h, emax)


@pytest.mark.parametrize("name,units,sparsities", [
    ("longctx_b1_128k", [(0, 0), (0, 5)], (0.4,)),
    ("sweep_b32_16k", [(0, 0), (31, 7)], (0.0, 0.4, 0.6)),
    ("llama8b_b8_32k", [(7, 3)], (0.4,)),
])
def test_full_size_sampled(name, units, sparsities):
    """Full workload sizes in the benchmark's launch configuration: every
    sequence and head runs on the GPU; sampled (sequence, KV head) units are
    checked against the oracle (pages bit-exact, channels bit-exact, output
    within tolerance)."""
    case = Case(W.workload(name))
    cache = case.gpu_cache()
    _check_pages(case, cache, units=units)
    for s in sparsities:
        _decode_and_compare(case, cache, s, steps=(0,), units=units)


@pytest.mark.parametrize("fused", [True, False])
def test_decode_step_graph_replay_matches_eager(fused):
    """The captured step (one fused launch, or append -> select -> decode)
    gives the same bytes and outputs as the same calls launched one by one."""
    wl = W.workload("llama8b_b8_32k", batch=2)
    case = Case(wl, n_ctx=400)
    A, Ai = dev64(case.A), dev64(case.Ai)
    steps = [kvq.DecodeStep(case.gpu_cache(), A, Ai, 0.4, wl.n_q_heads, fused=fused) for _ in range(2)]
    outs = [[], []]
    for i in range(4):
        kn, vn = W.make_step_kv(wl, i)
        q = case.q(i)
        for m, st in enumerate(steps):
            st.q.copy_(to_dev(q, "bf16"))
            st.k_new.copy_(to_dev(kn, "bf16"))
            st.v_new.copy_(to_dev(vn, "bf16"))
            outs[m].append(st.run().clone())
            if m == 1 and i == 0:
                torch.cuda.synchronize()
                st.capture()
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    assert torch.equal(steps[0].cache.pages, steps[1].cache.pages)
    assert steps[1].cache.seq_len.tolist() == [404, 404]


def test_small_append_capacity_and_lengths():
    """Decode-sized appends (one token) advance every sequence's length once
    per call, and stop at capacity with the flag set and the pages intact."""
    wl = W.workload("llama8b_b8_32k", batch=3)
    case = Case(wl, n_ctx=254, capacity=256)
    cache = case.gpu_cache()
    A = dev64(case.A)
    for i in range(2):
        kn, vn = W.make_step_kv(wl, i)
        kvq.append(cache, to_dev(kn, "bf16"), to_dev(vn, "bf16"), A)
    assert cache.seq_len.tolist() == [256, 256, 256] and kvq.read_status(cache) == 0
    before = cache.pages.clone()
    kn, vn = W.make_step_kv(wl, 5)
    kvq.append(cache, to_dev(kn, "bf16"), to_dev(vn, "bf16"), A)
    assert kvq.read_status(cache) & kvq.KVQ_DEV_CAPACITY
    assert cache.seq_len.tolist() == [256, 256, 256]
    assert torch.equal(before, cache.pages)
    # the counters the calls use are back at zero
    assert not cache.status[1:].any()


@pytest.mark.parametrize("name,n_ctx,bits,g", [("llama8b_b8_32k", 300, 2, 4), ("longctx_b1_128k", 5000, 2, 4),
                                              ("llama8b_b8_32k", 300, 4, 4), ("llama8b_b8_32k", 300, 2, 8)])
def test_decode_writes_stay_in_bounds(name, n_ctx, bits, g):
    """Sentinel words after the output and after the workspace survive."""
    wl = W.workload(name, bits=bits, n_q_heads=8 * g)
    case = Case(wl, n_ctx=n_ctx)
    cache = case.gpu_cache()
    q = case.q(0)
    sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), 0.4)
    n_out = wl.batch * wl.n_q_heads * 128
    guard = 4096
    out_buf = torch.full((n_out + guard,), float("nan"), dtype=torch.float32, device="cuda")
    wsb = kvq.decode_workspace_bytes(cache, wl.n_q_heads, sel.k)
    ws_buf = torch.full((wsb + 4 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    out = out_buf[:n_out].view(wl.batch, wl.n_q_heads, 128)
    for _ in range(2):
        kvq.decode_attn(cache, sel, out=out, ws=ws_buf)
    torch.cuda.synchronize()
    assert torch.isnan(out_buf[n_out:]).all()
    assert (ws_buf[wsb:] == 0xA5).all()
    assert torch.isfinite(out).all()
    ref, _, _ = case.oracle_decode(q, wl.batch - 1, wl.n_kv_heads - 1, 0.4)
    emax, _ = rel_errors(out[-1, -g:].cpu().numpy(), ref)
    assert emax <= TOL_MAX


@pytest.mark.parametrize("bits,g", [(2, 4), (4, 4), (2, 2)])
def test_decode_rejects_malformed_channel_list(bits, g):
    """A channel list that is not 0 followed by ascending channels in 1..127
    raises KVQ_DEV_INDEX; a valid list afterwards still decodes correctly and
    raises no flag."""
    wl = W.workload("llama8b_b8_32k", batch=1, bits=bits, n_q_heads=8 * g)
    case = Case(wl, n_ctx=260)
    cache = case.gpu_cache()
    q = case.q(0)
    sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), 0.5)
    assert kvq.read_status(cache) == 0
    good = sel.idx.clone()
    for bad in ("duplicate", "descending", "out_of_range", "first_not_zero"):
        idx = good.clone()
        if bad == "duplicate":
            idx[0, 3, 5] = idx[0, 3, 4]
        elif bad == "descending":
            idx[0, 0, 1:] = idx[0, 0, 1:].flip(0)
        elif bad == "out_of_range":
            idx[0, 7, -1] = 128
        else:
            idx[0, 2, 0] = 1
        sel.idx.copy_(idx)
        out = kvq.decode_attn(cache, sel)
        torch.cuda.synchronize()
        assert kvq.read_status(cache) & kvq.KVQ_DEV_INDEX, bad
        assert not cache.status[1:].any()
        cache.status.zero_()
    sel.idx.copy_(good)
    out = kvq.decode_attn(cache, sel).cpu().numpy()
    assert kvq.read_status(cache) == 0
    for h in range(wl.n_kv_heads):
        ref, _, _ = case.oracle_decode(q, 0, h, 0.5)
        emax, emean = rel_errors(out[0, h * g:(h + 1) * g], ref)
        assert emax <= TOL_MAX and emean <= TOL_MEAN

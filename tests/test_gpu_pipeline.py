"""The append + decode pipeline workload at full size: a 131072-token prefill
of heavy-tailed (Student-t(4)) keys and values, then 256 decode steps that
each append one token and decode (INT2 through the fused step; INT4 through
the three calls).  After the last step the whole page buffer (8 KV heads x
1026 pages) equals the oracle's byte for byte, the channel lists of the last
step equal the oracle's, and sampled outputs of the last step are within the
decode tolerance."""
import numpy as np
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W
from oracle import oracle as orc

from helpers import Case, dev64, rel_errors, to_dev

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-3
TOL_MEAN = 1e-3


@pytest.mark.parametrize("bits", [2, 4])
def test_pipeline_prefill_and_256_steps_full_buffer(bits):
    wl = W.workload("pipeline_128k_t4", bits=bits)
    assert wl.n_ctx == 131072 and wl.n_steps == 256
    case = Case(wl)
    cache = case.gpu_cache()                                   # the prefill
    A, Ai = dev64(case.A), dev64(case.Ai)
    step_k, step_v = [], []
    for i in range(wl.n_steps):
        kn, vn = W.make_step_kv(wl, i)
        step_k.append(kn)
        step_v.append(vn)
        q = case.q(i)
        out, sel = kvq.decode_step(cache, to_dev(q, wl.dtype), to_dev(kn, wl.dtype), to_dev(vn, wl.dtype), A, Ai,
                                   wl.sparsity)
    torch.cuda.synchronize()
    n = wl.n_ctx + wl.n_steps
    assert cache.seq_len.tolist() == [n]
    assert kvq.read_status(cache) == 0
    pages = cache.all_pages().cpu().numpy()
    out = out.cpu().numpy()
    q = case.q(wl.n_steps - 1)
    g = wl.group_size
    k = orc.num_selected(wl.sparsity)
    for h in range(wl.n_kv_heads):
        Kf = np.concatenate([W.as_float(case.K[0, h], wl.dtype)] + [W.as_float(x[0, h], wl.dtype) for x in step_k])
        Vf = np.concatenate([W.as_float(case.V[0, h], wl.dtype)] + [W.as_float(x[0, h], wl.dtype) for x in step_v])
        unit = orc.new_unit(case.capacity, bits)
        orc.append_unit(unit, bits, 0, orc.transform(Kf, case.A[h]), Vf)
        assert np.array_equal(pages[0, h], unit), f"KV head {h}: page bytes differ"
        qp = orc.transform(W.as_float(q[0, h * g:(h + 1) * g], wl.dtype), case.Ai[h])
        idx, _ = orc.select(qp, k)
        assert np.array_equal(sel.idx[0, h].cpu().numpy(), idx), h
        if h in (0, 5):
            want = orc.decode_dense(*orc.dequant_unit(unit, bits, n), qp, idx)
            emax, emean = rel_errors(out[0, h * g:(h + 1) * g], want)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (h, emax, emean)

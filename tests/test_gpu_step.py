"""lrkv_decode_step (append one token, then attend, with the query fold done
by the append kernel) against the two-call path and the oracle.

The append work is the same kernel code in both paths, so the caches must
match bit for bit; the folded queries are summed in another order, so the
outputs agree with the two-call path to within the isolated-attention bar
and with the oracle to within the end-to-end bar.
"""
import numpy as np
import pytest
import torch

from rank_kv_cache_lrkv_b200 import workloads as wk
from tests import lrkv_testutil as tu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


CASES = [
    ("llama_anchors", wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=2, T=700, n_decode=70, window=32)),
    ("qwen_no_anchors", wk.QWEN3_LAYER_8K.with_(B=3, T=300, n_decode=40)),
    ("tiny_fp32", wk.TINY_SINGLE_HEAD.with_(T=200, n_decode=20, append_before_attend=True)),
]


@pytest.mark.parametrize("name,wl", CASES, ids=[c[0] for c in CASES])
def test_decode_step_matches_two_calls_and_oracle(lrkv, name, wl):
    inp = tu.Inputs(wl)
    dt = tu.torch_dtype(wl)
    K, V = inp.K.cuda(), inp.V.cuda()
    Pk, Pv = inp.Pk.cuda(), inp.Pv.cuda()
    caches, outs = [], []
    for fused in (False, True):
        cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, wl.T + wl.n_decode, wl.n_sink,
                                 wl.window, dtype=dt)
        lrkv.compress(cache, K[:, :, :wl.T], V[:, :, :wl.T], Pk, Pv)
        ws = lrkv.decode_workspace(cache, wl.H_q)
        o_s = []
        for s in range(wl.n_decode):
            t = wl.T + s
            q = inp.q[s].cuda().contiguous()
            o = torch.empty_like(q)
            if fused:
                lrkv.decode_step(cache, K[:, :, t:t + 1], V[:, :, t:t + 1], q, Pk, Pv, wl.scale,
                                 o, ws)
            else:
                lrkv.compress(cache, K[:, :, t:t + 1], V[:, :, t:t + 1], Pk, Pv)
                lrkv.decode_attn(cache, q, Pk, Pv, wl.scale, o, ws)
            o_s.append(o.double().cpu().numpy())
        torch.cuda.synchronize()
        assert lrkv.workspace_error(ws) == 0
        caches.append(cache)
        outs.append(o_s)
    a, b = caches
    assert torch.equal(a.seq_len, b.seq_len)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.anchors, b.anchors)
    _, refs = tu.run_oracle(wl, inp)
    for s in range(wl.n_decode):
        assert tu.row_rel_err(outs[1][s], outs[0][s]) < tu.TOL_ISO[wl.dtype], s
        assert tu.row_rel_err(outs[1][s], refs[s]) < tu.TOL[wl.dtype], s


def test_decode_step_refuses_what_it_does_not_serve(lrkv):
    q8 = lrkv.LatentCache(1, 2, 32, 32, 200, int8_codes=True)
    va = lrkv.LatentCache(1, 2, 32, 32, 200, amortised_values=True)
    k = torch.zeros(1, 2, 1, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    P = torch.zeros(2, 128, 32, device="cuda")
    ws = torch.zeros(1 << 22, dtype=torch.uint8, device="cuda")
    for cache in (q8, va):
        with pytest.raises(lrkv.LrkvError) as e:
            lrkv.decode_step(cache, k, k, q, P, P, 0.1, torch.empty_like(q), ws)
        assert e.value.status == -2
    plain = lrkv.LatentCache(1, 2, 32, 32, 200)
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(lrkv.LrkvError) as e:
        lrkv.decode_step(plain, k, k, q, P, P, 0.1, torch.empty_like(q), small)
    assert e.value.status == -4
    assert int(plain.seq_len.sum()) == 0  # nothing was launched

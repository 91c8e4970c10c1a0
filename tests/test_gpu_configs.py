"""The configured workloads at full size on the GPU against the oracle.

Where the oracle would take too long over every (sequence, KV head) unit,
it simulates sampled units on their own (units are independent: each has its
own codes, anchors and softmax), and their outputs and codes are compared
element by element.  Tolerances are those of tests/lrkv_testutil.py.
"""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_lrkv_b200 import workloads as wk
from tests import lrkv_testutil as tu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _sampled(lrkv, wl, units, page_perm=None):
    inp = tu.Inputs(wl)
    cache, outs = tu.run_gpu(wl, inp, lrkv=lrkv, page_perm=page_perm)
    res = tu.run_oracle(wl, inp, units=units)
    G = wl.G
    worst = 0.0
    for (b, h), (oc, refs) in res.items():
        for o, ref in zip(outs, refs):
            worst = max(worst, tu.row_rel_err(o[b, h * G:(h + 1) * G], ref))
        n = oc.codes_k[0][0].shape[0]
        for kind, refc in (("k", oc.codes_k[0][0]), ("v", oc.codes_v[0][0])):
            got = tu.gather_codes(cache, b, h, n, kind)
            den = np.maximum(np.max(np.abs(refc), axis=1), 1e-30)
            assert np.max(np.max(np.abs(got - refc), axis=1) / den) < tu.TOL_CODE[wl.dtype]
    assert worst < tu.TOL[wl.dtype], worst
    return worst


def test_qwen3_layer_8k_full():
    """Qwen3-1.7B-shaped layer, B=4, T=8192, r 64/32, RoPE 1e6, compress the
    whole prompt then 64 decode steps; every output checked."""
    from rank_kv_cache_lrkv_b200 import lrkv
    tu.run_and_compare(lrkv, wk.QWEN3_LAYER_8K)


def test_llama31_layer_32k_anchors_sampled(lrkv):
    """Llama-3.1-8B-shaped layer at 32K with sink + 128-token window; the
    pages scattered by a permuted block table; 8 decode steps."""
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(n_decode=8)
    npages = wl.B * -(-(wl.T + 8 - 129) // 64)
    perm = torch.from_numpy(wk.page_permutation(wl, npages))
    _sampled(lrkv, wl, [(0, 0), (1, 3), (3, 7)], page_perm=perm)


@pytest.mark.parametrize("r_k,r_v,B", [(96, 64, 8), (32, 32, 32), (64, 32, 1)])
def test_qwen3_rank_batch_sweep_points(lrkv, r_k, r_v, B):
    wl = wk.qwen3_sweep_point(r_k, r_v, B).with_(n_decode=2)
    _sampled(lrkv, wl, [(0, 0), (B - 1, 7)])


def test_qwen3_28_layer_stack_with_oja():
    """28 Qwen3-shaped layers, B=2, T=32768, r 48/48, per-layer random
    orthonormal initial basis adapted per sequence by Oja over the prompt
    (eta 1e-3, QR every 256 tokens), then 128 decode steps (the decode-time
    update every 512 generated tokens does not fire).  At every layer one
    (sequence, KV head) unit is replayed by the oracle: its Oja bases (plain-C
    float64 loop) and its decode outputs."""
    from rank_kv_cache_lrkv_b200 import lrkv
    wl = wk.QWEN3_STACK_OJA
    B, H, T, r, G = wl.B, wl.H_kv, wl.T, wl.r_k, wl.G
    bs = H * 128 * r
    worst_out, worst_P = 0.0, 0.0
    for layer in range(wl.layers):
        d = wk.layer_inputs(wl, layer)
        qs = wk.layer_queries(wl, layer)
        K, V = d["K"].cuda(), d["V"].cuda()
        total = K.shape[2]
        Pk = d["P_k"][None].repeat(B, 1, 1, 1).contiguous().cuda()
        Pv = d["P_v"][None].repeat(B, 1, 1, 1).contiguous().cuda()
        lrkv.oja_update(Pk.view(B * H, 128, r), K.view(B * H, total, 128)[:, :T],
                        wl.oja_eta, wl.oja_qr_every, 0)
        lrkv.oja_update(Pv.view(B * H, 128, r), V.view(B * H, total, 128)[:, :T],
                        wl.oja_eta, wl.oja_qr_every, 0)
        cache = lrkv.LatentCache(B, H, r, r, T + wl.n_decode)
        lrkv.compress(cache, K[:, :, :T], V[:, :, :T], Pk, Pv, basis_batch_stride=bs)
        ws = lrkv.decode_workspace(cache, wl.H_q)
        outs = []
        for s in range(wl.n_decode):
            lrkv.compress(cache, K[:, :, T + s:T + s + 1], V[:, :, T + s:T + s + 1], Pk, Pv,
                          basis_batch_stride=bs)
            q = qs[s].cuda().contiguous()
            o = torch.empty_like(q)
            lrkv.decode_attn(cache, q, Pk, Pv, wl.scale, o, ws, basis_batch_stride=bs)
            outs.append(o)
        torch.cuda.synchronize()
        assert lrkv.workspace_error(ws) == 0
        # oracle replay of one unit
        b, h = layer % B, (3 * layer) % H
        Kn = d["K"][b, h].float().numpy()
        Vn = d["V"][b, h].float().numpy()
        Pk_ref = orc.oja_update_streams(d["P_k"][h][None].double().numpy(), Kn[None, :T],
                                        wl.oja_eta, wl.oja_qr_every, 0)[0]
        Pv_ref = orc.oja_update_streams(d["P_v"][h][None].double().numpy(), Vn[None, :T],
                                        wl.oja_eta, wl.oja_qr_every, 0)[0]
        for got, ref in ((Pk[b, h], Pk_ref), (Pv[b, h], Pv_ref)):
            worst_P = max(worst_P, float(np.max(np.abs(got.cpu().double().numpy() - ref))
                                         / np.max(np.abs(ref))))
        oc = orc.LatentCacheOracle(1, 1, r, r)
        Pk4, Pv4 = Pk_ref[None, None], Pv_ref[None, None]
        oc.append(Kn[None, None, :T].astype(np.float64), Vn[None, None, :T].astype(np.float64),
                  Pk4, Pv4)
        for s in range(wl.n_decode):
            oc.append(Kn[None, None, T + s:T + s + 1].astype(np.float64),
                      Vn[None, None, T + s:T + s + 1].astype(np.float64), Pk4, Pv4)
            q = qs[s][b:b + 1, h * G:(h + 1) * G].double().numpy()
            ref = oc.attend(q, Pk4, Pv4, wl.scale)[0]
            worst_out = max(worst_out, tu.row_rel_err(
                outs[s][b, h * G:(h + 1) * G].double().cpu().numpy(), ref))
        del K, V, cache, outs
    assert worst_P <= 1e-3, worst_P
    assert worst_out < tu.TOL["bf16"], worst_out

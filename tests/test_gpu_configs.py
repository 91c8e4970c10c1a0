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
from tests.test_tolerances import TOL_P_STACK

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _sampled(lrkv, wl, units, page_perm=None, inp=None, inp_gpu=None):
    inp = tu.Inputs(wl) if inp is None else inp
    cache, outs = tu.run_gpu(wl, inp if inp_gpu is None else inp_gpu, lrkv=lrkv,
                             page_perm=page_perm)
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


class _Slice:
    """Inputs of a sweep point cut from the largest point's draws."""

    def __init__(self, K, V, Pk, Pv, q):
        self.K, self.V, self.Pk, self.Pv, self.q = K, V, Pk, Pv, q


@pytest.fixture(scope="module")
def sweep_inputs():
    """The sweep's seeded draws at the largest batch and ranks.  A stream
    depends only on its (sequence, KV head) seed and a basis of rank r is the
    first r columns of the rank-96 (keys) or rank-64 (values) SVD basis, so
    every point's inputs are slices of these."""
    rk_max = max(r for r, _ in wk.SWEEP_RANKS)
    rv_max = max(r for _, r in wk.SWEEP_RANKS)
    wl = wk.qwen3_sweep_point(rk_max, rv_max, max(wk.SWEEP_BATCHES)).with_(n_decode=2)
    cpu = tu.Inputs(wl)
    gpu = _Slice(cpu.K.cuda(), cpu.V.cuda(), cpu.Pk, cpu.Pv, cpu.q)
    return cpu, gpu


@pytest.mark.parametrize("r_k,r_v", wk.SWEEP_RANKS)
@pytest.mark.parametrize("B", wk.SWEEP_BATCHES)
def test_qwen3_rank_batch_sweep_points(lrkv, sweep_inputs, r_k, r_v, B):
    """Every point of the rank x batch sweep at T=16384: two decode steps;
    the first and last (sequence, KV head) units and one in the middle are
    replayed by the oracle."""
    wl = wk.qwen3_sweep_point(r_k, r_v, B).with_(n_decode=2)
    cpu, gpu = sweep_inputs
    Pk = cpu.Pk[:, :, :r_k].contiguous()
    Pv = cpu.Pv[:, :, :r_v].contiguous()
    assert torch.equal(Pk[0], torch.from_numpy(wk.basis(wl, "k", 0, 0)))
    inp = _Slice(cpu.K[:B], cpu.V[:B], Pk, Pv, cpu.q[:, :B])
    inp_gpu = _Slice(gpu.K[:B], gpu.V[:B], Pk, Pv, cpu.q[:, :B])
    units = sorted({(0, 0), (B // 2, 3), (B - 1, 7)})
    _sampled(lrkv, wl, units, inp=inp, inp_gpu=inp_gpu)


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
    # fp32 against float64 over 32,768 tokens and 128 QRs: a float32
    # restatement of the loop drifts a few 1e-6 (tests/test_tolerances.py);
    # 1e-4 leaves more than an order of magnitude for the GPU's summation order
    print(f"28-layer stack: worst basis deviation {worst_P:.3e}, worst output {worst_out:.3e}")
    assert worst_P <= TOL_P_STACK, worst_P
    assert worst_out < tu.TOL["bf16"], worst_out

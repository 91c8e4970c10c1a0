"""Per-token int8 codes (LRKV_BF16_Q8) against the oracle.

The oracle stores each code row as its dequantised int8 form (scale =
max |c| / 127, codes rounded half to even, decided in fp32) and attends over
those rows; the GPU compresses into int8 pages and dequantises inside the
decode.  Checks: end to end at the bf16 bar, stored codes within one
quantum of the oracle's (a quantum is 1/127 of the row's largest code, so
rows agree to the code tolerance), attention over the GPU's own int8 codes
at the attention-alone bar, and bit-exact codes and scales where both sides
see the same fp32 codes (a basis of unit vectors makes the codes the input
coordinates themselves).
"""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_lrkv_b200 import workloads as wk
from tests import lrkv_testutil as tu

pytestmark = pytest.mark.gpu

# Attention alone over the GPU's own int8 codes: the bf16 bar (one rounding
# of o, 2^-9, plus fp32 sums) and one more bf16 rounding of every dequantised
# code inside the decode (2^-9 of each code, carried to o through the
# softmax weights and P_v), so twice the bf16 attention-alone bar.
TOL_ISO_Q8 = 2 * tu.TOL_ISO["bf16"]


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _deq(cache, b, h, n, kind):
    q, s = tu.gather_q8(cache, b, h, n, kind)
    return orc.dequantize_codes(q, s)


def _check_codes(wl, cache, oc):
    for b in range(wl.B):
        for h in range(wl.H_kv):
            n = oc.codes_k[b][h].shape[0]
            for kind, ref in (("k", oc.codes_k[b][h]), ("v", oc.codes_v[b][h])):
                if n == 0:
                    continue
                got = _deq(cache, b, h, n, kind)
                den = np.maximum(np.max(np.abs(ref), axis=1), 1e-30)
                err = np.max(np.max(np.abs(got - ref), axis=1) / den)
                assert err < tu.TOL_CODE["bf16"], (b, h, kind, err)


def _isolated(wl, inp, cache, L, q, o_gpu):
    _, lat, _ = orc.partition(L, wl.n_sink, wl.window)
    slots = tu.window_slots(L, wl.n_sink, wl.window)
    Ck = [[_deq(cache, b, h, len(lat), "k") for h in range(wl.H_kv)] for b in range(wl.B)]
    Cv = [[_deq(cache, b, h, len(lat), "v") for h in range(wl.H_kv)] for b in range(wl.B)]
    z = np.zeros((0, 128))
    Ka = [[tu.gather_anchor_slots(cache, b, h, slots, "k") if slots else z
           for h in range(wl.H_kv)] for b in range(wl.B)]
    Va = [[tu.gather_anchor_slots(cache, b, h, slots, "v") if slots else z
           for h in range(wl.H_kv)] for b in range(wl.B)]
    ref = orc.decode_from_parts(q, inp.Pk.double().numpy()[None], inp.Pv.double().numpy()[None],
                                Ck, Cv, Ka, Va, wl.G, wl.scale)
    return tu.row_rel_err(o_gpu, ref)


@pytest.mark.parametrize("kw", [
    dict(B=2, T=700, n_decode=5),                          # sink + window, evictions
    dict(B=3, T=1000, n_decode=3, n_sink=0, window=0, r_k=32, r_v=64),
    dict(B=2, T=400, n_decode=3, H_q=64, r_k=128, r_v=128),
])
def test_int8_codes_end_to_end(lrkv, kw):
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(**kw)
    inp = tu.Inputs(wl)
    cache, outs = tu.run_gpu(wl, inp, lrkv=lrkv, int8_codes=True)
    oc, refs = tu.run_oracle(wl, inp, quant_bits=8)
    errs = [tu.row_rel_err(o, r) for o, r in zip(outs, refs)]
    assert max(errs) < tu.TOL["bf16"], errs
    _check_codes(wl, cache, oc)
    L = wl.T + wl.n_decode
    e = _isolated(wl, inp, cache, L, inp.q[-1].double().numpy(), outs[-1])
    assert e < TOL_ISO_Q8, e


def test_int8_codes_bit_exact_under_unit_vector_basis(lrkv):
    """P = the first r unit vectors: every code is an input coordinate (a bf16
    value, exact in fp32 on both sides), so the quantisation decisions must
    agree bit for bit, through the prefill kernel and through evictions."""
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=2, T=500, n_decode=3, window=32)
    d = wk.layer_inputs(wl)
    r_k, r_v = wl.r_k, wl.r_v
    Pk = torch.zeros(wl.H_kv, 128, r_k)
    Pv = torch.zeros(wl.H_kv, 128, r_v)
    Pk[:, torch.arange(r_k), torch.arange(r_k)] = 1.0
    Pv[:, torch.arange(r_v), torch.arange(r_v)] = 1.0
    cache = lrkv.LatentCache(wl.B, wl.H_kv, r_k, r_v, wl.T + wl.n_decode, wl.n_sink, wl.window,
                             int8_codes=True)
    K, V = d["K"].cuda(), d["V"].cuda()
    lrkv.compress(cache, K[:, :, :wl.T], V[:, :, :wl.T], Pk.cuda(), Pv.cuda())
    for s in range(wl.n_decode):
        t = wl.T + s
        lrkv.compress(cache, K[:, :, t:t + 1], V[:, :, t:t + 1], Pk.cuda(), Pv.cuda())
    torch.cuda.synchronize()
    L = wl.T + wl.n_decode
    _, lat, _ = orc.partition(L, wl.n_sink, wl.window)
    for b in range(wl.B):
        for h in range(wl.H_kv):
            for kind, X, r in (("k", d["K"], r_k), ("v", d["V"], r_v)):
                rows = X[b, h, lat, :r].double().numpy()
                q_ref, s_ref = orc.quantize_codes(rows, 8)
                q, s = tu.gather_q8(cache, b, h, len(lat), kind)
                assert np.array_equal(q, q_ref), (b, h, kind)
                assert np.array_equal(s, s_ref), (b, h, kind)


def test_int8_cache_refuses_rebase_and_ranks_off_16(lrkv):
    cache = lrkv.LatentCache(1, 2, 32, 32, 200, int8_codes=True)
    P = torch.zeros(2, 128, 32, device="cuda")
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(lrkv.LrkvError) as e:
        lrkv.rebase(cache, P, P, None, None, ws)
    assert e.value.status == -2
    bad = lrkv.LatentCache(1, 2, 24, 32, 200, int8_codes=True)
    k = torch.zeros(1, 2, 40, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lrkv.LrkvError) as e:
        lrkv.compress(bad, k, k, torch.zeros(2, 128, 24, device="cuda"), P)
    assert e.value.status == -2


def test_int8_codes_llama_32k_sampled(lrkv):
    """The Llama-3.1-8B-shaped layer at 32K with int8 codes: four decode
    steps, three (sequence, KV head) units replayed by the oracle."""
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(n_decode=4)
    inp = tu.Inputs(wl)
    cache, outs = tu.run_gpu(wl, inp, lrkv=lrkv, int8_codes=True)
    units = [(0, 0), (1, 5), (3, 7)]
    res = tu.run_oracle(wl, inp, units=units, quant_bits=8)
    G = wl.G
    worst = 0.0
    for (b, h), (oc, refs) in res.items():
        for o, ref in zip(outs, refs):
            worst = max(worst, tu.row_rel_err(o[b, h * G:(h + 1) * G], ref))
        n = oc.codes_k[0][0].shape[0]
        for kind, refc in (("k", oc.codes_k[0][0]), ("v", oc.codes_v[0][0])):
            got = _deq(cache, b, h, n, kind)
            den = np.maximum(np.max(np.abs(refc), axis=1), 1e-30)
            assert np.max(np.max(np.abs(got - refc), axis=1) / den) < tu.TOL_CODE["bf16"]
    assert worst < tu.TOL["bf16"], worst

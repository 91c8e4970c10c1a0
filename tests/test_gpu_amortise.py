"""Value amortisation (LRKV_BF16_VA) against the oracle.

Schedule on both sides: the prompt is appended (key codes only on the GPU),
the per-(sequence, KV head) value predictors are fitted over the prompt's
latent tokens and each prompt page keeps the residuals of its 16 worst-
predicted tokens; every decode step appends a token (an evicted window
token's residual competes for its page's slots) and attends over the
amortised value codes A^T c_k + kept residual.  Checks: the GPU's
predictions close to the oracle's (both fit the same least-squares problem,
the GPU from bf16 key codes in fp32/fp64); the kept slots are each page's
top 16 under the oracle's residual norms, up to near-ties that the GPU's
fp32 norms of bf16-code residuals may order the other way; every output at
the bf16 bar against the oracle's arithmetic over the slots the GPU kept.
Comparing against the oracle's own top-16 instead would test the tie
breaks: with these synthetic values a single swapped near-tie can move an
output row by 10 % or more, since a token's value code is either its
prediction or its exact code.
"""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_lrkv_b200 import workloads as wk
from tests import lrkv_testutil as tu

pytestmark = pytest.mark.gpu

KEEP = 16
NEAR_TIE = 2e-2  # relative gap in residual norm under which two tokens may swap


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _slot_rows(codes, bt, b, h, n, rk, rv):
    """Per page of unit (b, h): the token rows its residual slots hold (-1:
    unused), from a host copy of the code pool."""
    off = 64 * rk * 2 + KEEP * rv * 2
    out = []
    for p0 in range(0, n, 64):
        slab = codes[int(bt[b, p0 // 64]), h]
        out.append(slab[off:off + 4 * KEEP].view(np.int32).copy())
    return out


def _kept_mask(slots, n):
    """Latent tokens whose residual a slot holds, as a mask [n]."""
    kept = np.zeros(n, bool)
    for pi, idx in enumerate(slots):
        for r in idx:
            if 0 <= r and pi * 64 + r < n:
                kept[pi * 64 + r] = True
    return kept


def _run(lrkv, wl):
    inp = tu.Inputs(wl)
    K, V = inp.K.cuda(), inp.V.cuda()
    Pk, Pv = inp.Pk.cuda(), inp.Pv.cuda()
    cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, wl.T + wl.n_decode, wl.n_sink,
                             wl.window, amortised_values=True)
    lrkv.compress(cache, K[:, :, :wl.T], V[:, :, :wl.T], Pk, Pv)
    A = torch.zeros(wl.B, wl.H_kv, wl.r_k, wl.r_v, device="cuda")
    lrkv.amortise(cache, V[:, :, :wl.T], Pv, A)
    ws = lrkv.decode_workspace(cache, wl.H_q)
    bt = cache.block_table.cpu().numpy()
    outs, pools = [], []
    for s in range(wl.n_decode):
        t = wl.T + s
        lrkv.compress_amortised(cache, K[:, :, t:t + 1], V[:, :, t:t + 1], Pk, Pv, A)
        q = inp.q[s].cuda().contiguous()
        o = torch.empty_like(q)
        lrkv.decode_attn_amortised(cache, q, Pk, Pv, A, wl.scale, o, ws)
        outs.append(o.double().cpu().numpy())
        pools.append(cache.codes.cpu().numpy())  # the slots this step attended over
    torch.cuda.synchronize()
    assert lrkv.workspace_error(ws) == 0
    # the oracle
    Kn, Vn = inp.K.double().numpy(), inp.V.double().numpy()
    Pkn, Pvn = inp.Pk.double().numpy()[None], inp.Pv.double().numpy()[None]
    oc = orc.LatentCacheOracle(wl.B, wl.H_kv, wl.r_k, wl.r_v, wl.n_sink, wl.window,
                               value_keep=KEEP)
    oc.append(Kn[:, :, :wl.T], Vn[:, :, :wl.T], Pkn, Pvn)
    oc.amortise()
    checks = []
    for s in range(wl.n_decode):
        t = wl.T + s
        oc.append(Kn[:, :, t:t + 1], Vn[:, :, t:t + 1], Pkn, Pvn)
        q = inp.q[s].double().numpy()
        # the oracle's arithmetic over the residual slots the GPU kept: the
        # top-16 choice is a floating-point decision whose near-ties (checked
        # below) may fall either way
        Ck, Cv, Ka, Va, sel = [], [], [], [], []
        for b in range(wl.B):
            ck_, cv_, ka_, va_, sel_ = [], [], [], [], []
            for h in range(wl.H_kv):
                ck, cv = oc.codes_k[b][h], oc.codes_v[b][h]
                kept = _kept_mask(_slot_rows(pools[s], bt, b, h, ck.shape[0], wl.r_k, wl.r_v),
                                  ck.shape[0])
                pred = ck @ oc.A[b][h]
                ck_.append(ck)
                cv_.append(pred + np.where(kept[:, None], cv - pred, 0.0))
                ka, va = oc.anchors(b, h)
                ka_.append(ka)
                va_.append(va)
                sel_.append(kept)
            Ck.append(ck_); Cv.append(cv_); Ka.append(ka_); Va.append(va_); sel.append(sel_)
        ref = orc.decode_from_parts(q, Pkn, Pvn, Ck, Cv, Ka, Va, wl.G, wl.scale)
        checks.append((ref, sel))
    return A.double().cpu().numpy(), outs, oc, checks


def _check_selection(oc, b, h, kept_gpu):
    """The GPU's kept residuals are each page's top 16 under the oracle's
    residual norms, up to near-ties at the page's cut."""
    Ck, Cv = oc.codes_k[b][h], oc.codes_v[b][h]
    nrm = np.linalg.norm(Cv - Ck @ oc.A[b][h], axis=1)
    _, want = orc.amortised_value_codes(Ck, Cv, oc.A[b][h], KEEP)
    for p0 in range(0, Ck.shape[0], 64):
        rows = np.arange(p0, min(p0 + 64, Ck.shape[0]))
        assert kept_gpu[rows].sum() == want[rows].sum(), (b, h, p0)
        cut = nrm[rows][want[rows]].min()
        for r in rows[kept_gpu[rows] != want[rows]]:
            assert abs(nrm[r] - cut) <= NEAR_TIE * cut, (b, h, p0, r, nrm[r], cut)


@pytest.mark.parametrize("kw", [
    dict(B=2, T=700, n_decode=5, window=32),
    dict(B=3, T=900, n_decode=70, n_sink=0, window=0, r_k=48, r_v=48),  # fresh pages at decode
])
def test_amortised_values_match_oracle(lrkv, kw):
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(**kw)
    A, outs, oc, checks = _run(lrkv, wl)
    for b in range(wl.B):
        for h in range(wl.H_kv):
            Ck, Cv = oc.codes_k[b][h], oc.codes_v[b][h]
            pred_gpu, pred_ref = Ck @ A[b, h], Ck @ oc.A[b][h]
            assert np.max(np.abs(pred_gpu - pred_ref)) < 1e-2 * np.max(np.abs(Cv)), (b, h)
            _check_selection(oc, b, h, checks[-1][1][b][h])
    errs = [tu.row_rel_err(o, ref) for o, (ref, _) in zip(outs, checks)]
    assert max(errs) < tu.TOL["bf16"], (max(errs), int(np.argmax(errs)))


def test_amortised_cache_refuses_the_other_entry_points(lrkv):
    cache = lrkv.LatentCache(1, 2, 32, 32, 200, amortised_values=True)
    plain = lrkv.LatentCache(1, 2, 32, 32, 200)
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    P = torch.zeros(2, 128, 32, device="cuda")
    A = torch.zeros(1, 2, 32, 32, device="cuda")
    ws = torch.zeros(1 << 22, dtype=torch.uint8, device="cuda")
    for call in (lambda: lrkv.decode_attn(cache, q, P, P, 0.1, o, ws),
                 lambda: lrkv.decode_attn_amortised(plain, q, P, P, A, 0.1, o, ws),
                 lambda: lrkv.rebase(cache, P, P, None, None, ws)):
        with pytest.raises(lrkv.LrkvError) as e:
            call()
        assert e.value.status == -2

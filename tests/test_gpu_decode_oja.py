"""Decode-time Oja at a cadence that fires, against the oracle.

The OjaKV article adapts the basis comprehensively during the prompt and
lightly, periodically, during decoding.  Schedule (both sides):
  1. every (sequence, KV head) basis starts from the workload's random
     orthonormal basis and is adapted by Oja over the prompt tokens (keys for
     P_k, values for P_v), QR every 64 tokens seen;
  2. the prompt is compressed with the adapted bases;
  3. each decode step appends its token (the oldest window token is evicted
     into codes with the current bases) and attends with the current bases;
  4. after every 32nd generated token the bases are updated by Oja over those
     32 tokens, the token count carried on; then either the stored codes are
     re-based onto the new bases (lrkv_rebase) or left as stored, per the two
     readings of what happens to them.
Every step's output is compared with the float64 oracle at the bf16 bar, and
the final bases at the fp32 Oja bar.
"""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_lrkv_b200 import workloads as wk
from tests import lrkv_testutil as tu

pytestmark = pytest.mark.gpu

TOL_P = 1e-4   # fp32 Oja bases against the float64 loop (as in test_gpu_oja)


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _oracle(wl, d, qs, rebase):
    B, H, T, r, N = wl.B, wl.H_kv, wl.T, wl.r_k, wl.oja_decode_every
    K, V = d["K"].double().numpy(), d["V"].double().numpy()
    Pk = np.repeat(d["P_k"].double().numpy()[None], B, 0)      # [B, H, 128, r]
    Pv = np.repeat(d["P_v"].double().numpy()[None], B, 0)

    def oja(P, X, seen):
        out = orc.oja_update_streams(P.reshape(B * H, 128, r), X.reshape(B * H, -1, 128),
                                     wl.oja_eta, wl.oja_qr_every, seen)
        return out.reshape(B, H, 128, r)

    Pk, Pv = oja(Pk, K[:, :, :T], 0), oja(Pv, V[:, :, :T], 0)
    oc = orc.LatentCacheOracle(B, H, r, r, wl.n_sink, wl.window)
    oc.append(K[:, :, :T], V[:, :, :T], Pk, Pv)
    outs = []
    for s in range(wl.n_decode):
        t = T + s
        oc.append(K[:, :, t:t + 1], V[:, :, t:t + 1], Pk, Pv)
        outs.append(oc.attend(qs[s].double().numpy(), Pk, Pv, wl.scale))
        if (s + 1) % N == 0:
            lo = t + 1 - N
            Pk_new = oja(Pk, K[:, :, lo:t + 1], lo)
            Pv_new = oja(Pv, V[:, :, lo:t + 1], lo)
            if rebase:
                oc.rebase(Pk, Pk_new, Pv, Pv_new)
            Pk, Pv = Pk_new, Pv_new
    return outs, Pk, Pv, oc


def _gpu(lrkv, wl, d, qs, rebase):
    B, H, T, r, N = wl.B, wl.H_kv, wl.T, wl.r_k, wl.oja_decode_every
    K, V = d["K"].cuda(), d["V"].cuda()
    total = K.shape[2]
    Pk = d["P_k"][None].repeat(B, 1, 1, 1).contiguous().cuda()
    Pv = d["P_v"][None].repeat(B, 1, 1, 1).contiguous().cuda()
    bs = H * 128 * r
    Ks, Vs = K.view(B * H, total, 128), V.view(B * H, total, 128)
    lrkv.oja_update(Pk.view(B * H, 128, r), Ks[:, :T], wl.oja_eta, wl.oja_qr_every, 0)
    lrkv.oja_update(Pv.view(B * H, 128, r), Vs[:, :T], wl.oja_eta, wl.oja_qr_every, 0)
    cache = lrkv.LatentCache(B, H, r, r, T + wl.n_decode, wl.n_sink, wl.window)
    lrkv.compress(cache, K[:, :, :T], V[:, :, :T], Pk, Pv, basis_batch_stride=bs)
    ws = lrkv.decode_workspace(cache, wl.H_q)
    rws = lrkv.rebase_workspace(cache)
    outs = []
    for s in range(wl.n_decode):
        t = T + s
        lrkv.compress(cache, K[:, :, t:t + 1], V[:, :, t:t + 1], Pk, Pv, basis_batch_stride=bs)
        o = torch.empty_like(qs[s]).cuda()
        lrkv.decode_attn(cache, qs[s].cuda().contiguous(), Pk, Pv, wl.scale, o, ws,
                         basis_batch_stride=bs)
        outs.append(o)
        if (s + 1) % N == 0:
            lo = t + 1 - N
            Pk_old, Pv_old = Pk.clone(), Pv.clone()
            lrkv.oja_update(Pk.view(B * H, 128, r), Ks[:, lo:t + 1], wl.oja_eta,
                            wl.oja_qr_every, lo)
            lrkv.oja_update(Pv.view(B * H, 128, r), Vs[:, lo:t + 1], wl.oja_eta,
                            wl.oja_qr_every, lo)
            if rebase:
                lrkv.rebase(cache, Pk_old, Pk, Pv_old, Pv, rws, basis_batch_stride=bs)
    torch.cuda.synchronize()
    assert lrkv.workspace_error(ws) == 0 and lrkv.workspace_error(rws) == 0
    return [o.double().cpu().numpy() for o in outs], Pk.double().cpu().numpy(), \
        Pv.double().cpu().numpy(), cache


@pytest.mark.parametrize("rebase", [False, True])
def test_decode_time_oja_every_32_tokens_matches_oracle(lrkv, rebase):
    wl = wk.QWEN3_DECODE_OJA_SMALL
    assert wl.n_decode // wl.oja_decode_every >= 3
    d = wk.layer_inputs(wl)
    qs = wk.layer_queries(wl)
    ref, Pk_ref, Pv_ref, oc = _oracle(wl, d, qs, rebase)
    got, Pk, Pv, cache = _gpu(lrkv, wl, d, qs, rebase)
    errs = [tu.row_rel_err(o, r) for o, r in zip(got, ref)]
    assert max(errs) < tu.TOL["bf16"], (max(errs), int(np.argmax(errs)))
    for P, R in ((Pk, Pk_ref), (Pv, Pv_ref)):
        assert np.max(np.abs(P - R)) / np.max(np.abs(R)) < TOL_P
    # stored codes and anchors as the oracle holds them: re-based or not.  The
    # GPU stores bf16 and rounds again at every re-basing while the oracle
    # keeps float64: after k re-basings a stored code carries up to k + 1
    # roundings of 2^-9, and a re-basing also carries the earlier roundings of
    # a row through R (a near-rotation, rows of |R| summing to about 2).
    k = wl.n_decode // wl.oja_decode_every if rebase else 0
    tol = max(tu.TOL_CODE["bf16"], 2 * (k + 1) * 2.0 ** -9)
    tu.check_state(wl, d_inputs(d, qs), cache, oc, wl.T + wl.n_decode, tol_code=tol)
    # the schedule is discriminating: under the other reading the stored key
    # codes differ by several times the code tolerance
    _, _, _, oc_other = _oracle(wl, d, qs, not rebase)
    ck, ck_other = oc.codes_k[0][0], oc_other.codes_k[0][0]
    row = np.max(np.abs(ck - ck_other), axis=1) / np.max(np.abs(ck), axis=1)
    assert np.max(row) > 3 * tu.TOL_CODE["bf16"]


class d_inputs:
    """The attributes check_state reads, from the drawn inputs."""

    def __init__(self, d, qs):
        self.K, self.V, self.Pk, self.Pv, self.q = d["K"], d["V"], d["P_k"], d["P_v"], qs

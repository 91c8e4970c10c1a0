"""GPU parity of lrkv_rebase (stored codes re-expressed under new bases,
c' = P_new^T (P_old c)) against the float64 oracle.

Codes: the oracle re-bases the GPU's own stored codes (read back before the
call), so the comparison isolates the re-basing: the GPU multiplies in fp32
and rounds once to the cache dtype, i.e. within 1e-2 (bf16) or 1e-5 (fp32)
of each row's largest code, as for compress.  Decode after re-basing is
compared end to end with the oracle cache (append under P_old, re-base,
attend under P_new) at the stated bars: 2e-2 for bf16 codes, 1e-4 for fp32.
"""
import math

import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from tests import lrkv_testutil as tu

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _orth(gen, *lead, r):
    """Random orthonormal bases [*lead, 128, r] (float32, on the GPU)."""
    x = torch.randn(*lead, D, r, generator=gen, dtype=torch.float64)
    q, rr = torch.linalg.qr(x)
    q = q * torch.sign(torch.diagonal(rr, dim1=-2, dim2=-1)).unsqueeze(-2)
    return q.float().cuda().contiguous()


def _n_lat(L, n_sink, W):
    sink = min(L, n_sink)
    return L - sink - min(L - sink, W)


def _row_err(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    if a.size == 0:
        return 0.0
    den = np.maximum(np.abs(b).max(axis=1), 1e-30)
    return float((np.abs(a - b).max(axis=1) / den).max())


def _case(lrkv, *, dtype, B, H_kv, G, rk, rv, n_sink, W, lens, per_seq, sides="kv",
          same_span=False, seed=0, contiguous=False):
    gen = torch.Generator().manual_seed(seed)
    T = max(lens)
    perm = torch.randperm(B * math.ceil(max(1, T - n_sink - W) / 64), generator=gen)
    cache = lrkv.LatentCache(B, H_kv, rk, rv, T, n_sink, W, dtype=dtype,
                             page_perm=None if contiguous else perm)
    K = torch.randn(B, H_kv, T, D, generator=gen).to(dtype).cuda()
    V = torch.randn(B, H_kv, T, D, generator=gen).to(dtype).cuda()
    Bp = B if per_seq else 1
    Pk0, Pv0 = _orth(gen, Bp, H_kv, r=rk), _orth(gen, Bp, H_kv, r=rv)
    if same_span:  # the same subspaces in other coordinates
        Rk = torch.linalg.qr(torch.randn(Bp, H_kv, rk, rk, generator=gen, dtype=torch.float64))[0]
        Rv = torch.linalg.qr(torch.randn(Bp, H_kv, rv, rv, generator=gen, dtype=torch.float64))[0]
        Pk1 = (Pk0.double() @ Rk.cuda()).float().contiguous()
        Pv1 = (Pv0.double() @ Rv.cuda()).float().contiguous()
    else:
        Pk1, Pv1 = _orth(gen, Bp, H_kv, r=rk), _orth(gen, Bp, H_kv, r=rv)
    bs = H_kv * D * rk if per_seq else 0
    assert not per_seq or rk == rv  # one batch stride serves both bases
    n_new = torch.tensor(lens, dtype=torch.int32).cuda()
    lrkv.compress(cache, K, V, Pk0, Pv0, basis_batch_stride=bs, n_new=n_new)
    torch.cuda.synchronize()
    before = {(b, h, s): tu.gather_codes(cache, b, h, _n_lat(lens[b], n_sink, W), s)
              for b in range(B) for h in range(H_kv) for s in "kv"}
    q = torch.randn(B, H_kv * G, D, generator=gen).to(dtype).cuda()
    o_before = torch.empty_like(q)
    wsd = lrkv.decode_workspace(cache, H_kv * G)
    lrkv.decode_attn(cache, q, Pk0, Pv0, 1 / math.sqrt(D), o_before, wsd, basis_batch_stride=bs)

    ws = lrkv.rebase_workspace(cache)
    lrkv.rebase(cache, Pk0 if "k" in sides else None, Pk1 if "k" in sides else None,
                Pv0 if "v" in sides else None, Pv1 if "v" in sides else None, ws,
                basis_batch_stride=bs)
    o_after = torch.empty_like(q)
    Pk_use = Pk1 if "k" in sides else Pk0
    Pv_use = Pv1 if "v" in sides else Pv0
    lrkv.decode_attn(cache, q, Pk_use, Pv_use, 1 / math.sqrt(D), o_after, wsd,
                     basis_batch_stride=bs)
    torch.cuda.synchronize()
    assert lrkv.workspace_error(ws) == 0 and lrkv.workspace_error(wsd) == 0
    key = "bf16" if dtype == torch.bfloat16 else "f32"

    # codes: the oracle re-bases the GPU's own codes
    P = {"k": (Pk0.double().cpu().numpy(), Pk1.double().cpu().numpy()),
         "v": (Pv0.double().cpu().numpy(), Pv1.double().cpu().numpy())}
    for (b, h, s), c0 in before.items():
        got = tu.gather_codes(cache, b, h, c0.shape[0], s)
        if s not in sides:
            assert np.array_equal(got, c0)  # untouched side: bit for bit
            continue
        bb = b if per_seq else 0
        want = orc.rebase_codes(P[s][0][bb, h], P[s][1][bb, h], c0)
        assert _row_err(got, want) < tu.TOL_CODE[key], (b, h, s)

    # decode after re-basing, end to end against the oracle cache
    Kn, Vn = K.double().cpu().numpy(), V.double().cpu().numpy()
    qn = q.double().cpu().numpy()
    for b in range(B):
        bb = b if per_seq else 0
        oc = orc.LatentCacheOracle(1, H_kv, rk, rv, n_sink, W)
        oc.append(Kn[b:b + 1, :, :lens[b]], Vn[b:b + 1, :, :lens[b]],
                  P["k"][0][bb:bb + 1], P["v"][0][bb:bb + 1])
        oc.rebase(P["k"][0][bb:bb + 1] if "k" in sides else None, P["k"][1][bb:bb + 1],
                  P["v"][0][bb:bb + 1] if "v" in sides else None, P["v"][1][bb:bb + 1])
        Pk_o = P["k"][1 if "k" in sides else 0][bb:bb + 1]
        Pv_o = P["v"][1 if "v" in sides else 0][bb:bb + 1]
        ref = oc.attend(qn[b:b + 1], Pk_o, Pv_o, 1 / math.sqrt(D))
        assert tu.row_rel_err(o_after[b:b + 1].double().cpu().numpy(), ref) < tu.TOL[key], b
    return o_before, o_after


def test_rebase_fp32_per_sequence_bases(lrkv):
    """fp32 codes, one basis per sequence, pages in a permuted pool, ragged
    lengths with partial last pages."""
    _case(lrkv, dtype=torch.float32, B=3, H_kv=2, G=2, rk=32, rv=32, n_sink=1, W=16,
          lens=[300, 129, 64 + 17 + 5], per_seq=True, seed=1)


def test_rebase_bf16_shared_basis_with_empty_and_all_anchor_sequences(lrkv):
    """bf16 codes at r 64/32 (the decode rank class), a shared basis; one
    sequence is empty and one holds only anchors (nothing to re-base)."""
    _case(lrkv, dtype=torch.bfloat16, B=4, H_kv=4, G=4, rk=64, rv=32, n_sink=1, W=128,
          lens=[1000, 0, 100, 700], per_seq=False, seed=2)


def test_rebase_keys_only_leaves_value_codes_bitwise(lrkv):
    _case(lrkv, dtype=torch.bfloat16, B=2, H_kv=2, G=2, rk=48, rv=64, n_sink=0, W=0,
          lens=[520, 333], per_seq=False, sides="k", seed=3)


def test_rebase_within_the_same_span_keeps_decode_output(lrkv):
    """P_new = P_old Q spans the same subspaces: decode output before and
    after re-basing agree within one rounding of the codes."""
    o0, o1 = _case(lrkv, dtype=torch.float32, B=2, H_kv=2, G=4, rk=64, rv=64, n_sink=1, W=32,
                   lens=[640, 400], per_seq=False, same_span=True, seed=4)
    assert tu.row_rel_err(o1.double().cpu().numpy(), o0.double().cpu().numpy()) < 1e-4


def test_rebase_wide_ranks(lrkv):
    """r_k = r_v = 128 (the largest rank; one R per side staged at a time)."""
    _case(lrkv, dtype=torch.bfloat16, B=2, H_kv=1, G=8, rk=128, rv=128, n_sink=1, W=8,
          lens=[200, 75], per_seq=False, seed=5)


def test_rebase_bf16_consecutive_pages(lrkv):
    """bf16 codes at r 64/32 in a pool whose pages follow one another, so
    page pairs arrive by one tensor load (about 4 pages per CTA); odd page
    counts, partial last pages and range ends leave single-page jobs on the
    chunk copies, and one sequence holds only anchors."""
    _case(lrkv, dtype=torch.bfloat16, B=4, H_kv=4, G=4, rk=64, rv=32, n_sink=1, W=128,
          lens=[4000, 64 * 5 + 129 + 7, 100, 64 * 40 + 129], per_seq=False, seed=6,
          contiguous=True)


def test_rebase_bf16_consecutive_pages_equal_ranks(lrkv):
    """The same at r_k = r_v = 64 (16 chunks per page, a 32 KB box), about
    3.5 pages per CTA."""
    _case(lrkv, dtype=torch.bfloat16, B=2, H_kv=4, G=2, rk=64, rv=64, n_sink=1, W=8,
          lens=[8000, 64 * 3 + 9 + 1], per_seq=False, seed=7, contiguous=True)

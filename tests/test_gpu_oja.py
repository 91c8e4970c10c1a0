"""GPU parity of the Oja subspace update and QR re-orthonormalisation against
the float64 oracle (plain-C loop, OjaKV article: Oja's rule for online PCA).

The kernel runs in fp32.  Tolerance: max |P - P_ref| <= 1e-4 * max |P_ref|
(the stated bar for fp32 paths); QR with diag(R) > 0 makes P unique, so P
itself is compared, not only its projector.
"""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_lrkv_b200 import workloads as wk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def _setup(S, r, n, dtype, seed=0):
    g = np.random.default_rng(seed)
    P0 = np.stack([wk.haar_orthogonal(g)[:, :r] for _ in range(S)]).astype(np.float32)
    X = (g.standard_normal((S, n, 128)) * wk.spectrum("k")[None, None, :]) @ wk.haar_orthogonal(g)
    Xt = torch.from_numpy(X.astype(np.float32))
    if dtype == "bf16":
        Xt = Xt.to(torch.bfloat16)
    return P0, Xt


@pytest.mark.parametrize("r,dtype,qr_every,seen", [(48, "bf16", 256, 100), (32, "f32", 64, 0),
                                                   (8, "bf16", 0, 0), (128, "f32", 100, 7),
                                                   (64, "bf16", 128, 0), (56, "f32", 200, 3)])
def test_oja_matches_oracle(lrkv, r, dtype, qr_every, seen):
    S, n, eta = 5, 700, 1e-3
    P0, X = _setup(S, r, n, dtype)
    P = torch.from_numpy(P0).cuda()
    lrkv.oja_update(P, X.cuda(), eta, qr_every, seen)
    ref = orc.oja_update_streams(P0.astype(np.float64), X.float().numpy(), eta, qr_every, seen)
    assert _rel(P.cpu().double().numpy(), ref) <= 1e-4


def test_oja_split_calls_equal_one_call(lrkv):
    S, r, n = 3, 48, 512
    P0, X = _setup(S, r, n, "bf16", seed=1)
    Xd = X.cuda()
    one = torch.from_numpy(P0).cuda()
    lrkv.oja_update(one, Xd, 1e-3, 100, 0)
    two = torch.from_numpy(P0).cuda()
    lrkv.oja_update(two, Xd[:, :200].contiguous(), 1e-3, 100, 0)
    lrkv.oja_update(two, Xd[:, 200:].contiguous(), 1e-3, 100, 200)
    assert torch.equal(one, two)


def test_qr_gives_orthonormal_basis_with_positive_diagonal(lrkv):
    g = np.random.default_rng(2)
    A = g.standard_normal((4, 128, 40)).astype(np.float32)
    P = torch.from_numpy(A).cuda()
    lrkv.qr_orthonormalize(P)
    Q = P.cpu().double().numpy()
    for s in range(4):
        ref = orc.qr_positive(A[s].astype(np.float64))
        assert np.max(np.abs(Q[s] - ref)) < 1e-5
        assert np.max(np.abs(Q[s].T @ Q[s] - np.eye(40))) < 1e-5


def test_oja_strided_streams(lrkv):
    """x streams taken from a [B, H_kv, T, 128] cache view (stride T * 128)."""
    S, r, n, T = 4, 16, 300, 512
    P0, X = _setup(S, r, T, "bf16", seed=3)
    P = torch.from_numpy(P0).cuda()
    Xd = X.cuda()
    lrkv.oja_update(P, Xd[:, :n], 2e-3, 128, 0)
    ref = orc.oja_update_streams(P0.astype(np.float64), X[:, :n].float().numpy(), 2e-3, 128, 0)
    assert _rel(P.cpu().double().numpy(), ref) <= 1e-4

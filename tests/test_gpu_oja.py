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


def _blocked_ref(P0, X, eta, qr_every, seen, chunk):
    return np.stack([orc.oja_update_blocked(P0[s].astype(np.float64), X[s].float().numpy(), eta,
                                            qr_every, seen, chunk) for s in range(P0.shape[0])])


@pytest.mark.parametrize("r,dtype,qr_every,seen,chunk", [
    (48, "bf16", 256, 100, 64), (32, "f32", 64, 0, 16), (8, "bf16", 0, 0, 64),
    (64, "bf16", 128, 5, 64), (56, "f32", 100, 3, 7), (48, "bf16", 256, 0, 1)])
def test_chunked_oja_matches_oracle(lrkv, r, dtype, qr_every, seen, chunk):
    """lrkv_oja_update_chunked against the oracle's chunked rule (fp32 bar);
    chunk 7 and QR every 100 make chunks end early at QR points."""
    S, n, eta = 5, 700, 1e-3
    P0, X = _setup(S, r, n, dtype, seed=3)
    P = torch.from_numpy(P0).cuda()
    lrkv.oja_update_chunked(P, X.cuda(), eta, qr_every, seen, chunk)
    ref = _blocked_ref(P0, X, eta, qr_every, seen, chunk)
    assert _rel(P.cpu().double().numpy(), ref) <= 1e-4


def test_chunked_oja_split_calls_equal_one_call(lrkv):
    """Splitting the tokens at a chunk boundary changes nothing."""
    S, r, n = 3, 48, 640
    P0, X = _setup(S, r, n, "bf16", seed=4)
    Xd = X.cuda()
    one = torch.from_numpy(P0).cuda()
    lrkv.oja_update_chunked(one, Xd, 1e-3, 256, 0, 64)
    two = torch.from_numpy(P0).cuda()
    lrkv.oja_update_chunked(two, Xd[:, :256].contiguous(), 1e-3, 256, 0, 64)
    lrkv.oja_update_chunked(two, Xd[:, 256:].contiguous(), 1e-3, 256, 256, 64)
    assert torch.equal(one, two)


def test_chunked_oja_rejects_wide_ranks(lrkv):
    P = torch.zeros(1, 128, 96, device="cuda")
    x = torch.zeros(1, 64, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lrkv.LrkvError) as e:
        lrkv.oja_update_chunked(P, x, 1e-3, 0, 0, 64)
    assert e.value.status == -2

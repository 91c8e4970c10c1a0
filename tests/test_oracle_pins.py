"""Pins of the float64 oracle to facts that do not come from the oracle.

Each test ties one oracle function to a closed form, an invariant of the
mathematics, a value printed on the pages (tests/golden/), or an
independent pure-Python loop, so that a dropped term, a wrong sign or index
or a transposed operand fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import bruteforce as bf
from oracle import lrkv_oracle as orc
from rank_kv_cache_lrkv_b200 import workloads as wk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D = 128


def _orth(rng, n, r):
    q, rr = np.linalg.qr(rng.standard_normal((n, r)))
    return q * np.sign(np.diag(rr))[None, :]


# ------------------------------------------------------------ attention

def test_full_rank_orthonormal_basis_reproduces_dense_attention():
    """Half the Memory, section 04: routing the uncompressed cache through
    the path reproduces the model's output.  r = 128 with an orthonormal
    basis is that case: latent attention must equal dense attention."""
    rng = np.random.default_rng(1)
    Pk, Pv = _orth(rng, D, D), _orth(rng, D, D)
    K, V = rng.standard_normal((40, D)), rng.standard_normal((40, D))
    q = rng.standard_normal(D)
    o_lat = orc.latent_attention(q, Pk, Pv, orc.project(Pk, K), orc.project(Pv, V),
                                 np.zeros((0, D)), np.zeros((0, D)), 0.3)
    o_dense = orc.dense_attention(q, K, V, 0.3)
    assert np.max(np.abs(o_lat - o_dense)) < 1e-12 * np.max(np.abs(o_dense)) + 1e-13


def test_latent_equals_reconstructed_for_any_basis():
    """Section 08: attending on the codes is algebraically equal to
    attending over reconstructed tensors; true for any (non-orthonormal) P."""
    rng = np.random.default_rng(2)
    Pk = rng.standard_normal((D, 24)) * 0.2
    Pv = rng.standard_normal((D, 16)) * 0.2
    Ck, Cv = rng.standard_normal((30, 24)), rng.standard_normal((30, 16))
    Ka, Va = rng.standard_normal((5, D)), rng.standard_normal((5, D))
    q = rng.standard_normal(D)
    a = orc.latent_attention(q, Pk, Pv, Ck, Cv, Ka, Va, 0.2)
    b = orc.reconstructed_attention(q, Pk, Pv, Ck, Cv, Ka, Va, 0.2)
    assert np.max(np.abs(a - b)) < 1e-12 * np.max(np.abs(b))


def test_bruteforce_loops_match_vectorised_oracle():
    """Independent pure-Python loops on tiny inputs (T <= 16, r <= 8)."""
    rng = np.random.default_rng(3)
    for trial in range(3):
        rk, rv, n, na = 8, 4 + trial, 9 + 3 * trial, trial
        Pk, Pv = rng.standard_normal((D, rk)), rng.standard_normal((D, rv))
        Xk, Xv = rng.standard_normal((n, D)), rng.standard_normal((n, D))
        Ck, Cv = orc.project(Pk, Xk), orc.project(Pv, Xv)
        assert np.max(np.abs(Ck - np.array(bf.codes(Pk.tolist(), Xk.tolist())))) < 1e-12
        Ka, Va = rng.standard_normal((na, D)), rng.standard_normal((na, D))
        q = rng.standard_normal(D)
        o = orc.latent_attention(q, Pk, Pv, Ck, Cv, Ka, Va, 0.125)
        ob = bf.attention(q.tolist(), Pk.tolist(), Pv.tolist(), Ck.tolist(),
                          Cv.tolist(), Ka.tolist(), Va.tolist(), 0.125)
        assert np.max(np.abs(o - np.array(ob))) < 1e-13 * max(1.0, np.max(np.abs(o)))


def test_softmax_rows_sum_to_one_and_survive_huge_scores():
    rng = np.random.default_rng(4)
    for scale in [1.0, 1e3, 1e6]:
        p = orc.softmax(rng.standard_normal(1000) * scale)
        assert abs(p.sum() - 1.0) < 1e-15 * 1000
        assert np.all(np.isfinite(p)) and np.all(p >= 0)


def test_single_token_returns_its_reconstructed_value():
    rng = np.random.default_rng(5)
    Pk, Pv = rng.standard_normal((D, 8)), rng.standard_normal((D, 8))
    ck, cv = rng.standard_normal((1, 8)), rng.standard_normal((1, 8))
    o = orc.latent_attention(rng.standard_normal(D), Pk, Pv, ck, cv,
                             np.zeros((0, D)), np.zeros((0, D)), 1.0)
    assert np.max(np.abs(o - Pv @ cv[0])) < 1e-14 * np.max(np.abs(o))
    va = rng.standard_normal((1, D))
    o2 = orc.latent_attention(rng.standard_normal(D), Pk, Pv, np.zeros((0, 8)),
                              np.zeros((0, 8)), rng.standard_normal((1, D)), va, 1.0)
    assert np.array_equal(o2, va[0])


def test_zero_query_gives_mean_of_values():
    """q = 0 makes every score 0, so softmax is uniform."""
    rng = np.random.default_rng(6)
    Pk, Pv = rng.standard_normal((D, 8)), rng.standard_normal((D, 6))
    Ck, Cv = rng.standard_normal((7, 8)), rng.standard_normal((7, 6))
    Ka, Va = rng.standard_normal((3, D)), rng.standard_normal((3, D))
    o = orc.latent_attention(np.zeros(D), Pk, Pv, Ck, Cv, Ka, Va, 1.0)
    mean = (np.sum(Cv @ Pv.T, 0) + np.sum(Va, 0)) / 10.0
    assert np.max(np.abs(o - mean)) < 1e-14 * np.max(np.abs(mean))


def test_token_permutation_does_not_change_output():
    rng = np.random.default_rng(7)
    Pk, Pv = rng.standard_normal((D, 16)), rng.standard_normal((D, 8))
    Ck, Cv = rng.standard_normal((50, 16)), rng.standard_normal((50, 8))
    q = rng.standard_normal(D)
    z = np.zeros((0, D))
    a = orc.latent_attention(q, Pk, Pv, Ck, Cv, z, z, 0.1)
    perm = rng.permutation(50)
    b = orc.latent_attention(q, Pk, Pv, Ck[perm], Cv[perm], z, z, 0.1)
    assert np.max(np.abs(a - b)) < 1e-14 * np.max(np.abs(a))


def test_gqa_head_h_reads_kv_head_h_over_G():
    rng = np.random.default_rng(8)
    B, Hkv, G = 2, 3, 2
    c = orc.LatentCacheOracle(B, Hkv, 8, 8)
    Pk = rng.standard_normal((1, Hkv, D, 8))
    Pv = rng.standard_normal((1, Hkv, D, 8))
    k, v = rng.standard_normal((B, Hkv, 6, D)), rng.standard_normal((B, Hkv, 6, D))
    c.append(k, v, Pk, Pv)
    q = rng.standard_normal((B, Hkv * G, D))
    o = c.attend(q, Pk, Pv, 0.1)
    for b in range(B):
        for h in range(Hkv * G):
            g = h // G
            ref = orc.dense_attention(q[b, h], orc.reconstruct(Pk[0, g], orc.project(Pk[0, g], k[b, g])),
                                      orc.reconstruct(Pv[0, g], orc.project(Pv[0, g], v[b, g])), 0.1)
            assert np.max(np.abs(o[b, h] - ref)) < 1e-12 * np.max(np.abs(ref))


# ------------------------------------------------------------ cache / anchors

def test_all_anchor_cache_is_dense_attention_and_stores_inputs_bitwise():
    """OjaKV anchors are kept full-rank: a cache whose tokens are all anchors
    must be ordinary attention, with the anchor rows equal to the inputs."""
    rng = np.random.default_rng(9)
    T = 20
    c = orc.LatentCacheOracle(1, 1, 8, 8, n_sink=1, window=T)
    k, v = rng.standard_normal((1, 1, T, D)), rng.standard_normal((1, 1, T, D))
    P = rng.standard_normal((1, 1, D, 8))
    c.append(k, v, P, P)
    Ka, Va = c.anchors(0, 0)
    assert np.array_equal(Ka, k[0, 0]) and np.array_equal(Va, v[0, 0])
    assert c.codes_k[0][0].shape[0] == 0
    q = rng.standard_normal((1, 1, D))
    o = c.attend(q, P, P, 0.2)
    assert np.max(np.abs(o[0, 0] - orc.dense_attention(q[0, 0], k[0, 0], v[0, 0], 0.2))) < 1e-13


@pytest.mark.parametrize("n_sink,W", [(0, 0), (1, 0), (0, 5), (1, 5), (1, 64)])
def test_partition_and_chunked_appends(n_sink, W):
    """First token (sink) and the W most recent tokens full-rank, the rest
    compressed in order; appending in any chunking gives the same state."""
    rng = np.random.default_rng(10 + W)
    B, Hkv, T = 2, 2, 37
    k, v = rng.standard_normal((B, Hkv, T, D)), rng.standard_normal((B, Hkv, T, D))
    P = rng.standard_normal((1, Hkv, D, 8))
    one = orc.LatentCacheOracle(B, Hkv, 8, 8, n_sink, W)
    one.append(k, v, P, P)
    chunked = orc.LatentCacheOracle(B, Hkv, 8, 8, n_sink, W)
    pos = 0
    for n in [1, 3, 0, 10, 2, 21]:
        chunked.append(k[:, :, pos:pos + n], v[:, :, pos:pos + n], P, P)
        pos += n
    assert pos == T
    sink, lat, win = orc.partition(T, n_sink, W)
    assert len(sink) + len(lat) + len(win) == T
    for b in range(B):
        for h in range(Hkv):
            for c in (one, chunked):
                assert np.allclose(c.codes_k[b][h], k[b, h, lat] @ P[0, h], rtol=0, atol=1e-12)
                Ka, Va = c.anchors(b, h)
                assert np.array_equal(Ka, k[b, h, sink + win])
                assert np.array_equal(Va, v[b, h, sink + win])


def test_evicted_tokens_use_the_basis_current_at_eviction():
    rng = np.random.default_rng(11)
    k, v = rng.standard_normal((1, 1, 6, D)), rng.standard_normal((1, 1, 6, D))
    P1, P2 = rng.standard_normal((1, 1, D, 4)), rng.standard_normal((1, 1, D, 4))
    c = orc.LatentCacheOracle(1, 1, 4, 4, 0, 2)
    c.append(k[:, :, :4], v[:, :, :4], P1, P1)   # tokens 0,1 evicted with P1
    c.append(k[:, :, 4:], v[:, :, 4:], P2, P2)   # tokens 2,3 evicted with P2
    exp = np.concatenate([k[0, 0, :2] @ P1[0, 0], k[0, 0, 2:4] @ P2[0, 0]])
    assert np.allclose(c.codes_k[0][0], exp, rtol=0, atol=1e-12)


# ------------------------------------------------------------ re-basing

def test_rebase_is_the_least_squares_code_of_the_reconstruction():
    # pin against a different formulation: lstsq solves min ||P_new y - x^||
    rng = np.random.default_rng(21)
    P_old, P_new = _orth(rng, D, 16), _orth(rng, D, 16)
    C = rng.standard_normal((9, 16))
    got = orc.rebase_codes(P_old, P_new, C)
    xhat = C @ P_old.T
    want = np.linalg.lstsq(P_new, xhat.T, rcond=None)[0].T
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_rebase_onto_the_same_basis_is_the_identity():
    rng = np.random.default_rng(22)
    P = _orth(rng, D, 24)
    C = rng.standard_normal((7, 24))
    assert np.allclose(orc.rebase_codes(P, P, C), C, rtol=0, atol=1e-12)


def test_rebase_within_the_same_span_keeps_reconstruction_and_attention():
    # P_new = P_old Q spans the same subspace: every reconstruction, hence
    # every score and output, is unchanged
    rng = np.random.default_rng(23)
    r = 12
    P_k, P_v = _orth(rng, D, r)[None, None], _orth(rng, D, r)[None, None]
    Qk, Qv = _orth(rng, r, r), _orth(rng, r, r)
    P_k2, P_v2 = P_k @ Qk, P_v @ Qv
    c = orc.LatentCacheOracle(1, 1, r, r, 1, 3)
    k, v = rng.standard_normal((1, 1, 20, D)), rng.standard_normal((1, 1, 20, D))
    c.append(k, v, P_k, P_v)
    q = rng.standard_normal((1, 2, D))
    before = c.attend(q, P_k, P_v, 1 / math.sqrt(D))
    rec = c.codes_k[0][0] @ P_k[0, 0].T
    c.rebase(P_k, P_k2, P_v, P_v2)
    assert np.allclose(c.codes_k[0][0] @ P_k2[0, 0].T, rec, rtol=0, atol=1e-12)
    after = c.attend(q, P_k2, P_v2, 1 / math.sqrt(D))
    assert np.allclose(after, before, rtol=0, atol=1e-12)


def test_rebase_residual_is_the_part_outside_the_new_span():
    # ||P_new c' - x^||^2 = ||x^||^2 - ||c'||^2 for orthonormal P_new
    # (orthogonal projection), and the residual is orthogonal to span(P_new)
    rng = np.random.default_rng(24)
    P_old, P_new = _orth(rng, D, 20), _orth(rng, D, 20)
    C = rng.standard_normal((5, 20))
    xhat = C @ P_old.T
    c2 = orc.rebase_codes(P_old, P_new, C)
    res = c2 @ P_new.T - xhat
    assert np.allclose((res ** 2).sum(1), (xhat ** 2).sum(1) - (c2 ** 2).sum(1),
                       rtol=1e-10, atol=1e-10)
    assert np.abs(res @ P_new).max() < 1e-12


def test_rebase_pin_catches_a_transposed_operand():
    # a planted mistake in a copy of the oracle's arithmetic must fail the
    # least-squares pin: projecting with P_old^T P_new instead
    rng = np.random.default_rng(25)
    P_old, P_new = _orth(rng, D, 16), _orth(rng, D, 16)
    C = rng.standard_normal((9, 16))
    wrong = C @ (P_old.T @ P_new).T
    want = np.linalg.lstsq(P_new, (C @ P_old.T).T, rcond=None)[0].T
    assert not np.allclose(wrong, want, rtol=0, atol=1e-6)


# ------------------------------------------------------------ basis

def test_eckart_young_tail_energy_with_planted_spectrum():
    """Rank-r reconstruction error of the top-r SVD basis equals the sum of
    the squared tail singular values, which are planted here (not computed)."""
    rng = np.random.default_rng(12)
    n = 300
    U = _orth(rng, n, D)
    Vt = _orth(rng, D, D).T
    sig = np.exp(-np.arange(D) / 10.0) * 3.0
    X = (U * sig[None, :]) @ Vt
    for r in [8, 32, 64, 127]:
        P = orc.svd_basis(X, r)
        err = np.sum((X - orc.reconstruct(P, orc.project(P, X))) ** 2)
        tail = np.sum(sig[r:] ** 2)
        assert abs(err - tail) <= 1e-10 * tail + 1e-13 * np.sum(sig ** 2)
        assert np.max(np.abs(P.T @ P - np.eye(r))) < 1e-12


def test_generator_tail_energy_matches_its_spectrum():
    """The seeded generator's decaying spectrum: relative tail energy of a
    rank-r SVD basis is sum_{i>=r} s_i^2 / sum s_i^2 (statistically)."""
    wl = wk.TINY_SINGLE_HEAD
    for kind, r in [("k", 64), ("v", 32), ("k", 16)]:
        s2 = wk.spectrum(kind) ** 2
        expect = s2[r:].sum() / s2.sum()
        X = wk.stream(wl, kind, 0, 0, 0, n=2048)
        P = wk.basis(wl.with_(r_k=r, r_v=r), kind, 0, 0).astype(np.float64)
        rel = np.sum((X - orc.reconstruct(P, orc.project(P, X))) ** 2) / np.sum(X ** 2)
        assert 0.8 * expect < rel < 1.25 * expect, (kind, r, rel, expect)


# ------------------------------------------------------------ Oja

def test_oja_single_step_closed_form():
    """P = e1 (r = 1), x = a e1 + b e2: y = a, x - P y = b e2, so the new
    basis is e1 + eta a b e2 (worked by hand)."""
    a, b, eta = 2.0, 3.0, 0.1
    P = np.zeros((D, 1))
    P[0, 0] = 1.0
    x = np.zeros(D)
    x[0], x[1] = a, b
    out = orc.oja_update(P, x[None, :], eta, 0)
    exp = P.copy()
    exp[1, 0] = eta * a * b
    assert np.array_equal(out, exp)
    out_c = orc.oja_update_streams(P[None], x[None, None, :], eta, 0)[0]
    assert np.array_equal(out_c, exp)


def test_oja_in_span_is_a_fixed_point():
    rng = np.random.default_rng(13)
    P = _orth(rng, D, 6)
    X = rng.standard_normal((20, 6)) @ P.T
    out = orc.oja_update(P, X, 0.05, 0)
    assert np.max(np.abs(out - P)) < 1e-14


def test_oja_step_matches_bruteforce_loops():
    rng = np.random.default_rng(14)
    P = rng.standard_normal((D, 5)) * 0.1
    x = rng.standard_normal(D)
    a = orc.oja_update(P, x[None], 0.01, 0)
    b = np.array(bf.oja_step(P.tolist(), x.tolist(), 0.01))
    assert np.max(np.abs(a - b)) < 1e-14


def test_oja_qr_orthonormal_with_positive_diagonal():
    rng = np.random.default_rng(15)
    P = rng.standard_normal((D, 12))
    Q = orc.qr_positive(P)
    assert np.max(np.abs(Q.T @ Q - np.eye(12))) < 1e-13
    R = Q.T @ P
    assert np.max(np.abs(np.tril(R, -1))) < 1e-12 and np.all(np.diag(R) > 0)
    assert np.max(np.abs(Q @ R - P)) < 1e-12


def test_oja_c_loop_matches_numpy_loop_with_qr():
    rng = np.random.default_rng(16)
    S, r, n = 3, 8, 70
    P0 = np.stack([_orth(rng, D, r) for _ in range(S)])
    X = rng.standard_normal((S, n, D)).astype(np.float32)
    Pc = orc.oja_update_streams(P0, X, 0.02, 16, tokens_seen=5)
    for s in range(S):
        Pn = orc.oja_update(P0[s], X[s].astype(np.float64), 0.02, 16, tokens_seen=5)
        assert np.max(np.abs(Pc[s] - Pn)) < 1e-12


def test_oja_two_half_calls_equal_one_call():
    rng = np.random.default_rng(17)
    P0 = _orth(rng, D, 8)
    X = rng.standard_normal((100, D))
    one = orc.oja_update(P0, X, 0.01, 32)
    two = orc.oja_update(orc.oja_update(P0, X[:50], 0.01, 32), X[50:], 0.01, 32,
                         tokens_seen=50)
    assert np.max(np.abs(one - two)) < 1e-12


def test_oja_is_rotation_equivariant():
    """P -> P R (R orthogonal) maps the trajectory to P_t R without QR; with
    QR the projector P P^T is unchanged."""
    rng = np.random.default_rng(18)
    P0 = _orth(rng, D, 6)
    R = _orth(rng, 6, 6)
    X = rng.standard_normal((60, D))
    a = orc.oja_update(P0, X, 0.01, 0)
    b = orc.oja_update(P0 @ R, X, 0.01, 0)
    assert np.max(np.abs(a @ R - b)) < 1e-12
    a = orc.oja_update(P0, X, 0.01, 20)
    b = orc.oja_update(P0 @ R, X, 0.01, 20)
    assert np.max(np.abs(a @ a.T - b @ b.T)) < 1e-12


def test_oja_tracks_a_planted_subspace():
    """On data drawn from a planted r-dim subspace plus small noise the
    projector distance to the planted subspace shrinks while it is far above
    the noise floor, and ends near that floor."""
    rng = np.random.default_rng(19)
    r = 4
    U = _orth(rng, D, r)
    P = _orth(rng, D, r)
    X = rng.standard_normal((3000, r)) @ (U.T * 3.0) + 0.01 * rng.standard_normal((3000, D))
    dist = [np.linalg.norm(P @ P.T - U @ U.T)]
    for c in range(6):
        P = orc.oja_update(P, X[c * 100:(c + 1) * 100], 0.001, 50, tokens_seen=c * 100)
        dist.append(np.linalg.norm(P @ P.T - U @ U.T))
    assert all(dist[i + 1] < dist[i] for i in range(len(dist) - 1)), dist
    P = orc.oja_update(P, X[600:], 0.01, 50, tokens_seen=600)
    assert np.linalg.norm(P @ P.T - U @ U.T) < 0.05 * dist[0]


# ------------------------------------------------------------ sizes

def test_llama_kv_cache_is_16_gib():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_sizes.json")))["llama31_8b_dense_32k_b4"]
    n = orc.kv_cache_bytes(g["layers"], g["kv_heads"], g["head_dim"], g["tokens"],
                           g["batch"], g["bytes_per_elem"])
    assert n == g["exact_gib"] * 2 ** 30
    assert abs(n / 1e9 - g["stated_gb_approx"]) / g["stated_gb_approx"] < 0.1


def test_two_x_compression_halves_the_cache_and_values_at_quarter():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_sizes.json")))
    h = g["halved_at_2x"]
    assert orc.compression_ratio(h["r_k_plus_r_v"] // 2, h["r_k_plus_r_v"] // 2) == h["ratio"]
    dense = orc.kv_cache_bytes(1, 8, 128, 4096, 2)
    lat = orc.latent_cache_bytes(1, 8, 64, 64, 4096, 2)
    assert dense == 2 * lat
    q = g["values_at_quarter"]
    assert q["r_v"] / q["head_dim"] == q["fraction"]
    assert math.isclose(orc.compression_ratio(64, 32), 256 / 96)


# ------------------------------------------------------------ decode from parts

def _parts_case(rng, B, Hkv, G, rk, rv, lens, n_anc, per_seq_basis):
    """Explicit per-(sequence, KV head) parts with ragged latent and anchor
    counts, and per-sequence bases when asked."""
    Bp = B if per_seq_basis else 1
    Pk = rng.standard_normal((Bp, Hkv, D, rk)) * 0.3
    Pv = rng.standard_normal((Bp, Hkv, D, rv)) * 0.3
    Ck = [[rng.standard_normal((lens[b][h], rk)) for h in range(Hkv)] for b in range(B)]
    Cv = [[rng.standard_normal((lens[b][h], rv)) for h in range(Hkv)] for b in range(B)]
    Ka = [[rng.standard_normal((n_anc[b][h], D)) for h in range(Hkv)] for b in range(B)]
    Va = [[rng.standard_normal((n_anc[b][h], D)) for h in range(Hkv)] for b in range(B)]
    q = rng.standard_normal((B, Hkv * G, D))
    return q, Pk, Pv, Ck, Cv, Ka, Va


@pytest.mark.parametrize("G", [1, 2, 4])
def test_decode_from_parts_matches_independent_loops(G):
    """Half the Memory, section 08 (attention on the codes) with OjaKV
    anchors: every (sequence, q head) output of decode_from_parts must equal
    the pure-Python loop over reconstructed rows of KV head h // G, with the
    basis of its own sequence.  Ragged latent and anchor counts per unit, one
    unit with no latent tokens, and r_k == r_v so that a swap of the key and
    value codes would still run (and must fail here)."""
    rng = np.random.default_rng(300 + G)
    B, Hkv, rk, rv = 2, 2, 6, 6
    lens = [[5, 0], [3, 7]]
    n_anc = [[2, 3], [0, 1]]
    q, Pk, Pv, Ck, Cv, Ka, Va = _parts_case(rng, B, Hkv, G, rk, rv, lens, n_anc, True)
    o = orc.decode_from_parts(q, Pk, Pv, Ck, Cv, Ka, Va, G, 0.2)
    assert o.shape == (B, Hkv * G, D)
    for b in range(B):
        for h in range(Hkv * G):
            g = h // G
            ref = bf.attention(q[b, h].tolist(), Pk[b, g].tolist(), Pv[b, g].tolist(),
                               Ck[b][g].tolist(), Cv[b][g].tolist(), Ka[b][g].tolist(),
                               Va[b][g].tolist(), 0.2)
            ref = np.array(ref)
            assert np.max(np.abs(o[b, h] - ref)) < 1e-12 * np.max(np.abs(ref)), (b, h)


def test_decode_from_parts_pin_catches_planted_mistakes():
    """The loop comparison above is discriminating: the plausible mistakes
    (head map h % G, key and value codes swapped, the shared basis of
    sequence 0 used for every sequence) each move the output far beyond
    the 1e-12 bar on the same data."""
    rng = np.random.default_rng(310)
    B, Hkv, G, r = 2, 2, 2, 6
    lens = [[5, 4], [3, 7]]
    n_anc = [[2, 3], [1, 1]]
    q, Pk, Pv, Ck, Cv, Ka, Va = _parts_case(rng, B, Hkv, G, r, r, lens, n_anc, True)
    o = orc.decode_from_parts(q, Pk, Pv, Ck, Cv, Ka, Va, G, 0.2)
    b, h = 1, 1                      # h % G = 1 but h // G = 0
    good = orc.latent_attention(q[b, h], Pk[b, 0], Pv[b, 0], Ck[b][0], Cv[b][0],
                                Ka[b][0], Va[b][0], 0.2)
    wrong = [
        orc.latent_attention(q[b, h], Pk[b, 1], Pv[b, 1], Ck[b][1], Cv[b][1], Ka[b][1],
                             Va[b][1], 0.2),
        orc.latent_attention(q[b, h], Pk[b, 0], Pv[b, 0], Cv[b][0], Ck[b][0], Ka[b][0],
                             Va[b][0], 0.2),
        orc.latent_attention(q[b, h], Pk[0, 0], Pv[0, 0], Ck[b][0], Cv[b][0], Ka[b][0],
                             Va[b][0], 0.2),
    ]
    scale = np.max(np.abs(good))
    assert np.max(np.abs(o[b, h] - good)) < 1e-12 * scale
    for w in wrong:
        assert np.max(np.abs(w - good)) > 1e-3 * scale


@pytest.mark.parametrize("G", [1, 2, 4])
def test_decode_from_parts_equals_cache_attend(G):
    """Parts read out of a LatentCacheOracle (sink + window + codes, per
    sequence bases) decode to exactly what the cache's own attend gives."""
    rng = np.random.default_rng(320 + G)
    B, Hkv, rk, rv = 2, 2, 8, 4
    c = orc.LatentCacheOracle(B, Hkv, rk, rv, n_sink=1, window=3)
    Pk = rng.standard_normal((B, Hkv, D, rk)) * 0.3
    Pv = rng.standard_normal((B, Hkv, D, rv)) * 0.3
    k, v = rng.standard_normal((B, Hkv, 13, D)), rng.standard_normal((B, Hkv, 13, D))
    c.append(k, v, Pk, Pv)
    q = rng.standard_normal((B, Hkv * G, D))
    Ck = [[c.codes_k[b][h] for h in range(Hkv)] for b in range(B)]
    Cv = [[c.codes_v[b][h] for h in range(Hkv)] for b in range(B)]
    Ka = [[c.anchors(b, h)[0] for h in range(Hkv)] for b in range(B)]
    Va = [[c.anchors(b, h)[1] for h in range(Hkv)] for b in range(B)]
    o = orc.decode_from_parts(q, Pk, Pv, Ck, Cv, Ka, Va, G, 0.15)
    ref = c.attend(q, Pk, Pv, 0.15)
    assert np.max(np.abs(o - ref)) < 1e-13 * np.max(np.abs(ref))


# ------------------------------------------------------------ quantised codes

def test_quantize_codes_worked_example():
    """By hand: the largest magnitude maps to 127 and sets the scale; the
    rest round half to even."""
    C = np.array([[0.5, -1.27, 0.01, 0.005],
                  [0.0, 0.0, 0.0, 0.0],
                  [2.0, 1.0, -0.5, 0.25]])
    q, s = orc.quantize_codes(C, 8)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert np.isclose(s[0], 0.01, rtol=1e-6) and s[1] == 0 and np.isclose(s[2], 2.0 / 127, rtol=1e-6)
    assert q[0].tolist() == [50, -127, 1, 0]          # 0.5 -> 0 (half to even)
    assert q[1].tolist() == [0, 0, 0, 0]
    assert q[2].tolist() == [127, 64, -32, 16]        # 63.5 -> 64, 15.875 -> 16


def test_quantize_codes_round_trip_bound_and_extremes():
    """Every row: |c - q s| <= s / 2 (plus fp32 rounding of c), the largest
    entry is reproduced to fp32 precision, and |q| <= 127."""
    rng = np.random.default_rng(400)
    C = rng.standard_normal((200, 24)) * np.exp(-np.arange(24) / 8.0)[None, :]
    C[7] *= 1e-30                       # tiny row: still its own scale
    q, s = orc.quantize_codes(C, 8)
    Ch = orc.dequantize_codes(q, s)
    err = np.abs(Ch - C)
    assert np.all(err <= s[:, None] / 2 * (1 + 1e-6) + np.abs(C) * 2 ** -23)
    assert np.all(np.abs(q.astype(int)) <= 127)
    j = np.argmax(np.abs(C), axis=1)
    assert np.all(np.abs(q[np.arange(200), j].astype(int)) == 127)
    assert np.allclose(Ch[np.arange(200), j], C[np.arange(200), j], rtol=1e-6, atol=0)


def test_quantised_cache_attends_over_dequantised_codes():
    """The quantised cache keeps each code row as its dequantised int8 form;
    attention reads those rows, anchors stay exact."""
    rng = np.random.default_rng(401)
    P = rng.standard_normal((1, 1, D, 16)) * 0.2
    k, v = rng.standard_normal((1, 1, 40, D)), rng.standard_normal((1, 1, 40, D))
    cq = orc.LatentCacheOracle(1, 1, 16, 16, n_sink=1, window=4, quant_bits=8)
    cq.append(k, v, P, P)
    lat = list(range(1, 36))
    ref_k = orc.dequantize_codes(*orc.quantize_codes(k[0, 0, lat] @ P[0, 0], 8))
    assert np.array_equal(cq.codes_k[0][0], ref_k)
    Ka, _ = cq.anchors(0, 0)
    assert np.array_equal(Ka, k[0, 0, [0, 36, 37, 38, 39]])
    q = rng.standard_normal((1, 1, D))
    o = cq.attend(q, P, P, 0.1)
    o_ref = orc.latent_attention(q[0, 0], P[0, 0], P[0, 0], ref_k, cq.codes_v[0][0], Ka,
                                 cq.anchors(0, 0)[1], 0.1)
    assert np.max(np.abs(o[0, 0] - o_ref)) < 1e-14 * np.max(np.abs(o_ref))
    # close to the unquantised cache (8-bit codes: well inside the bf16 bar)
    c = orc.LatentCacheOracle(1, 1, 16, 16, n_sink=1, window=4)
    c.append(k, v, P, P)
    o_full = c.attend(q, P, P, 0.1)
    assert np.max(np.abs(o - o_full)) < 2e-2 * np.max(np.abs(o_full))


# ------------------------------------------------------------ chunked Oja

def test_blocked_oja_with_chunk_one_is_the_sequential_rule():
    rng = np.random.default_rng(500)
    P0 = _orth(rng, D, 12)
    X = rng.standard_normal((300, D)) * np.exp(-np.arange(D) / 16.0)[None, :]
    a = orc.oja_update_blocked(P0, X, 0.01, 64, tokens_seen=30, chunk=1)
    b = orc.oja_update(P0, X, 0.01, 64, tokens_seen=30)
    assert np.max(np.abs(a - b)) < 1e-13


def test_blocked_oja_one_chunk_is_the_covariance_form():
    """One chunk, written through the chunk's second moment C = X^T X:
    P + eta (C P - P P^T C P) -- the frozen-basis sum of Oja's per-token
    updates, spelled without Y or Z."""
    rng = np.random.default_rng(501)
    P0 = rng.standard_normal((D, 8)) * 0.1
    X = rng.standard_normal((40, D))
    C = X.T @ X
    ref = P0 + 0.003 * (C @ P0 - P0 @ (P0.T @ C @ P0))
    got = orc.oja_update_blocked(P0, X, 0.003, 0, chunk=64)
    assert np.max(np.abs(got - ref)) < 1e-12 * np.max(np.abs(ref))


def test_blocked_oja_chunks_stop_at_qr_points():
    """tokens_seen = 50, QR every 64: chunks of 64 end at tokens 14, 78, ...,
    so the result equals explicit calls on those pieces with a QR after each
    piece that reaches a multiple of 64."""
    rng = np.random.default_rng(502)
    P0 = _orth(rng, D, 8)
    X = rng.standard_normal((200, D)) * 0.3
    got = orc.oja_update_blocked(P0, X, 0.02, 64, tokens_seen=50, chunk=64)
    P = P0.copy()
    for lo, hi in [(0, 14), (14, 78), (78, 142), (142, 200)]:
        P = orc.oja_update_blocked(P, X[lo:hi], 0.02, 0, chunk=64)
        if (50 + hi) % 64 == 0:
            P = orc.qr_positive(P)
    assert np.max(np.abs(got - P)) < 1e-13


def test_blocked_oja_span_is_a_fixed_point_and_tracks_a_planted_subspace():
    rng = np.random.default_rng(503)
    P = _orth(rng, D, 6)
    X = rng.standard_normal((50, 6)) @ P.T           # rows inside span(P)
    assert np.max(np.abs(orc.oja_update_blocked(P, X, 0.05, 0) - P)) < 1e-13
    U = _orth(rng, D, 6)                              # planted subspace
    Xs = rng.standard_normal((4000, 6)) * 3.0 @ U.T + 0.05 * rng.standard_normal((4000, D))
    P1 = orc.oja_update_blocked(_orth(rng, D, 6), Xs, 2e-3, 256, chunk=32)
    s = np.linalg.svd(U.T @ P1, compute_uv=False)
    assert np.min(s) > 0.99                           # cosines of the principal angles


def test_blocked_oja_departs_from_sequential_in_proportion_to_the_chunk():
    """Freezing P over a chunk of b tokens changes each chunk's update by a
    term of order eta^2 b: over the same tokens the distance to the
    sequential rule grows in proportion to b (chunk 1 is the rule itself)."""
    rng = np.random.default_rng(504)
    P0 = _orth(rng, D, 16)
    X = rng.standard_normal((2048, D)) * np.exp(-np.arange(D) / 16.0)[None, :]
    seq = orc.oja_update(P0, X, 1e-3, 256)
    d = {b: np.max(np.abs(orc.oja_update_blocked(P0, X, 1e-3, 256, chunk=b) - seq))
         for b in (1, 8, 64)}
    assert d[1] < 1e-13
    assert 5 < d[64] / d[8] < 11
    assert d[8] < 1e-3


# ------------------------------------------------------------ value amortisation

def test_value_predictor_residual_is_orthogonal_to_the_key_codes():
    """Least squares, checked through its normal equations: C_k^T (C_k A - C_v) = 0."""
    rng = np.random.default_rng(600)
    Ck, Cv = rng.standard_normal((300, 16)), rng.standard_normal((300, 8))
    A = orc.fit_value_predictor(Ck, Cv)
    assert A.shape == (16, 8)
    assert np.max(np.abs(Ck.T @ (Ck @ A - Cv))) < 1e-10 * np.max(np.abs(Ck.T @ Cv))


def test_value_predictor_recovers_an_exact_linear_map():
    rng = np.random.default_rng(601)
    Ck = rng.standard_normal((200, 12))
    A_true = rng.standard_normal((12, 6))
    A = orc.fit_value_predictor(Ck, Ck @ A_true)
    assert np.max(np.abs(A - A_true)) < 1e-12
    vals, kept = orc.amortised_value_codes(Ck, Ck @ A_true, A, keep=0)
    assert np.max(np.abs(vals - Ck @ A_true)) < 1e-12 and not kept.any()


def test_amortised_selection_worked_example():
    """Pages of 4 tokens, keep 2: residual norms (by hand) 3, 1, 5, 1 | 2, 2, 0;
    page one keeps tokens 2 and 0, page two keeps 4 and 5 (tie: earlier)."""
    Ck = np.zeros((7, 1))
    Cv = np.array([[3.0], [1.0], [-5.0], [1.0], [2.0], [-2.0], [0.0]])
    A = np.zeros((1, 1))
    vals, kept = orc.amortised_value_codes(Ck, Cv, A, keep=2, page=4)
    assert kept.tolist() == [True, False, True, False, True, True, False]
    assert vals[:, 0].tolist() == [3.0, 0.0, -5.0, 0.0, 2.0, -2.0, 0.0]


def test_amortised_values_with_every_residual_kept_are_the_value_codes():
    rng = np.random.default_rng(602)
    Ck, Cv = rng.standard_normal((150, 16)), rng.standard_normal((150, 8))
    A = orc.fit_value_predictor(Ck, Cv)
    vals, kept = orc.amortised_value_codes(Ck, Cv, A, keep=64)
    assert kept.all() and np.max(np.abs(vals - Cv)) < 1e-12


def test_amortised_cache_attends_over_predicted_values_plus_kept_residuals():
    """An amortised cache reads the value code A^T c_k + kept residual; the
    predictor is fitted over the prompt and applies to later evictions."""
    rng = np.random.default_rng(603)
    P = rng.standard_normal((1, 1, D, 16)) * 0.2
    k, v = rng.standard_normal((1, 1, 200, D)), rng.standard_normal((1, 1, 200, D))
    c = orc.LatentCacheOracle(1, 1, 16, 16, n_sink=1, window=8, value_keep=16)
    c.append(k[:, :, :150], v[:, :, :150], P, P)
    c.amortise()
    n0 = c.codes_k[0][0].shape[0]
    A = orc.fit_value_predictor(c.codes_k[0][0], c.codes_v[0][0])
    c.append(k[:, :, 150:], v[:, :, 150:], P, P)          # evictions after the fit
    assert np.array_equal(c.A[0][0], A) and c.codes_k[0][0].shape[0] > n0
    vals, kept = orc.amortised_value_codes(c.codes_k[0][0], c.codes_v[0][0], A, 16)
    q = rng.standard_normal((1, 1, D))
    Ka, Va = c.anchors(0, 0)
    ref = orc.latent_attention(q[0, 0], P[0, 0], P[0, 0], c.codes_k[0][0], vals, Ka, Va, 0.1)
    assert np.max(np.abs(c.attend(q, P, P, 0.1)[0, 0] - ref)) < 1e-14 * np.max(np.abs(ref))
    assert kept.sum() == sum(min(16, len(range(p, min(p + 64, len(kept)))))
                             for p in range(0, len(kept), 64))

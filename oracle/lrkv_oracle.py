"""Float64 CPU oracle of the low-rank latent KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may call it.  It shares no code with the CUDA library; the only thing
both sides share is the seeded input module, which holds no arithmetic of
the method.

What it computes, and where the pages state it:

* Codes.  Each token's post-RoPE key and its value (128 dims per KV head)
  are projected per (layer, head) to r-dim codes, c = P^T x, and only the
  codes are stored (Half the Memory, section 04).
* Latent attention.  Attention can run directly on the codes instead of on
  reconstructed tensors; the two are algebraically the same (Half the
  Memory, section 08): with q~ = P_k^T q, s_t = q~ . c_k,t * scale and
  o = P_v sum_t softmax(s)_t c_v,t.  The scale is 1/sqrt(128), the original
  head dim (the pages do not state it; latent == reconstructed requires it).
* Anchors.  The first token and the most recent tokens stay full-rank and
  all intermediate tokens are compressed (OjaKV page, the question on which
  tokens to compress, and its bullet list).  Anchors join the same softmax
  with full-rank scores q . k * scale and add p_t v_t to the output.
* Window dynamics (the pages leave them open; plain reading): a fixed window
  of the W most recent tokens; the token that leaves it is compressed with
  the basis current at that moment and never re-encoded.
* Oja.  The basis adapts online with Oja's rule for online PCA, during the
  prompt and periodically during decoding (OjaKV page, the question on
  online subspace adaptation): for each token x in order, y = P^T x and
  P <- P + eta (x - P y) y^T; after every qr_every-th token P is replaced by
  the Q factor of its QR decomposition with diag(R) > 0.

Every pin that checks this file lives in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import collections
import ctypes
import os
from typing import Optional

import numpy as np

HEAD_DIM = 128


# ---------------------------------------------------------------- basics

def project(P: np.ndarray, X: np.ndarray) -> np.ndarray:
    """Codes of the rows of X [n, 128] under basis P [128, r]: rows of X P.

    Half the Memory, section 04: project each 128-dim vector to r dims and
    store the small r-dim code.
    """
    return np.asarray(X, np.float64) @ np.asarray(P, np.float64)


def reconstruct(P: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Rank-r reconstruction C P^T of codes C [n, r] (section 04's
    'reconstruct on the fly'; also the Palu abstract)."""
    return np.asarray(C, np.float64) @ np.asarray(P, np.float64).T


def rebase_codes(P_old: np.ndarray, P_new: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Codes C [n, r] stored under basis P_old, re-expressed under P_new.

    The pages adapt the basis online (OjaKV page, the question on online
    subspace adaptation) but leave open what happens to codes stored under
    the old basis.  Plain reading: a stored code stands for its rank-r
    reconstruction x^ = P_old c (section 04's reconstruction), and re-basing
    gives that vector's code in the new basis, c' = P_new^T x^; for an
    orthonormal P_new this is the least-squares code of x^.  Written as the
    two steps, reconstruct then project.
    """
    return project(P_new, reconstruct(P_old, C))


def svd_basis(X: np.ndarray, r: int) -> np.ndarray:
    """Top-r right singular vectors of X [n, 128] as columns [128, r]
    (Half the Memory, section 05: plain SVD projections)."""
    _, _, vt = np.linalg.svd(np.asarray(X, np.float64), full_matrices=False)
    return vt[:r].T.copy()


def softmax(s: np.ndarray) -> np.ndarray:
    """Softmax of a score vector with max subtraction."""
    s = np.asarray(s, np.float64)
    if s.size == 0:
        return s.copy()
    e = np.exp(s - s.max())
    return e / e.sum()


def dense_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray,
                    scale: float) -> np.ndarray:
    """One head of ordinary attention: softmax(K q * scale)^T V."""
    p = softmax(np.asarray(K, np.float64) @ np.asarray(q, np.float64) * scale)
    return p @ np.asarray(V, np.float64)


def latent_attention(q, P_k, P_v, C_k, C_v, K_anc, V_anc, scale):
    """One q head attending over latent codes plus full-rank anchors.

    q~ = P_k^T q; latent scores q~ . c_k * scale, anchor scores q . k * scale;
    one softmax over the union; o = P_v (sum p_t c_v,t) + sum p_a v_a.
    (Half the Memory, section 08; anchors: OjaKV page.)
    """
    q = np.asarray(q, np.float64)
    C_k = np.asarray(C_k, np.float64).reshape(-1, np.shape(P_k)[1])
    C_v = np.asarray(C_v, np.float64).reshape(-1, np.shape(P_v)[1])
    K_anc = np.asarray(K_anc, np.float64).reshape(-1, HEAD_DIM)
    V_anc = np.asarray(V_anc, np.float64).reshape(-1, HEAD_DIM)
    q_lat = np.asarray(P_k, np.float64).T @ q
    s = np.concatenate([C_k @ q_lat * scale, K_anc @ q * scale])
    if s.size == 0:
        return np.zeros(HEAD_DIM)
    p = softmax(s)
    n = C_k.shape[0]
    return np.asarray(P_v, np.float64) @ (p[:n] @ C_v) + p[n:] @ V_anc


def reconstructed_attention(q, P_k, P_v, C_k, C_v, K_anc, V_anc, scale):
    """The same head attending over reconstructed tensors (the form the
    latent one is algebraically equal to, section 08)."""
    K = np.concatenate([reconstruct(P_k, np.reshape(C_k, (-1, np.shape(P_k)[1]))),
                        np.reshape(K_anc, (-1, HEAD_DIM))])
    V = np.concatenate([reconstruct(P_v, np.reshape(C_v, (-1, np.shape(P_v)[1]))),
                        np.reshape(V_anc, (-1, HEAD_DIM))])
    if K.shape[0] == 0:
        return np.zeros(HEAD_DIM)
    return dense_attention(q, K, V, scale)


# ---------------------------------------------------------------- cache

def _basis_of(P: np.ndarray, b: int, h: int) -> np.ndarray:
    """P is [Bp, H_kv, 128, r] with Bp == 1 (shared) or Bp == B."""
    P = np.asarray(P)
    return np.asarray(P[0 if P.shape[0] == 1 else b, h], np.float64)


class LatentCacheOracle:
    """Per-sequence hybrid cache: sink, full-rank window, latent codes.

    Tokens arrive in order.  With n_sink == 1 the first token of a sequence
    is the sink.  Every later token enters the window of the W most recent
    tokens; when the window overflows, its oldest token is projected with
    the basis passed to that append and joins the latent codes (OjaKV page:
    first and most recent tokens full-rank, the rest compressed).
    """

    def __init__(self, B: int, H_kv: int, r_k: int, r_v: int,
                 n_sink: int = 0, window: int = 0):
        self.B, self.H_kv, self.r_k, self.r_v = B, H_kv, r_k, r_v
        self.n_sink, self.W = n_sink, window
        self.seq_len = [0] * B
        self.sink_k = [[] for _ in range(B)]   # list of [H_kv, 128]
        self.sink_v = [[] for _ in range(B)]
        self.win_k = [collections.deque() for _ in range(B)]
        self.win_v = [collections.deque() for _ in range(B)]
        self.codes_k = [[np.zeros((0, r_k)) for _ in range(H_kv)] for _ in range(B)]
        self.codes_v = [[np.zeros((0, r_v)) for _ in range(H_kv)] for _ in range(B)]

    def append(self, k: np.ndarray, v: np.ndarray, P_k: np.ndarray,
               P_v: np.ndarray) -> None:
        """Append n tokens per sequence; k, v are [B, H_kv, n, 128]."""
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        for b in range(self.B):
            evict_k, evict_v = [], []
            for t in range(k.shape[2]):
                kt, vt = k[b, :, t, :], v[b, :, t, :]
                if len(self.sink_k[b]) < self.n_sink:
                    self.sink_k[b].append(kt)
                    self.sink_v[b].append(vt)
                else:
                    self.win_k[b].append(kt)
                    self.win_v[b].append(vt)
                    if len(self.win_k[b]) > self.W:
                        evict_k.append(self.win_k[b].popleft())
                        evict_v.append(self.win_v[b].popleft())
                self.seq_len[b] += 1
            if evict_k:
                ek, ev = np.stack(evict_k, 1), np.stack(evict_v, 1)  # [H, n, 128]
                for h in range(self.H_kv):
                    self.codes_k[b][h] = np.concatenate(
                        [self.codes_k[b][h], project(_basis_of(P_k, b, h), ek[h])])
                    self.codes_v[b][h] = np.concatenate(
                        [self.codes_v[b][h], project(_basis_of(P_v, b, h), ev[h])])

    def rebase(self, P_k_old, P_k_new, P_v_old, P_v_new) -> None:
        """Re-express every stored code under the new bases (rebase_codes);
        a pair given as None leaves that side's codes as they are."""
        for b in range(self.B):
            for h in range(self.H_kv):
                if P_k_old is not None:
                    self.codes_k[b][h] = rebase_codes(_basis_of(P_k_old, b, h),
                                                      _basis_of(P_k_new, b, h),
                                                      self.codes_k[b][h])
                if P_v_old is not None:
                    self.codes_v[b][h] = rebase_codes(_basis_of(P_v_old, b, h),
                                                      _basis_of(P_v_new, b, h),
                                                      self.codes_v[b][h])

    def anchors(self, b: int, h: int):
        """Full-rank anchor rows (sink first, then window oldest first)."""
        ks = [x[h] for x in self.sink_k[b]] + [x[h] for x in self.win_k[b]]
        vs = [x[h] for x in self.sink_v[b]] + [x[h] for x in self.win_v[b]]
        if not ks:
            return np.zeros((0, HEAD_DIM)), np.zeros((0, HEAD_DIM))
        return np.stack(ks), np.stack(vs)

    def attend(self, q: np.ndarray, P_k: np.ndarray, P_v: np.ndarray,
               scale: float) -> np.ndarray:
        """Decode attention of q [B, H_q, 128] over the cache (GQA: q head h
        reads KV head h // (H_q / H_kv))."""
        q = np.asarray(q, np.float64)
        B, H_q, _ = q.shape
        G = H_q // self.H_kv
        o = np.zeros((B, H_q, HEAD_DIM))
        for b in range(B):
            for h in range(H_q):
                g = h // G
                Ka, Va = self.anchors(b, g)
                o[b, h] = latent_attention(
                    q[b, h], _basis_of(P_k, b, g), _basis_of(P_v, b, g),
                    self.codes_k[b][g], self.codes_v[b][g], Ka, Va, scale)
        return o


def partition(seq_len: int, n_sink: int, window: int):
    """Token indices of (sink, latent, window) for a sequence of seq_len
    tokens under the fixed-window reading of the OjaKV anchors."""
    sink = list(range(min(seq_len, n_sink)))
    rest = seq_len - len(sink)
    n_win = min(rest, window)
    latent = list(range(len(sink), seq_len - n_win))
    win = list(range(seq_len - n_win, seq_len))
    return sink, latent, win


def decode_from_parts(q, P_k, P_v, C_k, C_v, K_anc, V_anc, G, scale):
    """Decode output [B, H_q, 128] from explicit per-(b, kv head) parts.

    C_k[b][g] etc. are arrays; used to decode a cache whose codes were
    produced elsewhere (the oracle then checks attention alone).
    """
    q = np.asarray(q, np.float64)
    B, H_q, _ = q.shape
    o = np.zeros((B, H_q, HEAD_DIM))
    for b in range(B):
        for h in range(H_q):
            g = h // G
            o[b, h] = latent_attention(q[b, h], _basis_of(P_k, b, g),
                                       _basis_of(P_v, b, g), C_k[b][g],
                                       C_v[b][g], K_anc[b][g], V_anc[b][g], scale)
    return o


# ---------------------------------------------------------------- Oja

def qr_positive(P: np.ndarray) -> np.ndarray:
    """Q factor of the thin QR of P with the signs chosen so diag(R) > 0."""
    Q, R = np.linalg.qr(np.asarray(P, np.float64))
    d = np.sign(np.diag(R))
    d[d == 0] = 1.0
    return Q * d[None, :]


def oja_update(P: np.ndarray, X: np.ndarray, eta: float, qr_every: int,
               tokens_seen: int = 0) -> np.ndarray:
    """Sequential Oja subspace rule over the rows of X (OjaKV page).

    For each token x in order: y = P^T x; P <- P + eta (x - P y) y^T.  When
    the running token count (tokens_seen + j + 1) is a multiple of qr_every,
    P is re-orthonormalised by QR with diag(R) > 0.  Returns a new array.
    """
    P = np.array(P, np.float64, copy=True)
    X = np.asarray(X, np.float64)
    for j in range(X.shape[0]):
        x = X[j]
        y = P.T @ x
        P += eta * np.outer(x - P @ y, y)
        if qr_every > 0 and (tokens_seen + j + 1) % qr_every == 0:
            P = qr_positive(P)
    return P


_OJA_LIB = None


def _oja_lib():
    global _OJA_LIB
    if _OJA_LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_oja_ref.so")
        if not os.path.exists(path):
            from . import build_oracle
            build_oracle.build()
        lib = ctypes.CDLL(path)
        lib.oja_ref_f64.restype = None
        lib.oja_ref_f64.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_long]
        lib.oja_ref_threads.restype = ctypes.c_int
        _OJA_LIB = lib
    return _OJA_LIB


def oja_update_streams(P: np.ndarray, X: np.ndarray, eta: float,
                       qr_every: int, tokens_seen: int = 0) -> np.ndarray:
    """The same rule as oja_update for S independent streams at once, run by
    the plain-C float64 loop in oja_ref.c (OpenMP over streams).

    P: [S, 128, r]; X: [S, n, 128] (any float dtype; converted to float32,
    which holds bf16 and fp32 inputs exactly).  Returns float64 [S, 128, r].
    """
    P = np.ascontiguousarray(P, np.float64).copy()
    X = np.ascontiguousarray(X, np.float32)
    S, d, r = P.shape
    assert d == HEAD_DIM and X.shape[0] == S and X.shape[2] == HEAD_DIM
    _oja_lib().oja_ref_f64(P.ctypes.data, X.ctypes.data, S, r, X.shape[1],
                           float(eta), int(qr_every), int(tokens_seen))
    return P


def oja_threads() -> int:
    return int(_oja_lib().oja_ref_threads())


# ---------------------------------------------------------------- sizes

def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int,
                   batch: int, bytes_per_elem: int = 2) -> int:
    """Dense KV cache size: K and V for every layer, head, token, sequence
    (the OjaKV page's Llama-3.1-8B figure is this at 32 layers, 8 KV heads,
    128 dims, 32K tokens, batch 4, 2-byte elements)."""
    return 2 * layers * kv_heads * head_dim * tokens * batch * bytes_per_elem


def latent_cache_bytes(layers: int, kv_heads: int, r_k: int, r_v: int,
                       tokens: int, batch: int, bytes_per_elem: int = 2) -> int:
    """Durable size of a cache holding only r_k + r_v dim codes per token and
    head (Half the Memory, section 08: halved at every context length at 2x)."""
    return layers * kv_heads * (r_k + r_v) * tokens * batch * bytes_per_elem


def compression_ratio(r_k: int, r_v: int, head_dim: int = HEAD_DIM) -> float:
    """Dense-to-latent byte ratio per token and head: 2 d / (r_k + r_v)."""
    return 2.0 * head_dim / (r_k + r_v)

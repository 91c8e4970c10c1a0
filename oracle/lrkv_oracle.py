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
* Value amortisation (the LowRAM abstract: within a head values are largely
  predictable from their keys; a light per-head predictor is fitted at test
  time and residuals are stored only for the tokens it reconstructs worst).
  The pages give no predictor form or selection rule; the plain reading
  taken here, in the codes' space: per (sequence, KV head) a linear map A
  (r_k x r_v) fitted by least squares over the prompt's latent tokens,
  C_k A ~ C_v; residual e_t = c_v,t - A^T c_k,t; in each 64-token page the
  `keep` tokens with the largest ||e_t|| (ties: the earlier token) keep
  their residual, and attention reads the value code A^T c_k,t (+ e_t).
* Quantised codes.  Low-rank codes compose with quantisation (the Palu
  abstract: quantisation-friendly low-rank codes; the LowRAM abstract: the
  pipeline composes with quantisation).  The pages give no scheme; the plain
  reading taken here is symmetric per-token integer codes: for each stored
  token and side, s = max_j |c_j| / (2^(bits-1) - 1) and q_j = round(c_j / s)
  (round half to even), and attention reads the dequantised code q s.  The
  decision q is an integer decided from floating point, so it is taken in
  fp32, the precision the CUDA path takes it in.

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


def quantize_codes(C: np.ndarray, bits: int = 8):
    """Symmetric per-token integer codes of C [n, r] (one scale per row).

    s = max_j |c_j| / (2^(bits-1) - 1) and q_j = round(c_j / s), round half
    to even, both in fp32 (the quantisation decision is taken in the
    precision of the CUDA path); a row of zeros gets s = 0 and q = 0.
    Returns (q as int8 [n, r], s as float32 [n]).
    """
    qmax = np.float32(2 ** (bits - 1) - 1)
    C32 = np.asarray(C, np.float64).astype(np.float32)
    amax = np.max(np.abs(C32), axis=1) if C32.shape[1] else np.zeros(C32.shape[0], np.float32)
    s = (amax / qmax).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.rint((C32 / safe[:, None]).astype(np.float32))
    q = np.clip(q, -qmax, qmax)
    q[s == 0] = 0
    return q.astype(np.int8), s


def dequantize_codes(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """The codes a quantised row stands for: q_j s, in float64."""
    return np.asarray(q, np.float64) * np.asarray(s, np.float64)[:, None]


def fit_value_predictor(C_k: np.ndarray, C_v: np.ndarray) -> np.ndarray:
    """Least-squares linear predictor of value codes from key codes:
    A = argmin ||C_k A - C_v||_F, shape [r_k, r_v] (LowRAM abstract: a
    lightweight per-head predictor fitted at test time)."""
    return np.linalg.lstsq(np.asarray(C_k, np.float64), np.asarray(C_v, np.float64),
                           rcond=None)[0]


def amortised_value_codes(C_k: np.ndarray, C_v: np.ndarray, A: np.ndarray, keep: int,
                          page: int = 64):
    """Value codes as an amortised cache holds them: the prediction A^T c_k
    for every token, plus the residual c_v - A^T c_k for the `keep` tokens of
    each `page`-token page with the largest residual norm (ties: the earlier
    token).  Returns (value codes [n, r_v], kept mask [n])."""
    C_k = np.asarray(C_k, np.float64)
    C_v = np.asarray(C_v, np.float64)
    pred = C_k @ np.asarray(A, np.float64)
    E = C_v - pred
    norms = np.linalg.norm(E, axis=1)
    kept = np.zeros(C_k.shape[0], bool)
    for p0 in range(0, C_k.shape[0], page):
        idx = sorted(range(p0, min(p0 + page, C_k.shape[0])), key=lambda t: (-norms[t], t))
        kept[idx[:keep]] = True
    return pred + np.where(kept[:, None], E, 0.0), kept


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
                 n_sink: int = 0, window: int = 0, quant_bits: int = 0,
                 value_keep: int = 0):
        self.B, self.H_kv, self.r_k, self.r_v = B, H_kv, r_k, r_v
        self.n_sink, self.W = n_sink, window
        # 0: codes kept as computed; 8: every stored code row is replaced by
        # its dequantised per-token int8 form (quantize_codes)
        self.quant_bits = quant_bits
        # value amortisation: residuals kept per 64-token page once amortise()
        # has fitted the predictors (None until then)
        self.value_keep = value_keep
        self.A = None
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
                        [self.codes_k[b][h], self._stored(project(_basis_of(P_k, b, h), ek[h]))])
                    self.codes_v[b][h] = np.concatenate(
                        [self.codes_v[b][h], self._stored(project(_basis_of(P_v, b, h), ev[h]))])

    def _stored(self, C: np.ndarray) -> np.ndarray:
        """What the cache keeps of freshly computed codes C."""
        if not self.quant_bits:
            return C
        return dequantize_codes(*quantize_codes(C, self.quant_bits))

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

    def amortise(self) -> None:
        """Fit every unit's value predictor over its latent tokens so far
        (the prompt) and from now on attend over amortised value codes
        (fit_value_predictor, amortised_value_codes)."""
        self.A = [[fit_value_predictor(self.codes_k[b][h], self.codes_v[b][h])
                   for h in range(self.H_kv)] for b in range(self.B)]

    def value_codes(self, b: int, h: int) -> np.ndarray:
        """The value codes attention reads for unit (b, h)."""
        if self.A is None:
            return self.codes_v[b][h]
        return amortised_value_codes(self.codes_k[b][h], self.codes_v[b][h], self.A[b][h],
                                     self.value_keep)[0]

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
                    self.codes_k[b][g], self.value_codes(b, g), Ka, Va, scale)
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


def oja_update_blocked(P: np.ndarray, X: np.ndarray, eta: float, qr_every: int,
                       tokens_seen: int = 0, chunk: int = 64) -> np.ndarray:
    """Chunked form of the Oja rule: the tokens are taken in chunks of
    `chunk`, and within a chunk every token's update uses the basis of the
    chunk's start.

    The OjaKV page adapts the basis over the prompt token by token; done so,
    the prompt pass is one long chain of dependent steps.  Freezing P within
    a chunk keeps Oja's per-token update, y = P^T x and (x - P y) y^T, and
    sums it over the chunk, so a chunk is three matrix products:
    Y = X P, Z = X - Y P^T, P <- P + eta Z^T Y.  With chunk = 1 this is the
    sequential rule.  A chunk never straddles a QR point: chunks end where the
    running token count (tokens_seen + tokens so far) reaches a multiple of
    qr_every, and P is then replaced by the Q of its QR with diag(R) > 0.
    Returns a new array.
    """
    P = np.array(P, np.float64, copy=True)
    X = np.asarray(X, np.float64)
    j = 0
    while j < X.shape[0]:
        n = min(chunk, X.shape[0] - j)
        if qr_every > 0:
            n = min(n, qr_every - (tokens_seen + j) % qr_every)
        Xc = X[j:j + n]
        Y = Xc @ P
        Z = Xc - Y @ P.T
        P = P + eta * (Z.T @ Y)
        j += n
        if qr_every > 0 and (tokens_seen + j) % qr_every == 0:
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

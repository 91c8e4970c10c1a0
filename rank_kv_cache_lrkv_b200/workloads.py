"""Seeded synthetic inputs for the latent-KV decode path.

This module only draws and shapes inputs. It holds none of the method's
arithmetic (no projection to codes, no attention, no Oja step), so both the
CUDA path and the float64 oracle can consume exactly the same arrays.

Recipe (shared by every workload):

* Keys of one (layer, sequence, KV head) stream are ``K = Z diag(s) Q`` with
  ``Z ~ N(0, 1)`` of shape [n, 128], ``s_i = exp(-i/16)`` and ``Q`` a seeded
  Haar-random orthogonal 128x128 matrix (QR of a Gaussian, columns signed so
  that diag(R) > 0).  Values are built the same way with ``s_i = exp(-i/8)``
  and an independent ``Q``.  ``Q`` is per (layer, KV head) and is shared by
  every sequence and by the calibration draw: it stands for that head's
  statistics.
* Keys are rotated with RoPE (rotate-half pairing of dims i and i+64,
  inverse frequency theta^(-2i/128)) at their token position when the
  workload names a theta; the library always receives post-RoPE keys
  ("keys compressed after RoPE", Half the Memory, section 04).
* Queries are ``q ~ N(0, 1/128)`` per (sequence, q head, decode step), rotated
  at the position of the token being decoded.
* The projection basis is an input to the library.  For SVD workloads it is
  the top-r right singular vectors of a separate seeded calibration draw of
  the same head ("plain SVD projections, the top-r directions of each head's
  statistics", Half the Memory, section 05); for the Oja workload it is a
  seeded random orthonormal matrix.
* bf16 workloads round K, V and q to bf16 (round to nearest even) before
  either side sees them; fp32 workloads round them to fp32.

Workload shapes follow the pages' models: a Qwen3-1.7B-shaped layer
(H_q=16, H_kv=8, d=128) and a Llama-3.1-8B-shaped layer (H_q=32, H_kv=8).
The pages' accuracy numbers come from a private simulator that is not
available; these seeded draws stand in for its activations.
"""
from __future__ import annotations

import dataclasses
import functools
from typing import Optional

import numpy as np

HEAD_DIM = 128

# Seed-sequence tags: every random draw is keyed by
# (workload id, tag, layer, sequence, kv head).
TAG_QK = 1        # orthogonal Q of the key stream
TAG_QV = 2        # orthogonal Q of the value stream
TAG_ZK = 3        # key noise
TAG_ZV = 4        # value noise
TAG_CAL_K = 5     # calibration draw for the key basis
TAG_CAL_V = 6     # calibration draw for the value basis
TAG_QUERY = 7     # decode queries
TAG_BASIS_K = 8   # random orthonormal initial key basis
TAG_BASIS_V = 9   # random orthonormal initial value basis
TAG_PAGES = 10    # permutation of the page pool (block table)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, ranks, anchors and schedule."""

    name: str
    wid: int                 # seed namespace
    B: int
    H_q: int
    H_kv: int
    T: int                   # prompt tokens
    r_k: int
    r_v: int
    dtype: str               # 'f32' or 'bf16': K/V/q/codes/anchors/o
    rope_theta: Optional[float] = None
    n_sink: int = 0          # full-rank first token (0 or 1)
    window: int = 0          # full-rank most recent tokens
    n_decode: int = 1        # decode steps after the prompt
    n_cal: int = 2048        # calibration tokens for the SVD basis
    basis: str = "svd"       # 'svd' or 'random'
    layers: int = 1
    oja_eta: float = 0.0
    oja_qr_every: int = 0
    oja_decode_every: int = 0
    prefill_oja: bool = False
    append_before_attend: bool = True   # decode token joins the cache first
    seq0: int = 0            # global index of sequence 0 (a replica's shard)

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(HEAD_DIM))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads, named for what they are.
TINY_SINGLE_HEAD = Workload(
    name="tiny_single_head_fp32", wid=0, B=1, H_q=4, H_kv=1, T=512,
    r_k=64, r_v=32, dtype="f32", n_decode=1, n_cal=2048,
    append_before_attend=False)
QWEN3_LAYER_8K = Workload(
    name="qwen3_1.7b_layer_T8192", wid=1, B=4, H_q=16, H_kv=8, T=8192,
    r_k=64, r_v=32, dtype="bf16", rope_theta=1e6, n_decode=64, n_cal=4096)
LLAMA31_LAYER_32K_ANCHORS = Workload(
    name="llama3.1_8b_layer_T32768_anchors", wid=2, B=4, H_q=32, H_kv=8,
    T=32768, r_k=64, r_v=32, dtype="bf16", rope_theta=5e5, n_sink=1,
    window=128, n_decode=64, n_cal=4096)


def qwen3_sweep_point(r_k: int, r_v: int, B: int) -> Workload:
    """One point of the rank x batch sweep on a Qwen3-1.7B-shaped layer."""
    return Workload(
        name=f"qwen3_1.7b_layer_T16384_rk{r_k}_rv{r_v}_B{B}", wid=3, B=B,
        H_q=16, H_kv=8, T=16384, r_k=r_k, r_v=r_v, dtype="bf16",
        rope_theta=1e6, n_decode=8, n_cal=4096)


SWEEP_RANKS = [(96, 64), (96, 32), (64, 64), (64, 32), (32, 64), (32, 32)]
SWEEP_BATCHES = [1, 8, 32, 64]

QWEN3_STACK_OJA = Workload(
    name="qwen3_1.7b_28layer_T32768_oja", wid=4, B=2, H_q=16, H_kv=8,
    T=32768, r_k=48, r_v=48, dtype="bf16", rope_theta=1e6, n_decode=128,
    basis="random", layers=28, oja_eta=1e-3, oja_qr_every=256,
    oja_decode_every=512, prefill_oja=True)

# Small variant of the Oja workload whose decode-time update fires: the basis
# of every (sequence, KV head) is adapted over the prompt, then every 32
# generated tokens over those 32 tokens, with a QR every 64 tokens seen.
# Sink + window anchors make evictions cross basis updates.  The rate is
# larger than the stack's 1e-3 so that a 32-token update moves the basis
# visibly (eta * |x|^2 stays below 0.2, well inside Oja's stable range).
QWEN3_DECODE_OJA_SMALL = Workload(
    name="qwen3_1.7b_layer_T512_decode_oja32", wid=5, B=2, H_q=8, H_kv=2,
    T=512, r_k=32, r_v=32, dtype="bf16", rope_theta=1e6, n_sink=1, window=32,
    n_decode=96, basis="random", oja_eta=2e-2, oja_qr_every=64,
    oja_decode_every=32, prefill_oja=True)

ALL = {w.name: w for w in [TINY_SINGLE_HEAD, QWEN3_LAYER_8K,
                           LLAMA31_LAYER_32K_ANCHORS, QWEN3_STACK_OJA]}


# ---------------------------------------------------------------- draws

def _rng(wl: Workload, tag: int, layer: int = 0, b: int = 0, h: int = 0):
    return np.random.default_rng(
        np.random.SeedSequence([wl.wid, tag, layer, b, h, 0x1a2b]))


def haar_orthogonal(rng: np.random.Generator, n: int = HEAD_DIM) -> np.ndarray:
    """Haar-random orthogonal matrix: QR of a Gaussian with diag(R) > 0."""
    a = rng.standard_normal((n, n))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def spectrum(kind: str) -> np.ndarray:
    """Singular-value profile s_i of the synthetic key/value generator."""
    i = np.arange(HEAD_DIM, dtype=np.float64)
    return np.exp(-i / (16.0 if kind == "k" else 8.0))


@functools.lru_cache(maxsize=8)
def _rope_table(n: int, theta: float):
    half = HEAD_DIM // 2
    inv_freq = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / HEAD_DIM)
    ang = np.arange(n, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang), np.sin(ang)


def rope_rotate(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE of rows of x [n, 128] at integer positions [n]."""
    half = HEAD_DIM // 2
    positions = np.asarray(positions)
    if positions.ndim == 1 and len(positions) and np.array_equal(
            positions, np.arange(len(positions))):
        cos, sin = _rope_table(len(positions), float(theta))
    else:
        inv_freq = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / HEAD_DIM)
        ang = positions.astype(np.float64)[:, None] * inv_freq[None, :]
        cos, sin = np.cos(ang), np.sin(ang)
    x1, x2 = x[:, :half], x[:, half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=1)


def head_q(wl: Workload, kind: str, layer: int, kvh: int) -> np.ndarray:
    return haar_orthogonal(_rng(wl, TAG_QK if kind == "k" else TAG_QV, layer, 0, kvh))


def stream(wl: Workload, kind: str, layer: int, b: int, kvh: int,
           n: Optional[int] = None, Q: Optional[np.ndarray] = None) -> np.ndarray:
    """Float64 key ('k') or value ('v') rows of one stream, tokens 0..n-1.

    The stream always draws T + n_decode rows so that token t is the same
    whatever prefix is asked for.  Keys are post-RoPE when theta is set.
    """
    total = wl.T + wl.n_decode
    n = total if n is None else n
    if Q is None:
        Q = head_q(wl, kind, layer, kvh)
    z = _rng(wl, TAG_ZK if kind == "k" else TAG_ZV, layer, wl.seq0 + b, kvh).standard_normal(
        (total, HEAD_DIM))[:n]
    x = (z * spectrum(kind)[None, :]) @ Q
    if kind == "k" and wl.rope_theta is not None:
        x = rope_rotate(x, np.arange(n), wl.rope_theta)
    return x


def calibration_draw(wl: Workload, kind: str, layer: int, kvh: int,
                     Q: Optional[np.ndarray] = None) -> np.ndarray:
    """Separate seeded draw of n_cal tokens of one head (post-RoPE keys)."""
    if Q is None:
        Q = head_q(wl, kind, layer, kvh)
    z = _rng(wl, TAG_CAL_K if kind == "k" else TAG_CAL_V, layer, 0, kvh
             ).standard_normal((wl.n_cal, HEAD_DIM))
    x = (z * spectrum(kind)[None, :]) @ Q
    if kind == "k" and wl.rope_theta is not None:
        x = rope_rotate(x, np.arange(wl.n_cal), wl.rope_theta)
    return x


def basis(wl: Workload, kind: str, layer: int, kvh: int) -> np.ndarray:
    """Input basis [128, r] in fp32 for one (layer, KV head)."""
    r = wl.r_k if kind == "k" else wl.r_v
    if wl.basis == "random":
        g = _rng(wl, TAG_BASIS_K if kind == "k" else TAG_BASIS_V, layer, 0, kvh)
        return haar_orthogonal(g)[:, :r].astype(np.float32)
    x = calibration_draw(wl, kind, layer, kvh)
    _, _, vt = np.linalg.svd(x, full_matrices=False)
    return np.ascontiguousarray(vt[:r].T).astype(np.float32)


def queries(wl: Workload, layer: int, step: int) -> np.ndarray:
    """Float64 queries [B, H_q, 128] for decode step `step` (post-RoPE)."""
    q = np.empty((wl.B, wl.H_q, HEAD_DIM))
    pos = wl.T + step if wl.append_before_attend else wl.T
    for b in range(wl.B):
        g = _rng(wl, TAG_QUERY, layer, wl.seq0 + b, step)
        qb = g.standard_normal((wl.H_q, HEAD_DIM)) / np.sqrt(HEAD_DIM)
        if wl.rope_theta is not None:
            qb = rope_rotate(qb, np.full(wl.H_q, pos), wl.rope_theta)
        q[b] = qb
    return q


def page_permutation(wl: Workload, num_pages: int) -> np.ndarray:
    """Seeded permutation used to scatter sequences over the page pool."""
    return _rng(wl, TAG_PAGES).permutation(num_pages).astype(np.int32)


# ---------------------------------------------------------------- rounding

def round_to(x: np.ndarray, dtype: str):
    """Round float64 values to the workload dtype.

    Returns (torch tensor in that dtype on CPU, float64 numpy of the rounded
    values).  bf16 rounding is round-to-nearest-even (torch's cast).
    """
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t, t.to(torch.float64).numpy()


def layer_inputs(wl: Workload, layer: int = 0, threads: Optional[int] = None):
    """All K/V streams of one layer, rounded to the workload dtype.

    Returns dict with torch CPU tensors K, V [B, H_kv, T + n_decode, 128] in
    the workload dtype, and fp32 bases P_k [H_kv, 128, r_k], P_v.  Streams are
    drawn in parallel threads; each stream's values depend only on its seed.
    """
    import concurrent.futures
    import os
    import torch
    total = wl.T + wl.n_decode
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    K = torch.empty((wl.B, wl.H_kv, total, HEAD_DIM), dtype=tdt)
    V = torch.empty_like(K)
    Pk = np.empty((wl.H_kv, HEAD_DIM, wl.r_k), np.float32)
    Pv = np.empty((wl.H_kv, HEAD_DIM, wl.r_v), np.float32)
    Qs = {(kind, h): head_q(wl, kind, layer, h) for kind in "kv" for h in range(wl.H_kv)}
    if wl.rope_theta is not None:
        _rope_table(total, float(wl.rope_theta))

    def one(job):
        kind, b, h = job
        dst = K if kind == "k" else V
        dst[b, h] = round_to(stream(wl, kind, layer, b, h, Q=Qs[(kind, h)]), wl.dtype)[0]

    def bases(h):
        Pk[h] = basis(wl, "k", layer, h)
        Pv[h] = basis(wl, "v", layer, h)

    jobs = [(kind, b, h) for kind in "kv" for b in range(wl.B) for h in range(wl.H_kv)]
    n = threads or min(16, os.cpu_count() or 4)
    with concurrent.futures.ThreadPoolExecutor(n) as ex:
        list(ex.map(one, jobs))
        list(ex.map(bases, range(wl.H_kv)))
    return {"K": K, "V": V, "P_k": torch.from_numpy(Pk), "P_v": torch.from_numpy(Pv)}


def layer_queries(wl: Workload, layer: int = 0):
    """Rounded queries for every decode step: [n_decode, B, H_q, 128]."""
    import torch
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    out = torch.empty((wl.n_decode, wl.B, wl.H_q, HEAD_DIM), dtype=tdt)
    for s in range(wl.n_decode):
        out[s] = round_to(queries(wl, layer, s), wl.dtype)[0]
    return out

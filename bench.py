"""Decode benchmark of the latent-KV cache (one process per GPU).

Workload (default): the Llama-3.1-8B-shaped layer with hybrid anchors,
B=4, H_q=32, H_kv=8, d=128, 32K-token prompt, token 0 and the 128 most
recent tokens full-rank bf16, all other tokens r_k=64 / r_v=32 bf16 codes.
A step is one decode step of every sequence: lrkv_compress of the new token
(window append + eviction of the oldest window token into codes) and
lrkv_decode_attn (q-fold, split-K over the codes and anchors, merge with the
value up-projection).

Prints one JSON line (rank 0).  `value` is decode tokens/s over all ranks
(B * steps * N / max-over-ranks time, device time with CUDA events around a
CUDA graph of the timed steps).  Extra keys: the lrkv_decode_attn roofline
(algorithmic bytes: codes + anchors + q + o), the dense bf16 decode baseline
measured in the same run, an end-to-end number through the Python API with
host buffers, the oracle on the host cores, and SM clocks sampled during the
timed region.

--impl reference runs the float64 oracle (the only reference this method
has) on the host cores instead.
"""
import argparse
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEAD_DIM = 128


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=256)
    p.add_argument("--warmup", type=int, default=8)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="llama32k", choices=["llama32k", "qwen8k"])
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--context", type=int, default=0,
                   help="override the prompt length (small cases for profiler captures)")
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-oja", action="store_true",
                   help="skip the Oja-update timing of the 28-layer stack")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the other workloads (tiny, Qwen3 8K, the rank x batch sweep, "
                        "the 28-layer stack)")
    p.add_argument("--profile", type=int, default=0,
                   help="profiling run: prefill, then this many eager decode steps "
                        "(append + decode attention) and one re-basing, no timing and no "
                        "JSON line")
    return p.parse_args()


def workload(name):
    from rank_kv_cache_lrkv_b200 import workloads as wk
    return {"llama32k": wk.LLAMA31_LAYER_32K_ANCHORS, "qwen8k": wk.QWEN3_LAYER_8K}[name]


def config_of(wl):
    return {"workload": wl.name, "B": wl.B, "H_q": wl.H_q, "H_kv": wl.H_kv, "head_dim": HEAD_DIM,
            "T": wl.T, "r_k": wl.r_k, "r_v": wl.r_v, "n_sink": wl.n_sink, "window": wl.window,
            "codes": wl.dtype, "accumulate": "fp32",
            "l2": "no flush: every decode step streams the whole code cache, larger than L2"}


def step_bytes(wl, L):
    """Algorithmic bytes of one decode-attention call at sequence length L:
    latent codes + full-rank anchors + q + o (bf16)."""
    es = 2 if wl.dtype == "bf16" else 4
    sink = min(L, wl.n_sink)
    win = min(L - sink, wl.window)
    lat = L - sink - win
    units = wl.B * wl.H_kv
    return (units * lat * (wl.r_k + wl.r_v) * es + units * (sink + win) * 2 * HEAD_DIM * es
            + 2 * wl.B * wl.H_q * HEAD_DIM * es)


# DRAM bytes (read + write) of one decode-attention call (q-fold + split +
# merge), summed from an ncu capture of `bench.py --profile 6`
# (dram__bytes_read.sum + dram__bytes_write.sum per launch).  Valid only while
# the decode sources hash to the recorded values; scaled to the bench's
# context by the algorithmic bytes.
TRAFFIC = {
    # ncu, one split_kernel launch with cold caches (1 pass):
    # dram__bytes_read.sum + dram__bytes_write.sum
    "llama3.1_8b_layer_T32768_anchors": {
        "bytes": 206470000, "context": 32771,
        "sources": {"decode.cu": "a5708206b9e5ec2d4f59d747935ec2f2276c7f63e0d2a388568107ff63295215",
                    "common.cuh": "867648f72ac4bef6638f39474ad2af8cef852d6f55e4d265fffd4c7212795edf"},
    },
}
# The same kernel with caches left as the previous launch left them (ncu
# --cache-control none, one pass): what a replayed call reads from DRAM.
TRAFFIC_WARM = {
    "llama3.1_8b_layer_T32768_anchors": {
        "bytes": 199030000, "context": 32773,
        "sources": {"decode.cu": "a5708206b9e5ec2d4f59d747935ec2f2276c7f63e0d2a388568107ff63295215",
                    "common.cuh": "867648f72ac4bef6638f39474ad2af8cef852d6f55e4d265fffd4c7212795edf"},
    },
}


def measured_traffic(wl, L, table=None):
    import hashlib
    rec = (TRAFFIC if table is None else table).get(wl.name)
    if rec is None:
        return None
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rank_kv_cache_lrkv_b200", "csrc")
    for f, h in rec["sources"].items():
        with open(os.path.join(csrc, f), "rb") as fh:
            if hashlib.sha256(fh.read()).hexdigest() != h:
                return None
    return int(round(rec["bytes"] * step_bytes(wl, L) / step_bytes(wl, rec["context"])))


def time_oja(lrkv, dev, world):
    """Prefill Oja update of the 28-layer Qwen3 stack: every (layer, sequence,
    KV head) key and value stream (2 * 28 * 2 * 8 = 896 streams) over the
    32,768-token prompt, r = 48, eta = 1e-3, QR every 256 tokens, in one call.
    The update is sequential per stream, so this is latency-bound: wall time
    and stream steps per second.  Rows are drawn on the device (Gaussian
    with the key spectrum exp(-i/16) under a random rotation, in bf16); the
    cost does not depend on the values."""
    import torch
    from rank_kv_cache_lrkv_b200 import replicas
    from rank_kv_cache_lrkv_b200 import workloads as wk
    wl = wk.QWEN3_STACK_OJA
    S, n, r = 2 * wl.layers * wl.B * wl.H_kv, wl.T, wl.r_k
    g = torch.Generator(device=dev)
    g.manual_seed(4242)
    Q, _ = torch.linalg.qr(torch.randn(HEAD_DIM, HEAD_DIM, device=dev, generator=g))
    spec = torch.exp(-torch.arange(HEAD_DIM, device=dev, dtype=torch.float32) / 16.0)
    x = torch.empty(S, n, HEAD_DIM, device=dev, dtype=torch.bfloat16)
    for s0 in range(0, S, 32):
        z = torch.randn(min(32, S - s0), n, HEAD_DIM, device=dev, generator=g)
        x[s0:s0 + 32] = ((z * spec) @ Q).to(torch.bfloat16)
        del z
    P0, _ = torch.linalg.qr(torch.randn(S, HEAD_DIM, r, device=dev, generator=g))
    P = P0.contiguous()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lrkv.oja_update(P[:4].clone(), x[:4, :512], wl.oja_eta, wl.oja_qr_every, 0)  # warm-up
    torch.cuda.synchronize()
    e0.record()
    lrkv.oja_update(P, x, wl.oja_eta, wl.oja_qr_every, 0)
    e1.record()
    torch.cuda.synchronize()
    ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    ok = bool(torch.isfinite(P).all().item())
    # the chunked form (P frozen within 64-token chunks) on the same rows
    Pc = P0.clone().contiguous()
    lrkv.oja_update_chunked(Pc[:4].clone(), x[:4, :512], wl.oja_eta, wl.oja_qr_every, 0, 64)
    torch.cuda.synchronize()
    e0.record()
    lrkv.oja_update_chunked(Pc, x, wl.oja_eta, wl.oja_qr_every, 0, 64)
    e1.record()
    torch.cuda.synchronize()
    cms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    # how far the chunked bases are from the sequential ones (projector gap)
    gap = float(torch.linalg.matrix_norm(P @ P.transpose(1, 2) - Pc @ Pc.transpose(1, 2),
                                         ord=2).max().item())
    del x, P, P0, Pc
    torch.cuda.empty_cache()
    return {"workload": wl.name, "streams": S, "tokens_per_stream": n, "rank": r,
            "eta": wl.oja_eta, "qr_every": wl.oja_qr_every, "ms": round(ms, 3),
            "stream_steps_per_s": round(S * n / (ms * 1e-3), 1),
            "us_per_token_step": round(ms * 1e3 / n, 4), "finite": ok,
            "chunked": {"chunk": 64, "ms": round(cms, 3), "speedup": round(ms / cms, 2),
                        "max_projector_gap_to_sequential": round(gap, 6)}}


def device_kv(dev, g, B, H_kv, n, dtype):
    """Timing inputs drawn on the device: keys and values [B, H_kv, n, 128]
    with the workload recipe's spectra (exp(-i/16) keys, exp(-i/8) values)
    under a random rotation per KV head.  Decode and compress time do not
    depend on the values; parity is tested on the oracle's own draws."""
    import torch
    out = []
    for decay in (16.0, 8.0):
        spec = torch.exp(-torch.arange(HEAD_DIM, device=dev, dtype=torch.float32) / decay)
        Q = torch.linalg.qr(torch.randn(H_kv, HEAD_DIM, HEAD_DIM, device=dev, generator=g))[0]
        x = torch.empty((B, H_kv, n, HEAD_DIM), device=dev, dtype=dtype)
        for b in range(B):
            z = torch.randn((H_kv, n, HEAD_DIM), device=dev, generator=g)
            x[b] = torch.bmm(z * spec, Q).to(dtype)
            del z
        out.append(x)
    return out


def device_basis(dev, g, lead, r):
    """Random orthonormal bases [*lead, 128, r] in fp32."""
    import torch
    z = torch.randn(tuple(lead) + (HEAD_DIM, r), device=dev, generator=g)
    return torch.linalg.qr(z)[0].contiguous()


def time_layer_decode(lrkv, dev, wl, steps, calls, world, clk, seed):
    """One layer of workload wl on device draws: prefill compress, then
    `steps` decode steps (append + decode attention) captured in a CUDA graph
    and timed, then `calls` decode-attention calls alone (the roofline)."""
    import torch
    from rank_kv_cache_lrkv_b200 import replicas
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    n = wl.T + steps + 1
    Kd, Vd = device_kv(dev, g, wl.B, wl.H_kv, n, dt)
    Pk, Pv = device_basis(dev, g, (wl.H_kv,), wl.r_k), device_basis(dev, g, (wl.H_kv,), wl.r_v)
    qs = (torch.randn((steps + 1, wl.B, wl.H_q, HEAD_DIM), device=dev, generator=g)
          / HEAD_DIM ** 0.5).to(dt)
    cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, n, wl.n_sink, wl.window, dtype=dt,
                             device=dev)
    lrkv.compress(cache, Kd[:, :, :wl.T], Vd[:, :, :wl.T], Pk, Pv)
    ws = lrkv.decode_workspace(cache, wl.H_q, device=dev)
    o = torch.empty_like(qs[0])

    def step(s):
        t = wl.T + s
        lrkv.compress(cache, Kd[:, :, t:t + 1], Vd[:, :, t:t + 1], Pk, Pv)
        lrkv.decode_attn(cache, qs[s], Pk, Pv, wl.scale, o, ws)

    step(0)  # warm: module loading, attributes
    torch.cuda.synchronize()
    gs = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gs, capture_error_mode="relaxed"):
        for s in range(1, steps + 1):
            step(s)
    saved = cache.seq_len.clone()
    gs.replay()
    torch.cuda.synchronize()
    cache.seq_len.copy_(saved)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        gs.replay()
        e1.record()
        torch.cuda.synchronize()
    ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    ga = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ga, capture_error_mode="relaxed"):
        for _ in range(calls):
            lrkv.decode_attn(cache, qs[0], Pk, Pv, wl.scale, o, ws)
    ga.replay()
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        ga.replay()
        e1.record()
        torch.cuda.synchronize()
    attn_ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev) / calls
    assert lrkv.workspace_error(ws) == 0
    L = wl.T + steps + 1
    nbytes = step_bytes(wl, L)
    del gs, ga, cache, Kd, Vd
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(wl.B * steps * world / (ms * 1e-3), 1),
            "us_per_step": round(ms * 1e3 / steps, 3),
            "attn_us": round(attn_ms * 1e3, 3), "bytes_per_call": nbytes,
            "attn_GBs": round(nbytes / (attn_ms * 1e-3) / 1e9, 1), "context": L}


def time_code_variants(lrkv, dev, world, clk, hbm, wl, calls):
    """Decode attention over the same Llama-3.1-8B-shaped layer with per-token
    int8 codes and with value amortisation (key codes + 16 residual slots per
    page, predictors fitted over the prompt): microseconds per call, the
    bytes one call streams, and the fraction of the measured copy peak."""
    import torch
    from rank_kv_cache_lrkv_b200 import replicas
    g = torch.Generator(device=dev)
    g.manual_seed(99)
    n = wl.T + 2
    Kd, Vd = device_kv(dev, g, wl.B, wl.H_kv, n, torch.bfloat16)
    Pk, Pv = device_basis(dev, g, (wl.H_kv,), wl.r_k), device_basis(dev, g, (wl.H_kv,), wl.r_v)
    q = (torch.randn((wl.B, wl.H_q, HEAD_DIM), device=dev, generator=g) / HEAD_DIM ** 0.5).to(
        torch.bfloat16)
    o = torch.empty_like(q)
    L = wl.T + 1
    sink = min(L, wl.n_sink)
    win = min(L - sink, wl.window)
    lat = L - sink - win
    units = wl.B * wl.H_kv
    pages = -(-lat // 64)
    anchors = units * (sink + win) * 2 * HEAD_DIM * 2 + 2 * wl.B * wl.H_q * HEAD_DIM * 2
    out = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for name in ("int8_codes", "amortised_values"):
        cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, n, wl.n_sink, wl.window,
                                 device=dev, **{name: True})
        lrkv.compress(cache, Kd[:, :, :wl.T], Vd[:, :, :wl.T], Pk, Pv)
        ws = lrkv.decode_workspace(cache, wl.H_q, device=dev)
        if name == "amortised_values":
            A = torch.zeros(wl.B, wl.H_kv, wl.r_k, wl.r_v, device=dev)
            lrkv.amortise(cache, Vd[:, :, :wl.T], Pv, A)
            lrkv.compress_amortised(cache, Kd[:, :, wl.T:L], Vd[:, :, wl.T:L], Pk, Pv, A)
            call = lambda: lrkv.decode_attn_amortised(cache, q, Pk, Pv, A, wl.scale, o, ws)
            slab = 64 * wl.r_k * 2 + 16 * wl.r_v * 2 + 128
        else:
            lrkv.compress(cache, Kd[:, :, wl.T:L], Vd[:, :, wl.T:L], Pk, Pv)
            call = lambda: lrkv.decode_attn(cache, q, Pk, Pv, wl.scale, o, ws)
            slab = 64 * (wl.r_k + wl.r_v) + 512
        call()
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, capture_error_mode="relaxed"):
            for _ in range(calls):
                call()
        gr.replay()
        torch.cuda.synchronize()
        with clk.region():
            e0.record()
            gr.replay()
            e1.record()
            torch.cuda.synchronize()
        us = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev) * 1e3 / calls
        assert lrkv.workspace_error(ws) == 0
        nbytes = units * pages * slab + anchors
        out[name] = {"attn_us": round(us, 3), "bytes_per_call": nbytes,
                     "attn_GBs": round(nbytes / (us * 1e-6) / 1e9, 1),
                     "frac": round(nbytes / (us * 1e-6) / 1e9 / hbm, 4),
                     "page_slab_bytes": slab,
                     "bf16_page_slab_bytes": 64 * (wl.r_k + wl.r_v) * 2}
        del gr, cache
    del Kd, Vd
    torch.cuda.empty_cache()
    out["workload"] = wl.name
    out["inputs"] = "device draws with the recipe's spectra; random orthonormal bases"
    return out


def time_sweep(lrkv, dev, world, clk, hbm, steps, calls):
    """Rank x batch sweep on the Qwen3-1.7B-shaped layer at T=16384: decode
    tokens/s and the roofline fraction of decode attention per point."""
    from rank_kv_cache_lrkv_b200 import workloads as wk
    pts = []
    for B in wk.SWEEP_BATCHES:
        for r_k, r_v in wk.SWEEP_RANKS:
            wl = wk.qwen3_sweep_point(r_k, r_v, B)
            res = time_layer_decode(lrkv, dev, wl, steps, calls, world, clk,
                                    seed=1000 + 7 * B + r_k + r_v)
            res.update({"B": B, "r_k": r_k, "r_v": r_v,
                        "frac": round(res["attn_GBs"] / hbm, 4)})
            pts.append(res)
    return {"workload": "qwen3_1.7b_layer_T16384 rank x batch sweep", "T": 16384, "H_q": 16,
            "H_kv": 8, "steps": steps, "calls": calls,
            "inputs": "device draws with the recipe's spectra; random orthonormal bases",
            "points": pts}


def time_stack(lrkv, dev, world, clk, steps):
    """The 28-layer Qwen3-1.7B-shaped stack (B=2, T=32768, r 48/48, bases per
    sequence): decode tokens/s over all layers (a step appends one token and
    attends at every layer), then one decode-time basis update of the whole
    stack: Oja over 512 generated tokens for every (layer, K|V, sequence, KV
    head) stream (896 streams) followed by re-basing every layer's codes."""
    import torch
    from rank_kv_cache_lrkv_b200 import replicas
    from rank_kv_cache_lrkv_b200 import workloads as wk
    wl = wk.QWEN3_STACK_OJA
    B, H, r, T, Lyr = wl.B, wl.H_kv, wl.r_k, wl.T, wl.layers
    g = torch.Generator(device=dev)
    g.manual_seed(2828)
    P = device_basis(dev, g, (Lyr, 2, B, H), r)        # [layer][K|V][b][h][128][r]
    bs = H * HEAD_DIM * r
    caches, news = [], []
    for layer in range(Lyr):
        Kd, Vd = device_kv(dev, g, B, H, T + steps + 1, torch.bfloat16)
        c = lrkv.LatentCache(B, H, r, r, T + steps + 1, dtype=torch.bfloat16, device=dev)
        lrkv.compress(c, Kd[:, :, :T], Vd[:, :, :T], P[layer, 0], P[layer, 1],
                      basis_batch_stride=bs)
        caches.append(c)
        news.append((Kd[:, :, T:].clone(), Vd[:, :, T:].clone()))
        del Kd, Vd
    qs = (torch.randn((steps + 1, Lyr, B, wl.H_q, HEAD_DIM), device=dev, generator=g)
          / HEAD_DIM ** 0.5).to(torch.bfloat16)
    ws = [lrkv.decode_workspace(c, wl.H_q, device=dev) for c in caches]
    o = torch.empty_like(qs[0, 0])

    def step(s):
        for layer in range(Lyr):
            kn, vn = news[layer]
            lrkv.compress(caches[layer], kn[:, :, s:s + 1], vn[:, :, s:s + 1], P[layer, 0],
                          P[layer, 1], basis_batch_stride=bs)
            lrkv.decode_attn(caches[layer], qs[s, layer], P[layer, 0], P[layer, 1], wl.scale, o,
                             ws[layer], basis_batch_stride=bs)

    step(0)
    torch.cuda.synchronize()
    gs = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gs, capture_error_mode="relaxed"):
        for s in range(1, steps + 1):
            step(s)
    saved = [c.seq_len.clone() for c in caches]
    gs.replay()
    torch.cuda.synchronize()
    for c, sv in zip(caches, saved):
        c.seq_len.copy_(sv)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        gs.replay()
        e1.record()
        torch.cuda.synchronize()
    ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    assert all(lrkv.workspace_error(w) == 0 for w in ws)
    del gs
    stack_bytes = Lyr * step_bytes(wl, T + steps + 1)
    out = {"workload": wl.name, "layers": Lyr, "B": B, "T": T, "r_k": r, "r_v": r,
           "steps": steps, "tokens_per_s": round(B * steps * world / (ms * 1e-3), 1),
           "us_per_step": round(ms * 1e3 / steps, 2),
           "GBs_per_step": round(stack_bytes / (ms * 1e-3 / steps) / 1e9, 1)}
    # decode-time update of the whole stack (eta 1e-3, QR every 256, tokens
    # counted on from the prompt), then every layer's codes re-based
    n_upd = wl.oja_decode_every
    S = Lyr * 2 * B * H
    x = torch.empty((S, n_upd, HEAD_DIM), device=dev, dtype=torch.bfloat16)
    for s0 in range(0, S, 64):
        x[s0:s0 + 64] = device_kv(dev, g, 1, min(64, S - s0), n_upd, torch.bfloat16)[0][0]
    Pflat = P.view(S, HEAD_DIM, r)
    rws = [lrkv.rebase_workspace(c, device=dev) for c in caches]
    P_old = torch.empty_like(P)

    def update():
        P_old.copy_(P)
        lrkv.oja_update(Pflat, x, wl.oja_eta, wl.oja_qr_every, T)
        for layer in range(Lyr):
            lrkv.rebase(caches[layer], P_old[layer, 0], P[layer, 0], P_old[layer, 1],
                        P[layer, 1], rws[layer], basis_batch_stride=bs)

    update()  # warm
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        update()
        e1.record()
        torch.cuda.synchronize()
    ums = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    assert all(lrkv.workspace_error(w) == 0 for w in rws)
    out["decode_oja"] = {"streams": S, "tokens": n_upd, "rank": r, "ms": round(ums, 3),
                         "note": "Oja over the last 512 generated tokens of every stream, "
                                 "then lrkv_rebase of all 28 layers; once per 512 steps",
                         "share_of_512_steps": round(ums / (512 * ms / steps), 4)}
    del caches, news, x, P, P_old
    torch.cuda.empty_cache()
    return out


def dense_step_bytes(wl, L):
    es = 2 if wl.dtype == "bf16" else 4
    return wl.B * wl.H_kv * L * 2 * HEAD_DIM * es + 2 * wl.B * wl.H_q * HEAD_DIM * es


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls NVML (the library nvidia-smi reads) for SM clock and throttle
    reasons while the timed region runs."""

    def __init__(self, index=0, period=0.002):
        self.samples, self.period, self.index = [], period, index
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        self.active = False     # set around each timed region
        self.regions = 0
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            if self.active:
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    if self.active:
                        self.samples.append((mhz, rs))
                except Exception:
                    pass
            time.sleep(self.period)

    def region(self):
        """Context manager marking one timed region (sampled while open)."""
        clk = self

        class _Region:
            def __enter__(self_inner):
                clk.active = True
                clk.regions += 1

            def __exit__(self_inner, *a):
                clk.active = False
        return _Region()

    def __enter__(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        nv = self.nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        mhz = sorted(s[0] for s in self.samples)
        seen = set()
        for _, rs in self.samples:
            for n, bit in names.items():
                if rs & bit and n != "gpu_idle":
                    seen.add(n)
        return {"sm_mhz": mhz[len(mhz) // 2] if mhz else None, "sm_max_mhz": self.max_mhz,
                "samples": len(mhz), "timed_regions": self.regions, "reasons": sorted(seen),
                "note": "NVML polled every 2 ms while any timed region of this run was open"}


# ------------------------------------------------------------------ oracle
class OracleUnit:
    """The float64 oracle on one (sequence, KV head) unit of the workload:
    its prompt is compressed once; a decode step appends one token and
    attends with the unit's G query heads."""

    def __init__(self, wl, inp):
        import numpy as np
        from oracle import lrkv_oracle as orc
        self.np, self.wl = np, wl
        self.Pk = inp["P_k"][0:1].double().numpy()[None]
        self.Pv = inp["P_v"][0:1].double().numpy()[None]
        self.K = inp["K"][0:1, 0:1].double().numpy()
        self.V = inp["V"][0:1, 0:1].double().numpy()
        self.oc = orc.LatentCacheOracle(1, 1, wl.r_k, wl.r_v, wl.n_sink, wl.window)
        self.oc.append(self.K[:, :, :wl.T], self.V[:, :, :wl.T], self.Pk, self.Pv)
        self.rng = np.random.default_rng(0)
        self.n = 0

    def run(self, seconds):
        """Decode steps for about `seconds`; returns (steps, seconds per step)."""
        wl, np = self.wl, self.np
        n, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < seconds or n == 0:
            t = wl.T + (self.n % (self.K.shape[2] - wl.T))
            self.oc.append(self.K[:, :, t:t + 1], self.V[:, :, t:t + 1], self.Pk, self.Pv)
            q = self.rng.standard_normal((1, wl.G, HEAD_DIM)) / np.sqrt(HEAD_DIM)
            self.oc.attend(q, self.Pk, self.Pv, wl.scale)
            n += 1
            self.n += 1
        return n, (time.perf_counter() - t0) / n


def host_cores():
    try:
        import threadpoolctl
        return max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_text(wl, n):
    units = wl.B * wl.H_kv
    return (f"{n} float64 oracle decode steps (append + attend) of 1 of the {units} "
            f"(sequence, KV head) units at {wl.T}-token context; a full step is taken "
            f"as {units} x the unit time")


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist
    from rank_kv_cache_lrkv_b200 import lrkv
    from rank_kv_cache_lrkv_b200 import replicas
    from rank_kv_cache_lrkv_b200 import workloads as wk

    base = workload(args.workload)
    if args.context:
        base = base.with_(T=args.context)
    W, K = args.warmup, args.steps
    E = 0 if args.no_e2e else min(K, 64)
    # this rank's own B sequences (weak scaling; no data-path collective)
    wl = replicas.shard(base.with_(n_decode=W + K + E + 2), rank, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = wk.layer_inputs(wl)
    qs = wk.layer_queries(wl).to(dev)
    Kd, Vd = inp["K"].to(dev), inp["V"].to(dev)
    Pk, Pv = inp["P_k"].to(dev), inp["P_v"].to(dev)
    cap = wl.T + wl.n_decode
    cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, cap, wl.n_sink, wl.window,
                             dtype=Kd.dtype, device=dev)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(dev.index)
    clk.__enter__()
    # warm the prefill kernels (module loading) on a small cache first
    small = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, 1024, wl.n_sink, wl.window,
                             dtype=Kd.dtype, device=dev)
    lrkv.compress(small, Kd[:, :, :1024], Vd[:, :, :1024], Pk, Pv)
    torch.cuda.synchronize()
    del small
    with clk.region():
        e0.record()
        lrkv.compress(cache, Kd[:, :, :wl.T], Vd[:, :, :wl.T], Pk, Pv)
        e1.record()
        torch.cuda.synchronize()
    # eager: includes the host's launch work (tensor maps, launches) between the events
    prefill_eager_ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    # device time: the same call replayed from a CUDA graph into the emptied cache
    cache.seq_len.zero_()
    gp = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gp, capture_error_mode="relaxed"):
        lrkv.compress(cache, Kd[:, :, :wl.T], Vd[:, :, :wl.T], Pk, Pv)
    cache.seq_len.zero_()
    gp.replay()
    torch.cuda.synchronize()
    cache.seq_len.zero_()
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        gp.replay()
        e1.record()
        torch.cuda.synchronize()
    prefill_ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    del gp
    # prefill bytes: K and V rows read, codes and anchors written
    n_lat = wl.T - wl.n_sink - wl.window
    prefill_bytes = (wl.B * wl.H_kv * wl.T * 2 * 128 * Kd.element_size()
                     + wl.B * wl.H_kv * n_lat * (wl.r_k + wl.r_v) * Kd.element_size()
                     + wl.B * wl.H_kv * (wl.n_sink + wl.window) * 2 * 128 * Kd.element_size())
    ws = lrkv.decode_workspace(cache, wl.H_q, device=dev)
    o = torch.empty_like(qs[0])

    def step(s, fused=False):
        t = wl.T + s
        if fused:  # lrkv_decode_step: append + query fold, split-K, merge
            lrkv.decode_step(cache, Kd[:, :, t:t + 1], Vd[:, :, t:t + 1], qs[s], Pk, Pv,
                             wl.scale, o, ws)
        else:      # two calls: append; q-fold, split-K, merge
            lrkv.compress(cache, Kd[:, :, t:t + 1], Vd[:, :, t:t + 1], Pk, Pv)
            lrkv.decode_attn(cache, qs[s], Pk, Pv, wl.scale, o, ws)

    if args.profile:
        for s in range(min(args.profile, wl.n_decode)):
            step(s)
        # one re-basing onto a rotated basis of the same span (a profiler
        # selects it by kernel name)
        g = torch.Generator().manual_seed(7)
        Qk = torch.linalg.qr(torch.randn(wl.r_k, wl.r_k, generator=g, dtype=torch.float64))[0]
        Pk2 = (Pk.double() @ Qk.to(dev)).float().contiguous()
        rb_ws = lrkv.rebase_workspace(cache, device=dev)
        lrkv.rebase(cache, Pk, Pk2, Pv, Pv, rb_ws)
        # a chunked and a sequential Oja update, 64 streams x 2048 tokens, r 48
        g2 = torch.Generator(device=dev)
        g2.manual_seed(11)
        xo = (torch.randn(64, 2048, HEAD_DIM, device=dev, generator=g2) * 0.3).to(torch.bfloat16)
        Po = torch.linalg.qr(torch.randn(64, HEAD_DIM, 48, device=dev, generator=g2))[0]
        lrkv.oja_update_chunked(Po.contiguous(), xo, 1e-3, 256, 0, 64)
        lrkv.oja_update(Po.contiguous(), xo, 1e-3, 256, 0)
        torch.cuda.synchronize()
        assert lrkv.workspace_error(ws) == 0 and lrkv.workspace_error(rb_ws) == 0
        clk.__exit__()
        print(f"profile run: {wl.name}, prefill + {args.profile} decode steps, one re-basing, "
              "a chunked and a sequential Oja update")
        return None

    for s in range(W):
        step(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        for s in range(W, W + K):
            step(s)
    torch.cuda.synchronize()
    # One untimed replay uploads the graph; restoring seq_len makes the timed
    # replay append the same tokens into the same slots and pages again.
    saved_len = cache.seq_len.clone()
    g.replay()
    torch.cuda.synchronize()
    cache.seq_len.copy_(saved_len)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
    ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    if world > 1:
        dist.barrier()
    assert lrkv.workspace_error(ws) == 0
    # the same steps through lrkv_decode_step, for comparison
    g1 = torch.cuda.CUDAGraph()
    cache.seq_len.copy_(saved_len)
    with torch.cuda.graph(g1, capture_error_mode="relaxed"):
        for s in range(W, W + K):
            step(s, fused=True)
    cache.seq_len.copy_(saved_len)
    g1.replay()
    torch.cuda.synchronize()
    cache.seq_len.copy_(saved_len)
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        g1.replay()
        e1.record()
        torch.cuda.synchronize()
    ms_two = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    del g1

    # roofline of lrkv_decode_attn alone: the same call replayed (state fixed)
    R = 200
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, capture_error_mode="relaxed"):
        for _ in range(R):
            lrkv.decode_attn(cache, qs[0], Pk, Pv, wl.scale, o, ws)
    g2.replay()
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        g2.replay()
        e1.record()
        torch.cuda.synchronize()
    attn_ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev) / R
    L_now = wl.T + W + K
    abytes = step_bytes(wl, L_now)

    # lrkv_rebase over the whole cache, timed as round trips to bases of the
    # same span and back (the cache holds equivalent codes afterwards)
    rb_ws = lrkv.rebase_workspace(cache, device=dev)
    gq = torch.Generator().manual_seed(7)

    def rotated(P):
        Q = torch.linalg.qr(torch.randn(P.shape[-1], P.shape[-1], generator=gq,
                                        dtype=torch.float64))[0]
        return (P.double() @ Q.to(P.device)).float().contiguous()

    Pk2, Pv2 = rotated(Pk), rotated(Pv)
    RB = 4
    lrkv.rebase(cache, Pk, Pk2, Pv, Pv2, rb_ws)
    lrkv.rebase(cache, Pk2, Pk, Pv2, Pv, rb_ws)
    torch.cuda.synchronize()
    with clk.region():
        e0.record()
        for rep in range(RB):
            lrkv.rebase(cache, Pk, Pk2, Pv, Pv2, rb_ws)
            lrkv.rebase(cache, Pk2, Pk, Pv2, Pv, rb_ws)
        e1.record()
        torch.cuda.synchronize()
    assert lrkv.workspace_error(rb_ws) == 0
    rb_ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev) / (2 * RB)
    es = 2 if wl.dtype == "bf16" else 4
    n_lat = max(0, L_now - wl.n_sink - wl.window)
    rb_bytes = 2 * wl.B * wl.H_kv * n_lat * (wl.r_k + wl.r_v) * es
    pk = peaks()
    hbm = pk["hbm_gbs"] if pk else 6650.0
    achieved = abytes / (attn_ms * 1e-3) / 1e9
    out = {
        "metric": "latent-KV decode tokens/s and achieved HBM GB/s (fraction of ~8 TB/s) at 1 GPU",
        "value": round(replicas.aggregate_tokens_per_s(wl.B, K, world, ms), 2),
        "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": dict(config_of(wl), parallelism=f"replicas{world}",
                       step="lrkv_compress then lrkv_decode_attn (append; q-fold, split-K, "
                            "merge)"),
        "gpu_launches": 4 * K,
        "decode_step_call": {"ms_per_step": round(ms_two / K, 5),
                             "tokens_per_s": round(replicas.aggregate_tokens_per_s(
                                 wl.B, K, world, ms_two), 2),
                             "note": "the same steps through lrkv_decode_step (3 launches: "
                                     "append + query fold, split-K, merge); e2e uses this call"},
        "roofline": {"kernel": "lrkv_decode_attn (qfold + split + merge)", "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "frac_of_8TBs": round(achieved / 8000, 4),
                     "peak_source": "MEASURED_PEAKS.json hbm_gbs" if pk else "fallback",
                     "bytes_per_call": abytes, "us_per_call": round(attn_ms * 1e3, 3),
                     "context": L_now, "traffic": measured_traffic(wl, L_now),
                     "traffic_warm": measured_traffic(wl, L_now, TRAFFIC_WARM)},
        "prefill_compress": {"tokens": wl.T * wl.B, "ms": round(prefill_ms, 3),
                             "eager_ms": round(prefill_eager_ms, 3),
                             "timing": "CUDA-graph replay (device time); eager_ms adds the "
                                       "host's launch work between the events",
                             "tokens_per_s": round(wl.T * wl.B / (prefill_ms * 1e-3), 1),
                             "bytes": prefill_bytes,
                             "achieved_GBs": round(prefill_bytes / (prefill_ms * 1e-3) / 1e9, 1),
                             "frac": round(prefill_bytes / (prefill_ms * 1e-3) / 1e9 / hbm, 4)},
        "rebase": {"us_per_call": round(rb_ms * 1e3, 2), "bytes_per_call": rb_bytes,
                   "achieved_GBs": round(rb_bytes / (rb_ms * 1e-3) / 1e9, 1),
                   "frac": round(rb_bytes / (rb_ms * 1e-3) / 1e9 / hbm, 4),
                   "note": "every latent code read and written once; per-unit r x r products"},
    }

    if not args.no_oja:
        with clk.region():
            out["oja_update"] = time_oja(lrkv, dev, world)

    if not args.no_dense:
        dc = lrkv.DenseCache(wl.B, wl.H_kv, cap, dtype=Kd.dtype, device=dev)
        lrkv.dense_append(dc, Kd[:, :, :wl.T + W], Vd[:, :, :wl.T + W])
        dws = lrkv.dense_decode_workspace(dc, wl.H_q, device=dev)
        g3 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g3, capture_error_mode="relaxed"):
            for s in range(W, W + K):
                t = wl.T + s
                lrkv.dense_append(dc, Kd[:, :, t:t + 1], Vd[:, :, t:t + 1])
                lrkv.dense_decode_attn(dc, qs[s], wl.scale, o, dws)
        torch.cuda.synchronize()
        with clk.region():
            e0.record()
            g3.replay()
            e1.record()
            torch.cuda.synchronize()
        dms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
        g4 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g4, capture_error_mode="relaxed"):
            for _ in range(R):
                lrkv.dense_decode_attn(dc, qs[0], wl.scale, o, dws)
        g4.replay()
        torch.cuda.synchronize()
        with clk.region():
            e0.record()
            g4.replay()
            e1.record()
            torch.cuda.synchronize()
        dattn = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev) / R
        db = dense_step_bytes(wl, L_now)
        out["dense_baseline"] = {
            "tokens_per_s": round(wl.B * K / (dms * 1e-3), 2), "ms_per_step": round(dms / K, 5),
            "attn_us": round(dattn * 1e3, 3), "attn_GBs": round(db / (dattn * 1e-3) / 1e9, 1),
            "bytes_per_call": db, "speedup_latent_over_dense": round(dms / ms, 3)}
        del dc, g3, g4

    if E:
        # End to end through the public API with host buffers: per step the
        # new k, v and q (packed in one pinned host buffer) are copied to the
        # device in one transfer, and o is read back.
        a0 = wl.T + W + K
        nk = wl.B * wl.H_kv * HEAD_DIM
        nq = wl.B * wl.H_q * HEAD_DIM
        host_in = torch.empty((E, 2 * nk + nq), dtype=Kd.dtype).pin_memory()
        host_in[:, :nk] = inp["K"][:, :, a0:a0 + E].permute(2, 0, 1, 3).reshape(E, nk)
        host_in[:, nk:2 * nk] = inp["V"][:, :, a0:a0 + E].permute(2, 0, 1, 3).reshape(E, nk)
        host_in[:, 2 * nk:] = wk.layer_queries(wl)[W + K:W + K + E].reshape(E, nq)
        oh = torch.empty((E,) + tuple(o.shape), dtype=o.dtype).pin_memory()
        dev_in = torch.empty((2 * nk + nq,), dtype=Kd.dtype, device=dev)
        kd = dev_in[:nk].view(wl.B, wl.H_kv, 1, HEAD_DIM)
        vd = dev_in[nk:2 * nk].view(wl.B, wl.H_kv, 1, HEAD_DIM)
        qd = dev_in[2 * nk:].view(wl.B, wl.H_q, HEAD_DIM)
        torch.cuda.synchronize()
        with clk.region():
            e0.record()
            for s in range(E):
                dev_in.copy_(host_in[s], non_blocking=True)
                lrkv.decode_step(cache, kd, vd, qd, Pk, Pv, wl.scale, o, ws)
                oh[s].copy_(o, non_blocking=True)
            e1.record()
            torch.cuda.synchronize()
        ems = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
        es = Kd.element_size()
        out["e2e"] = {"value": round(replicas.aggregate_tokens_per_s(wl.B, E, world, ems), 2),
                      "unit": "tokens/s",
                      "h2d_bytes_per_step": (2 * nk + nq) * es,
                      "d2h_bytes_per_step": o.numel() * es, "steps": E}

    # the other workloads: decode tokens/s and roofline fraction of each
    if not args.no_workloads:
        S2, C2 = min(max(K, 8), 32), 50
        del g, g2
        torch.cuda.empty_cache()
        extra = {}
        for key, w in (("tiny_single_head_fp32", wk.TINY_SINGLE_HEAD),
                       ("qwen3_1.7b_layer_T8192", wk.QWEN3_LAYER_8K)):
            shard = replicas.shard(w, rank, world)
            res = time_layer_decode(lrkv, dev, shard, S2, C2, world, clk, seed=77)
            res.update({"B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "T": w.T, "r_k": w.r_k,
                        "r_v": w.r_v, "dtype": w.dtype,
                        "frac": round(res["attn_GBs"] / hbm, 4)})
            extra[key] = res
        out["workloads"] = extra
        out["code_variants"] = time_code_variants(lrkv, dev, world, clk, hbm, base, C2)
        out["sweep"] = time_sweep(lrkv, dev, world, clk, hbm, S2, C2)
        out["stack"] = time_stack(lrkv, dev, world, clk, min(max(K, 4), 16))
    clk.__exit__()
    out["clocks"] = clk.summary()
    if rank == 0 and world == 1 and not args.no_cpu:
        n, per_unit = OracleUnit(wl, inp).run(args.cpu_seconds)
        rate = wl.B / (per_unit * wl.B * wl.H_kv)
        out["cpu_baseline"] = {"value": round(rate, 4), "unit": "tokens/s", "cores": host_cores(),
                               "kind": "oracle", "sample": oracle_sample_text(wl, n)}
    return out


def run_reference(args, rank, world):
    """The oracle arm: float64 decode steps on the host cores."""
    from rank_kv_cache_lrkv_b200 import workloads as wk
    base = workload(args.workload)
    K, W = args.steps, args.warmup
    wl = base.with_(n_decode=16)
    # Inputs of one unit suffice for the bounded sample.
    inp = wk.layer_inputs(wl.with_(B=1, H_kv=1, H_q=wl.G))
    unit = OracleUnit(wl, inp)
    per = max(0.2, min(2.0, 120.0 / max(1, K + W)))
    rates, total = [], 0
    for i in range(W + K):
        n, dt = unit.run(per)
        if i >= W:
            rates.append(wl.B / (dt * wl.B * wl.H_kv))
            total += n
    rate = sorted(rates)[len(rates) // 2]
    cores, sample = host_cores(), oracle_sample_text(wl, total)
    step_ms = wl.B / rate * 1e3
    return {"impl": "reference",
            "metric": "latent-KV decode tokens/s and achieved HBM GB/s (fraction of ~8 TB/s) at 1 GPU",
            "value": round(rate, 4), "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": round(step_ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config_of(wl), parallelism="host cores"),
            "cpu_baseline": {"value": round(rate, 4), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(rate, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    import datetime
    import torch
    import torch.distributed as dist
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    try:
        out = run_ours(args, rank, world)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

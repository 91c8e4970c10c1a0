"""The allocation-free decode entry point, checked against the regular one.

lrkv_decode_attn_static is for callers that cannot allocate device memory
or pass a workspace (for example a plugin whose host framework owns every
allocation); it uses scratch compiled into the library instead.  Two decode
steps in a row go through both entry points on the same cache and inputs;
the outputs must agree within the attention-alone tolerance of the other
GPU tests.  This file sorts last so a run that stops at the first failure
has already run every other test.
"""
import numpy as np
import pytest
import torch

from rank_kv_cache_lrkv_b200 import workloads as wk

pytestmark = pytest.mark.gpu

TOL = 5e-3  # attention-alone tolerance for bf16 outputs


def _row_err(a, b):
    a = a.double().cpu().numpy().reshape(-1, 128)
    b = b.double().cpu().numpy().reshape(-1, 128)
    den = np.maximum(np.max(np.abs(b), axis=1), 1e-30)
    return float(np.max(np.max(np.abs(a - b), axis=1) / den))


def test_static_scratch_decode_matches_workspace_decode():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=2, T=700, n_decode=2)
    d = wk.layer_inputs(wl)
    qs = wk.layer_queries(wl)
    cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, wl.T + wl.n_decode, wl.n_sink,
                             wl.window)
    K, V, Pk, Pv = d["K"].cuda(), d["V"].cuda(), d["P_k"].cuda(), d["P_v"].cuda()
    lrkv.compress(cache, K[:, :, :wl.T], V[:, :, :wl.T], Pk, Pv)
    ws = lrkv.decode_workspace(cache, wl.H_q)
    for s in range(2):
        t = wl.T + s
        lrkv.compress(cache, K[:, :, t:t + 1], V[:, :, t:t + 1], Pk, Pv)
        q = qs[s].cuda().contiguous()
        o_ws = torch.empty_like(q)
        o_static = torch.full_like(q, float("nan"))
        lrkv.decode_attn(cache, q, Pk, Pv, wl.scale, o_ws, ws)
        lrkv.decode_attn_static(cache, q, Pk, Pv, wl.scale, o_static)
        torch.cuda.synchronize()
        assert torch.isfinite(o_static).all()
        assert _row_err(o_static, o_ws) <= TOL, s

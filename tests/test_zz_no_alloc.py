"""The allocation-free decode entry point, checked against the regular one.

lrkv_decode_attn_static is for callers that cannot allocate device memory
or pass a workspace (for example a plugin whose host framework owns every
allocation); it uses scratch compiled into the library instead.  Two decode
steps in a row go through both entry points on the same cache and inputs.
Both run the same kernels with the same plan on the same inputs, so their
outputs must be bit-identical (a stale-scratch bug of any size fails).  A
configuration whose scratch would exceed the built-in array must be refused
before anything is launched.  This file sorts last so a run that stops at
the first failure has already run every other test.
"""
import pytest
import torch

from rank_kv_cache_lrkv_b200 import workloads as wk

pytestmark = pytest.mark.gpu

STATIC_BYTES = 4 << 20  # LRKV_STATIC_WORKSPACE_BYTES


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
    assert 0 < lrkv.decode_workspace_bytes(cache, wl.H_q) <= STATIC_BYTES
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
        assert torch.equal(o_static, o_ws), s
    assert lrkv.workspace_error(ws) == 0


def test_static_scratch_refuses_configurations_beyond_its_size():
    """256 sequences x 8 KV heads at ranks 128/128 and 4 q heads per KV head
    need tens of MB of split-K records: the call must raise
    'workspace too small' and leave o untouched."""
    from rank_kv_cache_lrkv_b200 import lrkv
    B, H_kv, H_q, r = 256, 8, 32, 128
    cache = lrkv.LatentCache(B, H_kv, r, r, 64)
    assert lrkv.decode_workspace_bytes(cache, H_q) > STATIC_BYTES
    q = torch.zeros((B, H_q, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, float("nan"))
    Pk = torch.zeros((H_kv, 128, r), dtype=torch.float32, device="cuda")
    with pytest.raises(lrkv.LrkvError) as e:
        lrkv.decode_attn_static(cache, q, Pk, Pk, 0.088, o)
    assert e.value.status == -4
    torch.cuda.synchronize()
    assert torch.isnan(o).all()

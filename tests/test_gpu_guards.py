"""Corrupt block-table entries, injected on the host.

Every kernel range-checks a page id before it touches the page: writes to an
out-of-range page are skipped, and decode and re-basing set error word 2
(a block-table entry out of range) and still return.  The pools here sit
between guard bands of a known byte pattern, so any stray write outside the
pool would show.  Pages the bad entries do not name must hold exactly what a
clean run stores.
"""
import pytest
import torch

from rank_kv_cache_lrkv_b200 import workloads as wk

pytestmark = pytest.mark.gpu

GUARD = 1 << 16     # bytes of canary on each side of a pool
CANARY = 0xA5
ERR_BAD_PAGE = 2


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available()
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _guarded(t: torch.Tensor):
    """A zeroed copy of t's shape and dtype living between two canary bands;
    returns (view, whole byte buffer)."""
    nbytes = t.numel() * t.element_size()
    buf = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device=t.device)
    view = buf[GUARD:GUARD + nbytes].view(t.dtype).view(t.shape)
    view.zero_()
    return view, buf


def _bands_intact(buf: torch.Tensor) -> bool:
    return bool((buf[:GUARD] == CANARY).all() and (buf[-GUARD:] == CANARY).all())


def _guard_latent(cache):
    cache.codes, cbuf = _guarded(cache.codes)
    cache.anchors, abuf = _guarded(cache.anchors)
    cache.desc.codes = cache.codes.data_ptr()
    cache.desc.anchors = cache.anchors.data_ptr()
    return cbuf, abuf


def _run(lrkv, wl, d, qs, bad):
    """Prefill, then two decode steps (append + attention), then a re-basing
    onto rotated bases and one more attention; `bad` maps (b, page index) to
    the id written into the block table before anything runs."""
    cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, wl.T + wl.n_decode, wl.n_sink,
                             wl.window)
    cbuf, abuf = _guard_latent(cache)
    for (b, i), page in bad.items():
        cache.block_table[b, i] = page
    K, V, Pk, Pv = d["K"].cuda(), d["V"].cuda(), d["P_k"].cuda(), d["P_v"].cuda()
    lrkv.compress(cache, K[:, :, :wl.T], V[:, :, :wl.T], Pk, Pv)
    ws = lrkv.decode_workspace(cache, wl.H_q)
    o = torch.empty_like(qs[0]).cuda()
    for s in range(2):
        t = wl.T + s
        lrkv.compress(cache, K[:, :, t:t + 1], V[:, :, t:t + 1], Pk, Pv)
        lrkv.decode_attn(cache, qs[s].cuda().contiguous(), Pk, Pv, wl.scale, o, ws)
    g = torch.Generator().manual_seed(5)
    Q = torch.linalg.qr(torch.randn(wl.r_k, wl.r_k, generator=g, dtype=torch.float64))[0]
    Pk2 = (Pk.double() @ Q.cuda()).float().contiguous()
    rws = lrkv.rebase_workspace(cache)
    lrkv.rebase(cache, Pk, Pk2, None, None, rws)
    lrkv.decode_attn(cache, qs[1].cuda().contiguous(), Pk2, Pv, wl.scale, o, ws)
    torch.cuda.synchronize()
    return cache, cbuf, abuf, lrkv.workspace_error(ws), lrkv.workspace_error(rws)


def test_out_of_range_pages_are_skipped_and_reported(lrkv):
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=3, T=700, n_decode=2, window=64)
    d = wk.layer_inputs(wl)
    qs = wk.layer_queries(wl)
    clean, cbuf0, abuf0, e0, r0 = _run(lrkv, wl, d, qs, {})
    assert (e0, r0) == (0, 0)
    assert _bands_intact(cbuf0) and _bands_intact(abuf0)
    npages = clean.num_pages
    bad = {(1, 2): npages + 7, (2, 0): -3}
    cache, cbuf, abuf, e, r = _run(lrkv, wl, d, qs, bad)
    assert e == ERR_BAD_PAGE and r == ERR_BAD_PAGE
    assert _bands_intact(cbuf), "a write landed outside the code pool"
    assert _bands_intact(abuf), "a write landed outside the anchor tiles"
    # every page no bad entry displaced holds what the clean run stored
    bt = clean.block_table.cpu()
    skipped = {int(bt[b, i]) for (b, i) in bad}
    keep = torch.tensor([p for p in range(npages) if p not in skipped], device="cuda")
    assert torch.equal(cache.codes[keep], clean.codes[keep])
    assert torch.equal(cache.anchors, clean.anchors)


def test_dense_baseline_out_of_range_page_is_reported(lrkv):
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=2, T=200, n_decode=1)
    d = wk.layer_inputs(wl)
    qs = wk.layer_queries(wl)
    dc = lrkv.DenseCache(wl.B, wl.H_kv, wl.T + 1)
    dc.kv_pages, buf = _guarded(dc.kv_pages)
    dc.desc.kv_pages = dc.kv_pages.data_ptr()
    dc.block_table[1, 3] = dc.num_pages + 100
    lrkv.dense_append(dc, d["K"].cuda()[:, :, :wl.T + 1], d["V"].cuda()[:, :, :wl.T + 1])
    ws = lrkv.dense_decode_workspace(dc, wl.H_q)
    o = torch.empty_like(qs[0]).cuda()
    lrkv.dense_decode_attn(dc, qs[0].cuda().contiguous(), wl.scale, o, ws)
    torch.cuda.synchronize()
    assert lrkv.workspace_error(ws) == ERR_BAD_PAGE
    assert _bands_intact(buf)

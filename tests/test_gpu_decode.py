"""GPU parity: the CUDA path through the C ABI against the float64 oracle on
the same seeded inputs.

Tolerances (max over rows of ||o - o_ref||_inf / ||o_ref||_inf):
  * bf16 codes, fp32 accumulation, end to end vs the oracle's float64 codes:
    2e-2 (the stated bar for bf16 codes).
  * fp32 path end to end: 1e-4 (the stated bar for fp32 paths).
  * attention alone (the oracle decodes the GPU's own stored codes and
    anchors): 5e-3 for bf16 outputs (one bf16 rounding of o is 2^-9 of
    ||o||_inf, plus fp32 accumulation) and 2e-5 for fp32.
  * codes: bf16 storage rounds each code to 2^-9 relative; rows are checked
    at 1e-2 of the row's largest code.  fp32 codes at 1e-5.
"""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_lrkv_b200 import workloads as wk
from tests import lrkv_testutil as tu

pytestmark = pytest.mark.gpu

TOL, TOL_ISO, TOL_CODE = tu.TOL, tu.TOL_ISO, tu.TOL_CODE
_run_and_compare = tu.run_and_compare


@pytest.fixture(scope="module")
def lrkv():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def test_tiny_single_head_fp32(lrkv):
    """B=1, H_q=4, H_kv=1, T=512, r 64/32, fp32, one decode step."""
    _run_and_compare(lrkv, wk.TINY_SINGLE_HEAD)


def test_qwen_layer_ragged_prompt(lrkv):
    """Qwen3-1.7B-shaped layer, prompt not a multiple of the page, a few
    decode steps, pages scattered by a permuted block table."""
    wl = wk.QWEN3_LAYER_8K.with_(B=2, T=1000, n_decode=3)
    perm = wk.page_permutation(wl, 2 * ((1003 + 63) // 64))
    _run_and_compare(lrkv, wl, page_perm=torch.from_numpy(perm))


def test_llama_layer_anchors_small(lrkv):
    """Sink + 128-token window + latent middle, evictions at every step."""
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=2, T=700, n_decode=5)
    _run_and_compare(lrkv, wl)


@pytest.mark.parametrize("case", [
    dict(T=1, n_sink=1, window=128),             # only the sink
    dict(T=60, n_sink=1, window=128),            # all anchors, no latent token
    dict(T=130, n_sink=0, window=5),             # window without sink
    dict(T=200, n_sink=1, window=0),             # sink only
    dict(T=65, n_sink=0, window=0),              # one token on a second page
    dict(T=300, H_q=8, H_kv=8),                  # G = 1 (MHA)
    dict(T=300, H_q=64, H_kv=8),                 # G = 8
    dict(T=250, r_k=48, r_v=96),                 # uneven ranks
    dict(T=250, r_k=128, r_v=8),
    dict(T=400, r_k=40, r_v=24),                 # ranks not multiples of 16
    dict(B=37, T=150, window=16),                # more sequences than a warp's lanes
])
def test_edge_cases(lrkv, case):
    kw = dict(B=2, n_decode=2, n_sink=0, window=0)
    kw.update(case)
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(**kw)
    _run_and_compare(lrkv, wl)


def test_prefill_in_chunks_equals_one_shot(lrkv):
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=2, T=900, n_decode=2, window=40)
    _run_and_compare(lrkv, wl, chunks=[1, 15, 300, 7, 577])


def test_full_rank_orthonormal_basis_matches_dense_gpu(lrkv):
    """r = 128 with an orthonormal basis: latent decode equals dense decode
    (Half the Memory, section 04's plumbing check), here in fp32."""
    wl = wk.TINY_SINGLE_HEAD.with_(r_k=128, r_v=128, T=300)
    inp = tu.Inputs(wl)
    Q = torch.from_numpy(np.linalg.qr(np.random.default_rng(0).standard_normal((128, 128)))[0]
                         .astype(np.float32))
    inp.Pk = Q[None].contiguous()
    inp.Pv = Q[None].contiguous()
    _, outs = tu.run_gpu(wl, inp, lrkv=lrkv)
    K, V = inp.K.double().numpy(), inp.V.double().numpy()
    q = inp.q[0].double().numpy()
    ref = np.stack([orc.dense_attention(q[0, h], K[0, 0, :wl.T], V[0, 0, :wl.T], wl.scale)
                    for h in range(wl.H_q)])
    assert tu.row_rel_err(outs[0][0], ref) < 1e-4


def test_ragged_batch_and_empty_sequence(lrkv):
    """Per-sequence append counts: lengths 0, 1, 700, 1300 in one batch."""
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=4, T=1300, n_decode=1)
    inp = tu.Inputs(wl)
    lens = [0, 1, 700, 1300]
    cache = lrkv.LatentCache(wl.B, wl.H_kv, wl.r_k, wl.r_v, wl.T, wl.n_sink, wl.window)
    K, V = inp.K.cuda(), inp.V.cuda()
    Pk, Pv = inp.Pk.cuda(), inp.Pv.cuda()
    n_new = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lrkv.compress(cache, K[:, :, :wl.T], V[:, :, :wl.T], Pk, Pv, n_new=n_new)
    q = inp.q[0].cuda().contiguous()
    o = torch.empty_like(q)
    ws = lrkv.decode_workspace(cache, wl.H_q)
    lrkv.decode_attn(cache, q, Pk, Pv, wl.scale, o, ws)
    assert cache.seq_len.cpu().tolist() == lens
    o = o.double().cpu().numpy()
    assert np.all(o[0] == 0)
    for b in range(1, 4):
        oc = orc.LatentCacheOracle(1, wl.H_kv, wl.r_k, wl.r_v, wl.n_sink, wl.window)
        oc.append(inp.K[b:b + 1, :, :lens[b]].double().numpy(),
                  inp.V[b:b + 1, :, :lens[b]].double().numpy(),
                  inp.Pk.double().numpy()[None], inp.Pv.double().numpy()[None])
        ref = oc.attend(inp.q[0][b:b + 1].double().numpy(), inp.Pk.double().numpy()[None],
                        inp.Pv.double().numpy()[None], wl.scale)
        assert tu.row_rel_err(o[b], ref[0]) < TOL["bf16"], b


def test_workspace_too_small_is_rejected(lrkv):
    wl = wk.QWEN3_LAYER_8K.with_(B=1, T=100)
    cache = lrkv.LatentCache(1, wl.H_kv, 64, 32, 200)
    ws = torch.empty(lrkv.decode_workspace_bytes(cache, wl.H_q) - 256, dtype=torch.uint8,
                     device="cuda")
    q = torch.zeros(1, wl.H_q, 128, dtype=torch.bfloat16, device="cuda")
    P = torch.zeros(wl.H_kv, 128, 64, device="cuda")
    with pytest.raises(lrkv.LrkvError) as e:
        lrkv.decode_attn(cache, q, P, P, 0.1, torch.empty_like(q), ws)
    assert e.value.status == -4


def test_dense_baseline_matches_oracle(lrkv):
    wl = wk.LLAMA31_LAYER_32K_ANCHORS.with_(B=3, T=777, n_decode=1)
    inp = tu.Inputs(wl)
    dc = lrkv.DenseCache(wl.B, wl.H_kv, wl.T + 1,
                         page_perm=torch.from_numpy(wk.page_permutation(wl, 3 * 25)))
    K, V = inp.K.cuda(), inp.V.cuda()
    lrkv.dense_append(dc, K[:, :, :500], V[:, :, :500])
    lrkv.dense_append(dc, K[:, :, 500:778], V[:, :, 500:778])
    q = inp.q[0].cuda().contiguous()
    o = torch.empty_like(q)
    ws = lrkv.dense_decode_workspace(dc, wl.H_q)
    lrkv.dense_decode_attn(dc, q, wl.scale, o, ws)
    o = o.double().cpu().numpy()
    Kn, Vn, qn = inp.K.double().numpy(), inp.V.double().numpy(), inp.q[0].double().numpy()
    ref = np.stack([[orc.dense_attention(qn[b, h], Kn[b, h // wl.G, :778], Vn[b, h // wl.G, :778],
                                         wl.scale) for h in range(wl.H_q)] for b in range(wl.B)])
    assert tu.row_rel_err(o, ref) < 5e-3

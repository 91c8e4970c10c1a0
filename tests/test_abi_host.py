"""The C ABI without a GPU: the library loads, exports every function the
header declares, its structs have the header's layout, and bad arguments
are rejected on the host before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lrkv.h")


@pytest.fixture(scope="module")
def lrkv():
    from rank_kv_cache_lrkv_b200 import lrkv as m
    return m


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lrkv_[a-z_0-9]+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["lrkv_compress", "lrkv_decode_attn", "lrkv_oja_update",
              "lrkv_decode_workspace_bytes", "lrkv_dense_decode_attn", "lrkv_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lrkv):
    lib = ctypes.CDLL(lrkv._LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) <= set(lrkv.EXPORTS) | set(_declared())
    assert lrkv.version() == 100
    assert lrkv.status_string(-4) == "workspace too small"


def test_struct_layout_matches_header(lrkv, tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "lrkv.h"\n'
        'int main(void){printf("%zu %zu %zu %zu %zu\\n", sizeof(lrkv_cache),'
        ' offsetof(lrkv_cache, codes), offsetof(lrkv_cache, append_counter),'
        ' sizeof(lrkv_dense_cache), offsetof(lrkv_dense_cache, append_counter));return 0;}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = list(map(int, subprocess.check_output([str(exe)]).split()))
    C, Dn = lrkv.CacheDesc, lrkv.DenseDesc
    assert got == [ctypes.sizeof(C), C.codes.offset, C.append_counter.offset,
                   ctypes.sizeof(Dn), Dn.append_counter.offset]


def _desc(lrkv, **kw):
    base = dict(batch=2, num_kv_heads=2, head_dim=128, rank_k=64, rank_v=32, dtype=0,
                n_sink=0, window=0, num_pages=4, max_pages_per_seq=2, codes=16,
                block_table=16, anchors=16, seq_len=16, append_counter=16)
    base.update(kw)
    return lrkv.CacheDesc(**base)


FAKE = ctypes.c_void_p(4096)  # never dereferenced: every case fails validation


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, -2), ("rank_k", 12, -2), ("rank_v", 0, -2), ("rank_k", 136, -2),
    ("dtype", 7, -2), ("batch", 0, -1), ("n_sink", 2, -1), ("window", -1, -1),
    ("codes", 0, -1), ("codes", 8, -1), ("num_pages", 0, -1), ("seq_len", 0, -1),
    ("append_counter", 0, -1)])
def test_compress_rejects_bad_cache(lrkv, field, value, status):
    d = _desc(lrkv, **{field: value})
    rc = lrkv._lib.lrkv_compress(ctypes.byref(d), FAKE, FAKE, 4, None, 512, 128, FAKE, FAKE, 0, None)
    assert rc == status


def test_compress_rejects_bad_calls(lrkv):
    d = _desc(lrkv)
    L = lrkv._lib
    assert L.lrkv_compress(None, FAKE, FAKE, 4, None, 0, 0, FAKE, FAKE, 0, None) == -1
    assert L.lrkv_compress(ctypes.byref(d), FAKE, FAKE, -1, None, 0, 0, FAKE, FAKE, 0, None) == -1
    assert L.lrkv_compress(ctypes.byref(d), None, FAKE, 4, None, 0, 0, FAKE, FAKE, 0, None) == -1
    assert L.lrkv_compress(ctypes.byref(d), FAKE, FAKE, 4, None, 0, 0, None, FAKE, 0, None) == -1
    assert L.lrkv_compress(ctypes.byref(d), FAKE, FAKE, 4, None, 0, 0, FAKE, FAKE, -3, None) == -1
    # 2 pages x 64 tokens is the capacity
    assert L.lrkv_compress(ctypes.byref(d), FAKE, FAKE, 129, None, 0, 0, FAKE, FAKE, 0, None) == -3
    # zero tokens is a no-op that launches nothing
    assert L.lrkv_compress(ctypes.byref(d), FAKE, FAKE, 0, None, 0, 0, FAKE, FAKE, 0, None) == 0
    anch = _desc(lrkv, window=4, anchors=0)
    assert L.lrkv_compress(ctypes.byref(anch), FAKE, FAKE, 4, None, 0, 0, FAKE, FAKE, 0, None) == -1


def test_decode_rejects_bad_calls(lrkv):
    d = _desc(lrkv)
    L = lrkv._lib
    args = lambda hq, ws=FAKE, q=FAKE: (ctypes.byref(d), q, hq, FAKE, FAKE, 0, 0.1, FAKE, ws, 1 << 20, None)
    assert L.lrkv_decode_attn(*args(3)) == -1          # H_q % H_kv != 0
    assert L.lrkv_decode_attn(*args(6)) == -2          # G = 3
    assert L.lrkv_decode_attn(*args(32)) == -2         # G = 16
    assert L.lrkv_decode_attn(*args(4, ws=None)) == -1
    assert L.lrkv_decode_attn(*args(4, q=None)) == -1
    assert L.lrkv_decode_attn(*args(4, ws=ctypes.c_void_p(4100))) == -1  # misaligned
    assert L.lrkv_decode_workspace_bytes(ctypes.byref(d), 3) == 0


def test_rebase_rejects_bad_calls(lrkv):
    d = _desc(lrkv)
    L = lrkv._lib
    n = L.lrkv_rebase_workspace_bytes(ctypes.byref(d))
    assert n == 256 + 2 * 2 * (64 * 64 + 32 * 32) * 4  # error word + R^T per unit and side

    def call(pko, pkn, pvo, pvn, ws=FAKE, bs=0, nb=n):
        return L.lrkv_rebase(ctypes.byref(d), pko, pkn, pvo, pvn, bs, ws, nb, None)

    assert call(FAKE, None, None, None) == -1                        # half a pair
    assert call(None, None, None, FAKE) == -1
    assert call(FAKE, FAKE, None, None, ws=None) == -1
    assert call(FAKE, FAKE, None, None, ws=ctypes.c_void_p(4100)) == -1  # misaligned
    assert call(ctypes.c_void_p(4104), FAKE, None, None) == -1         # misaligned basis
    assert call(FAKE, FAKE, None, None, bs=6) == -1                    # stride % 4
    assert call(FAKE, FAKE, FAKE, FAKE, nb=n - 1) == -4                # short workspace
    assert call(None, None, None, None) == 0                           # nothing to re-base
    assert L.lrkv_rebase(None, FAKE, FAKE, None, None, 0, FAKE, n, None) == -1
    assert L.lrkv_rebase_workspace_bytes(ctypes.byref(_desc(lrkv, rank_k=12))) == 0


def test_oja_and_dense_reject_bad_calls(lrkv):
    L = lrkv._lib
    assert L.lrkv_oja_update(None, 1, 8, 1024, FAKE, 0, 0, 4, 0.1, 0, 0, None) == -1
    assert L.lrkv_oja_update(FAKE, 0, 8, 1024, FAKE, 0, 0, 4, 0.1, 0, 0, None) == -1
    assert L.lrkv_oja_update(FAKE, 1, 200, 1 << 20, FAKE, 0, 0, 4, 0.1, 0, 0, None) == -1
    assert L.lrkv_oja_update(FAKE, 2, 8, 100, FAKE, 0, 0, 4, 0.1, 0, 0, None) == -1  # stride < 128 r
    assert L.lrkv_oja_update(FAKE, 1, 8, 1024, FAKE, 5, 0, 4, 0.1, 0, 0, None) == -2
    assert L.lrkv_oja_update(FAKE, 1, 8, 1024, None, 0, 0, 4, 0.1, 0, 0, None) == -1
    assert L.lrkv_oja_update(FAKE, 1, 8, 1024, FAKE, 0, 0, 4, 0.1, -1, 0, None) == -1
    assert L.lrkv_oja_update(FAKE, 1, 8, 1024, None, 0, 0, 0, 0.1, 0, 0, None) == 0
    assert L.lrkv_qr_orthonormalize(FAKE, 1, 0, 1024, None) == -1
    dd = lrkv.DenseDesc(batch=1, num_kv_heads=1, head_dim=100, dtype=0, num_pages=1,
                        max_pages_per_seq=1, kv_pages=16, block_table=16,
                        seq_len=16, append_counter=16)
    assert L.lrkv_dense_append(ctypes.byref(dd), FAKE, FAKE, 1, None, 0, 0, None) == -2
    dd.head_dim = 128
    assert L.lrkv_dense_append(ctypes.byref(dd), FAKE, FAKE, 33, None, 0, 0, None) == -3
    assert L.lrkv_dense_decode_attn(ctypes.byref(dd), FAKE, 3, 0.1, FAKE, FAKE, 1, None) == -2

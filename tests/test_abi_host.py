"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports exactly the entry points declared in include/dsa.h, and
rejects invalid arguments before any CUDA call (these calls launch nothing)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT
from sparse_long_context_03_b200 import build, dsa

HEADER = os.path.join(ROOT, "include", "dsa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
BOGUS = 0x1000  # never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dsa.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^DSA_API\s+[^(]*?\b(dsa_\w+)\(", text, flags=re.M)))


def exported_symbols(path):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    return sorted(line.split()[-1] for line in out.splitlines() if line.split()[-2] in ("T", "W"))


def test_exports_match_header(lib):
    decl = declared_symbols()
    assert len(decl) >= 12
    assert exported_symbols(dsa.LIB_PATH) == decl
    assert sorted(dsa.exported_symbols()) == decl
    for name in decl:
        assert hasattr(lib, name)


def test_version_and_status_strings(lib):
    assert dsa.version() == 100
    assert dsa.status_string(0) == "DSA_OK"
    assert dsa.status_string(5) == "DSA_ERR_TIMEOUT"
    assert dsa.status_string(99) == "DSA_ERR_UNKNOWN"


def test_indexer_rejects_bad_arguments(lib):
    f = lib.dsa_indexer_scores
    good = dict(L=512, HI=4, dI=32, rb=0, n=512, ld=512)

    def call(**kw):
        a = {**good, **kw}
        ptrs = [kw.get("p", BOGUS)] * 5
        return f(*ptrs, a["L"], a["HI"], a["dI"], a["rb"], a["n"], kw.get("out", BOGUS), a["ld"], None, None)

    assert call(HI=3) == UNSUPPORTED
    assert call(dI=48) == UNSUPPORTED
    assert call(n=-1) == INVALID
    assert call(rb=10, n=503) == INVALID       # past L
    assert call(ld=510) == INVALID             # ld < rows
    assert call(ld=514) == INVALID             # ld % 4
    assert call(p=None) == INVALID
    assert call(out=None) == INVALID
    assert call(n=0) == OK                     # empty chunk launches nothing


def test_topk_rejects_bad_arguments(lib):
    f = lib.dsa_topk
    assert f(BOGUS, 512, 0, 512, None, 512, 0, BOGUS, None, None, 0, None) == INVALID   # k < 1
    assert f(BOGUS, 512, 100, 500, None, 512, 64, BOGUS, None, None, 0, None) == INVALID  # rows past max_len
    assert f(BOGUS, 510, 0, 4, BOGUS, 512, 64, BOGUS, None, None, 0, None) == INVALID   # ld < max_len
    assert f(None, 512, 0, 4, BOGUS, 512, 64, BOGUS, None, None, 0, None) == INVALID
    assert f(BOGUS, 512, 0, 0, None, 512, 64, BOGUS, None, None, 0, None) == OK


def test_attention_rejects_bad_arguments(lib):
    f = lib.dsa_sparse_gqa_prefill
    assert f(BOGUS, BOGUS, BOGUS, BOGUS, 0, 8, 32, 5, 128, 64, 0.1, BOGUS, None, None) == UNSUPPORTED  # Hq % Hkv
    assert f(BOGUS, BOGUS, BOGUS, BOGUS, 0, 8, 32, 2, 128, 64, 0.1, BOGUS, None, None) == UNSUPPORTED  # G = 16
    assert f(BOGUS, BOGUS, BOGUS, BOGUS, 0, 8, 32, 4, 96, 64, 0.1, BOGUS, None, None) == UNSUPPORTED   # D
    assert f(BOGUS, BOGUS, BOGUS, BOGUS, 0, 8, 32, 4, 128, 0, 0.1, BOGUS, None, None) == INVALID
    assert f(None, BOGUS, BOGUS, BOGUS, 0, 8, 32, 4, 128, 64, 0.1, BOGUS, None, None) == INVALID
    assert f(BOGUS, BOGUS, BOGUS, BOGUS, 0, 2 ** 29, 32, 4, 128, 64, 0.1, BOGUS, None, None) == UNSUPPORTED  # grid


def test_decode_rejects_bad_arguments(lib):
    f = lib.dsa_sparse_gqa_decode
    need = lib.dsa_decode_workspace_size(4, 1000, 32, 4, 128, 64)
    assert need > 0

    def call(ws=BOGUS, ws_bytes=None, max_seq_len=1000, max_pages=16, HI=32, k=64):
        return f(*([BOGUS] * 9), max_pages, 100, BOGUS, max_seq_len, 4, 32, 4, 128, HI, 64, k, 0.1, ws,
                 need if ws_bytes is None else ws_bytes, BOGUS, None, None)

    assert call(ws=None) == WORKSPACE
    assert call(ws_bytes=need - 1) == WORKSPACE
    assert call(max_seq_len=16 * 64 + 1) == INVALID  # longer than the block table covers
    assert call(HI=12) == UNSUPPORTED
    assert call(k=0) == INVALID


def test_copies_in_16_byte_pieces_need_aligned_pointers(lib):
    # TMA boxes and 16-byte copies read these inputs: a pointer off a 16-byte
    # boundary is rejected before any launch.
    idx = lib.dsa_indexer_scores
    assert idx(BOGUS + 4, BOGUS, BOGUS, BOGUS, BOGUS, 512, 4, 32, 0, 8, BOGUS, 512, None, None) == INVALID  # q8
    assert idx(BOGUS, BOGUS, BOGUS, BOGUS + 8, BOGUS, 512, 4, 32, 0, 8, BOGUS, 512, None, None) == INVALID  # k8
    dec = lib.dsa_decode_indexer_scores

    def decode_scores(q8=BOGUS, k8c=BOGUS, skc=BOGUS):
        return dec(q8, BOGUS, BOGUS, k8c, skc, BOGUS, 16, 100, BOGUS, 1000, 4, 32, 64, BOGUS, 1000, None)

    assert decode_scores(q8=BOGUS + 4) == INVALID
    assert decode_scores(k8c=BOGUS + 16 + 8) == INVALID
    assert decode_scores(skc=BOGUS + 4) == INVALID
    chain = lib.dsa_sparse_gqa_decode
    need = lib.dsa_decode_workspace_size(4, 1000, 32, 4, 128, 64)

    def decode_chain(q8=BOGUS, k8c=BOGUS, skc=BOGUS):
        return chain(BOGUS, q8, BOGUS, BOGUS, k8c, skc, BOGUS, BOGUS, BOGUS, 16, 100, BOGUS, 1000, 4, 32, 4, 128,
                     32, 64, 64, 0.1, BOGUS, need, BOGUS, None, None)

    assert decode_chain(q8=BOGUS + 4) == INVALID
    assert decode_chain(k8c=BOGUS + 4) == INVALID
    assert decode_chain(skc=BOGUS + 8) == INVALID


def test_packed_prefill_rejects_bad_offsets():
    # checked on the host before any tensor is touched
    class Plan:
        L, D, fused = 100, 64, False

    class FusedPlan(Plan):
        fused = True

    for plan in (Plan(), FusedPlan()):
        # not starting at 0, decreasing, more tokens (or a longer sequence) than the plan holds
        for cu in ([1, 5], [0, 5, 3], [0, 50, 200]):
            with pytest.raises(dsa.DSAError):
                dsa.prefill_forward_packed(plan, cu, *([None] * 9), None)


def test_workspace_queries(lib):
    a = lib.dsa_decode_workspace_size(32, 262144, 32, 4, 128, 2048)
    b = lib.dsa_decode_workspace_size(32, 131072, 32, 4, 128, 2048)
    assert a > b > 32 * 131072 * 4
    assert lib.dsa_decode_attention_workspace_size(32, 32, 4, 128, 2048) > 0
    assert lib.dsa_topk_workspace_size(8, 1000, 0) == 0
    assert lib.dsa_row_stats_bytes(100) == 100 * 32

"""The C-ABI library without a GPU: it loads, exports every declared entry point, and rejects bad
arguments on the host before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_attention_12_b200 as dsa
from sparse_attention_12_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    return dsa.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dsa_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)
    assert set(dsa.EXPORTS) == set(names)


def test_abi_version_and_strings(lib):
    assert lib.dsa_abi_version() == 4
    for s in range(8):
        assert lib.dsa_status_string(s).decode() == dsa.STATUS[s]
    assert lib.dsa_status_string(99).decode() == "unknown status"


FAKE = 1 << 20  # an aligned, never-dereferenced "device" address: validation must fail first

# The validation tests below pass made-up device addresses that the host-side checks must reject
# before anything launches. They run only where no GPU can be reached, so that a change in the
# order of the checks can never send a kernel to those addresses.
no_gpu = pytest.mark.skipif(__import__("torch").cuda.is_available(),
                            reason="made-up device addresses: run where no GPU is reachable")


def batch(B=2, T=3, max_q=2, max_seq_len=300, max_pages=5, num_pages=10):
    return dsa.DsaBatchC(B, T, max_q, max_seq_len, max_pages, num_pages, FAKE, FAKE, FAKE)


@no_gpu
def test_plan_rejects_bad_arguments(lib):
    b = batch()
    n = lib.dsa_plan_workspace_size(ctypes.byref(b), 64)
    assert n > 64
    assert lib.dsa_plan(None, 64, FAKE, n, None) == 1
    assert lib.dsa_plan(ctypes.byref(b), 48, FAKE, n, None) == 2
    assert lib.dsa_plan(ctypes.byref(b), 64, FAKE + 4, n, None) == 1       # misaligned
    assert lib.dsa_plan(ctypes.byref(b), 64, FAKE, n - 1, None) == 3       # workspace
    bad = batch(max_pages=4)                                               # 300 positions need 5 pages
    assert lib.dsa_plan(ctypes.byref(bad), 64, FAKE, n, None) == 1
    nulls = dsa.DsaBatchC(2, 3, 2, 300, 5, 10, None, FAKE, FAKE)
    assert lib.dsa_plan(ctypes.byref(nulls), 64, FAKE, n, None) == 1


def test_empty_batch_is_a_no_op(lib):
    b = dsa.DsaBatchC(0, 0, 0, 0, 0, 0, None, None, None)
    assert lib.dsa_index_scores(ctypes.byref(b), None, None, None, None, 64, None, None, None, 0, None) == 0
    assert lib.dsa_topk(ctypes.byref(b), None, None, 0, 2048, None, None, 0, None) == 0
    assert lib.dsa_sparse_mla(ctypes.byref(b), None, None, 128, None, None, 2048, 0.07, None, None, None, 0,
                              None) == 0
    assert lib.dsa_layer(ctypes.byref(b), None, None, None, 64, None, None, None, 128, None, 2048, 0.07, None,
                         None, None, None, 0, None) == 0


@no_gpu
def test_index_scores_validation(lib):
    b = batch()
    call = lambda **kw: lib.dsa_index_scores(
        ctypes.byref(b), kw.get("plan", FAKE), kw.get("qI", FAKE), FAKE, FAKE, kw.get("nhI", 64),
        kw.get("kI", FAKE), FAKE, kw.get("scores", FAKE), kw.get("ld", 384), None)
    assert call(nhI=20) == 2
    assert call(qI=None) == 1
    assert call(kI=FAKE + 8) == 1
    assert call(ld=256) == 1          # ld < max_seq_len
    assert call(ld=302) == 1          # ld % 4
    assert call(scores=None) == 1


@no_gpu
def test_cache_write_validation(lib):
    b = batch()
    call = lambda **kw: lib.dsa_cache_write(ctypes.byref(b), kw.get("plan", FAKE), kw.get("k", FAKE), kw.get("c", FAKE),
                                            kw.get("kI", FAKE), kw.get("ks", FAKE), kw.get("kv", FAKE), None)
    assert call(k=None) == 1
    assert call(kv=None) == 1
    assert call(c=FAKE + 8) == 1        # misaligned
    assert call(plan=FAKE + 4) == 1
    empty = dsa.DsaBatchC(0, 0, 0, 0, 0, 0, None, None, None)
    assert lib.dsa_cache_write(ctypes.byref(empty), None, None, None, None, None, None, None) == 0


@no_gpu
def test_topk_and_mla_validation(lib):
    b = batch()
    assert lib.dsa_topk(ctypes.byref(b), FAKE, FAKE, 384, 0, FAKE, None, 0, None) == 2
    assert lib.dsa_topk(ctypes.byref(b), FAKE, FAKE, 384, 5000, FAKE, None, 0, None) == 2
    assert lib.dsa_topk(ctypes.byref(b), FAKE, FAKE, 100, 16, FAKE, None, 0, None) == 1
    assert lib.dsa_topk(ctypes.byref(b), FAKE, FAKE, 386, 16, FAKE, None, 0, None) == 1      # ld % 4
    assert lib.dsa_topk(ctypes.byref(b), FAKE, FAKE + 4, 384, 16, FAKE, None, 0, None) == 1  # misaligned scores
    long_rows = batch(max_seq_len=262145, max_pages=4097)
    assert lib.dsa_topk(ctypes.byref(long_rows), FAKE, FAKE, 262148, 16, FAKE, None, 0, None) == 2
    # few rows of 32769 .. 131072 positions: one cluster of CTAs per row, no workspace
    few = batch(max_seq_len=70000, max_pages=1094, num_pages=2000)
    assert lib.dsa_topk_workspace_size(ctypes.byref(few), 2047) == 0
    assert lib.dsa_topk_workspace_size(ctypes.byref(b), 2048) == 0
    # many long rows, or rows above 131072 positions: one CTA per row and 32768-position slice,
    # whose winners wait in the candidate workspace: positions and keys, T * slices * round4(k) each
    # (batches of many rows take 16384-position slices while the slices' winners fit one merge CTA)
    sliced = batch(B=1, T=1200, max_q=1200, max_seq_len=70000, max_pages=1094, num_pages=2000)
    need = lib.dsa_topk_workspace_size(ctypes.byref(sliced), 2047)
    assert need == 2 * 4 * 1200 * 5 * 2048
    wide_k = batch(B=1, T=1200, max_q=1200, max_seq_len=140000, max_pages=2188, num_pages=3000)
    # 9 slices of 16384 x 4096 winners > 32768: slices of 32768 instead
    assert lib.dsa_topk_workspace_size(ctypes.byref(wide_k), 4096) == 2 * 4 * 1200 * 5 * 4096
    longest = batch(max_seq_len=140000, max_pages=2188, num_pages=3000)
    assert lib.dsa_topk_workspace_size(ctypes.byref(longest), 2048) == 2 * 4 * 3 * 5 * 2048
    assert lib.dsa_topk(ctypes.byref(sliced), FAKE, FAKE, 70000, 2047, FAKE, None, 0, None) == 1      # no ws
    assert lib.dsa_topk(ctypes.byref(sliced), FAKE, FAKE, 70000, 2047, FAKE, FAKE, need - 1, None) == 3
    mla = lambda **kw: lib.dsa_sparse_mla(
        ctypes.byref(b), FAKE, kw.get("q", FAKE), kw.get("H", 128), FAKE, FAKE, kw.get("k", 2048),
        kw.get("scale", 0.07), FAKE, None, kw.get("ws", FAKE), kw.get("ws_bytes", 1 << 30), None)
    assert mla(H=0) == 2
    assert mla(H=129) == 2
    assert mla(k=0) == 2
    assert mla(scale=0.0) == 1
    assert mla(scale=float("nan")) == 1
    assert mla(q=FAKE + 2) == 1
    need = lib.dsa_sparse_mla_workspace_size(ctypes.byref(b), 128, 2048)
    assert need > 0          # 3 rows cannot fill the GPU: split partials need workspace
    assert mla(ws_bytes=need - 1) == 3
    # 16 heads or fewer run the few-head kernel: the same splits and partial-output layout
    # ([T][splits][H][512] fp32, then [T][splits][H] log-sum-exp), so the same size formula
    splits = min(74 // 3, 16, 2048 // 128)
    a16 = lambda x: (x + 15) // 16 * 16
    for H in (16, 5, 1):
        need_h = lib.dsa_sparse_mla_workspace_size(ctypes.byref(b), H, 2048)
        assert need_h == a16(4 * 3 * splits * H * 512) + a16(4 * 3 * splits * H)
        assert mla(H=H, ws_bytes=need_h - 1) == 3


@no_gpu
def test_layer_workspace_accounting(lib):
    b = batch()
    n = lib.dsa_layer_workspace_size(ctypes.byref(b), 64, 128, 2048)
    plan = lib.dsa_plan_workspace_size(ctypes.byref(b), 64)
    mla = lib.dsa_sparse_mla_workspace_size(ctypes.byref(b), 128, 2048)
    scores = 4 * 3 * 384
    S = 4 * 3 * 2048
    assert n >= plan + scores + S + mla
    assert n <= plan + scores + S + mla + 4 * 256
    args = [ctypes.byref(b), FAKE, FAKE, FAKE, 64, FAKE, FAKE, FAKE, 128, FAKE, 2048, 0.07, FAKE, None, None, FAKE]
    assert lib.dsa_layer(*args, n - 1, None) == 3
    assert lib.dsa_layer(*args[:4], 40, *args[5:], n, None) == 2


@no_gpu
def test_masked_mha_validation(lib):
    b = batch()
    need = lib.dsa_masked_mha_workspace_size(ctypes.byref(b), 16, 512)
    assert need == 4 * 3 * 12            # one bit per position: 300 positions -> 3 tiles of 4 words per row
    call = lambda **kw: lib.dsa_masked_mha(
        ctypes.byref(kw.get("b", b)), kw.get("plan", FAKE), kw.get("q", FAKE), kw.get("k", FAKE), kw.get("v", FAKE),
        kw.get("H", 16), kw.get("S", FAKE), kw.get("topk", 512), kw.get("scale", 0.07), kw.get("out", FAKE), None,
        kw.get("ws", FAKE), kw.get("ws_bytes", need), None)
    assert call(H=0) == 2
    assert call(H=129) == 2
    assert call(topk=0) == 2
    assert call(topk=4097) == 2
    assert call(v=None) == 1
    assert call(S=None) == 1
    assert call(k=FAKE + 2) == 1        # misaligned
    assert call(scale=-1.0) == 1
    assert call(ws=None) == 1
    assert call(ws_bytes=need - 1) == 3
    long_req = batch(max_seq_len=65537, max_pages=1025, num_pages=2000)
    assert call(b=long_req) == 2
    assert lib.dsa_masked_mha_workspace_size(ctypes.byref(long_req), 16, 512) == 0
    empty = dsa.DsaBatchC(0, 0, 0, 0, 0, 0, None, None, None)
    assert lib.dsa_masked_mha(ctypes.byref(empty), None, None, None, None, 16, None, 512, 0.07, None, None, None, 0,
                              None) == 0


@no_gpu
def test_noalloc_checks_arguments_like_layer(lib):
    """dsa_layer_noalloc returns what dsa_layer returns for every argument error, and only then
    applies its size limit (nothing launches in any of these calls)."""
    empty = dsa.DsaBatchC(0, 0, 0, 0, 0, 0, None, None, None)
    for nhI, H, k in [(48, 128, 2048), (64, 0, 2048), (64, 128, 0), (64, 128, 2048)]:
        want = lib.dsa_layer(ctypes.byref(empty), None, None, None, nhI, None, None, None, H, None, k, 0.07, None,
                             None, None, None, 0, None)
        got = lib.dsa_layer_noalloc(ctypes.byref(empty), None, None, None, nhI, None, None, None, H, None, k, 0.07,
                                    None, None, None, None)
        assert got == want == (0 if (nhI, H, k) == (64, 128, 2048) else 2)
    # 40000 query rows x 2048 positions of fp32 scores alone need 312 MiB of workspace
    big = dsa.DsaBatchC(1, 40000, 40000, 40000, 625, 700, FAKE, FAKE, FAKE)
    assert lib.dsa_layer_workspace_size(ctypes.byref(big), 64, 128, 2048) > (64 << 20)

    def noalloc(**kw):
        return lib.dsa_layer_noalloc(ctypes.byref(big), kw.get("qI", FAKE), FAKE, FAKE, 64, FAKE, FAKE, FAKE, 128,
                                     FAKE, 2048, ctypes.c_float(kw.get("scale", 0.07)), kw.get("out", FAKE), None,
                                     None, None)

    def layer(**kw):
        return lib.dsa_layer(ctypes.byref(big), kw.get("qI", FAKE), FAKE, FAKE, 64, FAKE, FAKE, FAKE, 128, FAKE, 2048,
                             ctypes.c_float(kw.get("scale", 0.07)), kw.get("out", FAKE), None, None, FAKE, 1 << 40,
                             None)

    for bad in ({"qI": None}, {"out": None}, {"qI": FAKE + 4}, {"scale": 0.0}):
        assert noalloc(**bad) == layer(**bad) == 1, bad
    assert noalloc() == 3  # valid arguments, above the 64 MiB static array: DSA_ERR_WORKSPACE


@no_gpu
def test_index_topk_support_and_validation(lib):
    def sup(B, T, max_q, L, nhI=64, k=2048):
        b = dsa.DsaBatchC(B, T, max_q, L, (L + 63) // 64, B * ((L + 63) // 64), FAKE, FAKE, FAKE)
        return lib.dsa_index_topk_supported(ctypes.byref(b), nhI, k)
    assert sup(64, 64, 1, 16384) == 1          # decode: one query per request
    assert sup(16, 32, 2, 131072) == 1         # MTP verify: two queries per request, long contexts
    assert sup(128, 128, 1, 131072) == 1
    assert sup(8, 32, 4, 32768) == 1           # four queries per request: one MMA group of 256 columns
    assert sup(8, 32, 4, 65536) == 0           # ... whose scores of 8192 positions per CTA leave < 3 key stages
    assert sup(8, 40, 5, 4096) == 0            # five do not fit one group of 64-head queries
    assert sup(8, 128, 16, 4096, nhI=16) == 1  # sixteen 16-head queries do
    assert sup(8, 32, 4, 131072) == 0          # four queries x 16384 positions per CTA: too much shared memory
    assert sup(1, 4096, 4096, 4096) == 0       # a prefill: not one group
    assert sup(64, 64, 1, 16384, nhI=48) == 0
    b = dsa.DsaBatchC(2, 3, 2, 300, 5, 10, FAKE, FAKE, FAKE)
    call = lambda **kw: lib.dsa_index_topk(ctypes.byref(kw.get("b", b)), FAKE, kw.get("qI", FAKE), FAKE, FAKE,
                                           kw.get("nhI", 64), FAKE, FAKE, kw.get("k", 256), kw.get("S", FAKE), None)
    assert call(S=None) == 1
    assert call(qI=FAKE + 4) == 1
    assert call(nhI=20) == 2
    assert call(k=0) == 2
    assert call(b=dsa.DsaBatchC(2, 6, 5, 300, 5, 10, FAKE, FAKE, FAKE)) == 2  # five queries in one request
    empty = dsa.DsaBatchC(0, 0, 0, 0, 0, 0, None, None, None)
    assert lib.dsa_index_topk(ctypes.byref(empty), None, None, None, None, 64, None, None, 256, None, None) == 0

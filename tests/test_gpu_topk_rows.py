"""Top-k on crafted score rows through the C ABI, compared exactly with the oracle's selection.

The indexer's own scores rarely tie; these rows do: flat rows, rows of three values, keys packed
into a few thousand ulps, magnitudes from 1e-30 to 1e30 of both signs, signed zeros and
infinities, at lengths around the 4096-position chunk, the 32768-key shared-memory cache and
k itself. Positions past a row's length hold +inf, so a read beyond the visible prefix would be
selected and caught.
"""
import numpy as np
import pytest
import torch

import sparse_attention_12_b200 as dsa
from oracle import dsa_oracle as O
from sparse_attention_12_b200 import build as dsa_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dsa_build.build()
    dsa.load()


def _row(kind, L, rng):
    if kind == "flat":
        return np.full(L, 0.37, np.float32)
    if kind == "three_values":
        return rng.integers(0, 3, L).astype(np.float32)
    if kind == "narrow":  # 3000 consecutive float values above 1.0
        return (1.0 + rng.integers(0, 3000, L) * 2.0 ** -23).astype(np.float32)
    if kind == "wide":
        mag = 10.0 ** rng.uniform(-30, 30, L)
        return (mag * rng.choice([-1.0, 1.0], L)).astype(np.float32)
    if kind == "zeros_inf":
        x = rng.standard_normal(L).astype(np.float32)
        x[rng.random(L) < 0.2] = 0.0
        x[rng.random(L) < 0.2] = -0.0
        x[rng.random(L) < 0.01] = np.inf
        x[rng.random(L) < 0.01] = -np.inf
        return x
    return rng.standard_normal(L).astype(np.float32)


def _run(k, rows, seed=0):
    rng = np.random.default_rng(seed)
    Ls = [L for _, L in rows]
    pages = [(L + 63) // 64 for L in Ls]
    max_pages = max(pages)
    bt = np.full((len(Ls), max_pages), -1, np.int32)
    nxt = 0
    for b, n in enumerate(pages):
        bt[b, :n] = np.arange(nxt, nxt + n)
        nxt += n
    batch = dsa.Batch.from_host(Ls, np.arange(len(Ls) + 1), bt, nxt)
    plan = dsa.plan(batch, 64)
    ld = (max(Ls) + 127) // 128 * 128
    host = np.full((len(Ls), ld), np.inf, np.float32)
    for t, (kind, L) in enumerate(rows):
        host[t, :L] = _row(kind, L, rng)
    scores = torch.from_numpy(host).cuda()
    S = dsa.topk(batch, plan, scores, k)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == 0
    got = S.cpu().numpy()
    for t, (kind, L) in enumerate(rows):
        want = O.topk_select(host[t, :L].astype(np.float64), k)
        take = min(k, L)
        np.testing.assert_array_equal(got[t, :take], np.sort(want[:take]), err_msg=f"{kind} L={L} k={k}")
        assert np.all(got[t, take:] == -1), f"{kind} L={L} k={k}: padding"


@pytest.mark.parametrize("k", [1, 256, 2048, 4096])
def test_topk_crafted_rows(k):
    rows = [("flat", 5000), ("three_values", 5000), ("narrow", 16384), ("wide", 16384), ("zeros_inf", 4097),
            ("normal", 4097), ("normal", k + 1), ("three_values", k + 1), ("normal", 100)]
    _run(k, rows, seed=k)


def test_topk_rows_beyond_the_cache():
    # 40000 and 131072 positions: no shared-memory cache, every pass re-reads the scores
    _run(2048, [("three_values", 40000), ("narrow", 40000), ("normal", 131072), ("flat", 32769)], seed=7)

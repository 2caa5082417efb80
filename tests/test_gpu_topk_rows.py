"""Top-k on crafted score rows through the C ABI, compared exactly with the oracle's selection.

The indexer's own scores rarely tie; these rows do: flat rows, rows of three values, keys packed
into a few thousand ulps, magnitudes from 1e-30 to 1e30 of both signs, signed zeros and
infinities, at lengths around the chunk sizes, the per-CTA slices and k itself. Positions past a
row's length hold +inf, so a read beyond the visible prefix would be selected and caught.

Rows of up to 32768 positions run the single-CTA kernel. Longer rows (up to 131072) in batches
whose clusters fit one wave run the cluster kernel, one cluster of up to 8 CTAs per row; otherwise
the single-CTA kernel's 32768-position slices and a merge over the slices' winners.
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
    if kind == "nans":  # NaN ranks below every other score, -inf included
        x = rng.standard_normal(L).astype(np.float32)
        x[rng.random(L) < 0.3] = np.nan
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
            ("normal", 4097), ("normal", k + 1), ("three_values", k + 1), ("normal", 100), ("nans", 3000),
            ("nans", k + 1)]
    _run(k, rows, seed=k)


def test_topk_rows_beyond_the_cache():
    # 40000 and 131072 positions in a batch of four rows: each row over the 8 CTAs of a cluster
    _run(2048, [("three_values", 40000), ("narrow", 40000), ("normal", 131072), ("flat", 32769)], seed=7)


def test_topk_cluster_rows_with_empty_slices():
    # one 131072-position row sets the cluster to 8 CTAs; in the short rows most CTAs hold no keys
    for k in (1, 2048):
        _run(k, [("normal", 131072), ("normal", 2049), ("three_values", 3), ("flat", 9), ("zeros_inf", 2050),
                 ("wide", 16385), ("narrow", 4095), ("nans", 40000)], seed=11 + k)


def test_topk_single_cta_path_long_rows():
    # a row above 131072 positions: the single-CTA kernel, 32768-position slices and a merge
    _run(2048, [("normal", 140000), ("three_values", 70000), ("narrow", 40000), ("normal", 3000),
                ("flat", 2049)], seed=9)


def test_topk_many_rows_single_cta_path():
    # 1200 rows: one CTA per row
    kinds = ["normal", "three_values", "narrow", "wide", "zeros_inf", "flat"]
    rows = [(kinds[i % len(kinds)], 400 + (i * 37) % 4700) for i in range(1200)]
    _run(512, rows, seed=5)


def test_topk_many_long_rows_slices_and_merge():
    # 40 rows of up to 131072 positions: too many clusters for one wave, so slices and a merge
    kinds = ["normal", "three_values", "narrow", "wide", "zeros_inf", "flat"]
    rows = [(kinds[i % len(kinds)], 32769 + (i * 2467) % 98000) for i in range(40)]
    _run(2048, rows, seed=6)


def test_topk_many_rows_with_long_ones_slices_of_16384():
    # 1200 rows, every 97th of them 40000 positions long: 512-thread CTAs over 16384-position slices,
    # a merge for the long rows
    kinds = ["normal", "three_values", "narrow", "wide", "zeros_inf", "nans"]
    rows = [(kinds[i % len(kinds)], 40000 if i % 97 == 0 else 300 + (i * 53) % 9000) for i in range(1200)]
    _run(2048, rows, seed=8)

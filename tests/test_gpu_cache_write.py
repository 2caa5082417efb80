"""Writing new positions into the caches, through the C ABI, against the oracle byte for byte.

The whole of all three caches is compared: the written slots (FP8 codes, scales, latent rows) must
match the oracle exactly and every other slot must be untouched. One key has max |k| = 448, so its
scale is exactly 1 and exact e4m3 midpoints reach the conversion unchanged (ties to even); one key
is all zeros (scale 1, codes 0 and 0x80 by sign); the others span 1e-3 .. 1e3 in magnitude.
"""
import numpy as np
import pytest
import torch

import sparse_attention_12_b200 as dsa
from oracle import dsa_oracle as O
from sparse_attention_12_b200 import build as dsa_build
from sparse_attention_12_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dsa_build.build()
    dsa.load()


def _new_rows(T, seed):
    rng = np.random.default_rng(seed)
    k_new = (rng.standard_normal((T, 128)) * np.exp(rng.uniform(-7, 7, (T, 1)))).astype(np.float32)
    k_new[0] = 0.0
    k_new[0, ::2] = -0.0
    if T > 1:
        row = rng.uniform(-400, 400, 128).astype(np.float32)
        row[:9] = [448.0, 1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -1.0625, 0.0, -0.0, 13.0]
        k_new[1] = row
    c_new = rng.integers(0, 1 << 16, (T, 576)).astype(np.uint16)
    return k_new, c_new


def _run(wl, seed, bad_rows=()):
    hb = synth.make_batch(wl, seed=seed, extra_pages=3)
    db = dsa.DeviceBatch(hb)
    plan = dsa.plan(db.batch, db.nhI)
    T = hb.total_q
    k_new, c_new = _new_rows(T, seed + 100)
    for i, t in enumerate(bad_rows):  # keys with no FP8 encoding: the row must not be written
        k_new[t, 5 + i] = [np.inf, -np.inf, np.nan][i % 3]
    dsa.cache_write(db.batch, plan, torch.from_numpy(k_new).cuda(),
                    torch.from_numpy(c_new.view(np.int16)).cuda().view(torch.bfloat16),
                    db.kI_cache, db.kI_scale, db.kv_cache)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == (7 if bad_rows else 0)  # DSA_ERR_DEVICE_VALUE
    good = [t for t in range(T) if t not in bad_rows]
    k_ok = np.where(np.isfinite(k_new), k_new, 0.0).astype(np.float32)
    want_kI, want_ks, want_kv = O.cache_write(hb.seq_lens, hb.cu_q, hb.block_table, k_ok, c_new, hb.kI_cache,
                                              hb.kI_scale, hb.kv_cache)
    req, pos = O.query_positions(hb.seq_lens, hb.cu_q)
    for t in bad_rows:  # the rejected rows keep the slots' old contents in all three caches
        (pg,), (sl,) = O.physical_rows(hb.block_table[req[t]], [pos[t]])
        want_kI[pg, sl], want_ks[pg, sl], want_kv[pg, sl] = hb.kI_cache[pg, sl], hb.kI_scale[pg, sl], hb.kv_cache[pg, sl]
    assert len(good) + len(bad_rows) == T
    got_kI = db.kI_cache.view(torch.uint8).cpu().numpy()
    got_ks = db.kI_scale.cpu().numpy()
    got_kv = db.kv_cache.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got_kI, want_kI), "FP8 key codes differ"
    assert np.array_equal(got_ks.view(np.uint32), want_ks.view(np.uint32)), "key scales differ"
    assert np.array_equal(got_kv, want_kv), "latent rows differ"


def test_cache_write_ragged_small():
    wl = synth.custom("cache_write", [300, 1000, 64, 1, 2100, 129], [1, 3, 64, 1, 5, 2], n_heads_index=64, topk=256,
                      n_heads=16)
    _run(wl, seed=11)


def test_cache_write_decode_64x16k():
    _run(synth.workload("decode_64x16k"), seed=12)


def test_cache_write_rejects_non_finite_keys():
    wl = synth.custom("cache_write_bad", [300, 1000, 64, 2100], [2, 3, 1, 4], n_heads_index=64, topk=256, n_heads=16)
    _run(wl, seed=13, bad_rows=(2, 5, 9))

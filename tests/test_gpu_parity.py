"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Small ragged cases are compared in full (every row, every score); the five workload shapes are
compared on all rows (prefill_32k: 512 sampled rows, including the dense/sparse boundary).
"""
import numpy as np
import pytest
import torch

import sparse_attention_12_b200 as dsa
from oracle import dsa_oracle as O
from sparse_attention_12_b200 import build as dsa_build
from sparse_attention_12_b200 import synth
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dsa_build.build()
    dsa.load()


def run_all_checks(wl, rows=None, seed=0, check_layer=True):
    hb = synth.make_batch(wl, seed=seed, extra_pages=3)
    db = dsa.DeviceBatch(hb)
    plan, scores, S = G.gpu_steps(db)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == 0
    T = hb.total_q
    rows = list(range(T)) if rows is None else list(rows)
    _, pos = O.query_positions(hb.seq_lens, hb.cu_q)
    ref = G.oracle_scores(hb, rows)
    sc = G.rows_to_host(scores, rows)
    Sg = G.rows_to_host(S, rows)
    G.check_scores(ref, sc, pos)
    G.check_topk_exact(sc, Sg, pos, db.k)
    G.check_index_sets(ref, Sg, pos, db.k)
    # attention on the oracle's index sets
    S_ref = np.full((T, db.k), -1, np.int32)
    for t in rows:
        S_ref[t] = O.topk_select(ref[t], db.k)
    lse = torch.empty((T, db.H), dtype=torch.float32, device="cuda")
    out = dsa.sparse_mla(db.batch, plan, db.q, db.kv_cache, torch.from_numpy(S_ref).cuda(), db.softmax_scale,
                         lse=lse)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == 0
    G.check_attention(hb, G.rows_to_host(out.float(), rows), G.rows_to_host(lse, rows),
                      {t: S_ref[t] for t in rows})
    if check_layer:
        S_out = torch.empty((T, db.k), dtype=torch.int32, device="cuda")
        lse2 = torch.empty((T, db.H), dtype=torch.float32, device="cuda")
        out2 = dsa.layer(db.batch, db.qI, db.qI_scale, db.wI, db.kI_cache, db.kI_scale, db.q, db.kv_cache, db.k,
                         db.softmax_scale, lse=lse2, S_out=S_out)
        torch.cuda.synchronize()
        S2 = G.rows_to_host(S_out, rows)
        for t in rows:
            assert np.array_equal(S2[t], Sg[t]), f"row {t}: fused layer picked other index sets than the steps"
        G.check_attention(hb, G.rows_to_host(out2.float(), rows), G.rows_to_host(lse2, rows), S2)
    return hb


# ---------------------------------------------------------------------------------------------
# small ragged cases (full comparison)

def test_decode_ragged_small():
    wl = synth.custom("decode_ragged", [300, 1000, 4097, 64, 1, 2100], [1] * 6, n_heads_index=64, topk=256,
                      n_heads=128, needles="decode", n_needles=4)
    run_all_checks(wl)


def test_mtp_two_queries_small():
    wl = synth.custom("mtp_small", [513, 2048, 130], [2, 2, 2], n_heads_index=64, topk=200, n_heads=128)
    run_all_checks(wl)


def test_prefill_small_16_heads():
    wl = synth.custom("prefill_small", [700], [700], n_heads_index=16, topk=128, n_heads=16,
                      needles="prefill", n_needles=4)
    run_all_checks(wl)


def test_chunked_prefill_with_history():
    # 5 queries at the end of a 900-position sequence, plus a request with no queries
    wl = synth.custom("chunk", [900, 77, 400], [5, 0, 7], n_heads_index=64, topk=300, n_heads=64)
    run_all_checks(wl)


def test_dense_fallback_every_row():
    wl = synth.custom("dense", [200, 50], [3, 1], n_heads_index=64, topk=2048, n_heads=128)
    hb = run_all_checks(wl)
    assert hb.total_q == 4


def test_k_equals_visible_positions():
    wl = synth.custom("k_eq", [256, 257], [1, 1], n_heads_index=64, topk=256, n_heads=128)
    run_all_checks(wl)


def test_prefill_two_splits_with_empty_units():
    # k = 4096 needs two units per query row (2048 entries each); rows before position 2048 have an
    # empty second unit, so the persistent clusters meet units without tiles between full ones
    wl = synth.custom("split_prefill", [2300], [2300], n_heads_index=16, topk=4096, n_heads=16,
                      needles="prefill", n_needles=4)
    run_all_checks(wl)


# ---------------------------------------------------------------------------------------------
# the workload shapes

def test_workload_prefill_2048():
    run_all_checks(synth.workload("prefill_2048"))


def test_workload_decode_64x16k():
    run_all_checks(synth.workload("decode_64x16k"))


def test_workload_mtp_16x128k():
    run_all_checks(synth.workload("mtp_16x128k"))


def test_workload_mixed_128():
    run_all_checks(synth.workload("mixed_128"))


def test_workload_prefill_32k_sampled():
    T = 32768
    rows = sorted(set(list(range(0, T, 64)) + list(range(2040, 2057)) + list(range(T - 16, T))))
    run_all_checks(synth.workload("prefill_32k"), rows=rows)

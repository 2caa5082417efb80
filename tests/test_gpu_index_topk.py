"""The fused indexer and top-k (dsa_index_topk) through the C ABI.

Two comparisons on the same seeded inputs:
  * with dsa_index_scores followed by dsa_topk on the GPU: identical index sets (the fused kernel
    computes each score with the same fp32 arithmetic, and both select exactly with the same tie
    rule), row by row and position by position;
  * with the oracle: every visible score recomputed in float64 and the index sets compared under
    the near-tie rule (the sets agree except where the oracle's scores are within 1e-3 relative of
    the k-th largest).
The workload shapes decode_64x16k, mtp_16x128k and mixed_128 run in full; small ragged cases cover
requests without queries, several queries per request, rows that take every visible position, and
16-head queries (16 of them per MMA group).
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


def run_fused(wl, seed=0, oracle_rows=None):
    hb = synth.make_batch(wl, seed=seed, extra_pages=2)
    db = dsa.DeviceBatch(hb)
    assert dsa.index_topk_supported(db.batch, db.nhI, db.k)
    plan, scores, S_ref = G.gpu_steps(db)
    S = torch.full_like(S_ref, -7)
    dsa.index_topk(db.batch, plan, db.qI, db.qI_scale, db.wI, db.kI_cache, db.kI_scale, db.k, S=S)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == 0
    assert torch.equal(S, S_ref), "fused sets differ from index_scores + topk"
    T = hb.total_q
    rows = list(range(T)) if oracle_rows is None else oracle_rows
    _, pos = O.query_positions(hb.seq_lens, hb.cu_q)
    G.check_index_sets(G.oracle_scores(hb, rows), G.rows_to_host(S, rows), pos, db.k)
    return hb


def test_fused_small_ragged():
    wl = synth.custom("fused_small", [300, 1000, 4097, 64, 1, 2100, 77, 9000], [1, 2, 1, 4, 1, 3, 0, 1],
                      n_heads_index=64, topk=256, n_heads=16, needles="decode", n_needles=3)
    run_fused(wl, seed=1)


def test_fused_sixteen_head_queries():
    wl = synth.custom("fused_16h", [2500, 700, 3000], [16, 3, 9], n_heads_index=16, topk=512, n_heads=16)
    run_fused(wl, seed=2)


def test_fused_k_at_and_above_the_visible_count():
    wl = synth.custom("fused_dense", [256, 257, 100], [1, 2, 1], n_heads_index=64, topk=256, n_heads=16)
    run_fused(wl, seed=3)


def test_fused_decode_64x16k():
    run_fused(synth.workload("decode_64x16k"))


def test_fused_mtp_16x128k():
    run_fused(synth.workload("mtp_16x128k"))


def test_fused_mixed_128():
    run_fused(synth.workload("mixed_128"))

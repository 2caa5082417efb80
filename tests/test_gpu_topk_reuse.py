"""Top-k reuse across adjacent layers, through the C ABI, against the oracle.

Some implementations let a layer reuse the index sets the previous layer selected and skip its own
indexer and top-k ("MTP 与稀疏注意力：NSA 与 DSA", section "对推理引擎的新要求": reuse of the selection
across adjacent layers). With this library that is a composition of calls: layer A runs the whole
path (dsa_layer, its S_t written out), and layer B runs only dsa_sparse_mla on its own queries and
latent cache with layer A's S_t and the batch's plan. The check: layer B's output equals the
oracle's sparse MLA of layer B's inputs on layer A's index sets, and the reused index sets are
exactly the ones layer A would select again.
"""
import dataclasses

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


def test_layer_b_reuses_layer_a_index_sets():
    wl = synth.custom("reuse", [3000, 700, 5000], [1, 2, 3], n_heads_index=64, topk=512, n_heads=128)
    layer_a = synth.make_batch(wl, seed=21, extra_pages=3)
    other = synth.make_batch(wl, seed=22, extra_pages=3)
    # layer B: the same requests and pages (one block table for every layer), its own queries and
    # latent cache
    layer_b = dataclasses.replace(layer_a, q=other.q, kv_cache=other.kv_cache)
    da, db = dsa.DeviceBatch(layer_a), dsa.DeviceBatch(layer_b)
    T = layer_a.total_q
    S_a = torch.empty((T, da.k), dtype=torch.int32, device="cuda")
    dsa.layer(da.batch, da.qI, da.qI_scale, da.wI, da.kI_cache, da.kI_scale, da.q, da.kv_cache, da.k,
              da.softmax_scale, S_out=S_a)
    plan = dsa.plan(db.batch, db.nhI)  # per batch: the same plan serves every layer
    lse_b = torch.empty((T, db.H), dtype=torch.float32, device="cuda")
    out_b = dsa.sparse_mla(db.batch, plan, db.q, db.kv_cache, S_a, db.softmax_scale, lse=lse_b)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == 0
    rows = list(range(T))
    S_host = G.rows_to_host(S_a, rows)
    # the reused sets are layer A's own selection (oracle scores of layer A, near-tie rule)
    _, pos = O.query_positions(layer_a.seq_lens, layer_a.cu_q)
    G.check_index_sets(G.oracle_scores(layer_a, rows), S_host, pos, da.k)
    # layer B's attention on them
    G.check_attention(layer_b, G.rows_to_host(out_b.float(), rows), G.rows_to_host(lse_b, rows), S_host)

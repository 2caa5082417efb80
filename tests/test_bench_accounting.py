"""The benchmark's algorithmic work per step (the numerators of its roofline fractions), checked
against counts derived by hand from the per-token sizes on the pages ("MTP 与稀疏注意力：NSA 与 DSA",
section "稀疏注意力：NSA 与 DSA": 128 FP8 bytes + a 4-byte scale of indexer key per token, a 576-wide
bf16 latent row per token, 2H(512+64) + 2H*512 FLOPs per selected pair, 2*64*128 per scored pair)."""
import types

import numpy as np

import bench


def _fake_batch(seq_lens, q_per_req, nhI, H, k):
    """Only the fields the accounting reads (no cache arrays: decode_64x16k's would be 1.2 GB)."""
    seq_lens = np.asarray(seq_lens, np.int32)
    cu_q = np.concatenate([[0], np.cumsum(q_per_req)]).astype(np.int32)
    T = int(cu_q[-1])

    def row_positions():
        req, pos = [], []
        for b, (n, m) in enumerate(zip(seq_lens, q_per_req)):
            req += [b] * m
            pos += [int(n) - m + i for i in range(m)]
        return np.asarray(req), np.asarray(pos, np.int64)

    return types.SimpleNamespace(seq_lens=seq_lens, cu_q=cu_q, total_q=T, row_positions=row_positions,
                                 qI=np.empty((T, nhI, 1)), q=np.empty((T, H, 1)),
                                 wl=types.SimpleNamespace(topk=k))


def test_decode_64x16k_bytes_and_flops():
    hb = _fake_batch([16384] * 64, [1] * 64, nhI=64, H=128, k=2048)
    w = bench.algorithmic(hb)
    keys = 16384 * (128 + 4)                 # every cached indexer key once, with its scale
    qw = 64 * 128 + 4 + 64 * 4               # FP8 query, its scale, the head weights
    scores = 16384 * 4                       # one fp32 score per visible position
    gather = 2048 * (576 * 2 + 4)            # selected latent rows and their indices
    q_mla, out = 128 * 576 * 2, 128 * 512 * 2
    assert w["index_scores"][0] == 64 * (keys + qw + scores)
    assert w["index_scores"][1] == 64 * 16384 * 2 * 64 * 128
    assert w["topk"][0] == 64 * (scores + 2048 * 4)
    assert w["sparse_mla"][0] == 64 * (gather + q_mla + out)
    assert w["sparse_mla"][1] == 64 * 2048 * (2 * 128 * 576 + 2 * 128 * 512)
    # the method's own traffic without the score and index round trips: 4.81 MB per request
    total = sum(w[n][0] for n in ("index_scores", "topk", "sparse_mla"))
    assert total - 64 * (2 * scores + 2 * 2048 * 4) == 64 * 4808964
    # fused indexer + top-k: no score row written or read, the index sets written
    assert w["index_topk"][0] == 64 * (keys + qw + 2048 * 4)


def test_causal_prefill_counts_visible_positions_only():
    L = 300
    hb = _fake_batch([L], [L], nhI=16, H=16, k=64)
    w = bench.algorithmic(hb)
    vis = L * (L + 1) // 2                   # query p sees p + 1 positions
    sel = sum(min(p + 1, 64) for p in range(L))
    assert w["index_scores"][1] == vis * 2 * 16 * 128
    assert w["sparse_mla"][1] == sel * (2 * 16 * 576 + 2 * 16 * 512)
    assert w["topk"][0] == vis * 4 + L * 64 * 4
    # the latent rows once (the whole cache of this request is named), indices, queries, output
    assert w["sparse_mla"][0] == L * 1152 + sel * 4 + L * 16 * 576 * 2 + L * 16 * 512 * 2


def test_mtp_rows_counted_once_per_request_at_most():
    # two queries of one request: at most 2k distinct rows, never more than the request holds
    hb = _fake_batch([131072, 3000], [2, 2], nhI=64, H=128, k=2048)
    w = bench.algorithmic(hb)
    rows = 2 * 2048 + 3000                   # request 1 holds 3000 positions, both of its rows see them all
    assert w["sparse_mla"][0] == rows * 1152 + (2 * 2048 + 2 * 2048) * 4 + 4 * 128 * (576 + 512) * 2


PEAKS = {"hbm_GBps": 6549.8, "bf16_TFLOPs": 1645.6, "fp8_TFLOPs": 3291.2}


def test_stage_bound_is_the_longer_roofline_time():
    # decode_64x16k's indexer: 124 FLOP per byte, below the FP8 ridge (~502) -> HBM-bound
    hb = _fake_batch([16384] * 64, [1] * 64, nhI=64, H=128, k=2048)
    w = bench.algorithmic(hb)
    r = bench.stage_roofline("index_scores", *w["index_scores"], 50.0, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["roofline_us"] - w["index_scores"][0] / 6549.8e9 * 1e6) < 1e-9
    assert abs(r["frac"] - r["roofline_us"] / 50.0) < 1e-12
    # a causal prefill's indexer: FLOPs grow with L^2, bytes with L -> FP8 tensor-bound
    hb = _fake_batch([32768], [32768], nhI=64, H=128, k=2048)
    w = bench.algorithmic(hb)
    r = bench.stage_roofline("index_scores", *w["index_scores"], 8000.0, PEAKS)
    assert r["bound"] == "tensor" and r["dtype"] == "fp8" and r["peak"] == 3291.2
    assert abs(r["achieved"] - w["index_scores"][1] / 8000e-6 / 1e12) < 1e-6
    # its sparse MLA at bf16, and the top-k (no contraction) always against HBM
    r = bench.stage_roofline("sparse_mla", *w["sparse_mla"], 30000.0, PEAKS)
    assert r["bound"] == "tensor" and r["dtype"] == "bf16" and r["peak"] == 1645.6
    r = bench.stage_roofline("topk", *w["topk"], 3000.0, PEAKS)
    assert r["bound"] == "hbm" and "tensor_frac" not in r


def test_both_arms_describe_the_same_config():
    from sparse_attention_12_b200 import synth
    wl = synth.workload("prefill_32k")
    c = bench.config_of(wl, 1)
    assert c["workload"] == "prefill_32k" and c["query_rows"] == 32768 and c["context"] == 32768
    assert set(c) >= {"workload", "page_size", "l2", "parallelism", "step"}

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
    total = sum(v[0] for v in w.values())
    assert total - 64 * (2 * scores + 2 * 2048 * 4) == 64 * 4808964


def test_causal_prefill_counts_visible_positions_only():
    L = 300
    hb = _fake_batch([L], [L], nhI=16, H=16, k=64)
    w = bench.algorithmic(hb)
    vis = L * (L + 1) // 2                   # query p sees p + 1 positions
    sel = sum(min(p + 1, 64) for p in range(L))
    assert w["index_scores"][1] == vis * 2 * 16 * 128
    assert w["sparse_mla"][1] == sel * (2 * 16 * 576 + 2 * 16 * 512)
    assert w["topk"][0] == vis * 4 + L * 64 * 4

"""Masked MHA mode for short prefill, through the C ABI, against the oracle.

The kernel computes dense 128 x 128 tiles over each query tile's causal range and masks them with
the bitmap of S_t; the oracle writes out softmax(tau q K^T + M) V with M = 0 on S_t, -inf elsewhere.
Tolerances as for the sparse MLA (bf16 output on fp32 accumulation, P rounded to bf16): max-abs
2e-2, mean-abs 2e-3, lse within 1e-3.
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


def _batch(seq_lens, q_per_req):
    """A device batch; the masked MHA mode reads no cache, so the block table is a plain layout."""
    pages = [(n + 63) // 64 for n in seq_lens]
    bt = np.full((len(seq_lens), max(pages)), -1, np.int32)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = np.arange(off, off + n)
        off += n
    cu = np.concatenate([[0], np.cumsum(q_per_req)]).astype(np.int32)
    return dsa.Batch.from_host(seq_lens, cu, bt, off), cu


def _bf16(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


def _run(lens, H, topk, seed, rows=None, sets=None):
    wl = synth.custom("mha", lens, lens, n_heads=H, topk=topk)
    x = synth.make_mha_inputs(wl, seed=seed)
    S = synth.random_index_sets(lens, lens, topk, seed=seed) if sets is None else sets
    batch, cu = _batch(lens, lens)
    plan = dsa.plan(batch, 16)
    T = int(cu[-1])
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    out = dsa.masked_mha(batch, plan, _bf16(x.q), _bf16(x.k), _bf16(x.v), torch.from_numpy(S).cuda(),
                         wl.softmax_scale, lse=lse)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == 0
    rows = list(range(T)) if rows is None else list(rows)
    ref_o, ref_l = O.masked_mha(lens, cu, x.q, x.k, x.v, S, wl.softmax_scale, rows=rows)
    idx = torch.as_tensor(rows, device="cuda")
    got_o = out.index_select(0, idx).float().cpu().numpy().astype(np.float64)
    got_l = lse.index_select(0, idx).cpu().numpy().astype(np.float64)
    err = np.abs(got_o - ref_o[rows])
    assert err.max() <= 2e-2, f"max-abs error {err.max():.3e}"
    assert err.mean() <= 2e-3, f"mean-abs error {err.mean():.3e}"
    np.testing.assert_allclose(got_l, ref_l[rows], rtol=0, atol=1e-3)
    return float(err.max()), float(err.mean())


def test_masked_mha_ragged_small():
    """Five whole prefills: tiles with a ragged tail, a one-token request, an exact tile, a request
    spanning 8 key tiles; sparse sets (k = 256 < most prefixes) and odd H."""
    _run([300, 1000, 1, 128, 129], H=3, topk=256, seed=1)


def test_masked_mha_dense_sets_are_causal_attention():
    """k above every prefix: S_t = [0, p], the mode is plain causal multi-head attention."""
    _run([700, 260], H=2, topk=1024, seed=2)


def test_masked_mha_single_position_sets():
    """|S_t| = 1 (position 0 for every row): the output is v_0 exactly (rounded to bf16)."""
    lens = [513]
    sets = np.full((513, 4), -1, np.int32)
    sets[:, 0] = 0
    _run(lens, H=2, topk=4, seed=3, sets=sets)


def test_masked_mha_prefill_2048_shape():
    """The short-prefill shape: L = 2048, 16 heads, k = 512; rows sampled across every query tile,
    both tile edges and the dense/sparse boundary at p = 511."""
    rows = sorted(set(list(range(0, 2048, 37)) + list(range(500, 520)) + [127, 128, 1023, 1024, 2046, 2047]))
    _run([2048], H=16, topk=512, seed=4, rows=rows)


def test_masked_mha_128_heads():
    """The model's head count (128 CTAs per query tile along the head axis), two requests, all rows."""
    _run([300, 77], H=128, topk=128, seed=6)


def test_masked_mha_ragged_many_heads():
    """64 heads over ragged requests (a partial last tile, a request of 1000 positions over eight
    query tiles, a request just past one tile); sparse sets (k = 300), rows sampled in every tile
    and at every tile edge."""
    lens = [600, 1000, 130]
    T = sum(lens)
    rows = sorted(set(list(range(0, T, 7)) + [127, 128, 255, 256, 599, 600, 727, 728, 855, 856, 1599, 1600, T - 1]))
    _run(lens, H=64, topk=300, seed=7, rows=rows)


def test_masked_mha_many_heads_dense_sets():
    """96 heads with k above every prefix: plain causal multi-head attention."""
    _run([520, 256], H=96, topk=1024, seed=8, rows=list(range(0, 776, 5)) + [255, 256, 511, 519, 775])


def test_masked_mha_rejects_requests_with_a_cached_prefix():
    """n_b != m_b is not a whole prefill: the kernel records DSA_ERR_DEVICE_INDEX and writes nothing."""
    lens, qs = [200], [100]
    wl = synth.custom("mha_bad", lens, lens, n_heads=2, topk=64)
    x = synth.make_mha_inputs(wl, seed=5)
    batch, _ = _batch(lens, qs)
    plan = dsa.plan(batch, 16)
    S = torch.from_numpy(synth.random_index_sets(lens, qs, 64, seed=5)).cuda()
    q = _bf16(x.q)[:100].contiguous()
    k = _bf16(x.k)[:100].contiguous()
    v = _bf16(x.v)[:100].contiguous()
    out = torch.full((100, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    dsa.masked_mha(batch, plan, q, k, v, S, wl.softmax_scale, out=out)
    assert dsa.status_read(plan) == 6
    assert bool((out == 7.0).all())


def test_masked_mha_rejects_a_cached_prefix_beside_a_whole_prefill():
    """128 heads, a cached-prefix request next to a whole prefill: the first is reported and left
    unwritten, the second computed."""
    lens, qs = [200, 300], [100, 300]
    wl = synth.custom("mha_bad2", lens, lens, n_heads=128, topk=64)
    x = synth.make_mha_inputs(wl, seed=9)
    batch, _ = _batch(lens, qs)
    plan = dsa.plan(batch, 16)
    S = torch.from_numpy(synth.random_index_sets(lens, qs, 64, seed=9)).cuda()
    sel = torch.cat([torch.arange(100, 200), torch.arange(200, 500)]).cuda()  # rows of the queries
    q = _bf16(x.q).index_select(0, sel).contiguous()
    k = _bf16(x.k).index_select(0, sel).contiguous()
    v = _bf16(x.v).index_select(0, sel).contiguous()
    out = torch.full((400, 128, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    dsa.masked_mha(batch, plan, q, k, v, S, wl.softmax_scale, out=out)
    assert dsa.status_read(plan) == 6
    assert bool((out[:100] == 7.0).all())

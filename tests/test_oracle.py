"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU needed).

Each check is chosen so that a plausible slip in the oracle fails it: a dropped ReLU or scale,
a wrong sign, an off-by-one in the causal set, a wrong page lookup, a transposed operand in the
attention, a wrong softmax scale or value width, a wrong tie rule.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from oracle import cost_model as CM
from sparse_attention_12_b200 import synth


# ---------------------------------------------------------------------------------------------
# storage decoders against torch's own conversions

def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # anchors from the OCP e4m3 definition
    assert O.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert O.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9
    assert O.e4m3_decode(np.uint8(0x08)) == 2.0 ** -6
    assert O.e4m3_decode(np.uint8(0x38)) == 1.0
    assert O.e4m3_decode(np.uint8(0xB8)) == -1.0


# ---------------------------------------------------------------------------------------------
# e4m3 encoder: round to nearest, ties to even, saturation at 448 (OCP E4M3)

def _finite_codes():
    return np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)


def test_e4m3_encode_round_trips_every_finite_code():
    codes = _finite_codes()
    vals = O.e4m3_decode(codes).astype(np.float32)
    vals[codes == 0x80] = np.float32(-0.0)  # the decoder folds -0 to 0.0 * -1 = -0.0 already
    assert np.array_equal(O.e4m3_encode(vals), codes)


def test_e4m3_encode_midpoints_go_to_the_even_code():
    mags = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    for c in range(0x7E):
        lo, hi = mags[c], mags[c + 1]
        mid = np.float32((lo + hi) / 2)           # at most 5 significant bits: exact in float32
        assert float(mid) == (lo + hi) / 2
        want = c if c % 2 == 0 else c + 1
        assert O.e4m3_encode([mid])[0] == want, (c, mid)
        assert O.e4m3_encode([-mid])[0] == want | 0x80
        below = np.nextafter(mid, np.float32(0.0), dtype=np.float32)
        above = np.nextafter(mid, np.float32(1e9), dtype=np.float32)
        assert O.e4m3_encode([below])[0] == c and O.e4m3_encode([above])[0] == c + 1


def test_e4m3_encode_saturates_and_keeps_zero_sign():
    enc = O.e4m3_encode(np.array([448.0, 464.0, 479.0, 1e30, -448.0, -1e30, 0.0, -0.0, 2.0 ** -12, -(2.0 ** -12)],
                                 np.float32))
    assert list(enc) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x00, 0x80, 0x00, 0x80]


def test_indexer_key_quantize_scale_and_error_bound():
    rng = np.random.default_rng(3)
    for k in [rng.standard_normal(128) * 3.0, rng.standard_normal(128) * 1e-3, np.zeros(128)]:
        k = k.astype(np.float32)
        codes, s = O.indexer_key_quantize(k)
        amax = np.float32(np.abs(k).max())
        assert s == (np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0))
        back = O.e4m3_decode(codes) * float(s)
        if amax > 0:
            assert (codes & 0x7F).max() == 0x7E   # the largest element maps to +-448
            # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
            normal = np.abs(k) / float(s) >= 2.0 ** -6
            assert np.all(np.abs(back - k)[normal] <= 2.0 ** -4 * np.abs(k)[normal] * (1 + 1e-6))
        else:
            assert np.all(codes == 0)


def test_indexer_key_quantize_agrees_with_the_synthetic_generator():
    # cross-check (not a pin): synth quantises with torch's float8 cast under the same reading
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((16, 128)) * np.exp(rng.uniform(-4, 4, (16, 1)))).astype(np.float32)
    codes, scale = synth.quantize_e4m3_per_token(x)
    for t in range(16):
        c, s = O.indexer_key_quantize(x[t])
        assert s == scale[t] and np.array_equal(c, codes[t])


def test_cache_write_places_rows_and_leaves_the_rest():
    rng = np.random.default_rng(5)
    P = 6
    kI = rng.integers(0, 256, (P, 64, 128)).astype(np.uint8)
    ks = rng.standard_normal((P, 64)).astype(np.float32)
    kv = rng.integers(0, 1 << 16, (P, 64, 576)).astype(np.uint16)
    seq_lens, cu_q = np.array([130, 64]), np.array([0, 2, 3])     # rows at positions 128, 129 and 63
    block_table = np.array([[4, 0, 2], [5, -1, -1]])
    k_new = rng.standard_normal((3, 128)).astype(np.float32)
    c_new = rng.integers(0, 1 << 16, (3, 576)).astype(np.uint16)
    kI2, ks2, kv2 = O.cache_write(seq_lens, cu_q, block_table, k_new, c_new, kI, ks, kv)
    where = [(2, 0), (2, 1), (5, 63)]                               # (page, slot) of each row
    for t, (pg, sl) in enumerate(where):
        codes, s = O.indexer_key_quantize(k_new[t])
        assert np.array_equal(kI2[pg, sl], codes) and ks2[pg, sl] == s
        assert np.array_equal(kv2[pg, sl], c_new[t])
    mask = np.ones((P, 64), bool)
    for pg, sl in where:
        mask[pg, sl] = False
    assert np.array_equal(kI2[mask], kI[mask]) and np.array_equal(ks2[mask], ks[mask])
    assert np.array_equal(kv2[mask], kv[mask])


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint16)
    ours = O.bf16_decode(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ---------------------------------------------------------------------------------------------
# indexer scores

def _hand_case(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "indexer_hand.json")))
    code = {float(k): v for k, v in g["e4m3_codes"].items()}
    P = 8
    kI = np.zeros((P, 64, 128), np.uint8)
    ks = np.ones((P, 64), np.float32)
    page = 5
    for j, (vec, s) in enumerate(zip(g["keys"]["vectors_first_two_dims"], g["keys"]["scales"])):
        kI[page, j, 0] = code[vec[0]] if vec[0] != 0 else 0
        kI[page, j, 1] = code[vec[1]] if vec[1] != 0 else 0
        ks[page, j] = s
    T = len(g["queries"])
    qI = np.zeros((T, 2, 128), np.uint8)
    qs = np.zeros(T, np.float32)
    w = np.zeros((T, 2), np.float32)
    for t, qq in enumerate(g["queries"]):
        for r, vec in enumerate(qq["heads_first_two_dims"]):
            qI[t, r, 0] = code[vec[0]] if vec[0] != 0 else 0
            qI[t, r, 1] = code[vec[1]] if vec[1] != 0 else 0
        qs[t] = qq["scale"]
        w[t] = qq["w"]
    bt = np.array([[page]], np.int32)
    seq_lens = np.array([3], np.int32)
    cu_q = np.array([0, 2], np.int32)
    expected = np.array([[float(x) for x in row] for row in g["expected_I"]])
    return dict(seq_lens=seq_lens, cu_q=cu_q, block_table=bt, qI=qI, qI_scale=qs, wI=w,
                kI_cache=kI, kI_scale=ks), expected


def test_index_scores_hand_computed(golden_dir):
    args, expected = _hand_case(golden_dir)
    got = O.index_scores(**args)
    assert got.shape == expected.shape
    assert np.array_equal(got, expected)


def test_query_positions_decode_and_mtp():
    req, pos = O.query_positions([5, 9, 3], [0, 1, 3, 6])
    assert list(req) == [0, 1, 1, 2, 2, 2]
    assert list(pos) == [4, 7, 8, 0, 1, 2]


def _small_batch(seq_lens, m, nhI=4, H=8, seed=3, extra_pages=2):
    wl = synth.custom("tiny", seq_lens, m, n_heads_index=nhI, topk=8, n_heads=H)
    return synth.make_batch(wl, seed=seed, extra_pages=extra_pages)


def _score_args(bt):
    return dict(seq_lens=bt.seq_lens, cu_q=bt.cu_q, block_table=bt.block_table, qI=bt.qI,
                qI_scale=bt.qI_scale, wI=bt.wI, kI_cache=bt.kI_cache, kI_scale=bt.kI_scale)


def test_index_scores_head_permutation_invariant():
    bt = _small_batch([70, 33], [3, 2], nhI=8)
    base = O.index_scores(**_score_args(bt))
    perm = np.random.default_rng(0).permutation(8)
    a = _score_args(bt)
    a["qI"] = bt.qI[:, perm]
    a["wI"] = bt.wI[:, perm]
    got = O.index_scores(**a)
    fin = np.isfinite(base)
    assert np.array_equal(np.isfinite(got), fin)
    np.testing.assert_allclose(got[fin], base[fin], rtol=1e-12, atol=1e-12)


def test_index_scores_positive_homogeneity_and_selection():
    bt = _small_batch([90], [4], nhI=4)
    a = _score_args(bt)
    base = O.index_scores(**a)
    a["qI_scale"] = bt.qI_scale * np.float32(4.0)
    got = O.index_scores(**a)
    fin = np.isfinite(base)
    np.testing.assert_allclose(got[fin], 4.0 * base[fin], rtol=1e-12)
    _, pos = O.query_positions(bt.seq_lens, bt.cu_q)
    assert np.array_equal(O.topk(base, pos, 8), O.topk(got, pos, 8))


def test_index_scores_single_head_is_textbook_dot():
    """1 head, w = 1, all products positive: I_tj = (s^q q) . (s^k k_j) exactly."""
    rng = np.random.default_rng(5)
    n = 10
    qf = np.abs(rng.standard_normal((1, 1, 128)).astype(np.float32))
    kf = np.abs(rng.standard_normal((1, 64, 128)).astype(np.float32))
    qc, qs = synth.quantize_e4m3_per_token(qf)
    kc, ksc = synth.quantize_e4m3_per_token(kf.reshape(64, 128))
    qv = torch.from_numpy(qc.reshape(1, 128)).view(torch.float8_e4m3fn).double().numpy() * qs[0]
    kv = torch.from_numpy(kc).view(torch.float8_e4m3fn).double().numpy() * ksc[:, None].astype(np.float64)
    want = np.array([float(np.dot(qv[0], kv[j])) for j in range(n)])
    got = O.index_scores(seq_lens=np.array([n], np.int32), cu_q=np.array([0, 1], np.int32),
                         block_table=np.array([[0]], np.int32), qI=qc, qI_scale=qs,
                         wI=np.ones((1, 1), np.float32), kI_cache=kc.reshape(1, 64, 128),
                         kI_scale=ksc.reshape(1, 64))
    np.testing.assert_allclose(got[0], want, rtol=1e-12)


def test_index_scores_paging_invariant():
    """Moving pages around the pool (and the block table with them) changes nothing."""
    bt = _small_batch([130, 64, 7], [2, 1, 3], nhI=4, extra_pages=3)
    base = O.index_scores(**_score_args(bt))
    P = bt.num_pages
    perm = np.random.default_rng(9).permutation(P)          # new slot of old page i is perm[i]
    kI2 = np.empty_like(bt.kI_cache)
    ks2 = np.empty_like(bt.kI_scale)
    kI2[perm] = bt.kI_cache
    ks2[perm] = bt.kI_scale
    table = np.where(bt.block_table >= 0, perm[np.maximum(bt.block_table, 0)], -1).astype(np.int32)
    a = _score_args(bt)
    a.update(kI_cache=kI2, kI_scale=ks2, block_table=table)
    got = O.index_scores(**a)
    assert np.array_equal(got, base)


def test_index_scores_causal_mask():
    bt = _small_batch([40, 12], [5, 12], nhI=2)
    sc = O.index_scores(**_score_args(bt))
    _, pos = O.query_positions(bt.seq_lens, bt.cu_q)
    for t in range(len(pos)):
        assert np.all(np.isfinite(sc[t, : pos[t] + 1]))
        assert np.all(np.isneginf(sc[t, pos[t] + 1:]))


# ---------------------------------------------------------------------------------------------
# TopK

def test_topk_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "topk_worked_example_p5.json")))
    s = np.array(g["scores_1based_positions_1_to_8"])
    S = O.topk_select(s, g["k"])
    assert sorted(S.tolist()) == g["expected_S_0based"]
    assert sorted((S + 1).tolist()) == g["expected_S_1based"]


def test_topk_worked_example_through_indexer():
    """t=8 (1-based), k=3: keys at positions 2, 5, 8 aligned with the query's positive head
    and all others anti-aligned give S_8 = {2, 5, 8} from the actual scoring function."""
    code_one, code_mone = 0x38, 0xB8
    kI = np.zeros((1, 64, 128), np.uint8)
    for j in range(8):
        kI[0, j, 0] = code_one if (j + 1) in (2, 5, 8) else code_mone
    ks = np.ones((1, 64), np.float32)
    ks[0, 1], ks[0, 4], ks[0, 7] = 3.0, 2.0, 1.0
    qI = np.zeros((1, 1, 128), np.uint8)
    qI[0, 0, 0] = code_one
    sc = O.index_scores(seq_lens=np.array([8], np.int32), cu_q=np.array([0, 1], np.int32),
                        block_table=np.array([[0]], np.int32), qI=qI, qI_scale=np.ones(1, np.float32),
                        wI=np.ones((1, 1), np.float32), kI_cache=kI, kI_scale=ks)
    S = O.topk_select(sc[0], 3)
    assert sorted((S + 1).tolist()) == [2, 5, 8]


def test_topk_matches_argpartition():
    rng = np.random.default_rng(11)
    for L, k in [(100, 7), (5000, 2048), (4096, 2048), (3000, 1)]:
        s = rng.standard_normal(L)
        S = O.topk_select(s, k)
        want = set(np.argpartition(-s, k - 1)[:k].tolist())
        assert set(S.tolist()) == want


def test_topk_dense_fallback_and_padding():
    s = np.array([0.3, -1.0, 2.0])
    S = O.topk_select(s, 5)
    assert sorted(S[:3].tolist()) == [0, 1, 2]
    assert S[3:].tolist() == [-1, -1]


def test_topk_ties_smaller_position_first():
    s = np.array([1.0, 5.0, 1.0, 1.0, 5.0, 1.0])
    assert O.topk_select(s, 3).tolist() == [1, 4, 0]


def test_needles_are_selected():
    wl = synth.custom("needles", [4096] * 2, [1, 2], n_heads_index=16, topk=256, n_heads=4,
                      needles="decode", n_needles=6)
    bt = synth.make_batch(wl, seed=0)
    req, pos = O.query_positions(bt.seq_lens, bt.cu_q)
    for t, j in bt.needles:
        I = O.index_scores_row(t, req, pos, bt.block_table, bt.qI, bt.qI_scale, bt.wI,
                               bt.kI_cache, bt.kI_scale)
        assert j in set(O.topk_select(I, 256).tolist())


# ---------------------------------------------------------------------------------------------
# sparse attention

def _sdpa(q, k, v, mask, scale):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=torch.from_numpy(mask),
        scale=scale).numpy()


def _mla_batch(L, H=4, seed=2):
    wl = synth.custom("mla", [L], [L], n_heads_index=2, topk=L, n_heads=H)
    return synth.make_batch(wl, seed=seed, extra_pages=1)


def _latent_rows(bt, b, n):
    pages, slots = O.physical_rows(bt.block_table[b], np.arange(n))
    return torch.from_numpy(bt.kv_cache[pages, slots].view(np.int16)).view(torch.bfloat16).double().numpy()


def test_sparse_mla_dense_when_k_covers_prefix():
    """With k >= p+1 the sparse output equals dense causal softmax attention (torch SDPA)."""
    L, H = 70, 4
    bt = _mla_batch(L, H)
    tau = O.default_softmax_scale()
    _, pos = O.query_positions(bt.seq_lens, bt.cu_q)
    S = np.full((L, L), -1, np.int32)
    for t in range(L):
        S[t, : t + 1] = np.arange(t + 1)[::-1]
    out, lse = O.sparse_mla(bt.seq_lens, bt.cu_q, bt.block_table, bt.q, bt.kv_cache, S, tau)
    c = _latent_rows(bt, 0, L)                                           # [L, 576]
    q = torch.from_numpy(bt.q.view(np.int16)).view(torch.bfloat16).double().numpy()   # [L, H, 576]
    qh = np.ascontiguousarray(q.transpose(1, 0, 2))                      # [H, L, 576]
    causal = np.where(np.tril(np.ones((L, L), bool)), 0.0, -np.inf)
    ref = _sdpa(qh, np.broadcast_to(c, (H, L, 576)).copy(),
                np.broadcast_to(c[:, :512], (H, L, 512)).copy(), causal, tau)
    np.testing.assert_allclose(out, ref.transpose(1, 0, 2), rtol=1e-10, atol=1e-12)
    logits = tau * np.einsum("thd,jd->thj", q, c) + causal[:, None, :]
    ref_lse = torch.logsumexp(torch.from_numpy(logits), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_sparse_mla_equals_masked_dense_form():
    """Gathering S_t equals softmax(QK^T/sqrt(d) + M) V with M = 0 on S_t, -inf elsewhere."""
    L, H = 90, 3
    bt = _mla_batch(L, H, seed=4)
    tau = O.default_softmax_scale()
    rng = np.random.default_rng(7)
    k = 11
    S = np.full((L, k), -1, np.int32)
    mask = np.full((L, L), -np.inf)
    for t in range(L):
        sel = rng.choice(t + 1, size=min(k, t + 1), replace=False)
        S[t, : sel.size] = sel
        mask[t, sel] = 0.0
    out, _ = O.sparse_mla(bt.seq_lens, bt.cu_q, bt.block_table, bt.q, bt.kv_cache, S, tau)
    c = _latent_rows(bt, 0, L)
    q = torch.from_numpy(bt.q.view(np.int16)).view(torch.bfloat16).double().numpy()
    ref = _sdpa(np.ascontiguousarray(q.transpose(1, 0, 2)), np.broadcast_to(c, (H, L, 576)).copy(),
                np.broadcast_to(c[:, :512], (H, L, 512)).copy(), mask, tau)
    np.testing.assert_allclose(out, ref.transpose(1, 0, 2), rtol=1e-10, atol=1e-12)


def test_sparse_mla_single_index_returns_value_row():
    L = 20
    bt = _mla_batch(L, 2, seed=6)
    S = np.full((L, 4), -1, np.int32)
    S[:, 0] = 3
    out, _ = O.sparse_mla(bt.seq_lens, bt.cu_q, bt.block_table, bt.q, bt.kv_cache, S, 0.1)
    c = _latent_rows(bt, 0, L)
    for t in range(L):
        assert np.array_equal(out[t], np.broadcast_to(c[3, :512], out[t].shape))


def test_sparse_mla_shift_invariant_and_order_free():
    L = 40
    bt = _mla_batch(L, 2, seed=8)
    rng = np.random.default_rng(1)
    S = np.stack([rng.permutation(L)[:16] for _ in range(L)]).astype(np.int32)
    o1, l1 = O.sparse_mla(bt.seq_lens, bt.cu_q, bt.block_table, bt.q, bt.kv_cache, S, 0.07)
    o2, l2 = O.sparse_mla(bt.seq_lens, bt.cu_q, bt.block_table, bt.q, bt.kv_cache, S[:, ::-1].copy(), 0.07)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)


# ---------------------------------------------------------------------------------------------
# masked MHA mode for short prefill: the expanded heads with the DSA mask

def _bf16_values(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def test_masked_mha_hand_worked():
    """One head, tau = 1, S_2 = {0, 1}: logits 0 and ln 3 give weights 1/4 and 3/4; position 2 has
    the largest logit but is not in S_2 and must not count."""
    q = np.zeros((3, 1, 2))
    q[2, 0] = [1.0, 0.0]
    k = np.array([[[0.0, 0.0]], [[math.log(3.0), 0.0]], [[5.0, 0.0]]])
    v = np.array([[[4.0, 0.0]], [[0.0, 8.0]], [[100.0, 100.0]]])
    S = np.array([[0, -1], [0, -1], [1, 0]], np.int32)
    out, lse = O.masked_mha([3], [0, 3], q, k, v, S, 1.0, rows=[2])
    np.testing.assert_allclose(out[2, 0], [1.0, 6.0], rtol=1e-14)
    np.testing.assert_allclose(lse[2, 0], math.log(4.0), rtol=1e-14)


def test_masked_mha_dense_when_sets_cover_prefix():
    """With S_t = [0, p] the masked mode is causal multi-head attention (torch SDPA, per request)."""
    lens, H = [37, 70], 3
    wl = synth.custom("mha", lens, lens, n_heads=H)
    x = synth.make_mha_inputs(wl, seed=3)
    tau = O.default_softmax_scale()
    cu = [0, lens[0], lens[0] + lens[1]]
    S = np.full((sum(lens), max(lens)), -1, np.int32)
    for b, n in enumerate(lens):
        for i in range(n):
            S[cu[b] + i, : i + 1] = np.arange(i + 1)
    out, lse = O.masked_mha(lens, cu, x.q, x.k, x.v, S, tau)
    q, k, v = (_bf16_values(a) for a in (x.q, x.k, x.v))
    for b, n in enumerate(lens):
        sl = slice(cu[b], cu[b] + n)
        per_head = lambda a: np.ascontiguousarray(a[sl].transpose(1, 0, 2))
        causal = np.where(np.tril(np.ones((n, n), bool)), 0.0, -np.inf)
        ref = _sdpa(per_head(q), per_head(k), per_head(v), causal, tau)
        np.testing.assert_allclose(out[sl], ref.transpose(1, 0, 2), rtol=1e-10, atol=1e-12)
        logits = tau * np.einsum("thd,jhd->thj", q[sl], k[sl]) + causal[:, None, :]
        np.testing.assert_allclose(lse[sl], torch.logsumexp(torch.from_numpy(logits), -1).numpy(), rtol=1e-12)


def test_masked_mha_emulates_absorbed_sparse_mla():
    """The masked MHA mode computes DSA: with k_jh = [W_UK_h c_j[:512], c_j[512:]], v_jh = W_UV_h c_j[:512]
    and the absorbed query [W_UK_h^T q_nope, q_rope], its output is the absorbed sparse MLA's output
    mapped by W_UV_h, on the same S_t (sparse sets, several heads, a ragged two-request batch)."""
    lens, H, kk = [50, 81], 3, 13
    wl = synth.custom("mha_vs_mla", lens, lens, n_heads_index=2, topk=kk, n_heads=H)
    bt = synth.make_batch(wl, seed=5, extra_pages=2)
    rng = np.random.default_rng(9)
    T = sum(lens)
    W_uk = rng.standard_normal((H, 128, 512)) / math.sqrt(512)
    W_uv = rng.standard_normal((H, 128, 512)) / math.sqrt(512)
    q_nope = rng.standard_normal((T, H, 128))
    q_rope = rng.standard_normal((T, H, 64))
    req, pos = O.query_positions(bt.seq_lens, bt.cu_q)
    c = np.zeros((T, 576))                      # latent row of every (request, position) = query row
    for t in range(T):
        c[t] = _latent_rows(bt, int(req[t]), int(pos[t]) + 1)[int(pos[t])]
    k_mha = np.concatenate([np.einsum("hde,te->thd", W_uk, c[:, :512]),
                            np.broadcast_to(c[:, None, 512:], (T, H, 64))], axis=2)
    v_mha = np.einsum("hde,te->thd", W_uv, c[:, :512])
    q_mha = np.concatenate([q_nope, q_rope], axis=2)
    q_abs = np.concatenate([np.einsum("hde,thd->the", W_uk, q_nope), q_rope], axis=2)
    S = synth.random_index_sets(lens, lens, kk, seed=2)
    tau = O.default_softmax_scale()
    o_mha, lse_mha = O.masked_mha(bt.seq_lens, bt.cu_q, q_mha, k_mha, v_mha, S, tau)
    o_mla, lse_mla = O.sparse_mla(bt.seq_lens, bt.cu_q, bt.block_table, q_abs, bt.kv_cache, S, tau)
    np.testing.assert_allclose(o_mha, np.einsum("hde,the->thd", W_uv, o_mla), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(lse_mha, lse_mla, rtol=1e-12, atol=1e-12)


def test_masked_mha_single_position_and_set_semantics():
    lens, H = [40], 2
    wl = synth.custom("mha1", lens, lens, n_heads=H)
    x = synth.make_mha_inputs(wl, seed=4)
    S = np.full((40, 6), -1, np.int32)
    S[:, 0] = 0
    out, _ = O.masked_mha(lens, [0, 40], x.q, x.k, x.v, S, 0.1)
    v = _bf16_values(x.v)
    for t in range(40):
        assert np.array_equal(out[t], v[0])
    S2 = synth.random_index_sets(lens, lens, 5, seed=1)
    dup = np.concatenate([S2, S2[:, :1]], axis=1)  # a position listed twice counts once
    o1, l1 = O.masked_mha(lens, [0, 40], x.q, x.k, x.v, S2, 0.1)
    o2, l2 = O.masked_mha(lens, [0, 40], x.q, x.k, x.v, dup, 0.1)
    np.testing.assert_allclose(o1, o2, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-14)


def test_random_index_sets_are_valid():
    S = synth.random_index_sets([300, 5], [300, 2], 64, seed=0)
    _, pos = O.query_positions([300, 5], [0, 300, 302])
    for t in range(S.shape[0]):
        sel = S[t][S[t] >= 0]
        assert sel.size == min(64, pos[t] + 1) and np.unique(sel).size == sel.size
        assert sel.max() <= pos[t] and np.all(S[t][sel.size:] == -1)


def test_softmax_scale_reading():
    assert O.default_softmax_scale() == 1.0 / math.sqrt(192.0)


# ---------------------------------------------------------------------------------------------
# cost model against the page's printed table

def test_cost_model_matches_printed_table(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "cost_table_p1.json")))
    assert round(CM.pair_flops_mla_absorbed() / 1e3) == g["pair_flops_mla_k"]
    assert round(CM.pair_flops_indexer() / 1e3) == g["pair_flops_indexer_k"]
    assert round(100 * CM.bytes_per_token_index() / CM.bytes_per_token_latent()) == g["index_cache_overhead_pct"]
    assert round(CM.pair_flops_mha_expanded() / 1e3) == g["pair_flops_mha_expanded_k"]
    assert round(CM.pair_flops_mla_absorbed() / CM.pair_flops_mha_expanded(), 1) == g["absorbed_over_expanded"]
    for row in g["rows"]:
        dec, rd, pre = CM.per_layer_costs(row["L"])
        assert [round(x / 1e9, 2) for x in dec] == row["decode_gflops"]
        assert round(dec[0] / dec[1], 1) == row["decode_ratio"]
        assert [round(x / 2 ** 20, 1) for x in rd] == row["read_mib"]
        assert round(rd[0] / rd[1], 1) == row["read_ratio"]
        assert [round(x / 1e12, 1) for x in pre] == row["prefill_tflops"]
        assert round(pre[0] / pre[1], 1) == row["prefill_ratio"]


def test_topk_nan_scores_rank_below_everything():
    """The pages leave NaN scores undefined; the library's reading: a NaN score ranks below every
    other score, -inf included, and NaNs tie (the smaller position first)."""
    s = np.array([1.0, np.nan, -np.inf, 2.0, np.nan, 0.0, -0.0])
    assert O.topk_select(s, 7).tolist() == [3, 0, 5, 6, 2, 1, 4]
    assert sorted(O.topk_select(s, 4).tolist()) == [0, 3, 5, 6]

"""CPU oracle of the DeepSeek Sparse Attention (DSA) hot path.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU-baseline leg
may import this module; the library never calls it and shares no code with it.

Plain, slow and written to be checked by eye against the formulas on the pages, in float64,
from the FP8 / bf16 storage codes (decoded here by this module's own routines). Positions are
0-based: the pages' C_t = {1..t} becomes j in [0, p].

Sources ("page" = title of the web page):
  [P5-LI]  "DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Lightning Indexer：为
           历史位置打分并选出 top-k": I_tj = sum_r w_tr ReLU(q_tr . k_j) over visible j <= t; one
           shared key per position; S_t = TopK_{j<=t}(I_tj, k); S_t shared by all attention heads;
           worked example t=8, k=3 -> S_8 = {2,5,8}.
  [P5-SA]  same page, section "Sparse Attention：在选中位置上计算 Attention": softmax(QK^T/sqrt(d_h)
           + M^DSA) V with M = 0 on S_t and -inf elsewhere, computed by reading only the rows in S_t.
  [P5-SWA] same page, section "SWA：让固定窗口沿序列移动": causal visibility C_t = {1..t}.
  [P1-DSA] "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA": 64 FP8 indexer heads of
           width 128, top 2048, absorbed MLA over a 576-wide latent (512 + 64 rope), per-pair FLOP
           counts; expanded head width 128 + 64 = 192; k = min(L, 2048); for short prefill,
           DeepSeek-V3.2 emulates DSA with a masked multi-head attention in the expanded form
           (q.k over 128 + 64 dims and p.v over 128 dims per head).

Readings where the pages leave a step open (each is listed in the design notes):
  * FP8 is OCP e4m3fn; per-token fp32 scales multiply the decoded codes (s^q_t for the query,
    s^k_j for the key). Positive scales pass through ReLU unchanged.
  * Query i of request b (m_b queries, n_b cached positions including them) sits at position
    p = n_b - m_b + i and sees j in [0, p] (self included).
  * TopK ties: higher score first, then smaller j. If p+1 <= k every visible position is selected.
  * Softmax scale tau = 1/sqrt(192) (expanded head width); V = first 512 latent dims.
"""
from __future__ import annotations

import math

import numpy as np

PAGE = 64
D_V = 512


# ---------------------------------------------------------------------------------------------
# storage decoders

def e4m3_decode(codes) -> np.ndarray:
    """Decode OCP FP8 E4M3 (e4m3fn) codes to float64.

    Bit layout s.eeee.mmm, exponent bias 7. Exponent field 0 gives subnormals (m/8)*2^-6;
    otherwise (1 + m/8)*2^(e-7). There are no infinities; s.1111.111 is NaN.
    """
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    mant = (c & 0x7).astype(np.float64)
    normal = (1.0 + mant / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    subnormal = (mant / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, subnormal, normal)
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, v)


_E4M3_TABLE = None


def e4m3_lookup(codes) -> np.ndarray:
    """e4m3_decode through a 256-entry table built by e4m3_decode itself (same values, faster)."""
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        _E4M3_TABLE = e4m3_decode(np.arange(256, dtype=np.uint8))
    return _E4M3_TABLE[np.asarray(codes).astype(np.uint8)]


def bf16_decode(bits) -> np.ndarray:
    """Decode bf16 bit patterns (the upper half of an IEEE float32) to float64."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _values(x) -> np.ndarray:
    """bf16 bit patterns (uint16 arrays) decoded to float64; float arrays are taken as values."""
    x = np.asarray(x)
    return bf16_decode(x) if x.dtype == np.uint16 else x.astype(np.float64)


def e4m3_encode(values) -> np.ndarray:
    """OCP FP8 E4M3 (e4m3fn) codes of finite float32 values: the nearest representable value,
    ties to the even code, magnitudes above 448 saturating to 448; the sign of zero is kept.

    Brute force over the magnitudes e4m3_decode gives codes 0x00..0x7E (0 .. 448), so the rounding
    can be checked by eye: among the magnitudes nearest to |v|, the even code wins.
    """
    v = np.asarray(values, np.float32).astype(np.float64)  # exact widening
    mags = e4m3_decode(np.arange(0x7F, dtype=np.uint8))     # 127 non-negative finite magnitudes
    codes_all = np.arange(0x7F)
    mag = np.minimum(np.abs(v), 448.0)
    dist = np.abs(mag[..., None] - mags)
    nearest = dist == dist.min(axis=-1, keepdims=True)     # one code, or two at an exact midpoint
    big = 1 << 20
    even = np.where(nearest & (codes_all % 2 == 0), codes_all, big).min(axis=-1)
    anyc = np.where(nearest, codes_all, big).min(axis=-1)
    code = np.where(even < big, even, anyc)
    return (code | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


# ---------------------------------------------------------------------------------------------
# batch geometry

def query_positions(seq_lens, cu_q):
    """(request b, position p) of every query row; query i of request b sits at n_b - m_b + i."""
    seq_lens = np.asarray(seq_lens, np.int64)
    cu_q = np.asarray(cu_q, np.int64)
    T = int(cu_q[-1]) if len(cu_q) else 0
    req = np.zeros(T, np.int64)
    pos = np.zeros(T, np.int64)
    for b in range(len(seq_lens)):
        m = int(cu_q[b + 1] - cu_q[b])
        for i in range(m):
            req[cu_q[b] + i] = b
            pos[cu_q[b] + i] = int(seq_lens[b]) - m + i
    return req, pos


def physical_rows(block_table_row, positions):
    """(page, slot) holding logical positions of one request: page = table[j // 64], slot = j % 64."""
    positions = np.asarray(positions, np.int64)
    pages = np.asarray(block_table_row, np.int64)[positions // PAGE]
    return pages, positions % PAGE


# ---------------------------------------------------------------------------------------------
# step 1: Lightning-Indexer scores  [P5-LI], FP8 per [P1-DSA]

def index_scores_row(t, req, pos, block_table, qI, qI_scale, wI, kI_cache, kI_scale) -> np.ndarray:
    """I_t = [I_t0 .. I_tp] for query row t, float64.

    I_tj = sum_r w_tr * ReLU( (s^q_t q_tr) . (s^k_j k_j) ).
    """
    b, p = int(req[t]), int(pos[t])
    pages, slots = physical_rows(block_table[b], np.arange(p + 1))
    k = e4m3_lookup(kI_cache[pages, slots]) * np.asarray(kI_scale, np.float64)[pages, slots][:, None]
    qt = e4m3_lookup(qI[t]) * float(qI_scale[t])            # [nhI, 128]
    logits = qt @ k.T                                        # [nhI, p+1]: q_tr . k_j
    return np.asarray(wI[t], np.float64) @ np.maximum(logits, 0.0)


def index_scores(seq_lens, cu_q, block_table, qI, qI_scale, wI, kI_cache, kI_scale, ld=None, rows=None):
    """Score matrix [T, ld] (float64); -inf at j > p (never visible). `rows` limits the work."""
    req, pos = query_positions(seq_lens, cu_q)
    T = len(req)
    if ld is None:
        ld = int(np.max(seq_lens)) if len(seq_lens) else 0
    out = np.full((T, ld), -np.inf)
    for t in (range(T) if rows is None else rows):
        out[t, : int(pos[t]) + 1] = index_scores_row(t, req, pos, block_table, qI, qI_scale, wI,
                                                     kI_cache, kI_scale)
    return out


# ---------------------------------------------------------------------------------------------
# step 2: TopK  [P5-LI]; k = min(L, TOPK) per [P1-DSA]

def topk_select(scores_row, k) -> np.ndarray:
    """S_t as int32[k]: positions of the min(k, L) largest scores (ties: smaller j first),
    in descending score order, padded with -1. `scores_row` holds exactly the L visible scores."""
    s = np.asarray(scores_row)
    L = s.shape[0]
    order = np.lexsort((np.arange(L), -s.astype(np.float64)))   # by -I, then by j
    out = np.full(k, -1, np.int32)
    take = min(k, L)
    out[:take] = np.asarray(order[:take], np.int32)
    return out


def topk(scores, pos, k, rows=None) -> np.ndarray:
    """Index sets for every row of a score matrix; row t sees its first pos[t]+1 columns."""
    T = scores.shape[0]
    out = np.full((T, k), -1, np.int32)
    for t in (range(T) if rows is None else rows):
        out[t] = topk_select(scores[t, : int(pos[t]) + 1], k)
    return out


# ---------------------------------------------------------------------------------------------
# step 3: sparse MLA on S_t  [P5-SA]; absorbed MLA form per [P1-DSA]

def sparse_mla_row(t, req, S_t, block_table, q, kv_cache, softmax_scale):
    """Attention of query row t over the latent rows in S_t (entries < 0 are padding).

    z_hj = tau * q_th . c_j (576 dims); o_th = sum_j softmax_j(z_hj) c_j[0:512];
    lse_th = log sum_j exp(z_hj). Returns (o [H, 512], lse [H]) in float64.
    """
    b = int(req[t])
    sel = np.asarray([j for j in S_t if j >= 0], np.int64)
    qt = _values(q[t])                                        # [H, 576]
    H = qt.shape[0]
    if sel.size == 0:
        return np.zeros((H, D_V)), np.full(H, -np.inf)
    pages, slots = physical_rows(block_table[b], sel)
    c = _values(kv_cache[pages, slots])                       # [|S_t|, 576]
    z = softmax_scale * (qt @ c.T)                            # [H, |S_t|]
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    denom = e.sum(axis=1, keepdims=True)
    o = (e @ c[:, :D_V]) / denom
    lse = zmax[:, 0] + np.log(denom[:, 0])
    return o, lse


def sparse_mla(seq_lens, cu_q, block_table, q, kv_cache, S, softmax_scale, rows=None):
    """Output [T, H, 512] and lse [T, H] (float64) for every (or the given) query row."""
    req, _ = query_positions(seq_lens, cu_q)
    T, H = q.shape[0], q.shape[1]
    out = np.zeros((T, H, D_V))
    lse = np.full((T, H), -np.inf)
    for t in (range(T) if rows is None else rows):
        out[t], lse[t] = sparse_mla_row(t, req, S[t], block_table, q, kv_cache, softmax_scale)
    return out, lse


# ---------------------------------------------------------------------------------------------
# writing new positions into the two caches: per token the latent row in bf16 and the indexer key
# as FP8 plus a 4-byte scale, the indexer keys paged like the latent rows [P1-DSA]; one indexer key
# per position, shared by every indexer head and kept in its own key cache [P5-LI]

def indexer_key_quantize(k_row):
    """(codes uint8[d], scale float32) of one new indexer key.

    Reading of "FP8 + a 4-byte scale per token": s = max_d |k_d| / 448 in float32 (1 when the key is
    all zeros), codes = e4m3(k_d / s) with the division in float32 (correctly rounded).
    """
    k = np.asarray(k_row, np.float32)
    amax = np.float32(np.max(np.abs(k)))
    s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
    return e4m3_encode((k / s).astype(np.float32)), s


def cache_write(seq_lens, cu_q, block_table, k_new, c_new_bits, kI_cache, kI_scale, kv_cache):
    """The three caches after writing every query row's own position (updated copies).

    Query row t (request b, position p) stores its indexer key at kI_cache[page][p % 64] with the
    scale at kI_scale[page][p % 64], and its latent row (bf16 bits) at kv_cache[page][p % 64],
    page = block_table[b][p // 64]. Every other slot keeps its contents.
    """
    req, pos = query_positions(seq_lens, cu_q)
    kI, ks, kv = np.array(kI_cache, copy=True), np.array(kI_scale, copy=True), np.array(kv_cache, copy=True)
    for t in range(len(req)):
        pages, slots = physical_rows(block_table[req[t]], [pos[t]])
        codes, s = indexer_key_quantize(k_new[t])
        kI[pages[0], slots[0]] = codes
        ks[pages[0], slots[0]] = s
        kv[pages[0], slots[0]] = c_new_bits[t]
    return kI, ks, kv


# ---------------------------------------------------------------------------------------------
# masked MHA mode for short prefill [P1-DSA]: the expanded multi-head form (per head, q and k of
# width 128 + 64, v of width 128) with the DSA mask of [P5-SA], M = 0 on S_t and -inf elsewhere

def masked_mha_row(t, req, pos, cu_q, seq_lens, S_t, q, k, v, softmax_scale):
    """Masked MHA of query row t, float64: (o [H, dv], lse [H]).

    Every request is a whole prefill (m_b = n_b): row cu_q[b] + j of k and v holds position j of
    request b. With K_b, V_b the request's rows,
        z_h = tau * q_th K_bh^T + M_t,   M_tj = 0 for j in S_t, -inf for every other j < n_b,
        o_th = softmax(z_h) V_bh,        lse_th = log sum_j exp(z_hj).
    Entries of S_t below 0 are padding; a position listed twice is still one position of the set.
    """
    b, p = int(req[t]), int(pos[t])
    n = int(seq_lens[b])
    lo = int(cu_q[b])
    assert int(cu_q[b + 1]) - lo == n, "masked MHA mode: every request is a whole prefill"
    sel = np.asarray([j for j in S_t if j >= 0], np.int64)
    assert np.all(sel <= p), "S_t holds visible positions only"
    qt = _values(q[t])                                        # [H, dqk]
    Kb = _values(k[lo:lo + n])                                # [n, H, dqk]
    Vb = _values(v[lo:lo + n])                                # [n, H, dv]
    H, dv = qt.shape[0], Vb.shape[2]
    M = np.full(n, -np.inf)
    M[sel] = 0.0
    if sel.size == 0:
        return np.zeros((H, dv)), np.full(H, -np.inf)
    z = softmax_scale * np.einsum("hd,jhd->hj", qt, Kb) + M[None, :]   # [H, n]
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)                                      # exp(-inf) = 0 off the mask
    denom = e.sum(axis=1, keepdims=True)
    o = np.einsum("hj,jhd->hd", e, Vb) / denom
    return o, zmax[:, 0] + np.log(denom[:, 0])


def masked_mha(seq_lens, cu_q, q, k, v, S, softmax_scale, rows=None):
    """Output [T, H, dv] and lse [T, H] (float64) of the masked MHA mode for every (or the given) row."""
    req, pos = query_positions(seq_lens, cu_q)
    T, H = q.shape[0], q.shape[1]
    dv = v.shape[2]
    out = np.zeros((T, H, dv))
    lse = np.full((T, H), -np.inf)
    for t in (range(T) if rows is None else rows):
        out[t], lse[t] = masked_mha_row(t, req, pos, cu_q, seq_lens, S[t], q, k, v, softmax_scale)
    return out, lse


# ---------------------------------------------------------------------------------------------
# the whole path

def dsa_layer(seq_lens, cu_q, block_table, qI, qI_scale, wI, kI_cache, kI_scale, q, kv_cache,
              k, softmax_scale, rows=None):
    """Indexer -> TopK -> sparse MLA for every (or the given) query row.

    Returns dict(scores [T, ld] f64, S [T, k] int32, out [T, H, 512] f64, lse [T, H] f64).
    """
    _, pos = query_positions(seq_lens, cu_q)
    scores = index_scores(seq_lens, cu_q, block_table, qI, qI_scale, wI, kI_cache, kI_scale, rows=rows)
    S = topk(scores, pos, k, rows=rows)
    out, lse = sparse_mla(seq_lens, cu_q, block_table, q, kv_cache, S, softmax_scale, rows=rows)
    return dict(scores=scores, S=S, out=out, lse=lse)


def default_softmax_scale() -> float:
    """tau = 1/sqrt(d_h) with the expanded head width d_h = 128 + 64 = 192 [P1-DSA], [P5-SA]."""
    return 1.0 / math.sqrt(128 + 64)

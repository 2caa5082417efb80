"""Seeded synthetic inputs for the DSA hot path.

This module only DRAWS inputs: random numbers, their storage encodings (FP8 e4m3 codes with a
per-token fp32 scale, bf16 bit patterns), the planted "needle" keys and the paged cache layout.
It holds none of the method's arithmetic (no scores, no selection, no attention); both the CPU
oracle and the CUDA path consume exactly what it returns.

Workload shapes follow the DSA configuration on the pages:
  * "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA": 64 indexer heads of width 128
    computed in FP8, top-2048 selection, absorbed MLA with 128 heads over a 512+64 latent, and an
    indexer key cache of 128 FP8 bytes plus a 4-byte scale per token.
  * "DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Lightning Indexer": one shared
    indexer key per position, per-query head weights w_t, causal visibility j <= t.
Page size 64 is the paged-cache granularity the serving commands on the pages use.

Random draws use numpy's PCG64: the page permutation and the needles from SeedSequence([seed,
workload_id]), every large array from SeedSequence([seed, workload_id, array tag]) in blocks of
whole rows, each block from its own spawned child (drawn on host threads; the values do not
depend on the thread count).
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

PAGE = 64          # positions per cache page
D_INDEX = 128      # indexer head width d_h^I
D_LATENT = 576     # MLA latent width: 512 "nope" + 64 rope
D_V = 512          # value width (first 512 latent dims)
FP8_MAX = 448.0    # largest finite e4m3fn magnitude


@dataclasses.dataclass(frozen=True)
class Workload:
    """Sizes of one synthetic DSA batch.

    seq_lens: n_b, positions cached for request b, its own query tokens included.
    q_per_req: m_b, query tokens of request b; query i sits at position n_b - m_b + i.
    """
    name: str
    wid: int                      # workload id, part of the seed
    seq_lens: tuple               # n_b per request
    q_per_req: tuple              # m_b per request
    n_heads_index: int            # n_h^I
    topk: int                     # k
    n_heads: int                  # H, MLA attention heads
    needles: str = "none"         # needle recipe
    n_needles: int = 0
    softmax_scale: float = 1.0 / math.sqrt(192.0)

    @property
    def batch(self) -> int:
        return len(self.seq_lens)

    @property
    def total_q(self) -> int:
        return int(sum(self.q_per_req))


def _log_uniform_lengths(rng: np.random.Generator, b: int, lo: int, hi: int) -> tuple:
    u = rng.uniform(math.log(lo), math.log(hi), size=b)
    return tuple(int(x) for x in np.floor(np.exp(u)).astype(np.int64))


def workload(name: str, seed: int = 0) -> Workload:
    """The five workload shapes, by name.

    prefill_2048      1 sequence, L=2048, 16 indexer heads, k=512, 16 MLA heads, 8 needles.
    decode_64x16k     64 requests x 16384 positions, 1 query each, k=2048, 32 needles/request.
    mtp_16x128k       16 requests x 131072 positions, 2 causal queries each (main + draft).
    prefill_32k       1 sequence, L=32768, k=2048, 64 needles at log-uniform distances.
    mixed_128         128 requests, lengths log-uniform in [4096, 131072], 1 query each.
    """
    if name == "prefill_2048":
        return Workload(name, 1, (2048,), (2048,), 16, 512, 16, "prefill", 8)
    if name == "decode_64x16k":
        return Workload(name, 2, (16384,) * 64, (1,) * 64, 64, 2048, 128, "decode", 32)
    if name == "mtp_16x128k":
        return Workload(name, 3, (131072,) * 16, (2,) * 16, 64, 2048, 128, "decode", 32)
    if name == "prefill_32k":
        return Workload(name, 4, (32768,), (32768,), 64, 2048, 128, "prefill_logdist", 64)
    if name == "mixed_128":
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 5, 1])))
        lens = _log_uniform_lengths(rng, 128, 4096, 131072)
        return Workload(name, 5, lens, (1,) * 128, 64, 2048, 128, "none", 0)
    if name.startswith("prefill_") and name[len("prefill_"):].isdigit():
        # prefill_32k's shape at another length L (smaller cases of the same kernels, for profiling)
        L = int(name[len("prefill_"):])
        return Workload(name, 6, (L,), (L,), 64, 2048, 128, "prefill_logdist", max(1, L // 512))
    raise KeyError(name)


WORKLOADS = ("prefill_2048", "decode_64x16k", "mtp_16x128k", "prefill_32k", "mixed_128")


def custom(name: str, seq_lens, q_per_req, n_heads_index=64, topk=2048, n_heads=128,
           needles="none", n_needles=0, wid=99) -> Workload:
    """A workload with explicit sizes (tests: ragged tails, tiny cases, edge cases)."""
    return Workload(name, wid, tuple(int(x) for x in seq_lens), tuple(int(x) for x in q_per_req),
                    n_heads_index, topk, n_heads, needles, n_needles)


# ---------------------------------------------------------------------------------------------
# storage encodings (input preparation, not part of the method)

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest even) and return the 16-bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def quantize_e4m3_per_token(x: np.ndarray):
    """Per-token FP8 quantisation: scale = absmax/448 over the trailing axes (1 if absmax is 0),
    codes = e4m3fn(x / scale) with round-to-nearest-even, saturating at +-448.

    The rounding itself is done by torch's float8_e4m3fn cast. Returns (codes uint8, scale f32).
    """
    import torch
    x = np.asarray(x, dtype=np.float32)
    lead = x.shape[0]
    flat = x.reshape(lead, -1)
    codes = np.empty(flat.shape, np.uint8)
    scale = np.empty(lead, np.float32)

    def work(lo, hi):
        amax = np.abs(flat[lo:hi]).max(axis=1)
        sc = np.where(amax > 0, amax / np.float32(FP8_MAX), np.float32(1.0)).astype(np.float32)
        y = np.clip(flat[lo:hi] / sc[:, None], -FP8_MAX, FP8_MAX).astype(np.float32)
        codes[lo:hi] = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        scale[lo:hi] = sc

    _row_blocks(work, lead, max(1, _BLOCK_ELEMS // max(1, flat.shape[1])))
    return codes.reshape(x.shape), scale


# ---------------------------------------------------------------------------------------------
# batch generation

@dataclasses.dataclass
class Batch:
    """One batch in the layouts the library takes (all numpy, host side).

    qI        uint8  [T, nhI, 128]    e4m3 codes of the indexer queries
    qI_scale  f32    [T]              per-token scale of qI
    wI        f32    [T, nhI]         per-query head weights w_t
    kI_cache  uint8  [P, 64, 128]     e4m3 codes of the indexer keys, paged
    kI_scale  f32    [P, 64]          per-token scale of kI
    q         uint16 [T, H, 576]      bf16 bits of the (absorbed) MLA queries
    kv_cache  uint16 [P, 64, 576]     bf16 bits of the latent rows, paged
    block_table int32 [B, max_pages]  physical page of logical page i of request b (-1 unused)
    seq_lens  int32  [B]
    cu_q      int32  [B+1]
    needles   list of (query row, key position)
    """
    wl: Workload
    qI: np.ndarray
    qI_scale: np.ndarray
    wI: np.ndarray
    kI_cache: np.ndarray
    kI_scale: np.ndarray
    q: np.ndarray
    kv_cache: np.ndarray
    block_table: np.ndarray
    seq_lens: np.ndarray
    cu_q: np.ndarray
    needles: list

    @property
    def total_q(self) -> int:
        return int(self.cu_q[-1])

    @property
    def num_pages(self) -> int:
        return int(self.kI_cache.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if len(self.seq_lens) else 0

    def row_positions(self):
        """(request, position) of every query row: query i of request b at n_b - m_b + i."""
        req = np.empty(self.total_q, np.int64)
        pos = np.empty(self.total_q, np.int64)
        for b in range(len(self.seq_lens)):
            lo, hi = int(self.cu_q[b]), int(self.cu_q[b + 1])
            req[lo:hi] = b
            pos[lo:hi] = int(self.seq_lens[b]) - (hi - lo) + np.arange(hi - lo)
        return req, pos


# Large arrays are drawn in blocks of whole leading rows (about _BLOCK_ELEMS values each), every
# block from its own child of the array's SeedSequence, on a pool of host threads. The values do
# not depend on the number of threads.
_BLOCK_ELEMS = 1 << 22


def _row_blocks(fn, n_rows: int, rows_per_block: int):
    """fn(lo, hi) over consecutive row blocks, on a thread pool (numpy and torch release the GIL)."""
    spans = [(lo, min(n_rows, lo + rows_per_block)) for lo in range(0, n_rows, rows_per_block)]
    if len(spans) <= 1:
        for lo, hi in spans:
            fn(lo, hi)
        return
    workers = max(1, min(32, len(os.sched_getaffinity(0)), len(spans)))
    with ThreadPoolExecutor(workers) as ex:
        for f in [ex.submit(fn, lo, hi) for lo, hi in spans]:
            f.result()


def _normal(ss: np.random.SeedSequence, shape, as_bf16: bool) -> np.ndarray:
    """N(0,1) draws of `shape`, float32 or stored as bf16 bits."""
    out = np.empty(shape, np.uint16 if as_bf16 else np.float32)
    n_rows = int(shape[0])
    flat = out.reshape(n_rows, -1)
    rows_per_block = max(1, _BLOCK_ELEMS // max(1, flat.shape[1]))
    children = ss.spawn((n_rows + rows_per_block - 1) // rows_per_block)

    def work(lo, hi):
        g = np.random.Generator(np.random.PCG64(children[lo // rows_per_block]))
        if as_bf16:
            flat[lo:hi] = f32_to_bf16_bits(g.standard_normal((hi - lo, flat.shape[1]), dtype=np.float32))
        else:
            g.standard_normal((hi - lo, flat.shape[1]), dtype=np.float32, out=flat[lo:hi])

    _row_blocks(work, n_rows, rows_per_block)
    return out


def _seq(seed: int, wl: "Workload", tag: int) -> np.random.SeedSequence:
    return np.random.SeedSequence([seed, wl.wid, tag])


def make_batch(wl: Workload, seed: int = 0, extra_pages: int = 0) -> Batch:
    """Draw one batch. Pages are a random permutation of the pool; slots past n_b on a request's
    last page hold random data too (they must never be read as visible positions)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, wl.wid])))
    B = wl.batch
    seq_lens = np.asarray(wl.seq_lens, np.int32)
    m = np.asarray(wl.q_per_req, np.int32)
    assert np.all(m >= 0) and np.all(m <= seq_lens), "each request needs m_b <= n_b"
    cu_q = np.zeros(B + 1, np.int32)
    cu_q[1:] = np.cumsum(m)
    T = int(cu_q[-1])
    pages_per_req = [(int(n) + PAGE - 1) // PAGE for n in seq_lens]
    P = int(sum(pages_per_req)) + int(extra_pages)
    max_pages = max(1, max(pages_per_req) if pages_per_req else 1)
    perm = rng.permutation(P).astype(np.int32)
    block_table = np.full((B, max_pages), -1, np.int32)
    off = 0
    for b, npg in enumerate(pages_per_req):
        block_table[b, :npg] = perm[off:off + npg]
        off += npg

    nhI, H = wl.n_heads_index, wl.n_heads
    # indexer queries and head weights
    qI_f = _normal(_seq(seed, wl, 1), (T, nhI, D_INDEX), False)
    wI = (_normal(_seq(seed, wl, 2), (T, nhI), False) / np.float32(math.sqrt(nhI))).astype(np.float32)
    # indexer keys, one per logical position, float before quantisation
    kI_f = _normal(_seq(seed, wl, 3), (P, PAGE, D_INDEX), False)

    # needles: k_j <- 0.8 * q_{t, r*} + 0.2 * noise, r* = argmax_r w_tr
    needles = []
    row0 = cu_q[:-1]
    if wl.needles != "none" and wl.n_needles > 0 and T > 0:
        for b in range(B):
            mb = int(m[b])
            if mb == 0:
                continue
            nb = int(seq_lens[b])
            count = wl.n_needles
            for _ in range(count):
                if wl.needles == "decode":
                    i = int(rng.integers(0, mb))
                    p = nb - mb + i
                    j = int(rng.integers(0, p + 1))
                elif wl.needles == "prefill":
                    i = int(rng.integers(1, mb))
                    p = nb - mb + i
                    j = int(rng.integers(0, p))
                elif wl.needles == "prefill_logdist":
                    i = int(rng.integers(2, mb))
                    p = nb - mb + i
                    d = int(math.floor(math.exp(rng.uniform(0.0, math.log(p)))))
                    d = min(max(d, 1), p)
                    j = p - d
                else:
                    raise ValueError(wl.needles)
                t = int(row0[b]) + i
                r = int(np.argmax(wI[t]))
                page = block_table[b, j // PAGE]
                kI_f[page, j % PAGE] = (np.float32(0.8) * qI_f[t, r]
                                        + np.float32(0.2) * rng.standard_normal(D_INDEX, dtype=np.float32))
                needles.append((t, j))

    qI, qI_scale = quantize_e4m3_per_token(qI_f)
    kI_codes, kI_scale = quantize_e4m3_per_token(kI_f.reshape(P * PAGE, D_INDEX))
    kI_cache = kI_codes.reshape(P, PAGE, D_INDEX)
    kI_scale = kI_scale.reshape(P, PAGE)

    q = _normal(_seq(seed, wl, 4), (T, H, D_LATENT), True)
    kv_cache = _normal(_seq(seed, wl, 5), (P, PAGE, D_LATENT), True)
    return Batch(wl, qI, qI_scale, wI, kI_cache, kI_scale, q, kv_cache, block_table,
                 seq_lens, cu_q, needles)


# ---------------------------------------------------------------------------------------------
# inputs of the masked MHA mode for short prefill (expanded heads: q and k of width 128 + 64,
# v of width 128, one row per position of each whole-prefill request)

D_QK_MHA = 128 + 64
D_V_MHA = 128


@dataclasses.dataclass
class MhaInputs:
    """q, k uint16 [T, H, 192] and v uint16 [T, H, 128]: bf16 bits of N(0,1) draws; row cu_q[b] + j
    of k and v is position j of request b (every request a whole prefill, m_b = n_b)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray


def make_mha_inputs(wl: Workload, seed: int = 0) -> MhaInputs:
    assert tuple(wl.seq_lens) == tuple(wl.q_per_req), "the masked MHA mode takes whole prefills"
    T, H = wl.total_q, wl.n_heads
    q = _normal(np.random.SeedSequence([seed, wl.wid, 7, 0]), (T, H, D_QK_MHA), True)
    k = _normal(np.random.SeedSequence([seed, wl.wid, 7, 1]), (T, H, D_QK_MHA), True)
    v = _normal(np.random.SeedSequence([seed, wl.wid, 7, 2]), (T, H, D_V_MHA), True)
    return MhaInputs(q, k, v)


def random_index_sets(seq_lens, q_per_req, k: int, seed: int = 0) -> np.ndarray:
    """int32 [T, k]: for every query row (request b, position p = n_b - m_b + i) min(k, p + 1)
    distinct positions drawn uniformly from [0, p], in random order, padded with -1."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 11])))
    T = int(sum(q_per_req))
    out = np.full((T, k), -1, np.int32)
    t = 0
    for n, m in zip(seq_lens, q_per_req):
        for i in range(int(m)):
            p = int(n) - int(m) + i
            take = min(k, p + 1)
            out[t, :take] = rng.choice(p + 1, size=take, replace=False) if take < p + 1 else rng.permutation(p + 1)
            t += 1
    return out

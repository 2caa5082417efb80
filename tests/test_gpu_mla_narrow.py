"""The sparse MLA for few heads (H <= 16: keys and value dimensions on the MMA's M axis, heads on N)
against the oracle, through the C ABI.

Every case runs the GPU's sparse MLA on the oracle's own index sets and compares every output row
and its log-sum-exp with the oracle (max-abs 2e-2, mean-abs 2e-3 on the bf16 output). The cases
cover what the kernel's pipeline distinguishes:
  * 16 heads and fewer (15, 8, 5, 1: the padding columns of the N = 16 MMAs are never written);
  * units of one tile, of a ragged last tile, and of the most tiles a unit takes (16);
  * splits of S_t (few query rows) with units that have no tiles, and the combine step;
  * query rows whose visible positions are fewer than k (padded index sets);
  * a reference maximum that moves by more than 2^8 in the middle of a unit, which rescales the
    O^T accumulator in TMEM: the rope dims of late positions are scaled by 16 (exact in bf16), so
    the tiles that hold them carry far larger scores than the first tiles of the same unit.
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


def scale_rope_from(position: int, factor: float):
    """A batch edit: the rope dims (512..575) of every request's positions >= `position` times
    `factor` (a power of two, so the bf16 values stay exact)."""
    def tweak(hb):
        kv = hb.kv_cache
        for b, n in enumerate(hb.seq_lens):
            for j in range(position, int(n)):
                page = hb.block_table[b, j // synth.PAGE]
                row = kv[page, j % synth.PAGE]
                f = (row[512:].astype(np.uint32) << np.uint32(16)).view(np.float32) * np.float32(factor)
                row[512:] = synth.f32_to_bf16_bits(f)
    return tweak


def check_mla(wl, seed=0, rows=None, tweak=None):
    hb = synth.make_batch(wl, seed=seed, extra_pages=2)
    if tweak is not None:
        tweak(hb)
    db = dsa.DeviceBatch(hb)
    plan, _, _ = G.gpu_steps(db)
    T = hb.total_q
    rows = list(range(T)) if rows is None else list(rows)
    ref = G.oracle_scores(hb, rows)
    S_ref = np.full((T, db.k), -1, np.int32)
    for t in rows:
        S_ref[t] = O.topk_select(ref[t], db.k)
    lse = torch.full((T, db.H), float("nan"), dtype=torch.float32, device="cuda")
    out = dsa.sparse_mla(db.batch, plan, db.q, db.kv_cache, torch.from_numpy(S_ref).cuda(), db.softmax_scale,
                         lse=lse)
    torch.cuda.synchronize()
    assert dsa.status_read(plan) == 0
    return G.check_attention(hb, G.rows_to_host(out.float(), rows), G.rows_to_host(lse, rows),
                             {t: S_ref[t] for t in rows})


@pytest.mark.parametrize("H", [16, 15, 8, 5, 1])
def test_narrow_head_counts(H):
    wl = synth.custom(f"narrow_h{H}", [700, 300, 1500], [40, 3, 17], n_heads_index=16, topk=256, n_heads=H,
                      needles="prefill", n_needles=3)
    check_mla(wl, seed=H)


def test_narrow_sixteen_tiles_per_unit():
    # 48 rows, k = 2048: one unit per row of up to 16 tiles (the most a unit takes)
    wl = synth.custom("narrow_long", [3000, 2100], [40, 8], n_heads_index=64, topk=2048, n_heads=16)
    check_mla(wl, seed=4)


def test_narrow_splits_and_empty_units():
    # 6 decode rows: S_t is split over several units, rows with few visible positions leave some
    # of their units without tiles, and the combine merges the rest
    wl = synth.custom("narrow_decode", [300, 1000, 4097, 64, 1, 2100], [1] * 6, n_heads_index=64, topk=256,
                      n_heads=16, needles="decode", n_needles=4)
    check_mla(wl, seed=5)


def test_narrow_splits_of_long_rows():
    wl = synth.custom("narrow_mtp", [5000, 2600], [2, 2], n_heads_index=64, topk=2048, n_heads=8)
    check_mla(wl, seed=6)


def test_narrow_rescales_the_accumulator_mid_unit():
    # index sets are emitted in increasing position order, so within a unit the tiles of positions
    # >= 1200 come last; their scores are much larger than those of the first tiles
    wl = synth.custom("narrow_rescale", [2000, 1600], [24, 8], n_heads_index=64, topk=1024, n_heads=16)
    check_mla(wl, seed=7, tweak=scale_rope_from(1200, 16.0))


def test_narrow_workload_prefill_2048():
    check_mla(synth.workload("prefill_2048"))

"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and compare it with
the CPU oracle on the same seeded inputs.

Tolerances (written out here, derived in the design notes):
  * scores: |I_gpu - I_oracle| <= 1e-3 * |I_oracle| + 1e-6 * max_j |I_oracle,tj| (the relative
    1e-3 asked for, with a floor for scores near 0, where signed head weights can cancel: FP8
    products are exact in fp32, the error is fp32 accumulation and summation order).
  * index sets: equal, except that every position in the symmetric difference has an oracle
    score within 1e-3 * |I_(k)| of the k-th largest oracle score I_(k) (near-ties).
  * top-k alone, fed the GPU's own fp32 scores: identical sets (both break ties by position).
  * attention output (bf16) on the oracle's index sets: max |diff| <= 2e-2, mean |diff| <= 2e-3;
    log-sum-exp within 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import sparse_attention_12_b200 as dsa
from oracle import dsa_oracle as O


def to_np_bf16(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def rows_to_host(x: torch.Tensor, rows) -> dict:
    idx = torch.as_tensor(list(rows), dtype=torch.long, device=x.device)
    sel = x.index_select(0, idx).cpu().numpy()
    return {t: sel[i] for i, t in enumerate(rows)}


def gpu_steps(db: "dsa.DeviceBatch"):
    """Plan, scores, top-k on the GPU; returns (plan, scores, S) device tensors."""
    plan = dsa.plan(db.batch, db.nhI)
    scores = dsa.index_scores(db.batch, plan, db.qI, db.qI_scale, db.wI, db.kI_cache, db.kI_scale)
    S = dsa.topk(db.batch, plan, scores, db.k)
    return plan, scores, S


def oracle_scores(hb, rows) -> dict:
    req, pos = O.query_positions(hb.seq_lens, hb.cu_q)
    return {t: O.index_scores_row(t, req, pos, hb.block_table, hb.qI, hb.qI_scale, hb.wI, hb.kI_cache, hb.kI_scale)
            for t in rows}


def check_scores(ref: dict, got: dict, pos) -> float:
    worst = 0.0
    for t, r in ref.items():
        g = got[t][: pos[t] + 1].astype(np.float64)
        err = np.abs(g - r)
        bound = 1e-3 * np.abs(r) + 1e-6 * float(np.max(np.abs(r)))
        ratio = float(np.max(err / np.maximum(bound, 1e-30)))
        worst = max(worst, ratio)
        assert ratio <= 1.0, f"row {t}: score error {err.max():.3e} exceeds the bound (ratio {ratio:.2f})"
    return worst


def check_index_sets(ref: dict, S_got: dict, pos, k) -> int:
    n_diff_rows = 0
    for t, r in ref.items():
        want = O.topk_select(r, k)
        got = S_got[t]
        L = int(pos[t]) + 1
        take = min(k, L)
        assert np.all(got[take:] == -1), f"row {t}: padding"
        g = got[:take]
        assert np.all((g >= 0) & (g < L)), f"row {t}: out-of-range position"
        assert len(set(g.tolist())) == take, f"row {t}: duplicate positions"
        diff = set(g.tolist()) ^ set(want[:take].tolist())
        if diff:
            n_diff_rows += 1
            kth = np.sort(r)[::-1][take - 1]
            for j in diff:
                assert abs(r[j] - kth) <= 1e-3 * abs(kth), \
                    f"row {t}: position {j} differs and is not a near-tie ({r[j]} vs k-th {kth})"
    return n_diff_rows


def check_topk_exact(scores_got: dict, S_got: dict, pos, k):
    for t, s in scores_got.items():
        L = int(pos[t]) + 1
        want = O.topk_select(s[:L].astype(np.float64), k)
        assert set(S_got[t].tolist()) == set(want.tolist()), f"row {t}: top-k differs on identical scores"
        sel = S_got[t][: min(k, L)]
        assert np.all(np.diff(sel) > 0), f"row {t}: positions not increasing"


def check_attention(hb, out_got: dict, lse_got, S: dict):
    req, _ = O.query_positions(hb.seq_lens, hb.cu_q)
    max_err, sum_err, n = 0.0, 0.0, 0
    for t, St in S.items():
        o, l = O.sparse_mla_row(t, req, St, hb.block_table, hb.q, hb.kv_cache, hb.wl.softmax_scale)
        err = np.abs(out_got[t].astype(np.float64) - o)
        max_err = max(max_err, float(err.max()))
        sum_err += float(err.sum())
        n += err.size
        if lse_got is not None:
            assert np.allclose(lse_got[t], l, rtol=0, atol=1e-3), f"row {t}: lse differs"
    mean_err = sum_err / max(n, 1)
    assert max_err <= 2e-2, f"attention max-abs error {max_err:.3e}"
    assert mean_err <= 2e-3, f"attention mean-abs error {mean_err:.3e}"
    return max_err, mean_err

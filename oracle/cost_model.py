"""Algorithmic work of the DSA path: FLOPs per (query, key) pair and bytes per token.

TEST INFRASTRUCTURE ONLY (see dsa_oracle.py). Restates the cost model of the page
"MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA" (the dense-vs-DSA comparison and
its printed table), so that the tests can check it against the values printed there.
"""
from __future__ import annotations

H, DC, ROPE = 128, 512, 64          # attention heads, latent "nope" width, rope width
IDX_H, IDX_D, TOPK = 64, 128, 2048  # indexer heads, indexer head width, selected positions


def pair_flops_mla_absorbed(h=H, dc=DC, rope=ROPE) -> int:
    """q.c over 576 dims plus p.v over 512 dims, for every head (multiply-add = 2 FLOPs)."""
    return 2 * h * (dc + rope) + 2 * h * dc


def pair_flops_mha_expanded(h=H, rope=ROPE, head=128) -> int:
    """Expanded (non-absorbed) heads of width 128 + 64 for q.k and 128 for p.v."""
    return 2 * h * (head + rope) + 2 * h * head


def pair_flops_indexer(nh=IDX_H, d=IDX_D) -> int:
    return 2 * nh * d


def bytes_per_token_latent(dc=DC, rope=ROPE) -> int:
    """bf16 latent row."""
    return (dc + rope) * 2


def bytes_per_token_index(d=IDX_D) -> int:
    """FP8 key plus a 4-byte scale."""
    return d + 4


def per_layer_costs(L: int, topk: int = TOPK):
    """(decode FLOPs dense, DSA), (decode bytes dense, DSA), (prefill FLOPs dense, DSA) at context L."""
    k = min(L, topk)
    pm, pe, pi = pair_flops_mla_absorbed(), pair_flops_mha_expanded(), pair_flops_indexer()
    kv, ib = bytes_per_token_latent(), bytes_per_token_index()
    dec = (L * pm, L * pi + k * pm)
    rd = (L * kv, L * ib + k * kv)
    pre = (L * L / 2 * pe, L * L / 2 * pi + L * k * pm)
    return dec, rd, pre

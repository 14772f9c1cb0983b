"""Decode-FLOPs model for full, token-sparse and page-sparse attention (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arms may use this.

The repro card (claim C2 in "What reproduces (and what does not)", and
"Layout": an exact decode-FLOPs model of the paper's Eqs. 6-11) reports a
54.5% reduction versus full attention for the 8B model at 32k context, and
("Key finding ...") a gap of 1-4% between the token-level method and the
page-level baseline at C = 2k tokens, the baseline's extra term being
2 q h (T/P).  The equations themselves are not printed; this reading
reproduces both numbers:

    F_full   = L (2 P_layer + 4 Hq d T)
    F_sparse = L (2 P_layer + 4 Hq d C)
    F_page   = F_sparse + L 2 Hq d (T / P)
    P_layer  = h Hq d + 2 h Hkv d + Hq d h + 3 h I   (q, k/v, o projections; gated MLP)

Embeddings, the LM head, norms and the predictor are left out.  The model
dimensions are the public Qwen3 configurations (not printed on the pages).
Pinned by tests/golden/flops_claims.txt (the pages' two numbers).
"""
from __future__ import annotations

QWEN3_8B = dict(hidden=4096, layers=36, n_q=32, n_kv=8, head_dim=128, inter=12288)
QWEN3_32B = dict(hidden=5120, layers=64, n_q=64, n_kv=8, head_dim=128, inter=25600)


def decode_flops(hidden, layers, n_q, n_kv, head_dim, inter, T, C, page=16):
    """FLOPs of one decode token -> dict(full, sparse, page, reduction, page_gap)."""
    p_layer = hidden * n_q * head_dim + 2 * hidden * n_kv * head_dim + n_q * head_dim * hidden + 3 * hidden * inter
    full = layers * (2 * p_layer + 4 * n_q * head_dim * T)
    sparse = layers * (2 * p_layer + 4 * n_q * head_dim * C)
    paged = sparse + layers * 2 * n_q * head_dim * (T / page)
    return dict(full=full, sparse=sparse, page=paged,
                reduction=1.0 - sparse / full,
                page_gap=(paged - sparse) / paged)

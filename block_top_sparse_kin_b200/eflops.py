"""eFLOPs cost model of one block top-k decode step.

"Kinetics: Rethinking Test-Time Scaling Law", response Q3 (Visualization of
eFLOPs): a workload of A FLOPs of computation and M bytes of memory access
takes T = A/C + M/B on hardware with peak compute C (FLOP/s) and memory
bandwidth B (bytes/s); with I = C/B, T = (A + I*M) / C, and A + I*M is the
workload's eFLOPs.  ("Kinetics: Memory-Aware Test-Time Scaling", eFLOPs
cost model, charges memory at about one FLOP per byte instead; the exact
form above is the one used here.)

The step's A and M are counted from the method's definition, per
(sequence, KV head) pair with nb = ceil(L / bs) blocks and g query heads:
  * scoring (only when nb > k): s_i = (1/sqrt(D)) sum_j q_j . m_i is 2 g D
    FLOPs per block; it reads the fp32 means (4 D bytes per block) and the
    g bf16 query rows;
  * top-k: comparisons only (no FLOPs counted); writes k int32 indices;
  * attention over the kept tokens T_p (k blocks, the last possibly
    partial; every token when k >= nb): 2 D FLOPs for q.K and 2 D for p.V
    per token and query head; reads the kept K and V rows (2 D bytes each)
    and the queries, writes the bf16 outputs;
  * append (when the step appends n tokens): writes n K and V rows per
    pair and re-reads the touched blocks' rows for their means (D FLOPs per
    row summed).
Pure host arithmetic: no GPU work and no part of the decode path.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class Cost:
    flops: float   # A
    bytes: float   # M

    def __add__(self, other: "Cost") -> "Cost":
        return Cost(self.flops + other.flops, self.bytes + other.bytes)


def step_costs(B: int, Hkv: int, Hq: int, D: int, bs: int, lens, k: int, n_append: int = 0,
               means_bytes: int = 4) -> dict:
    """A and M of each part of one decode step.  lens: the lengths the
    select and attention see (after the append); means_bytes: 4 for fp32
    block means, 2 for bf16."""
    g = Hq // Hkv
    lens = np.asarray(lens, dtype=np.int64)
    assert lens.shape == (B,)
    nb = -(-lens // bs)
    scanned = nb > k
    # scoring + top-k
    blocks_scanned = int((Hkv * nb[scanned]).sum())
    q_bytes = B * Hq * D * 2
    idx_bytes = B * Hkv * k * 4
    select = Cost(2.0 * g * D * blocks_scanned, float(blocks_scanned * D * means_bytes + q_bytes + idx_bytes))
    # attention over the kept tokens
    toks = np.where(scanned, (k - 1) * bs + (lens - (nb - 1) * bs), lens)
    kept = int((Hkv * toks).sum())
    attn = Cost(4.0 * D * g * kept, float(kept * D * 2 * 2 + q_bytes + B * Hq * D * 2 + idx_bytes))
    parts = {"select": select, "attn": attn}
    if n_append:
        l0 = lens - n_append
        first, last = l0 // bs, (lens - 1) // bs
        touched = rows = 0
        for b in range(B):  # touched blocks and their valid rows after the append
            for i in range(int(first[b]), int(last[b]) + 1):
                touched += 1
                rows += min((i + 1) * bs, int(lens[b])) - i * bs
        touched, rows = touched * Hkv, rows * Hkv
        new_rows = B * Hkv * n_append
        upd_bytes = (new_rows * D * 2 * 2        # read k_new, v_new
                     + new_rows * D * 2 * 2      # write the K, V cache rows
                     + (rows - new_rows) * D * 2  # re-read the touched blocks' older K rows
                     + touched * D * means_bytes)  # write their means
        parts["update"] = Cost(float(rows * D), float(upd_bytes))
    return parts


def token_step_costs(B: int, Hkv: int, Hq: int, D: int, lens, k_tokens: int) -> dict:
    """A and M of token-level top-k attention: every logit of every query
    head (2 D FLOPs per token and head, every K row read), then p.V over the
    k kept tokens of each head (2 D FLOPs, one V row each)."""
    lens = np.asarray(lens, dtype=np.int64)
    kept = np.minimum(k_tokens, lens)
    q_out = 2 * B * Hq * D * 2
    logits = Cost(2.0 * D * Hq * float(lens.sum()), float(Hkv * lens.sum() * D * 2))
    attn = Cost(2.0 * D * Hq * float(kept.sum()), float(Hq * kept.sum() * D * 2 + q_out))
    return {"logits": logits, "attn": attn}


def eflops(cost: Cost, peak_flops: float, bandwidth: float) -> dict:
    """eFLOPs = A + I M with I = C / B, and the predicted time T = eFLOPs / C
    (= A/C + M/B)."""
    intensity = peak_flops / bandwidth
    ef = cost.flops + intensity * cost.bytes
    return {
        "A_flops": cost.flops,
        "M_bytes": cost.bytes,
        "I_flop_per_byte": intensity,
        "eflops": ef,
        "t_pred_us": ef / peak_flops * 1e6,
        "t_compute_us": cost.flops / peak_flops * 1e6,
        "t_memory_us": cost.bytes / bandwidth * 1e6,
    }

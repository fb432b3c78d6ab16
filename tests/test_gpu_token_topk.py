"""Token-level top-k attention on the GPU (kin_token_topk_decode_attn)
against the fp64 oracle on the same bf16 inputs.

Kept token sets must equal the oracle's, except where the oracle's k-th and
(k+1)-th largest logits are within delta = 1e-4 max(|tau_k|, |tau_k+1|, eps)
of each other (eps: the logits' natural magnitude, the mean over tokens of
scale sum_d |q_d| |K_td|); there the GPU set may differ only as a top set of
logits perturbed by at most delta (kin_tiecheck).  Outputs are then compared
with the oracle recomputed on the GPU's set (max |err| <= 2e-2, mean
<= 2e-3; lse within 1e-3 + 1e-4 |lse|)."""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
import oracle
from kin_testlib import D, all_pairs, make_device_case
from kin_tiecheck import check_topk_set

pytestmark = pytest.mark.gpu
W = ki.Workload


def run_token(dc, kt, scale=0.0):
    w = dc.w
    ws = kin.alloc_token_workspace(dc.dims, kt)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    sel = torch.full((w.B, w.Hq, kt), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_token_topk_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, kt, scale, out, lse, ws,
                                   sel_tokens=sel, dev_status=st)
    torch.cuda.synchronize()
    return sel.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item())


def check_head(dc, b, j, kt, sel, out, lse, rows=None, scale=0.0):
    """One query head against the oracle; rows: its pair's (K, V) when the
    caller regenerated them already; scale as passed to the GPU (0 = the
    default 1/sqrt(D))."""
    w = dc.w
    h = j // w.g
    L = int(dc.lens_final[b])
    K, V = rows if rows is not None else ki.pair_rows(w, dc.hh, b, h, L)
    q = dc.q_host[b, j:j + 1]
    scale = scale if scale > 0 else 1 / math.sqrt(D)
    rsel, rout, rlse, z = oracle.token_topk_attend(q, K, V, L, kt, scale)
    n = min(kt, L)
    gsel = sel[b, j]
    assert np.all(gsel[n:] == -1), (b, j)
    g = gsel[:n]
    assert np.all(np.diff(g) > 0), (b, j, "not ascending")
    scale_eps = scale * (np.abs(oracle.bf16_bits_to_f64(q[0])) @ np.abs(oracle.bf16_bits_to_f64(K[:L])).T).mean()
    check_topk_set(z[0], np.arange(L), rsel[0], g, scale_eps, what=(b, j))
    if not np.array_equal(g, rsel[0]):
        # outputs against the oracle on the GPU's set
        zz = z[0, g]
        m = zz.max()
        wts = np.exp(zz - m)
        rout = ((wts[:, None] * oracle.bf16_bits_to_f64(V[g])).sum(0) / wts.sum())[None]
        rlse = np.array([m + np.log(wts.sum())])
    err = np.abs(out[b, j].astype(np.float64) - rout[0])
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (b, j, err.max(), err.mean())
    assert abs(lse[b, j] - rlse[0]) <= 1e-3 + 1e-4 * abs(rlse[0]), (b, j, lse[b, j], rlse[0])


@pytest.mark.parametrize("w,kt", [
    (W("tok_g4", 2, 2, 8, D, 16, 700, 1000, 8, 90, Lcap=1024), 96),
    (W("tok_g1_ragged", 3, 1, 1, D, 16, 20, 600, 8, 91, Lcap=640), 50),
    (W("tok_g8_long", 1, 1, 8, D, 16, 0, 0, 8, 92, Lcap=9000, lens=(8999,)), 700),
    (W("tok_dense_and_len1", 3, 1, 2, D, 16, 0, 0, 8, 93, Lcap=128, lens=(100, 1, 33)), 64),
    (W("tok_k1", 2, 2, 4, D, 16, 50, 300, 8, 94, Lcap=320), 1),
    # kept tokens over three segments of the attention kernel (2048, 2048, 404)
    (W("tok_g2_segments", 1, 2, 4, D, 16, 0, 0, 8, 96, Lcap=6000, lens=(5999,)), 4500),
    # rows longer than the 32768 keys kept in shared memory: keys in the
    # workspace scratch row, the emit in two rounds per warp
    (W("tok_long_scratch", 1, 1, 2, D, 16, 0, 0, 8, 97, Lcap=40000, lens=(39999,)), 3000),
], ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_token_topk_every_head(w, kt):
    dc = make_device_case(w)
    sel, out, lse, status = run_token(dc, kt)
    assert status == 0
    for b in range(w.B):
        for j in range(w.Hq):
            check_head(dc, b, j, kt, sel, out, lse)


@pytest.mark.parametrize("scale", [0.03, 0.5])
def test_token_topk_explicit_scale(scale):
    """An explicit softmax scale: kept tokens, out and lse against the
    oracle at that scale (the logits are rounded after scaling, so the set
    is checked by the near-tie rule at that scale, not against the default
    scale's set)."""
    w = W("tok_scale", 2, 2, 8, D, 16, 700, 1000, 8, 98, Lcap=1024)
    dc = make_device_case(w)
    sel, out, lse, status = run_token(dc, 96, scale)
    assert status == 0
    for b in range(w.B):
        for j in range(w.Hq):
            check_head(dc, b, j, 96, sel, out, lse, scale=scale)


def test_token_topk_bad_length_is_flagged():
    w = W("tok_bad", 2, 1, 2, D, 16, 0, 0, 8, 95, Lcap=128, lens=(100, 60))
    dc = make_device_case(w)
    dc.seq_lens[1] = 500
    sel, out, lse, status = run_token(dc, 16)
    assert status == 5
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1])) and np.all(sel[1] == -1)
    check_head(dc, 0, 0, 16, sel, out, lse)


def test_token_topk_32k_workload_every_head():
    """The 32K decode batch with a token budget equal to the block budget
    (256 blocks x 16 tokens = 4096 tokens per query head), every head
    against the oracle (host threads, one K/V regeneration per pair)."""
    w = ki.WORKLOADS["qwen3_8b_32k"]
    dc = make_device_case(w)
    kt = w.k * w.bs
    sel, out, lse, status = run_token(dc, kt)
    assert status == 0
    del dc.k_cache, dc.v_cache
    torch.cuda.empty_cache()

    def pair(bh):
        b, h = bh
        rows = ki.pair_rows(w, dc.hh, b, h, int(dc.lens_final[b]))
        for j in range(h * w.g, (h + 1) * w.g):
            check_head(dc, b, j, kt, sel, out, lse, rows)

    with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
        list(ex.map(pair, all_pairs(w)))

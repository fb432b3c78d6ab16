"""More GPU parity cases: minimal budgets, odd group sizes, multi-block
appends, very long block lists (the top-k path without a candidate list),
a multi-step decode loop (append -> select -> attend, checked every step),
and a whole step captured in a CUDA graph (as the benchmark replays it)."""
import math
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
import oracle
from kin_testlib import D, check_pair, gpu_step, make_device_case, to_dev_bf16

pytestmark = pytest.mark.gpu
W = ki.Workload


@pytest.mark.parametrize("w", [
    W("k2_ragged", 3, 2, 6, D, 16, 40, 700, 2, 40, Lcap=704),
    W("g3", 2, 3, 9, D, 16, 500, 900, 7, 41, Lcap=912),
    W("g6_bs32", 2, 2, 12, D, 32, 300, 1000, 5, 42, Lcap=1024),
    W("g7_bs64", 2, 1, 7, D, 64, 129, 1200, 4, 43, Lcap=1280),
    W("append_100_bs64", 2, 2, 4, D, 64, 0, 0, 5, 44, Lcap=640, n_append=100, lens=(300, 500)),
    W("append_130_bs128", 1, 2, 8, D, 128, 0, 0, 3, 45, Lcap=1024, n_append=130, lens=(900,)),
], ids=lambda w: w.name)
def test_edge_shapes_every_pair(w):
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    means = dc.means.cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            check_pair(dc, gr, b, h, w.k, gpu_means=means)


@pytest.mark.parametrize("mult", [0.5, 2.0, math.sqrt(D)], ids=["half", "double", "one"])
def test_explicit_softmax_scale(mult):
    """A softmax scale passed explicitly (mult / sqrt(D); sqrt(D) gives 1.0,
    a peaked softmax): out and lse against the oracle at the same scale, on
    pairs of three chunks (so the merge runs); the selection does not
    depend on it."""
    w = W("scale", 3, 2, 8, D, 16, 1500, 3000, 100, 50, Lcap=3072)
    dc = make_device_case(w)
    scale = mult / math.sqrt(D)
    gr = gpu_step(dc, w.k, scale=scale)
    assert gr.status == 0
    default = gpu_step(dc, w.k, build_means=False)
    assert np.array_equal(gr.sel, default.sel) and np.array_equal(gr.cnt, default.cnt)
    for b in range(w.B):
        for h in range(w.Hkv):
            check_pair(dc, gr, b, h, w.k, scale=scale)


def test_attention_without_lse_output():
    """lse is optional: with a null lse the outputs (a 2-block sequence and
    long ones whose pairs span many chunks, merged in the kernel) equal
    those of a call that writes lse, bit for bit."""
    w = W("no_lse", 3, 2, 8, D, 16, 0, 0, 100, 51, Lcap=3072, lens=(20, 908, 3072))
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    sel = torch.from_numpy(gr.sel).cuda()
    cnt = torch.from_numpy(gr.cnt).cuda()
    out = torch.empty((w.B, w.Hq, D), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = kin.alloc_workspace(dc.dims, w.k)
    kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, sel, cnt, w.k, 0.0,
                               out, None, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(out.float().cpu().numpy(), gr.out)


@pytest.mark.parametrize("k", [300, 32767])
def test_maximum_block_count(k):
    """The largest block count a sequence may have (ceil(Lcap / bs) = 32768
    at bs 16: 524288 tokens): the top-k over 32768 keys in shared memory,
    and a budget one block short of the whole sequence, whose 683 chunks per
    pair the attention merges in many staged batches; every pair against
    the oracle."""
    L = 32768 * 16
    w = W("max_blocks", 1, 2, 8, D, 16, 0, 0, k, 52, Lcap=L, lens=(L,))
    dc = make_device_case(w)
    gr = gpu_step(dc, k)
    assert gr.status == 0
    assert np.all(gr.cnt == k)
    for h in range(w.Hkv):
        check_pair(dc, gr, 0, h, k)


def test_long_block_list_with_all_equal_scores():
    """16384 blocks whose scores all tie: the top-k cannot keep a compact
    candidate list and must still pick blocks 0..k-2 and the last one."""
    L = 16384 * 16
    w = W("long_ties", 1, 2, 4, D, 16, 0, 0, 100, 46, Lcap=L, lens=(L,))
    dc = make_device_case(w)
    dc.q.zero_()
    dc.q_host[:] = 0
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    for h in range(w.Hkv):
        assert list(gr.sel[0, h]) == list(range(99)) + [16383]
        check_pair(dc, gr, 0, h, w.k)


def test_long_block_list_random():
    L = 16384 * 16 - 5
    w = W("long_rand", 1, 2, 8, D, 16, 0, 0, 300, 47, Lcap=16384 * 16, lens=(L,))
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    for h in range(w.Hkv):
        check_pair(dc, gr, 0, h, w.k)


def test_decode_loop_append_select_attend():
    """Three decode steps in a row on one stream (each kernel launched with
    programmatic dependent launch): every step's selection and output match
    the oracle on the grown cache."""
    w = W("loop", 2, 2, 8, D, 16, 0, 0, 6, 48, Lcap=400, lens=(200, 95))
    lens0 = np.array(w.lens, np.int32)
    steps = 3
    wf = w.with_(lens=tuple(int(x) + steps for x in lens0), n_append=steps)
    dc = make_device_case(wf)               # cache holds lens0 rows; the field runs to lens0 + 3
    kin.kin_block_means_build(dc.dims, dc.k_cache, dc.seq_lens, dc.means)
    ws = kin.alloc_workspace(dc.dims, w.k)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for s in range(steps):
        kn = dc.k_new[:, :, s:s + 1].contiguous()
        vn = dc.v_new[:, :, s:s + 1].contiguous()
        kin.kin_block_means_update(dc.dims, dc.k_cache, dc.v_cache, dc.means, dc.seq_lens, kn, vn, 1, st)
        sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
        cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
        out = torch.empty((w.B, w.Hq, D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        kin.kin_block_topk_select(dc.dims, dc.q, dc.means, dc.seq_lens, w.k, sel, cnt, ws, st)
        kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, sel, cnt, w.k, 0.0,
                                   out, lse, ws, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        lens = lens0 + s + 1
        assert np.array_equal(dc.seq_lens.cpu().numpy(), lens)
        sel_h, out_h = sel.cpu().numpy(), out.float().cpu().numpy()
        for b in range(w.B):
            L = int(lens[b])
            for h in range(w.Hkv):
                K, V = ki.pair_rows(wf, dc.hh, b, h, L)
                qg = dc.q_host[b, h * w.g:(h + 1) * w.g]
                ref_sel, c = oracle.select(oracle.block_scores(qg, oracle.block_means(K, L, w.bs)), w.k)
                assert np.array_equal(sel_h[b, h], ref_sel)
                o_ref, _ = oracle.attend(qg, K, V, L, w.bs, ref_sel[:c], 1 / math.sqrt(D))
                err = np.abs(out_h[b, h * w.g:(h + 1) * w.g] - o_ref)
                assert err.max() <= 2e-2 and err.mean() <= 2e-3


def test_step_captured_in_a_cuda_graph_matches_eager():
    w = W("graph", 4, 2, 8, D, 16, 2000, 4000, 40, 49, Lcap=4096)
    dc = make_device_case(w)
    kin.kin_block_means_build(dc.dims, dc.k_cache, dc.seq_lens, dc.means)
    ws = kin.alloc_workspace(dc.dims, w.k)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def bufs():
        return (torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda"),
                torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda"),
                torch.empty((w.B, w.Hq, D), dtype=torch.bfloat16, device="cuda"),
                torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda"))

    def step(sel, cnt, out, lse):
        kin.kin_block_topk_select(dc.dims, dc.q, dc.means, dc.seq_lens, w.k, sel, cnt, ws, st)
        kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, sel, cnt, w.k, 0.0,
                                   out, lse, ws, st)

    eager = bufs()
    step(*eager)
    torch.cuda.synchronize()
    graphed = bufs()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step(*graphed)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        for t in graphed:
            t.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(eager, graphed):
            assert torch.equal(a, b)
    assert int(st.item()) == 0


_THREADS = textwrap.dedent("""
    import sys, threading
    sys.path.insert(0, {root!r})
    sys.path.insert(0, {tests!r})
    import numpy as np, torch
    import block_top_sparse_kin_b200 as kin
    import kin_inputs as ki
    from kin_testlib import make_device_case
    W = ki.Workload
    # two shapes whose top-k kernels need different dynamic shared memory
    cases = [make_device_case(W("thr_a", 1, 1, 4, 128, 16, 0, 0, 8, 60, Lcap=9000, lens=(8999,))),
             make_device_case(W("thr_b", 1, 1, 2, 128, 16, 0, 0, 8, 61, Lcap=40000, lens=(39999,)))]
    torch.cuda.synchronize()

    def run(dc, kt, stream):
        w = dc.w
        with torch.cuda.stream(stream):
            ws = kin.alloc_token_workspace(dc.dims, kt)
            out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
            sel = torch.empty((w.B, w.Hq, kt), dtype=torch.int32, device="cuda")
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            kin.kin_token_topk_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, kt, 0.0, out, lse,
                                           ws, sel_tokens=sel, dev_status=st)
        stream.synchronize()
        return int(st.item()), sel.cpu().numpy(), out.view(torch.int16).cpu().numpy(), lse.cpu().numpy()

    n = 8
    gate = threading.Barrier(n)
    res, errs = [None] * n, []

    def worker(i):
        s = torch.cuda.Stream()
        try:
            gate.wait()
            res[i] = run(cases[i % 2], 700, s)
        except Exception as e:
            errs.append(repr(e))

    th = [threading.Thread(target=worker, args=(i,)) for i in range(n)]
    for t in th: t.start()
    for t in th: t.join()
    assert not errs, errs
    ref = [run(cases[j], 700, torch.cuda.current_stream()) for j in range(2)]
    for i, r in enumerate(res):
        assert r[0] == 0, (i, r[0])
        for a, b in zip(r[1:], ref[i % 2][1:]):
            assert np.array_equal(a, b), i
    print("threads ok")
""")


def test_concurrent_first_calls_from_host_threads():
    """Eight host threads, released together in a fresh process (so the
    library's per-device caches are cold), each on its own stream with its
    own buffers, on two shapes whose top-k kernels need different dynamic
    shared memory: every call succeeds and every result equals a serial
    run's, bit for bit."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = _THREADS.format(root=root, tests=os.path.join(root, "tests"))
    r = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "threads ok" in r.stdout, (r.stdout[-2000:], r.stderr[-3000:])

"""Benchmark: block top-k sparse decode attention on B200.

One step = the whole decode hot path for one batch: group-summed block scores
+ exact block top-k (kin_block_topk_select), then the split-K sparse decode
attention with its log-sum-exp merge (kin_sparse_decode_attn); workloads with
an append first run kin_block_means_update.  The block means and KV cache are
resident decode state built before timing.

Metric: query-heads/s = B * Hq / t_step (whole job: summed over ranks, time =
max over ranks).  Timing: the step is captured once as a CUDA graph and
replayed, with two timing events inside it around the step's kernels (CUDA
events on the launching stream); L2 flushed (a 256 MiB write then a 256 MiB
read, outside the events) before every step; W warm-up steps; barrier +
synchronize around the K timed steps.  Per-kernel times (for the roofline)
come from one graph per kernel family holding back-to-back calls; the e2e
figure runs the step eagerly through the public calls, with the copy of q
from pinned host memory and of the output back to it inside the events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--k K]
  python bench.py --impl reference ...   # the fp64 CPU oracle on host cores
Multi-GPU: torchrun, one rank per GPU, each rank an independent batch shard
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from dataclasses import dataclass

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kin_inputs as ki  # noqa: E402

DEFAULT_WORKLOAD = "qwen3_8b_32k"
METRIC = "block-top-k decode attn query-heads/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20  # > 2x the 126 MB L2
KERNEL_REPEATS = 4  # back-to-back calls per per-kernel timing graph


# ---------------------------------------------------------------- bytes model
def algorithmic_bytes(w: ki.Workload, k: int, lens: np.ndarray, means_bytes: int = 4):
    """Algorithmic HBM bytes per launch: (select, attention).

    select: fp32 means of every block (skipped when k >= nb), q, indices.
    attention: K+V rows of the kept tokens, q, bf16 out, indices.
    """
    nb = -(-lens.astype(np.int64) // w.bs)
    scan = nb > k
    means = int((w.Hkv * nb[scan] * w.D * means_bytes).sum())
    q_bytes = w.B * w.Hq * w.D * 2
    idx_bytes = w.B * w.Hkv * k * 4
    sel_bytes = means + q_bytes + idx_bytes
    # kept tokens per pair: k full blocks incl. the (maybe partial) last one
    toks = np.where(scan, (k - 1) * w.bs + (lens - (nb - 1) * w.bs), lens).astype(np.int64)
    kv = int((w.Hkv * toks * w.D * 2 * 2).sum())
    attn_bytes = kv + q_bytes + w.B * w.Hq * w.D * 2 + idx_bytes
    return sel_bytes, attn_bytes


def shared_algorithmic_bytes(w: ki.Workload, k: int, st, means_bytes: float = 4.0):
    """Algorithmic bytes when groups of samples share their prompt's pages
    and per-page means, each shared item read once: (select) the distinct
    mean rows (page, head) of the scanned sequences; (attention) the
    distinct kept K/V blocks (page, head) of each group, a full shared page
    counted once, plus q, out and indices.  Uses the step's selection."""
    lens = st["lens_final"].astype(np.int64)
    table = st["table_host"]
    sel = st["sel"].cpu().numpy()
    cnt = st["cnt"].cpu().numpy()
    nb = -(-lens // w.bs)
    scanned = nb > k
    pages = set()
    for b in np.nonzero(scanned)[0]:
        pages.update(table[b, :nb[b]].tolist())
    q_bytes = w.B * w.Hq * w.D * 2
    idx_bytes = w.B * w.Hkv * k * 4
    sel_bytes = len(pages) * w.Hkv * w.D * means_bytes + q_bytes + idx_bytes
    kept = {}  # (page, head) -> valid tokens
    for b in range(w.B):
        for h in range(w.Hkv):
            for blk in sel[b, h, :cnt[b, h]]:
                key = (int(table[b, blk]), h)
                kept[key] = max(kept.get(key, 0), int(min(w.bs, lens[b] - blk * w.bs)))
    attn_bytes = sum(kept.values()) * w.D * 2 * 2 + q_bytes + w.B * w.Hq * w.D * 2 + idx_bytes
    return sel_bytes, attn_bytes


def token_algorithmic_bytes(w: ki.Workload, kt: int, lens: np.ndarray):
    """Algorithmic HBM bytes of one token-level top-k step: every K row (the
    logits pass), the kept V rows of every query head, q and the bf16 out.
    The logits' round trip through workspace is reported as traffic, not
    counted here."""
    lens = lens.astype(np.int64)
    k_rows = int((w.Hkv * lens).sum())
    v_rows = int((w.Hq * np.minimum(kt, lens)).sum())
    return (k_rows + v_rows) * w.D * 2 + 2 * w.B * w.Hq * w.D * 2


def measured_bf16_peak():
    """Dense bf16 FLOP/s: the measured burst figure, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]) * 1e12, "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS * 1e12, "fallback"


def eflops_report(w, k, lens, ms_per_step, means_bytes=4, token_kt=0):
    """The eFLOPs model's predicted step time (T = A/C + M/B) beside the
    measured one, with the measured B200 peaks as C and B."""
    from block_top_sparse_kin_b200 import eflops as ef
    parts = (ef.token_step_costs(w.B, w.Hkv, w.Hq, w.D, lens, token_kt) if token_kt else
             ef.step_costs(w.B, w.Hkv, w.Hq, w.D, w.bs, lens, k, w.n_append, means_bytes))
    tot = ef.Cost(0.0, 0.0)
    for c in parts.values():
        tot = tot + c
    C, c_kind = measured_bf16_peak()
    Bw, b_kind = measured_peak()
    r = ef.eflops(tot, C, Bw * 1e9)
    r["t_meas_us"] = ms_per_step * 1e3
    r["meas_over_pred"] = r["t_meas_us"] / r["t_pred_us"]
    r["C_flops"] = C
    r["B_bytes_s"] = Bw * 1e9
    r["peaks"] = f"C = dense bf16 ({c_kind}), B = HBM copy ({b_kind})"
    return r


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_digest(name: str) -> str:
    path = os.path.join(ROOT, "block_top_sparse_kin_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_key(kernel_file: str, args) -> str:
    """The key a kernel family's captured traffic is stored under: the source
    file, plus the block-means kind for the select (fp32, bf16 and dual means
    move different bytes) and the KV layout when it is not the contiguous one
    (a paged or shared-prefix run has no capture of its own, so no figure)."""
    key = kernel_file
    if kernel_file == "kin_select.cu":
        key += "@" + means_kind(args)
    if getattr(args, "paged", False) or getattr(args, "shared_prefix", 1) > 1:
        key += "@paged"
    return key


def profiled_traffic(kernel_key: str, workload: str, k: int):
    """DRAM bytes per launch from a committed ncu summary, if it matches the
    current kernel source (profiles/traffic.txt: key workload k sha bytes; the
    key is the source file with the qualifiers traffic_key adds)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    digest = kernel_source_digest(kernel_key.split("@")[0])
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 5 and not line.startswith("#"):
                if parts[0] == kernel_key and parts[1] == workload and int(parts[2]) == k and parts[3] == digest:
                    return int(float(parts[4]))
    return None


# -------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event (throttle) reasons through NVML every
    millisecond while the timed region runs (the same counters nvidia-smi's
    clocks.sm / clocks_event_reasons.* report)."""

    REASONS = {  # NVML clocks-event reason bits
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40,
    }

    def __init__(self, local: int):
        self.local = local
        self.samples = []
        self.stop = threading.Event()
        self.handle = None
        self.max_mhz = None

    def __enter__(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.local).uuid)
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception as e:  # no NVML: report no samples
            self.error = repr(e)
        return self

    def poll(self):
        """One sample now (the timed loop also calls this after every step)."""
        if self.handle is None:
            return
        nv = self.nv
        try:
            mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
            try:
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            except AttributeError:
                rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
            self.samples.append((mhz, rs))
        except Exception:
            pass

    def _run(self):
        while not self.stop.is_set():
            self.poll()
            time.sleep(0.001)

    def __exit__(self, *a):
        self.stop.set()
        if self.handle is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml"}
        reasons = sorted(n for n, bit in self.REASONS.items() if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------- GPU arm
def setup_dist(args):
    """One process per GPU.  Under a launcher (WORLD_SIZE > 1) the ranks join
    one process group: NCCL on GPU hosts (gloo where no GPU is visible, which
    only the host-side tests use); it carries the barriers around the timed
    region and the max-over-ranks reduction, never data of the decode path."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        if torch.cuda.is_available():
            if local >= torch.cuda.device_count():
                raise SystemExit(f"rank {rank}: LOCAL_RANK {local} but only {torch.cuda.device_count()} GPUs visible")
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def _reduce_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def reduce_max(x: float, device=None) -> float:
    """Max of a per-rank number over all ranks (identity on one rank)."""
    return reduce_max_list([x], device)[0]


def reduce_max_list(xs, device=None):
    """Element-wise max over all ranks of a list of per-rank numbers, in one
    collective (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(x) for x in xs]
    t = torch.tensor([float(x) for x in xs], dtype=torch.float64, device=device or _reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu().tolist()]


def launch_ranks(args):
    """--gpus N.  Under a launcher, WORLD_SIZE must equal N (else exit 2).
    Without one, N > 1 runs this same command under torch.distributed.run
    with N ranks, one per GPU, on this node, and returns its exit code;
    None means this process is the (only) rank and runs the arm itself."""
    env_world = os.environ.get("WORLD_SIZE")
    if args.gpus < 1:
        raise SystemExit(2)
    if env_world is not None:
        if int(env_world) != args.gpus:
            print(f"bench.py: --gpus {args.gpus} disagrees with WORLD_SIZE={env_world}", file=sys.stderr)
            raise SystemExit(2)
        return None
    if args.gpus == 1:
        return None
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", sys.argv[0], *sys.argv[1:]]
    return subprocess.call(cmd)


def step_percentiles(step_ms) -> dict:
    """p10 / p50 / p90 of the timed steps (each step's max over ranks), in us."""
    p10, p50, p90 = np.percentile(np.asarray(step_ms, dtype=np.float64) * 1e3, [10, 50, 90])
    return {"p10": float(p10), "p50": float(p50), "p90": float(p90)}


def whole_job_value(world: int, qh_per_step: int, steps: int, max_total_ms: float) -> float:
    """Query heads decoded by all ranks per second of the slowest rank's time."""
    return world * qh_per_step * steps / (max_total_ms / 1e3)


def shard_workload(w: ki.Workload, rank: int) -> ki.Workload:
    """Weak scaling: every rank decodes its own batch of the same shape
    (independent sequences; seed offset by rank)."""
    return w.with_(seed=w.seed + 1000 * rank) if rank else w


SHARED_GEN_TOKENS = 2048  # tokens each Best-of-N sample generated after the shared prompt


def make_page_pool(st, seed: int, share_n: int = 1, shuffle: bool = True):
    """Moves the contiguous K/V caches into a shuffled page pool (page = one
    KV block, [num_pages, Hkv, bs, D]) with a block table [B, nbcap]: every
    block a sequence holds after the step's append gets a page, in random
    order.  share_n > 1: consecutive groups of share_n sequences are samples
    of one prompt; the prompt's blocks (all but the last SHARED_GEN_TOKENS
    tokens of the group's shortest sequence, whole blocks) map to the pages
    of the group's first sample.  shuffle=False keeps the pages in the order
    the sequences fill them (as a prefill allocator would).  Frees the
    contiguous caches."""
    import torch
    w = st["w"]
    B, Hkv, cap, D = st["k_cache"].shape
    bs, nbcap = w.bs, w.nbcap
    lens = st["lens_final"]
    nbs = [-(-int(L) // bs) for L in lens]
    owner = []
    table = np.full((B, nbcap), -1, np.int64)
    for b in range(B):
        first = b - b % share_n
        shared = 0
        if share_n > 1:
            group_min = int(min(lens[first:first + share_n]) - w.n_append)
            shared = max(0, (group_min - SHARED_GEN_TOKENS) // bs)
        for i in range(nbs[b]):
            if i < shared and b != first:
                table[b, i] = table[first, i]
            else:
                table[b, i] = len(owner)
                owner.append((b, i))
    P = len(owner)
    order = np.random.default_rng(seed).permutation(P) if shuffle else np.arange(P)
    table = np.where(table >= 0, order[np.maximum(table, 0)], -1).astype(np.int32)
    ib = np.array([o[0] for o in owner])
    ii = np.array([o[1] for o in owner])
    dst = torch.from_numpy(order.astype(np.int64)).cuda()
    tb, ti = torch.from_numpy(ib).cuda(), torch.from_numpy(ii).cuda()
    for name in ("k_cache", "v_cache"):
        cache = st.pop(name)
        if cap % bs:
            cache = torch.nn.functional.pad(cache, (0, 0, 0, nbcap * bs - cap))
        blocks = cache.view(B, Hkv, nbcap, bs, D)
        pool = torch.empty((P, Hkv, bs, D), dtype=torch.bfloat16, device="cuda")
        for c0 in range(0, len(ib), 1 << 16):  # bounded temporaries
            sl = slice(c0, c0 + (1 << 16))
            pool[dst[sl]] = blocks[tb[sl], :, ti[sl]]
        st[name.replace("cache", "pages")] = pool
        del cache, blocks
    st["table"] = torch.from_numpy(table).cuda()
    st["table_host"] = table
    st["num_pages"] = P
    torch.cuda.empty_cache()


def build_device_state(w: ki.Workload, k: int, paged: bool = False, means_bf16: bool = False, share_n: int = 1,
                       shuffle_pages: bool = True, means_dual: bool = False):
    import torch
    import block_top_sparse_kin_b200 as kin
    lens_final, lens_pre, hh = ki.case_meta(w)
    dims = kin.make_dims(w.B, w.Hkv, w.Hq, w.D, w.bs, w.cap)
    q_host = ki.fill_q(w.seed, w.B, w.Hq, w.D)
    st = dict(w=w, k=k, dims=dims, lens_final=lens_final, lens_pre=lens_pre, q_host=q_host)
    st["q"] = torch.from_numpy(q_host.view(np.int16)).cuda().view(torch.bfloat16)
    st["seq_pre"] = torch.from_numpy(lens_pre.copy()).cuda()
    st["seq"] = st["seq_pre"].clone()
    hh_dev = torch.from_numpy(hh).cuda()
    kc = torch.empty((w.B, w.Hkv, w.cap, w.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    ki.kv_cache_device(w.seed, True, w.B, w.Hkv, w.cap, w.D, w.bs, st["seq"], hh_dev, False, kc)
    ki.kv_cache_device(w.seed, False, w.B, w.Hkv, w.cap, w.D, w.bs, st["seq"], hh_dev, False, vc)
    st["k_cache"], st["v_cache"] = kc, vc
    if means_dual:  # fp32 means, their bf16 rounding and the rows' error radii in one buffer
        st["means"] = kin.alloc_dual_means(dims)
    else:
        st["means"] = torch.zeros((w.B, w.Hkv, w.nbcap, w.D), dtype=torch.bfloat16 if means_bf16 else torch.float32,
                                  device="cuda")
    if means_bf16 or means_dual:
        kin.kin_block_means_build_ex(dims, kc, st["seq"], st["means"])
    else:
        kin.kin_block_means_build(dims, kc, st["seq"], st["means"])
    if w.n_append:
        kn = np.empty((w.B, w.Hkv, w.n_append, w.D), np.uint16)
        vn = np.empty_like(kn)
        for b in range(w.B):
            for h in range(w.Hkv):
                t0 = int(lens_pre[b])
                kn[b, h] = ki.kv_rows(w.seed, True, b * w.Hkv + h, t0, t0 + w.n_append, w.D, w.bs, hh[b, h])
                vn[b, h] = ki.kv_rows(w.seed, False, b * w.Hkv + h, t0, t0 + w.n_append, w.D, w.bs, None)
        st["k_new"] = torch.from_numpy(kn.view(np.int16)).cuda().view(torch.bfloat16)
        st["v_new"] = torch.from_numpy(vn.view(np.int16)).cuda().view(torch.bfloat16)
    st["sel"] = torch.empty((w.B, w.Hkv, k), dtype=torch.int32, device="cuda")
    st["cnt"] = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    st["out"] = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    st["lse"] = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    st["status"] = torch.zeros(1, dtype=torch.int32, device="cuda")
    st["ws"] = kin.alloc_workspace(dims, k)
    if paged or share_n > 1:
        make_page_pool(st, w.seed, share_n, shuffle_pages)
    if share_n > 1:  # block means per page: the shared prompt's means exist once
        if means_dual:
            st["means"] = kin.alloc_dual_page_means(dims, st["num_pages"])
        else:
            st["means"] = torch.zeros((st["num_pages"], w.Hkv, w.D),
                                      dtype=torch.bfloat16 if means_bf16 else torch.float32, device="cuda")
        st["seq"].copy_(st["seq_pre"])
        kin.kin_block_means_build_ex(dims, st["k_pages"], st["seq"], st["means"], block_table=st["table"],
                                     per_page=True)
        st["page_means"] = True
    torch.cuda.synchronize()
    return st


def run_step(st, ev=None):
    """One decode step.  ev: optional list of 3 or 4 events to record between kernels."""
    w = st["w"]
    i = 0
    if ev is not None:
        ev[i].record(); i += 1
    if w.n_append:
        append(st)
        if ev is not None:
            ev[i].record(); i += 1
    if "token_kt" in st:
        token_step(st)
        return
    select(st)
    if ev is not None:
        ev[i].record(); i += 1
    attend(st)
    if ev is not None:
        ev[i].record()


def append(st):
    """The step's append: n new tokens per sequence, touched block means refreshed."""
    import block_top_sparse_kin_b200 as kin
    w = st["w"]
    paged = "table" in st
    k_rows, v_rows = (st["k_pages"], st["v_pages"]) if paged else (st["k_cache"], st["v_cache"])
    if "page_means" in st or str(st["means"].dtype) in ("torch.bfloat16", "torch.uint8"):
        kin.kin_block_means_update_ex(st["dims"], k_rows, v_rows, st["means"], st["seq"], st["k_new"], st["v_new"],
                                      w.n_append, block_table=st.get("table"), dev_status=st["status"],
                                      per_page="page_means" in st)
    elif paged:
        kin.kin_block_means_update_paged(st["dims"], k_rows, v_rows, st["table"], st["means"], st["seq"],
                                         st["k_new"], st["v_new"], w.n_append, st["status"])
    else:
        kin.kin_block_means_update(st["dims"], k_rows, v_rows, st["means"], st["seq"], st["k_new"], st["v_new"],
                                   w.n_append, st["status"])


def select(st):
    """The step's block scoring and top-k (fp32 means, or bf16 or dual means through the extended call)."""
    import block_top_sparse_kin_b200 as kin
    if "page_means" in st:
        kin.kin_block_topk_select_paged(st["dims"], st["q"], st["means"], st["table"], st["seq"], st["k"], st["sel"],
                                        st["cnt"], st["ws"], st["status"], num_pages=st["num_pages"])
    elif str(st["means"].dtype) in ("torch.bfloat16", "torch.uint8"):
        kin.kin_block_topk_select_ex(st["dims"], st["q"], st["means"], st["seq"], st["k"], st["sel"], st["cnt"],
                                     st["ws"], st["status"])
    else:
        kin.kin_block_topk_select(st["dims"], st["q"], st["means"], st["seq"], st["k"], st["sel"], st["cnt"],
                                  st["ws"], st["status"])


def token_step(st):
    """Token-level top-k attention (logits of every token, top-k per query head, attention)."""
    import block_top_sparse_kin_b200 as kin
    kin.kin_token_topk_decode_attn(st["dims"], st["q"], st["k_cache"], st["v_cache"], st["seq"], st["token_kt"], 0.0,
                                   st["out"], st["lse"], st["token_ws"], dev_status=st["status"])


def attend(st):
    """The step's attention call, over the contiguous cache or the page pool."""
    import block_top_sparse_kin_b200 as kin
    if "table" in st:
        kin.kin_sparse_decode_attn_paged(st["dims"], st["q"], st["k_pages"], st["v_pages"], st["table"], st["seq"],
                                         st["sel"], st["cnt"], st["k"], 0.0, st["out"], st["lse"], st["ws"],
                                         st["status"])
    else:
        kin.kin_sparse_decode_attn(st["dims"], st["q"], st["k_cache"], st["v_cache"], st["seq"], st["sel"],
                                   st["cnt"], st["k"], 0.0, st["out"], st["lse"], st["ws"], st["status"])


def reset_state(st):
    if st["w"].n_append:
        st["seq"].copy_(st["seq_pre"])


@dataclass
class RankRecord:
    """What one rank measured; report() reduces it over ranks.  Times in ms."""
    w0: ki.Workload                # the workload as named (every rank's shard has its shape)
    w: ki.Workload                 # this rank's shard
    k: int
    lens_final: np.ndarray
    per_step: list                 # device time of every timed step
    parts: list                    # [(name, algorithmic bytes per launch, source file)]
    part_ms: dict                  # name -> per-launch times
    upd_ms: list                   # the append update, per call (workloads with an append)
    e2e_ms: list                   # every e2e step (copies included)
    e2e: dict                      # how the e2e leg ran: mode, h2d/d2h bytes per step
    clocks: dict
    wall: float                    # host seconds around the timed loop
    status: int
    launches_per_step: int
    kv_layout: str
    token_kt: int = 0


def gpu_arm(args):
    import torch.distributed as dist
    rank, world, local = setup_dist(args)
    try:
        rec = measure_rank(args, rank, world, local)
        report(args, rank, world, rec)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


def measure_rank(args, rank, world, local) -> RankRecord:
    """Builds this rank's decode state on its GPU and times the step; the
    ranks meet only at the barriers around the timed regions."""
    import torch
    import torch.distributed as dist
    import block_top_sparse_kin_b200 as kin
    w0 = ki.WORKLOADS[args.workload]
    if args.batch:
        w0 = w0.with_(B=args.batch, name=f"{w0.name}_b{args.batch}")
    k = args.k or w0.k
    w = shard_workload(w0, rank)
    st = build_device_state(w, k, paged=args.paged, means_bf16=args.means_bf16,
                            means_dual=means_kind(args) == "dual", share_n=args.shared_prefix,
                            shuffle_pages=args.page_order == "shuffled")
    if args.token_topk:
        if args.paged or args.shared_prefix > 1:
            raise SystemExit("--token-topk reads the contiguous cache")
        st["token_kt"] = k * w.bs  # the block budget in tokens, per query head
        st["token_ws"] = kin.alloc_token_workspace(st["dims"], st["token_kt"])
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_sink = torch.zeros((), dtype=torch.float32, device="cuda")

    def flush_l2(i):
        """Write a buffer larger than L2, then read another one, so a timed
        step starts with a cold L2 holding no dirty lines to write back."""
        flush_w.fill_(i & 0xFF)
        flush_sink.copy_(flush_r.sum())

    def barrier():
        if world > 1:
            dist.barrier()

    # block path: scan + top-k, then attention; token path: logits, top-k,
    # attention; plus the append update
    launches_per_step = 4 if w.n_append else 3

    for _ in range(args.warmup):
        reset_state(st)
        run_step(st)
    torch.cuda.synchronize()
    if int(st["status"].item()) != 0:
        raise RuntimeError(f"device status {int(st['status'].item())} after warm-up")

    # A step is one CUDA graph, captured once and replayed every step as a
    # decode loop would, with two timing events inside it around the step's
    # kernels, so the kernels chain back to back.  Both this graph and the
    # per-kernel graphs below are replayed during warm-up, so no timed replay
    # pays a graph's first launch.  The L2 flush runs eagerly before every
    # replay, outside the events, and each replay's events are read back (a
    # host synchronize, also outside the events) before the next replay.
    def ext_events(n):
        return [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n)]

    # the step's kernel families: (name, call, algorithmic bytes, traffic key)
    means_bytes = means_bytes_per_dim(args)
    if args.token_topk:
        parts = [("token_topk_attn", lambda: token_step(st),
                  token_algorithmic_bytes(w, st["token_kt"], st["lens_final"]), traffic_key("kin_token.cu", args))]
    else:
        if args.shared_prefix > 1:  # shared items counted once (the step's selection, from warm-up)
            sel_b, attn_b = shared_algorithmic_bytes(w, k, st, means_bytes)
        else:
            sel_b, attn_b = algorithmic_bytes(w, k, st["lens_final"], means_bytes)
        parts = [("select", lambda: select(st), sel_b, traffic_key("kin_select.cu", args)),
                 ("attn", lambda: attend(st), attn_b, traffic_key("kin_attn.cu", args))]

    # Per-kernel times for the roofline: a graph per kernel family holding
    # KERNEL_REPEATS back-to-back calls between two events.  The means and the
    # kept K/V are larger than L2 and are streamed (means with evict-first
    # loads), so every call reads HBM; the events' few-us launch edges are
    # spread over the calls, as in a decode pipeline.  The append update is
    # timed once per replay (its calls would move the lengths).
    step_ev = ext_events(2)
    part_ev = [ext_events(2) for _ in parts]
    upd_ev = ext_events(2)
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            reset_state(st)
            step_ev[0].record()
            run_step(st)
            step_ev[1].record()
        part_graphs = []
        for (_, call, _, _), ev in zip(parts, part_ev):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                ev[0].record()
                for _ in range(KERNEL_REPEATS):
                    call()
                ev[1].record()
            part_graphs.append(g)
        upd_graph = None
        if w.n_append:
            upd_graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(upd_graph, stream=cap):
                reset_state(st)
                upd_ev[0].record()
                append(st)
                upd_ev[1].record()
    torch.cuda.current_stream().wait_stream(cap)
    diag = part_graphs + ([upd_graph] if upd_graph is not None else [])
    for _ in range(args.warmup):
        flush_l2(0)
        graph.replay()
        for g in diag:
            flush_l2(0)
            g.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    per_step = []
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for s in range(args.steps):
            flush_l2(s)                    # outside the events
            graph.replay()
            torch.cuda.synchronize()
            per_step.append(step_ev[0].elapsed_time(step_ev[1]))
            clk.poll()                     # the clock right after each step (outside the events)
        wall = time.perf_counter() - wall0
    barrier()
    part_ms = {name: [] for name, _, _, _ in parts}
    upd_ms = []
    for s in range(args.steps):            # per-kernel timing pass (not in `value`)
        for (name, _, _, _), g, ev in zip(parts, part_graphs, part_ev):
            flush_l2(s)
            g.replay()
            torch.cuda.synchronize()
            part_ms[name].append(ev[0].elapsed_time(ev[1]) / KERNEL_REPEATS)
        if upd_graph is not None:
            flush_l2(s)
            upd_graph.replay()
            torch.cuda.synchronize()
            upd_ms.append(upd_ev[0].elapsed_time(upd_ev[1]))
    reset_state(st)
    run_step(st)                           # leave the state as one step leaves it
    torch.cuda.synchronize()
    del graph, part_graphs, upd_graph, diag

    e2e_ms, e2e = e2e_leg(args, st, flush_l2, barrier)
    return RankRecord(
        w0=w0, w=w, k=k, lens_final=st["lens_final"], per_step=per_step,
        parts=[(name, nbytes, src) for name, _, nbytes, src in parts], part_ms=part_ms, upd_ms=upd_ms,
        e2e_ms=e2e_ms, e2e=e2e, clocks=clk.summary(), wall=wall, status=int(st["status"].item()),
        launches_per_step=launches_per_step, token_kt=st.get("token_kt", 0),
        kv_layout=(f"paged: {st['num_pages']} pages of one {w.bs}-token block, {args.page_order} pool"
                   f" + block table"
                   + (f"; groups of {args.shared_prefix} samples share their prompt's pages and"
                      f" per-page means" if args.shared_prefix > 1 else "")
                   if "table" in st else "contiguous [B][Hkv][Lcap][D]"))


def e2e_leg(args, st, flush_l2, barrier):
    """The step as a decode loop runs it from host buffers: the step's inputs
    (q, and the appended K/V rows where the workload appends) copied from
    pinned host memory, the step's kernels, and the output copied back to
    pinned host memory, all captured once in one CUDA graph and replayed.
    Each step is timed by CUDA events recorded on the stream around the
    replay (so the graph's launch edge on the device is inside), L2 flushed
    before.  Returns the per-step times and what was copied."""
    import torch
    w = st["w"]
    h2d = [(st["q"], torch.from_numpy(st["q_host"].view(np.int16)).view(torch.bfloat16).pin_memory())]
    if w.n_append:
        for name in ("k_new", "v_new"):
            h2d.append((st[name], st[name].cpu().pin_memory()))
    out_pin = torch.empty(st["out"].shape, dtype=torch.bfloat16).pin_memory()

    def body():
        reset_state(st)
        for dev, host in h2d:
            dev.copy_(host, non_blocking=True)
        run_step(st)
        out_pin.copy_(st["out"], non_blocking=True)

    for _ in range(args.warmup):
        body()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            body()
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(args.warmup):
        flush_l2(0)
        graph.replay()
    torch.cuda.synchronize()
    barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    stream = torch.cuda.current_stream()
    for s in range(args.steps):
        flush_l2(s)
        ev[s][0].record(stream)
        graph.replay()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in ev]
    # the copies really carried this step's data: the host copy of out is the device's
    if not torch.equal(out_pin.view(torch.int16), st["out"].cpu().view(torch.int16)):
        raise RuntimeError("e2e: the output copied to the host differs from the device output")
    del graph
    return times, {"mode": "graph replay: h2d copies + step + d2h copy",
                   "h2d_bytes_per_step": int(sum(host.numel() * host.element_size() for _, host in h2d)),
                   "d2h_bytes_per_step": int(out_pin.numel() * out_pin.element_size())}


L2_NOTE = ("GPU arm: L2 flushed before every step (256 MiB write + 256 MiB read, outside the timed events); "
           "oracle arm: host cores")


MEANS_KINDS = {
    "fp32": "fp32",
    "bf16": "bf16",
    "dual": "dual: the fp32 selection, read from a bf16 copy (fp32 + bf16 means + row error radii)",
}


def means_kind(args) -> str:
    """bf16 (--means-bf16), dual (--means-dual: the fp32 selection read from a
    bf16 copy), fp32 (--means-fp32); by default dual, except fp32 for
    per-page shared-prompt means, whose scan reads mostly from L2 (dual
    per-page means stay available with --means-dual)."""
    chosen = [f for f in ("means_bf16", "means_fp32", "means_dual") if getattr(args, f, False)]
    if len(chosen) > 1:
        raise SystemExit("--means-bf16, --means-fp32 and --means-dual exclude each other")
    if getattr(args, "means_bf16", False):
        return "bf16"
    if getattr(args, "means_dual", False):
        return "dual"
    if getattr(args, "means_fp32", False) or getattr(args, "shared_prefix", 1) > 1:
        return "fp32"
    return "dual"


def means_bytes_per_dim(args) -> float:
    """Block-mean bytes the select streams per head dim: fp32 4, bf16 2, dual
    2 + the row's 4-byte error radius spread over the 128 dims (the fp32 rows it
    rescores are counted as traffic, not here)."""
    return {"fp32": 4.0, "bf16": 2.0, "dual": 2.0 + 4.0 / 128}[means_kind(args)]


def workload_config(w0: ki.Workload, k: int, world: int, kv_layout: str = "contiguous [B][Hkv][Lcap][D]",
                    means: str = "fp32", token_kt: int = 0) -> dict:
    """The JSON line's config: the workload as named, the same in both arms."""
    return {
        "workload": w0.name, "batch": w0.B, "kv_heads": w0.Hkv, "q_heads": w0.Hq,
        "head_dim": w0.D, "context": [w0.Lmin, w0.Lmax], "block_size": w0.bs,
        "top_k_blocks": k, "append_tokens": w0.n_append,
        "global_batch": w0.B * world, "parallelism": f"dp{world}",
        "l2": L2_NOTE,
        "kv_layout": kv_layout,
        "block_means": MEANS_KINDS[means],
        **({"attention": f"token-level top-k, {token_kt} tokens per query head"} if token_kt else {}),
    }


def report(args, rank, world, rec: RankRecord):
    """Reduces the ranks' records (max over ranks) and prints the JSON line
    on rank 0."""
    import torch.distributed as dist
    names = [name for name, _, _ in rec.parts]
    means = [statistics.mean(rec.part_ms[n]) for n in names]
    upd = statistics.mean(rec.upd_ms) if rec.upd_ms else 0.0
    # one collective: totals, per-kernel means, then every step's time (the
    # step's max over ranks, for its percentiles)
    red = reduce_max_list([sum(rec.per_step), sum(rec.e2e_ms), rec.wall, upd, *means, *rec.per_step])
    total_ms, e2e_total, wall, upd = red[:4]
    avg = dict(zip(names, red[4:4 + len(names)]))
    step_max_ms = red[4 + len(names):]
    clocks_all = [rec.clocks]
    if world > 1:
        clocks_all = [None] * world
        dist.all_gather_object(clocks_all, rec.clocks)
        status = reduce_max(float(rec.status))
    else:
        status = rec.status
    if rank != 0:
        return
    w0, w, k = rec.w0, rec.w, rec.k
    steps = len(rec.per_step)
    ms_per_step = total_ms / steps
    qh_per_step = w.B * w.Hq
    value = whole_job_value(world, qh_per_step, steps, total_ms)
    e2e_value = whole_job_value(world, qh_per_step, len(rec.e2e_ms), e2e_total)
    peak, peak_kind = measured_peak()
    gbs = {name: nbytes / (avg[name] * 1e-3) / 1e9 for name, nbytes, _ in rec.parts}
    step_gbs = sum(nbytes for _, nbytes, _ in rec.parts) / (ms_per_step * 1e-3) / 1e9
    dominant, dom_bytes, dom_file = max(rec.parts, key=lambda pt: avg[pt[0]])
    dom_gbs = gbs[dominant]
    clocks = dict(rec.clocks)
    if world > 1:
        clocks["per_rank"] = clocks_all
        clocks["reasons"] = sorted(set(r for c in clocks_all for r in (c or {}).get("reasons", [])))
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "query-heads/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "step_us": step_percentiles(step_max_ms),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded Philox N(0,1) q/K/V, 5% heavy-hitter key-bias blocks)",
        "config": workload_config(w0, k, world, rec.kv_layout, means_kind(args), rec.token_kt),
        "impl": "kin",
        "gpu_launches": rec.launches_per_step * steps,  # in the timed region
        "kernel_ms": {**avg, **({"update": upd} if rec.upd_ms else {})},
        "hbm_gbs": {**gbs, "step": step_gbs},
        "hbm_frac": {**{n: v / peak for n, v in gbs.items()}, "step": step_gbs / peak,
                     "peak_gbs": peak, "peak_kind": peak_kind},
        "roofline": {
            "kernel": dominant, "bound": "hbm", "achieved": dom_gbs, "peak": peak, "unit": "GB/s",
            "frac": dom_gbs / peak, "peak_kind": peak_kind,
            "algorithmic_bytes_per_launch": dom_bytes,
            "traffic": profiled_traffic(dom_file, w0.name, k),
        },
        "e2e": {"value": e2e_value, "unit": "query-heads/s", **rec.e2e},
        "eflops": eflops_report(w, k, rec.lens_final, ms_per_step, means_bytes_per_dim(args), rec.token_kt),
        "clocks": clocks,
        "wall_s_timed_region": wall,
        "device_status": int(status),
    }
    if world == 1 and not args.no_cpu_baseline and not rec.token_kt:
        line["cpu_baseline"] = cpu_baseline(w0, k, budget_s=args.cpu_seconds)
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------- oracle (CPU) arm
def sample_pairs_default() -> int:
    """Pairs in the oracle's timing sample: two per host thread, at least 32,
    so every thread stays busy through a pass."""
    return max(32, 2 * (os.cpu_count() or 1))


class OracleSample:
    """A bounded sample of (batch, kv-head) pairs of a workload, prepared on
    the host for the fp64 oracle: K/V rows regenerated from the seeded
    generator and block means precomputed (resident state, as on the GPU)."""

    def __init__(self, w: ki.Workload, k: int, max_pairs: int):
        from concurrent.futures import ThreadPoolExecutor
        import oracle
        self.oracle = oracle
        self.w, self.k = w, k
        lens_final, _, hh = ki.case_meta(w)
        P = w.B * w.Hkv
        n = min(max_pairs, P)
        pairs = sorted(set(int(round(i * (P - 1) / max(n - 1, 1))) for i in range(n)))
        self.n, self.P = len(pairs), P
        Lmax = int(max(lens_final[p // w.Hkv] for p in pairs))
        nbcap = -(-Lmax // w.bs)
        q_all = ki.fill_q(w.seed, w.B, w.Hq, w.D)
        self.Kc = np.zeros((self.n, 1, Lmax, w.D), np.uint16)
        self.Vc = np.zeros_like(self.Kc)
        self.means = np.zeros((self.n, 1, nbcap, w.D))
        self.qs = np.zeros((self.n, w.g, w.D), np.uint16)
        self.lens = np.zeros(self.n, np.int32)
        self.threads = os.cpu_count() or 1

        def fill(i):  # the generator and the oracle are C calls that release the GIL
            b, h = divmod(pairs[i], w.Hkv)
            L = int(lens_final[b])
            self.Kc[i, 0, :L], self.Vc[i, 0, :L] = ki.pair_rows(w, hh, b, h, L)
            self.means[i, 0, :-(-L // w.bs)] = oracle.block_means(self.Kc[i, 0], L, w.bs)
            self.qs[i] = q_all[b, h * w.g:(h + 1) * w.g]
            self.lens[i] = L

        with ThreadPoolExecutor(self.threads) as ex:
            list(ex.map(fill, range(self.n)))

    def run_pass(self):
        w = self.w
        self.oracle.decode_pairs(Hkv=1, Hq=w.g, bs=w.bs, seq_lens=self.lens, q=self.qs, Kc=self.Kc,
                                 Vc=self.Vc, means=self.means, k=self.k, scale=1 / math.sqrt(w.D),
                                 pairs=np.arange(self.n), threads=self.threads)
        return self.n * w.g  # query heads processed

    def describe(self, passes, seconds):
        return (f"{self.n} of {self.P} (batch, kv-head) pairs of {self.w.name} (k={self.k}), {passes} "
                f"passes in {seconds:.3f} s on {self.threads} threads; scores + top-k + attention in fp64, "
                f"block means precomputed")


def cpu_baseline(w: ki.Workload, k: int, budget_s: float = 12.0, max_pairs: int = 0):
    """The oracle (as it stands) on the host cores: whole passes over the
    sample until `budget_s` has elapsed; query-heads/s."""
    smp = OracleSample(w, k, max_pairs or sample_pairs_default())
    t0 = time.perf_counter()
    passes, qh = 0, 0
    while True:
        qh += smp.run_pass()
        passes += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": qh / el, "unit": "query-heads/s", "cores": smp.threads, "kind": "oracle",
            "sample": smp.describe(passes, el)}


def reference_arm(args):
    """The oracle as the reference arm: each step is one pass over a bounded
    sample of the workload's pairs (the CPU baseline's sample by default),
    timed on the host clock.  ms_per_step is the time of that sampled pass,
    not of the whole batch; value (query-heads/s) is the sample's rate."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = ki.WORKLOADS[args.workload]
    k = args.k or w.k
    t0 = time.perf_counter()
    smp = OracleSample(w, k, max_pairs=args.ref_pairs or sample_pairs_default())
    for _ in range(args.warmup):
        smp.run_pass()
    el, qh, pass_ms = 0.0, 0, []
    for _ in range(args.steps):
        a = time.perf_counter()
        qh += smp.run_pass()
        pass_ms.append((time.perf_counter() - a) * 1e3)
        el += pass_ms[-1] / 1e3
    value = qh / el
    line = {
        "metric": METRIC, "value": value, "unit": "query-heads/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "step_us": step_percentiles(pass_ms),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, k, int(os.environ.get("WORLD_SIZE", "1")), means=means_kind(args)),
        "step": f"one pass over {smp.n} sampled (batch, kv-head) pairs ({smp.n * w.g} query heads)",
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "query-heads/s", "cores": smp.threads, "kind": "oracle",
                         "sample": smp.describe(args.steps, el)},
        "e2e": {"value": value, "unit": "query-heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kin", choices=["kin", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(ki.WORKLOADS))
    ap.add_argument("--k", type=int, default=0, help="override the workload's block budget")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-pairs", type=int, default=0,
                    help="(batch, kv-head) pairs per reference-arm step (default: the CPU baseline's sample)")
    ap.add_argument("--paged", action="store_true", help="KV cache in a shuffled page pool with a block table")
    ap.add_argument("--means-bf16", action="store_true", help="bf16 block means (the extended calls)")
    ap.add_argument("--means-fp32", action="store_true",
                    help="fp32 block means only: the plain select, which scans them in full (the default keeps dual "
                         "means and returns the same selection from a bf16 copy; see kin.h KIN_MEANS_DUAL)")
    ap.add_argument("--means-dual", action="store_true",
                    help="dual block means also with --shared-prefix (per page; the default elsewhere)")
    ap.add_argument("--page-order", default="shuffled", choices=["shuffled", "sequential"],
                    help="page pool order for --paged / --shared-prefix")
    ap.add_argument("--shared-prefix", type=int, default=1,
                    help="groups of N samples share a prompt (paged, block means per page)")
    ap.add_argument("--token-topk", action="store_true",
                    help="token-level top-k attention instead of the block path (budget = k blocks x bs tokens)")
    args = ap.parse_args(argv)
    rc = launch_ranks(args)
    if rc is not None:  # this process launched the ranks
        return rc
    if args.warmup < 3 and args.impl == "kin":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())

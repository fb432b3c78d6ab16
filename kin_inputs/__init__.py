"""Seeded synthetic decode-batch inputs for block top-k sparse decode attention.

This module is shared by the tests, the benchmark and the CPU baseline.  It
holds no arithmetic of the attention method itself: it only draws q, the K/V
caches, ragged sequence lengths and the heavy-hitter key bias from a
counter-based generator (Philox4x32-10 + Box-Muller, see ``csrc/kg_core.h``).
The host library (``libkg_host.so``, gcc) and the device library
(``libkg_cuda.so``, nvcc) produce identical bf16 bits, so an oracle can
regenerate any (batch, kv-head) slice of a cache that only exists on the GPU.

Workload recipe (the decode-layer shapes named by the Kinetics pages: Qwen3
models decoding with a 32K KV cache, "Kinetics: Rethinking Test-Time Scaling
Law", author response W2&Q2 "Real-world latency benchmarks"; block sizes and
budgets from the block-size ablation in response Q4):
  * q, K, V ~ N(0, 1) drawn in double, rounded to fp32 then to bf16 (RNE);
  * per (b, kv head) a bias vector beta ~ N(0, 2^2 I_D) is added to every key
    row of round(0.05 * nb) heavy-hitter blocks chosen uniformly without
    replacement (block 0 and the current block are eligible);
  * ragged lengths are uniform integers in [Lmin, Lmax].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_CSRC = os.path.join(_HERE, "csrc")
HOST_LIB = os.path.join(_HERE, "libkg_host.so")
CUDA_LIB = os.path.join(_HERE, "libkg_cuda.so")

TID_Q, TID_K, TID_V, TID_BETA, TID_HH, TID_LEN = 1, 2, 3, 4, 5, 6
BF16_NAN = 0x7FC0


def build(cuda: bool = True, verbose: bool = False) -> None:
    """Compile the host generator (gcc) and, if ``cuda``, the device one (nvcc)."""
    host_cmd = [
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
        "-fvisibility=hidden", "-I", _CSRC, os.path.join(_CSRC, "kg_host.c"),
        "-o", HOST_LIB, "-lm",
    ]
    _run(host_cmd, verbose)
    if cuda:
        cuda_cmd = [
            "nvcc", "-O3", "--fmad=false", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
            "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-I", _CSRC,
            os.path.join(_CSRC, "kg_cuda.cu"), "-o", CUDA_LIB,
        ]
        _run(cuda_cmd, verbose)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


_host_lib = None
_cuda_lib = None


def _host():
    global _host_lib
    if _host_lib is None:
        if not os.path.exists(HOST_LIB):
            build(cuda=False)
        lib = ctypes.CDLL(HOST_LIB)
        u32, i32, i64 = ctypes.c_uint32, ctypes.c_int, ctypes.c_int64
        vp = ctypes.c_void_p
        lib.kg_philox.argtypes = [vp, vp, vp]
        lib.kg_log_d.argtypes = [ctypes.c_double]
        lib.kg_log_d.restype = ctypes.c_double
        lib.kg_sincos_turns_d.argtypes = [ctypes.c_double, vp, vp]
        lib.kg_normal4_d.argtypes = [u32, u32, u32, u32, vp]
        lib.kg_bf16_from_f32.argtypes = [vp, i64, vp]
        lib.kg_fill_q.argtypes = [u32, i32, i32, i32, vp]
        lib.kg_seq_lens.argtypes = [u32, i32, i32, i32, vp]
        lib.kg_heavy_flags.argtypes = [u32, i32, i32, i32, i32, vp, i32, i32, vp]
        lib.kg_fill_kv_rows.argtypes = [u32, i32, u32, i32, i32, i32, i32, vp, vp]
        lib.kg_fill_kv_cache.argtypes = [u32, i32, i32, i32, i32, i32, i32, vp, vp, i32, i32, vp]
        _host_lib = lib
    return _host_lib


def _cuda():
    global _cuda_lib
    if _cuda_lib is None:
        if not os.path.exists(CUDA_LIB):
            raise RuntimeError(f"{CUDA_LIB} is missing: run kin_inputs.build()")
        lib = ctypes.CDLL(CUDA_LIB)
        u32, i32, vp = ctypes.c_uint32, ctypes.c_int, ctypes.c_void_p
        lib.kg_cuda_fill_kv_cache.argtypes = [u32, i32, i32, i32, i32, i32, i32, vp, vp, i32, i32, vp, vp]
        lib.kg_cuda_fill_kv_cache.restype = ctypes.c_int
        _cuda_lib = lib
    return _cuda_lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- primitives
def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    _host().kg_philox(_ptr(c), _ptr(k), _ptr(out))
    return out


def log_d(u: float) -> float:
    return _host().kg_log_d(float(u))


def sincos_turns(t: float):
    s, c = ctypes.c_double(), ctypes.c_double()
    _host().kg_sincos_turns_d(float(t), ctypes.byref(s), ctypes.byref(c))
    return s.value, c.value


def normal4(seed: int, tid: int, c0: int, c1: int) -> np.ndarray:
    z = np.zeros(4, dtype=np.float64)
    _host().kg_normal4_d(seed, tid, c0, c1, _ptr(z))
    return z


def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _host().kg_bf16_from_f32(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------- tensors
def fill_q(seed: int, B: int, Hq: int, D: int) -> np.ndarray:
    out = np.empty((B, Hq, D), dtype=np.uint16)
    _host().kg_fill_q(seed, B, Hq, D, _ptr(out))
    return out


def seq_lens(seed: int, B: int, Lmin: int, Lmax: int) -> np.ndarray:
    out = np.empty(B, dtype=np.int32)
    _host().kg_seq_lens(seed, B, Lmin, Lmax, _ptr(out))
    return out


def heavy_flags(seed: int, B: int, Hkv: int, nbcap: int, bs: int, lens: np.ndarray,
                num: int = 5, den: int = 100) -> np.ndarray:
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    out = np.empty((B, Hkv, nbcap), dtype=np.uint8)
    _host().kg_heavy_flags(seed, B, Hkv, nbcap, bs, _ptr(lens), num, den, _ptr(out))
    return out


def kv_rows(seed: int, is_k: bool, pair: int, t0: int, t1: int, D: int, bs: int,
            hh_pair: Optional[np.ndarray]) -> np.ndarray:
    out = np.empty((max(t1 - t0, 0), D), dtype=np.uint16)
    hp = None
    if hh_pair is not None:
        hh_pair = np.ascontiguousarray(hh_pair, dtype=np.uint8)
        hp = _ptr(hh_pair)
    if t1 > t0:
        _host().kg_fill_kv_rows(seed, int(is_k), pair, t0, t1, D, bs, hp, _ptr(out))
    return out


def kv_cache_host(seed: int, is_k: bool, B: int, Hkv: int, Lcap: int, D: int, bs: int,
                  lens: np.ndarray, hh: Optional[np.ndarray], poison: bool) -> np.ndarray:
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    out = np.empty((B, Hkv, Lcap, D), dtype=np.uint16)
    nbcap = hh.shape[-1] if hh is not None else 0
    hp = _ptr(np.ascontiguousarray(hh)) if hh is not None else None
    _host().kg_fill_kv_cache(seed, int(is_k), B, Hkv, Lcap, D, bs, _ptr(lens), hp, nbcap,
                             int(poison), _ptr(out))
    return out


def kv_cache_device(seed: int, is_k: bool, B: int, Hkv: int, Lcap: int, D: int, bs: int,
                    lens_dev, hh_dev, poison: bool, out_dev, stream: int = 0) -> None:
    """Fill a device cache tensor (any 2-byte dtype, [B,Hkv,Lcap,D]) in place."""
    nbcap = hh_dev.shape[-1] if hh_dev is not None else 0
    rc = _cuda().kg_cuda_fill_kv_cache(
        seed, int(is_k), B, Hkv, Lcap, D, bs, ctypes.c_void_p(lens_dev.data_ptr()),
        ctypes.c_void_p(hh_dev.data_ptr()) if hh_dev is not None else None, nbcap, int(poison),
        ctypes.c_void_p(out_dev.data_ptr()), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"kg_cuda_fill_kv_cache failed with CUDA error {rc}")


# ----------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Workload:
    """One synthetic decode-layer batch.

    Lengths are uniform in [Lmin, Lmax] (equal when Lmin == Lmax).  With
    ``n_append`` > 0 the cache initially holds ``L - n_append`` tokens per
    sequence and the step appends the next ``n_append`` rows of the same K/V
    field; heavy-hitter blocks are drawn on the final length.
    """
    name: str
    B: int
    Hkv: int
    Hq: int
    D: int
    bs: int
    Lmin: int
    Lmax: int
    k: int
    seed: int
    n_append: int = 0
    Lcap: int = 0
    hh_num: int = 5
    hh_den: int = 100
    lens: tuple = ()   # explicit final lengths (overrides the draw when given)

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def cap(self) -> int:
        return self.Lcap if self.Lcap else self.Lmax

    @property
    def nbcap(self) -> int:
        return -(-self.cap // self.bs)

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five decode workloads (sizes, seeds and distributions as stated above).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 4, 128, 16, 4096, 4096, 32, 0),
    "qwen3_8b_32k": Workload("qwen3_8b_32k", 32, 8, 32, 128, 16, 32768, 32768, 256, 1),
    "qwen3_14b_ragged": Workload("qwen3_14b_ragged", 64, 8, 40, 128, 16, 8192, 32768, 128, 2),
    "qwen3_32b_128k_append": Workload("qwen3_32b_128k_append", 16, 8, 64, 128, 32, 131072, 131072,
                                      128, 3, n_append=1),
    "qwen3_0p6b_sweep": Workload("qwen3_0p6b_sweep", 256, 8, 16, 128, 16, 16384, 16384, 128, 4),
}
SWEEP_K = (32, 64, 128, 256, 512, 1024)


@dataclass
class HostCase:
    """Host-materialised inputs of a Workload (bf16 as uint16 bit patterns)."""
    w: Workload
    q: np.ndarray            # [B,Hq,D]
    lens_final: np.ndarray   # [B] int32, length after the append
    lens_pre: np.ndarray     # [B] int32, length held by the cache before the step
    hh: np.ndarray           # [B,Hkv,nbcap] uint8
    k_cache: np.ndarray      # [B,Hkv,Lcap,D], rows >= lens_pre poisoned (NaN)
    v_cache: np.ndarray
    k_new: np.ndarray        # [B,Hkv,n_append,D]
    v_new: np.ndarray


def case_meta(w: Workload):
    if w.lens:
        lens_final = np.array(w.lens, dtype=np.int32)
        assert lens_final.shape == (w.B,)
    else:
        lens_final = seq_lens(w.seed, w.B, w.Lmin, w.Lmax)
    lens_pre = (lens_final - w.n_append).astype(np.int32)
    hh = heavy_flags(w.seed, w.B, w.Hkv, w.nbcap, w.bs, lens_final, w.hh_num, w.hh_den)
    return lens_final, lens_pre, hh


def make_host_case(w: Workload, poison: bool = True) -> HostCase:
    lens_final, lens_pre, hh = case_meta(w)
    q = fill_q(w.seed, w.B, w.Hq, w.D)
    kc = kv_cache_host(w.seed, True, w.B, w.Hkv, w.cap, w.D, w.bs, lens_pre, hh, poison)
    vc = kv_cache_host(w.seed, False, w.B, w.Hkv, w.cap, w.D, w.bs, lens_pre, hh, poison)
    n = w.n_append
    kn = np.empty((w.B, w.Hkv, n, w.D), dtype=np.uint16)
    vn = np.empty((w.B, w.Hkv, n, w.D), dtype=np.uint16)
    for b in range(w.B):
        for h in range(w.Hkv):
            p = b * w.Hkv + h
            t0 = int(lens_pre[b])
            kn[b, h] = kv_rows(w.seed, True, p, t0, t0 + n, w.D, w.bs, hh[b, h])
            vn[b, h] = kv_rows(w.seed, False, p, t0, t0 + n, w.D, w.bs, None)
    return HostCase(w, q, lens_final, lens_pre, hh, kc, vc, kn, vn)


def pair_rows(w: Workload, hh: np.ndarray, b: int, h: int, L: int):
    """Host regeneration of the first L rows of K and V for one (b, kv head)."""
    p = b * w.Hkv + h
    k = kv_rows(w.seed, True, p, 0, L, w.D, w.bs, hh[b, h])
    v = kv_rows(w.seed, False, p, 0, L, w.D, w.bs, None)
    return k, v

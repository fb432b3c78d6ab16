"""GPU parity on the block top-k's code paths and their boundaries, and on
seeded random shapes; every (batch, kv head) against the oracle.

The top-k CTA has 256, 512 or 1024 threads, picked from the block capacity
(up to 1024 / 2048 / 4096 blocks), and halved (down to 128) while the
capacity still fits 8 keys per thread and the pairs outnumber the resident
CTAs.  Each pair then
keeps its keys in registers, 4 or 8 per thread, or in shared memory beyond
8 per thread.  The cases below sit on both sides of every switch, so a
mistake in a boundary (an off-by-one in a key count, a halving that leaves
too few threads) shows up as a wrong selection.
"""
import numpy as np
import pytest
import torch

import kin_inputs as ki
from kin_testlib import D, all_pairs, check_pairs, gpu_step, make_device_case, random_shapes

pytestmark = pytest.mark.gpu
W = ki.Workload

BOUNDARY = [
    # name, B, Hkv, Hq, D, bs, Lmin, Lmax, k, seed, (extra); capacity = Lcap / 16 blocks
    W("cap1024_regs4_256", 2, 1, 4, D, 16, 0, 0, 100, 60, Lcap=1024 * 16, lens=(1024 * 16, 1023 * 16 + 1)),
    W("cap1025_regs4_512", 2, 1, 4, D, 16, 0, 0, 100, 61, Lcap=1025 * 16, lens=(1025 * 16, 700 * 16)),
    W("cap2048_regs4_512", 1, 2, 8, D, 16, 0, 0, 256, 62, Lcap=2048 * 16, lens=(2048 * 16,)),
    W("cap2049_regs4_1024", 1, 2, 8, D, 16, 0, 0, 256, 63, Lcap=2049 * 16, lens=(2049 * 16,)),
    W("cap4096_regs4_1024", 1, 2, 4, D, 16, 0, 0, 300, 64, Lcap=4096 * 16, lens=(4096 * 16,)),
    W("cap4097_regs8_1024", 1, 2, 4, D, 16, 0, 0, 300, 65, Lcap=4097 * 16, lens=(4097 * 16,)),
    W("cap8192_regs8_1024", 1, 1, 4, D, 16, 0, 0, 500, 66, Lcap=8192 * 16, lens=(8192 * 16,)),
    W("cap8193_memory_1024", 1, 1, 4, D, 16, 0, 0, 500, 67, Lcap=8193 * 16, lens=(8193 * 16,)),
    # one launch, every path: dense (nb <= k), 4 and 8 keys per thread, keys in memory
    W("ragged_every_path", 7, 1, 2, D, 16, 0, 0, 64, 68, Lcap=8193 * 16,
      lens=(1, 64 * 16, 100 * 16 + 3, 4096 * 16, 4097 * 16, 8192 * 16, 8193 * 16)),
]

# pairs beyond the resident CTAs: 2048 blocks at 512 threads halve to 256
# (8 keys per thread); 4096 blocks at 1024 halve to 512; 1024 blocks at 256
# halve to 128
HALVING = [
    W("halve_512_to_256", 38, 8, 8, D, 16, 16400, 32768, 128, 69, Lcap=32768),
    W("halve_1024_to_512", 19, 8, 8, D, 16, 16400, 65536, 128, 70, Lcap=65536),
    W("halve_256_to_128", 76, 8, 8, D, 16, 500, 16384, 64, 72, Lcap=16384),
]


def _every_pair(w):
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    means = dc.means.cpu().numpy()
    del dc.k_cache, dc.v_cache
    torch.cuda.empty_cache()
    near = check_pairs(dc, [(w.k, gr)], all_pairs(w), gpu_means=means)
    print(f"{w.name}: {w.B * w.Hkv} pairs against the oracle, {near} near-tie selections")


@pytest.mark.parametrize("w", BOUNDARY, ids=lambda w: w.name)
def test_topk_path_boundaries(w):
    _every_pair(w)


@pytest.mark.parametrize("w", HALVING, ids=lambda w: w.name)
def test_topk_thread_halving(w):
    _every_pair(w)


@pytest.mark.parametrize("w", random_shapes(12, seed=71), ids=lambda w: w.name)
def test_random_shapes_every_pair(w):
    _every_pair(w)

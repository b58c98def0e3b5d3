"""Data-parallel delayed scaling over torch.distributed: gloo, 2 ranks, CPU.

Each rank holds a shard of the rows of a tensor.  The protocol of
``fp8_delayed_scaling_02_b200.dp`` (local amax, MAX all-reduce of one float,
fold) must leave every rank with the ring one process gets from the whole
tensor.  The casts and folds here are the oracle's (the GPU kernels of the
same protocol are covered by tests/test_next_gpu.py); what this checks is the
host logic and the collective.
"""

import socket
from datetime import timedelta

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp8_delayed_scaling_02_b200 import dp
from fp8_delayed_scaling_02_b200 import synthetic as S
from oracle import recipe as R

WORLD = 2
ROWS = 64  # rows per rank
COLS = 96
STEPS = 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full(step):
    # Outlier magnitude changes with the step, so the rank that holds the
    # tensor's amax changes too.
    return S.normal_with_outliers((ROWS * WORLD, COLS), seed=300 + step, frac=0.01, mult=5.0 * (1 + step % 4))


def _ring_vector(ring):
    return np.concatenate([ring.history.astype(np.float64), [ring.scale, ring.scale_inv, ring.idx]])


def _worker(rank, port, fmt, results):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=timedelta(seconds=60))
    try:
        ring = R.Ring()
        codes = []
        for step in range(STEPS):
            shard = _full(step)[rank * ROWS:(rank + 1) * ROWS]
            out, _, a, sinv = R.quantize_local(shard, fmt, R.ROW, ring)
            assert sinv == np.float32(np.float32(1.0) / ring.scale)
            amax = torch.tensor([float(a)], dtype=torch.float32)
            dp.all_reduce_amax(amax)
            R.fold(ring, np.float32(amax.item()), fmt)
            codes.append(out)
        mine = torch.from_numpy(_ring_vector(ring))
        rings = [torch.zeros_like(mine) for _ in range(WORLD)]
        dist.all_gather(rings, mine)
        results.put((rank, [r.numpy() for r in rings], np.stack(codes)))
    finally:
        dist.destroy_process_group()


def _run(fmt):
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, fmt, results)) for r in range(WORLD)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(WORLD):
        rank, rings, codes = results.get(timeout=180)
        out[rank] = (rings, codes)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def _single_process(fmt, amax_of):
    """The ring after STEPS quantizes of the whole tensor, folding amax_of(full)."""
    ring = R.Ring()
    codes = []
    for step in range(STEPS):
        full = _full(step)
        out, _, _, _ = R.quantize_local(full, fmt, R.ROW, ring)
        R.fold(ring, amax_of(R.to_float32(full)), fmt)
        codes.append(out)
    return ring, np.stack(codes)


def test_dp_rings_match_the_whole_tensor_fold():
    for fmt in (R.F.E4M3, R.F.E5M2):
        out = _run(fmt)
        ref_ring, ref_codes = _single_process(fmt, R.amax)
        ref = _ring_vector(ref_ring)
        for rank, (rings, codes) in out.items():
            for r in rings:  # every rank ends with the same ring, bit for bit
                assert np.array_equal(r.astype(np.float32).view(np.uint32), ref.astype(np.float32).view(np.uint32))
            # each rank's codes are its rows of the whole tensor's codes
            assert np.array_equal(codes, ref_codes[:, rank * ROWS:(rank + 1) * ROWS])


def test_the_check_catches_a_local_or_summed_amax():
    """Folding only one shard's amax, or the sum of the shards', gives another ring."""
    ref = _ring_vector(_single_process(R.F.E4M3, R.amax)[0])
    local = _ring_vector(_single_process(R.F.E4M3, lambda xf: R.amax(xf[:ROWS]))[0])
    summed = _ring_vector(_single_process(R.F.E4M3, lambda xf: np.float32(R.amax(xf[:ROWS]) + R.amax(xf[ROWS:])))[0])
    assert not np.array_equal(ref, local)
    assert not np.array_equal(ref, summed)


# ---- the FP8-output GEMM's shard protocol (oracle arithmetic, gloo) ----------

from oracle import gemm as OG  # noqa: E402

K_GEMM, N_GEMM = 64, 48


def _gemm_full(step):
    a = S.fp8_codes((ROWS * WORLD, K_GEMM), seed=700 + step).numpy()
    b = S.fp8_codes((N_GEMM, K_GEMM), seed=800).numpy()
    return a, b


def _gemm_worker(rank, port, results):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=timedelta(seconds=60))
    try:
        ring = R.Ring()
        codes = []
        for step in range(STEPS):
            a, b = _gemm_full(step)
            ref, _ = OG.mm_fp8(a[rank * ROWS:(rank + 1) * ROWS], b, R.F.E4M3, R.F.E4M3, 2.0 ** -6, 2.0 ** -6)
            y = ref.astype(np.float32)  # the float64 sum is exact; every side rounds it to float32 alike
            codes.append(R.scaled_codes(y, ring.scale, R.F.E4M3))
            amax = torch.tensor([float(R.amax(y))], dtype=torch.float32)
            dp.all_reduce_amax(amax)
            R.fold(ring, np.float32(amax.item()), R.F.E4M3)
        mine = torch.from_numpy(_ring_vector(ring))
        rings = [torch.zeros_like(mine) for _ in range(WORLD)]
        dist.all_gather(rings, mine)
        results.put((rank, [r.numpy() for r in rings], np.stack(codes)))
    finally:
        dist.destroy_process_group()


def test_dp_fp8_output_rings_match_the_whole_output_fold():
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gemm_worker, args=(r, port, results)) for r in range(WORLD)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(WORLD):
        rank, rings, codes = results.get(timeout=180)
        out[rank] = (rings, codes)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ring = R.Ring()
    ref_codes = []
    for step in range(STEPS):
        a, b = _gemm_full(step)
        ref, _ = OG.mm_fp8(a, b, R.F.E4M3, R.F.E4M3, 2.0 ** -6, 2.0 ** -6)
        y = ref.astype(np.float32)
        ref_codes.append(R.scaled_codes(y, ring.scale, R.F.E4M3))
        R.fold(ring, R.amax(y), R.F.E4M3)
    ref_ring = _ring_vector(ring)
    assert ref_ring[R.HISTORY_LEN] != 1.0  # the scale moved: the fold saw real amaxes
    for rank, (rings, codes) in out.items():
        for r in rings:
            assert np.array_equal(r.astype(np.float32).view(np.uint32), ref_ring.astype(np.float32).view(np.uint32))
        assert np.array_equal(codes, np.stack(ref_codes)[:, rank * ROWS:(rank + 1) * ROWS])

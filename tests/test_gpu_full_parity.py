"""GPU parity at full size, every element: the quantizer (and its two
comparators, and the float32 transform) on every config at the sizes of the
benchmark's per-config table, compared element by element with the CPU
oracle.

The oracle runs in row chunks over a pool of spawned worker processes
(numpy only; a spawned process does not inherit this process's CUDA state).
Per config the test reports how many scale bytes and codes differ from the
oracle's, how many of those lie outside the literal reading of the rule (a
scaled value not within 1e-5 relative of an E2M1 midpoint, a block maximum
not within 1e-5 relative of a power of two), and how many float32
transformed values lie more than 1e-5 of their own value from the oracle's.
The test asserts the literal reading: no code or scale difference outside
its band, and no transformed value off by more than 1e-5 relative
(kq_transform computes in double).  With
``KQ_PARITY_REPORT=<path>`` the counts are also written there as JSON.
"""
import json
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

import workloads as w
from tests.parity import check_chunk, merge_stats

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")
DEV = "cuda:0"
CHUNK_ELEMENTS = 4 << 20
REPORT = {}


def _workers() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(32, n))


@pytest.fixture(scope="module")
def pool():
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    p = mp.get_context("spawn").Pool(_workers())
    yield p
    p.close()
    p.join()
    path = os.environ.get("KQ_PARITY_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(REPORT, f, indent=1, sort_keys=True)


def _gpu_outputs(c):
    x = c.x.to(DEV)
    p = torch.from_numpy(c.params).to(DEV)
    inv = torch.from_numpy(c.inv_s).to(DEV)
    q, s = kq.quantize(x, p)
    y = kq.transform(x, p)
    qh, sh = kq.quantize_hadamard(x)
    qs, ss = kq.quantize_smooth(x, inv)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in
           dict(q=q, s=s, y=y, qh=qh, sh=sh, qs=qs, ss=ss).items()}
    del x, q, s, y, qh, sh, qs, ss
    return out


@pytest.mark.parametrize("key", w.all_case_keys(), ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_full_size_every_element(pool, key):
    name, di, gi = key
    c = w.make_case(name, di, gi)
    out = _gpu_outputs(c)
    bits = c.x_bits()
    rows = max(1, CHUNK_ELEMENTS // c.d)
    jobs = []
    for r in range(0, c.M, rows):
        sl = slice(r, min(c.M, r + rows))
        jobs.append(("kron", bits[sl], c.params,
                     {"q": out["q"][sl], "s": out["s"][sl], "y": out["y"][sl]}))
        jobs.append(("hadamard", bits[sl], None, {"q": out["qh"][sl], "s": out["sh"][sl]}))
        jobs.append(("smooth", bits[sl], c.inv_s, {"q": out["qs"][sl], "s": out["ss"][sl]}))
    totals = {"kron": {}, "hadamard": {}, "smooth": {}}
    for job, st in zip(jobs, pool.imap(check_chunk, jobs)):
        merge_stats(totals[job[0]], st)
    REPORT[f"{name} d={c.d} gain={c.gain:g}"] = dict(totals, M=c.M, d=c.d)
    k, h, s = totals["kron"], totals["hadamard"], totals["smooth"]
    assert k["worst_transform_ratio"] < 1e-5
    # kq_transform runs in double: every value within 1e-5 of itself.
    assert k["transform_outside_relative"] == 0
    # A single float32 product is exact on both sides.
    assert s["scale_exempt"] == 0 and s["code_exempt"] == 0
    for st in (k, h):
        # The literal rule: a scale byte or code differs from the oracle's
        # only where the oracle's value lies within 1e-5 relative of a power
        # of two or of an E2M1 midpoint.  (The sign of a zero code is counted
        # apart: both signs stand for the value 0, and where the exact value
        # is a sum that cancels to about zero either is accepted.)
        assert st["scale_outside_literal"] == 0
        assert st["code_outside_literal"] == 0
        # Boundary cases are rare: at most one element in a million.
        assert st["scale_exempt"] <= max(2, st["blocks"] // 100000)
        assert st["code_exempt"] <= max(4, st["elements"] // 1000000)

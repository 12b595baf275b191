"""Per-head float64 oracle work for the full-size parity tests, run in a process pool.

Each task is one (batch, head) slice: the inputs and the GPU's outputs of that slice go
in as raw bits (bf16 as uint16, fp32 as float32), the oracle computes the head's exact
forward and backward, and only error sums come back (max |dO|, max |dlse|, squared error
and squared norm of dQ, dK, dV, and the head's weighted band torques, whose sum over
every head is the oracle's whole-problem dalpha).  Test infrastructure: it calls only
``oracle/`` and numpy.

The pool uses the ``spawn`` start method, so a worker never inherits a CUDA context, and
every worker's BLAS runs single-threaded (the elementwise work of the oracle is
single-threaded numpy anyway, so one head per core is the fastest split).
"""
import os

import numpy as np


def bf16_bits_to_f64(bits):
    """uint16 bf16 bit patterns -> the exact float64 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def head_task(task):
    """One head: exact oracle results for the slice, compared with the GPU's."""
    from oracle import rope_attn_ref as ref

    n, d, causal, base = task["n"], task["d"], task["causal"], task["base"]
    alpha = np.asarray(task["alpha"], dtype=np.float64)
    q, k, v, e = (bf16_bits_to_f64(task[x]) for x in ("q", "k", "v", "e"))
    _, th = ref.frequencies(d, base, alpha)
    phi = ref.angles(n, th)
    qt, kt = ref.rotate(q, phi), ref.rotate(k, phi)
    o, lse = ref.head_forward(qt, kt, v, causal)
    do = o - e
    dqt, dkt, dv = ref.head_backward(qt, kt, v, do, causal)
    dq = ref.rotate(dqt, phi, sign=-1.0)
    dk = ref.rotate(dkt, phi, sign=-1.0)
    pos = np.arange(n, dtype=np.float64)
    torque = pos @ (ref.band_torque(dqt, qt) + ref.band_torque(dkt, kt))

    out = {"head": task["head"], "torque": torque}
    g_o = bf16_bits_to_f64(task["g_o"])
    out["o_maxabs"] = float(np.max(np.abs(g_o - o)))
    out["lse_maxabs"] = float(np.max(np.abs(np.asarray(task["g_lse"], np.float64) - lse)))
    for name, ref_val in (("dq", dq), ("dk", dk), ("dv", dv)):
        g = bf16_bits_to_f64(task["g_" + name])
        out[name + "_err2"] = float(np.sum((g - ref_val) ** 2))
        out[name + "_norm2"] = float(np.sum(ref_val ** 2))
    return out


def _init_worker():
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"


def run_heads(tasks, processes=None):
    """head_task over every task in a spawn pool; results in task order."""
    import multiprocessing as mp

    if processes is None:
        try:
            processes = len(os.sched_getaffinity(0))
        except AttributeError:
            processes = os.cpu_count() or 1
    processes = max(1, min(processes, len(tasks)))
    # the children read these at numpy import time (set before the pool starts them)
    saved = {var: os.environ.get(var) for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                                 "MKL_NUM_THREADS")}
    for var in saved:
        os.environ[var] = "1"
    try:
        ctx = mp.get_context("spawn")
        with ctx.Pool(processes, initializer=_init_worker) as pool:
            return pool.map(head_task, tasks, chunksize=1)
    finally:
        for var, val in saved.items():
            if val is None:
                os.environ.pop(var, None)
            else:
                os.environ[var] = val

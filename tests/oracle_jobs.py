"""Oracle work for the GPU tests, run in worker processes.

Long prompts at the 4B width take the oracle minutes per prefill (its
attention loops over queries), so the GPU tests hand independent prefills to
a pool of spawned processes and run them while the GPU works.  Each job
rebuilds the seeded weights itself (nothing large crosses the process
boundary) and returns plain arrays: the last row's logits, the final state of
every chunk row and the cache contents, from which the calling process
continues decoding with its own copy of the oracle.

Only the oracle runs here; the CUDA library is never imported.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def model(shape, weight_seed):
    import numpy as np

    import oracle as O
    import synth
    return O.Model(shape, synth.make_weights(shape, weight_seed), dtype=np.float32)


def prefill(shape, weight_seed, prompt, k, mode, capacity):
    """Oracle prefill of one sequence: {"logits": last row, "s": s_k of every
    row, "kv": cache arrays by (layer, slot), "length": positions}."""
    import oracle as O
    om = model(shape, weight_seed)
    cache = O.Cache(om, capacity)
    tr = {}
    lg = O.forward_chunk(om, cache, prompt, k, mode, trace=tr)
    return {"logits": lg[-1], "s": tr["s"][-1], "kv": cache.kv, "length": cache.length}


def spec(shape, weight_seed, prompt, n_new, gamma, mode):
    """The oracle's self-speculative greedy generation (draft k=1, verify k=4)."""
    import oracle as O
    om = model(shape, weight_seed)
    toks, st = O.spec_generate(om, prompt, n_new, 1, 4, gamma, mode)
    return {"tokens": toks, "accepted_per_step": list(st.accepted_per_step)}


def restore(om, job):
    """An oracle cache holding a prefill job's result, for the calling process
    to continue decoding."""
    import oracle as O
    cache = O.Cache(om, job["kv"][next(iter(job["kv"]))][0].shape[0])
    cache.kv = job["kv"]
    cache.length = job["length"]
    return cache


def pool(workers, threads_each):
    """A process pool started with `spawn` (safe after CUDA is initialised);
    each worker's BLAS gets `threads_each` threads.  The environment is set
    only while the workers start."""
    ctx = mp.get_context("spawn")
    ex = ProcessPoolExecutor(max_workers=workers, mp_context=ctx)
    saved = {v: os.environ.get(v) for v in THREAD_VARS}
    for v in THREAD_VARS:
        os.environ[v] = str(threads_each)
    return ex, saved


def release_env(saved):
    for v, val in saved.items():
        if val is None:
            os.environ.pop(v, None)
        else:
            os.environ[v] = val

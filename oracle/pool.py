"""The oracle's serving step spread over host cores -- TEST INFRASTRUCTURE ONLY.

Used by bench.py's CPU-baseline leg to time the oracle on all host cores:
worker processes (spawned, so no CUDA state is inherited) attach to the
batch's indices and the window history in shared memory and each runs the
oracle's per-layer serving work -- count and redirect one layer's indices
with the plan in force, window sum, rebalance -- exactly as the
single-thread baseline does for every layer.  The arithmetic is the
oracle's (``oracle`` package); this module only distributes layers.
"""
from __future__ import annotations

from multiprocessing import shared_memory

import numpy as np

import oracle

_state: dict = {}


def init(idx_name: str, idx_shape, hist_name: str, hist_shape, P: int, G: int, N: int,
         gpus: int, X: int):
    """Pool initializer: attach the shared arrays."""
    from multiprocessing import resource_tracker
    shm_i = shared_memory.SharedMemory(name=idx_name)
    shm_h = shared_memory.SharedMemory(name=hist_name)
    # the creator owns the blocks: an attaching process must not unlink them
    # when it exits
    for shm in (shm_i, shm_h):
        resource_tracker.unregister(shm._name, "shared_memory")
    _state.update(idx=np.ndarray(idx_shape, np.int32, buffer=shm_i.buf),
                  hist=np.ndarray(hist_shape, np.int64, buffer=shm_h.buf),
                  shm=(shm_i, shm_h), params=(P, G, N, gpus, X), plans={})


def layer_step(layer: int) -> int:
    """One layer of the serving step (the plan in force is built once per
    layer from the history, as the single-thread baseline does)."""
    idx = _state["idx"][layer:layer + 1]
    hist = _state["hist"][:, layer:layer + 1]
    P, G, N, gpus, X = _state["params"]
    E = hist.shape[2]
    W = hist.shape[0] + 1
    plan = _state["plans"].get(layer)
    if plan is None:
        ring = np.concatenate([hist, np.zeros((1, 1, E), np.int64)], axis=0)
        plan = oracle.rebalance(oracle.window(ring, W, W - 1)[0], P, G, N, gpus, slots=X)
        _state["plans"][layer] = plan
    counts, _ = oracle.count_loads(idx, E)
    oracle.redirect(idx, plan[3], plan[2])
    ring = np.concatenate([hist, counts[None]], axis=0)
    loads = oracle.window(ring, W, W - 1)[0]
    oracle.rebalance(loads, P, G, N, gpus, slots=X)
    return layer


def main(argv=None):
    """``python -m oracle.pool '<json>'``: times the pool on inputs already in
    shared memory -- for ``seconds``, or ``steps`` steps after ``warmup`` --
    and prints one JSON object (value in layers per second)."""
    import json
    import multiprocessing as mp
    import sys
    import time
    a = json.loads((argv or sys.argv[1:])[0])
    L = a["idx_shape"][0]
    ctx = mp.get_context("spawn")
    with ctx.Pool(a["cores"], initializer=init,
                  initargs=(a["idx_name"], tuple(a["idx_shape"]), a["hist_name"],
                            tuple(a["hist_shape"]), a["P"], a["G"], a["N"], a["gpus"],
                            a["X"])) as p:
        p.map(layer_step, range(L), chunksize=1)  # plans in force, libraries loaded
        for _ in range(a.get("warmup", 0)):
            p.map(layer_step, range(L), chunksize=1)
        n, t0 = 0, time.perf_counter()
        while True:
            p.map(layer_step, range(L), chunksize=1)
            n += 1
            el = time.perf_counter() - t0
            if ("steps" in a and n >= a["steps"]) or ("steps" not in a and el >= a["seconds"]):
                break
    print(json.dumps({"steps": n, "seconds": el, "layers_per_s": L * n / el}), flush=True)


if __name__ == "__main__":
    main()

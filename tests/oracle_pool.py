"""Worker side of the full-size parity tests: one (sequence, KV head) unit
through the CPU oracle in a spawned process.  It imports numpy and the oracle
only (no torch, no CUDA), so a pool of these starts quickly and never touches
the GPU context of the test process."""
from __future__ import annotations

import numpy as np

import oracle


def unit(task):
    """task: dict with the unit's stored bytes as a single-head contiguous
    cache ("k", "v", optional "ks", "vs"), the full layer's query "qf"
    [1, G, d], the sparse layers' queries "qs" (list of [1, G, d]), the
    dtype codes, T, window, k_global and "local" -- the GPU's index list as
    positions (-1 padded).  Returns the oracle's full-layer output, scores and
    selected positions, and each sparse layer's output over the GPU's list."""
    T = task["T"]
    r = oracle.full_attn_select(task["qf"], task["q_dtype"], task["k"], task["v"], task["kv_dtype"],
                                np.array([T], np.int32), None, T, window=task["window"],
                                k_global=task["k_global"], k_scale=task.get("ks"), v_scale=task.get("vs"))
    local = np.asarray(task["local"], np.int32).reshape(1, 1, -1)
    sparse = [oracle.sparse_attn(q, task["q_dtype"], task["k"], task["v"], task["kv_dtype"], local,
                                 k_scale=task.get("ks"), v_scale=task.get("vs"))[0] for q in task["qs"]]
    return {"key": task["key"], "out": r["out"][0], "score": r["score"][0, 0], "idx": r["idx"][0, 0],
            "sparse": sparse}

"""Shared helpers of the parity tests: run the CUDA path through the C-ABI
binding and the oracle on the same seeded bytes, and compare them with the
tolerances of the Hybrid-Block decode path:
  * attention outputs: max-abs 1e-3 (fp32 cache), 2e-2 (bf16), 6e-2 (E4M3);
  * index sets: bit-exact, except positions whose oracle score lies within
    1e-6 relative of the oracle's k-th largest selectable score.
"""
from __future__ import annotations

import numpy as np
import torch

from long_context_decode_full_b200 import synth

TOL = {"f32": 1e-3, "bf16": 2e-2, "e4m3": 6e-2}
NEAR_TIE = 1e-6
DTYPE_CODE = {"f32": 0, "bf16": 1, "e4m3": 2}


def to_device(w: synth.Workload, device="cuda") -> synth.Workload:
    def mv(t):
        return None if t is None else t.to(device)
    return synth.Workload(w.spec, mv(w.q_full), mv(w.q_sparse), mv(w.k), mv(w.v), mv(w.k_scale), mv(w.v_scale),
                          mv(w.seq_lens), mv(w.page_table), w.page_size, w.needle_pos)


def garbage_workspace(w: synth.Workload, seed=0):
    """A workspace full of random bytes: every result must be independent of
    what an earlier call left behind."""
    from long_context_decode_full_b200 import hs2
    s = w.spec
    n = hs2.full_workspace_bytes(s.batch, s.num_kv_heads, s.group, s.head_dim, w.t_cap)
    g = torch.Generator(device=w.k.device)
    g.manual_seed(seed)
    ws = torch.randint(0, 256, (n,), dtype=torch.uint8, device=w.k.device, generator=g)
    ws[:256] = 0  # the sticky error flag starts clear
    return ws


def run_gpu(w: synth.Workload, q=None, window=None, k_global=None, workspace=None, fused=False):
    from long_context_decode_full_b200 import hs2
    s = w.spec
    if workspace is None:
        workspace = garbage_workspace(w)
    return hs2.full_attn_select(w.q_full if q is None else q, w.k, w.v, w.seq_lens, w.page_table, w.page_size,
                                s.window if window is None else window, s.k_global if k_global is None else k_global,
                                w.k_scale, w.v_scale, workspace=workspace, fused=fused)


def run_gpu_sparse(w: synth.Workload, q, idx):
    from long_context_decode_full_b200 import hs2
    return hs2.sparse_attn(q, w.k, w.v, idx, w.k_scale, w.v_scale, w.page_size)


def run_oracle(oracle, w: synth.Workload, q=None, window=None, k_global=None):
    s = w.spec
    q = w.q_full if q is None else q
    return oracle.full_attn_select(
        synth.raw(q), DTYPE_CODE[s.q_dtype], synth.raw(w.k), synth.raw(w.v), DTYPE_CODE[s.kv_dtype],
        synth.raw(w.seq_lens), synth.raw(w.page_table), w.page_size,
        window=s.window if window is None else window, k_global=s.k_global if k_global is None else k_global,
        k_scale=synth.raw(w.k_scale), v_scale=synth.raw(w.v_scale))


def run_oracle_sparse(oracle, w: synth.Workload, q, idx):
    s = w.spec
    return oracle.sparse_attn(synth.raw(q), DTYPE_CODE[s.q_dtype], synth.raw(w.k), synth.raw(w.v),
                              DTYPE_CODE[s.kv_dtype], np.asarray(idx, np.int32), k_scale=synth.raw(w.k_scale),
                              v_scale=synth.raw(w.v_scale))


def out_err(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu_out.detach().float().cpu().double().numpy()
    return float(np.nanmax(np.abs(g - ref))) if g.size else 0.0


def check_out(gpu_out, ref, kv_dtype, what="out"):
    assert np.all(np.isfinite(gpu_out.detach().float().cpu().numpy())), f"{what}: non-finite values"
    err = out_err(gpu_out, ref)
    assert err <= TOL[kv_dtype], f"{what}: max-abs error {err:.3g} > {TOL[kv_dtype]}"
    return err


def slot_to_pos(w: synth.Workload, b: int) -> dict:
    T = int(w.seq_lens[b])
    sl = synth.slots_of(w, b, torch.arange(T, device=w.k.device)).cpu().numpy()
    return {int(s): t for t, s in enumerate(sl)}


def check_idx_unit(gpu_row, ora_row, ora_score, T, window, k_global, s2p):
    """Compare one (sequence, kv head) index list.  gpu_row / ora_row: slots,
    ora_score: oracle scores of positions [0, T).  Returns the number of
    positions that differ (all inside the near-tie band)."""
    L = window + k_global
    n = min(T, L)
    g = np.asarray(gpu_row)
    assert len(g) == L
    assert np.all(g[n:] == -1), "padding must be -1"
    gv = g[:n]
    assert np.all(gv >= 0), "valid entries must be slots"
    gpos = np.array([s2p[int(s)] for s in gv])
    assert np.all(np.diff(gpos) > 0), "positions must be strictly ascending"
    opos = np.array([s2p[int(s)] for s in np.asarray(ora_row)[:n]])
    win = set(range(max(0, T - window), T))
    assert win <= set(gpos.tolist()), "forced window missing"
    diff = set(gpos.tolist()) ^ set(opos.tolist())
    if diff:
        nC = max(0, T - window)
        cand = np.sort(ora_score[:nC])[::-1]
        sk = cand[k_global - 1]
        bad = [t for t in diff if not (abs(ora_score[t] - sk) <= NEAR_TIE * sk)]
        assert not bad, (f"{len(bad)} positions differ outside the near-tie band, e.g. {bad[:5]} "
                         f"(scores {[ora_score[t] for t in bad[:5]]}, k-th {sk})")
    return len(diff)


def check_full(w: synth.Workload, gpu_out, gpu_idx, ora, window=None, k_global=None):
    s = w.spec
    W = s.window if window is None else window
    K = s.k_global if k_global is None else k_global
    err = check_out(gpu_out, ora["out"], s.kv_dtype)
    gi = gpu_idx.cpu().numpy()
    ndiff = 0
    for b in range(s.batch):
        T = int(w.seq_lens[b])
        s2p = slot_to_pos(w, b)
        for h in range(s.num_kv_heads):
            ndiff += check_idx_unit(gi[b, h], ora["idx"][b, h], ora["score"][b, h], T, W, K, s2p)
    return err, ndiff


def unit_oracle(oracle, w: synth.Workload, b: int, kvh: int, q=None):
    """Oracle of one (sequence, kv head) of a large workload: gathers the
    unit's rows into a contiguous single-head cache and runs the oracle there.
    Returns (result, slots) where slots[t] is the workload slot of position t."""
    s = w.spec
    T = int(w.seq_lens[b])
    dev = w.k.device
    slots = synth.slots_of(w, b, torch.arange(T, device=dev))
    G = s.group
    qq = (w.q_full if q is None else q)[b:b + 1, kvh * G:(kvh + 1) * G]
    k = w.k[slots, kvh:kvh + 1]
    v = w.v[slots, kvh:kvh + 1]
    ks = None if w.k_scale is None else w.k_scale[slots, kvh:kvh + 1]
    vs = None if w.v_scale is None else w.v_scale[slots, kvh:kvh + 1]
    r = oracle.full_attn_select(synth.raw(qq), DTYPE_CODE[s.q_dtype], synth.raw(k), synth.raw(v),
                                DTYPE_CODE[s.kv_dtype], np.array([T], np.int32), None, T,
                                window=s.window, k_global=s.k_global, k_scale=synth.raw(ks), v_scale=synth.raw(vs))
    return r, slots.cpu().numpy()


def unit_oracle_sparse(oracle, w: synth.Workload, b: int, kvh: int, q, local_idx):
    """Oracle sparse layer of one unit with positions as the index list."""
    s = w.spec
    T = int(w.seq_lens[b])
    slots = synth.slots_of(w, b, torch.arange(T, device=w.k.device))
    G = s.group
    qq = q[b:b + 1, kvh * G:(kvh + 1) * G]
    k = w.k[slots, kvh:kvh + 1]
    v = w.v[slots, kvh:kvh + 1]
    ks = None if w.k_scale is None else w.k_scale[slots, kvh:kvh + 1]
    vs = None if w.v_scale is None else w.v_scale[slots, kvh:kvh + 1]
    return oracle.sparse_attn(synth.raw(qq), DTYPE_CODE[s.q_dtype], synth.raw(k), synth.raw(v),
                              DTYPE_CODE[s.kv_dtype], np.asarray(local_idx, np.int32).reshape(1, 1, -1),
                              k_scale=synth.raw(ks), v_scale=synth.raw(vs))


def check_idx_positions(gpos_row, opos_row, ora_score, T, window, k_global):
    """check_idx_unit() on lists already mapped to logical positions: gpos_row
    is the GPU's list (-1 padding, -2 for a slot outside the sequence),
    opos_row the oracle's (-1 padded), ora_score its scores of [0, T).
    Returns the number of positions that differ (all inside the near-tie band)."""
    L = window + k_global
    n = min(T, L)
    g = np.asarray(gpos_row)
    assert len(g) == L
    assert np.all(g[n:] == -1), "padding must be -1"
    gv = g[:n]
    assert np.all(gv >= 0), "valid entries must be slots of the sequence"
    assert np.all(np.diff(gv) > 0), "positions must be strictly ascending"
    ov = np.asarray(opos_row)[:n]
    win = set(range(max(0, T - window), T))
    assert win <= set(gv.tolist()), "forced window missing"
    diff = set(gv.tolist()) ^ set(ov.tolist())
    if diff:
        nC = max(0, T - window)
        cand = np.sort(ora_score[:nC])[::-1]
        sk = cand[k_global - 1]
        bad = [t for t in diff if not (abs(ora_score[t] - sk) <= NEAR_TIE * sk)]
        assert not bad, (f"{len(bad)} positions differ outside the near-tie band, e.g. {bad[:5]} "
                         f"(scores {[ora_score[t] for t in bad[:5]]}, k-th {sk})")
    return len(diff)


def check_block_positions(gpos_row, opos_row, ora_score, T, window, k_global, block):
    """Block-level index lists as positions: the GPU's (gpos_row, -1 padded)
    against the oracle's (opos_row).  Both must hold the window and whole
    blocks in ascending order; a block may differ only when its oracle block
    sum lies within 1e-6 relative of the oracle's (k_global / block)-th block
    sum.  Returns the number of blocks that differ."""
    L = window + k_global
    g = np.asarray(gpos_row)
    assert len(g) == L
    gv = g[g >= 0]
    assert np.all(g[len(gv):] == -1), "padding must be -1 and last"
    assert np.all(np.diff(gv) > 0), "positions must be strictly ascending"
    nC = max(0, T - window)
    win = set(range(nC, T))
    assert win <= set(gv.tolist()), "forced window missing"
    ov = np.asarray(opos_row)
    ov = ov[ov >= 0]
    gblk = {int(t) // block for t in gv if t < nC}
    oblk = {int(t) // block for t in ov if t < nC}
    for j in gblk:  # whole blocks only
        lo, hi = j * block, min((j + 1) * block, nC)
        assert set(range(lo, hi)) <= set(gv.tolist()), f"block {j} taken in part"
    diff = gblk ^ oblk
    if diff:
        nblk = (nC + block - 1) // block
        sums = np.array([ora_score[j * block:min((j + 1) * block, nC)].sum() for j in range(nblk)])
        keep = k_global // block
        sk = np.sort(sums)[::-1][keep - 1]
        bad = [j for j in diff if not (abs(sums[j] - sk) <= NEAR_TIE * sk)]
        assert not bad, f"{len(bad)} blocks differ outside the near-tie band, e.g. {bad[:5]} (k-th sum {sk})"
    return len(diff)

"""Parity of the CUDA path (through the C-ABI) with the CPU oracle on small
seeded workloads that still span many tiles, several CTAs per sequence and
ragged tails, plus the edge cases of the method.

Full layer (attention + token selection) and sparse layers (attention over the
selected rows) of the HySparse2 Hybrid Block; tolerances in hs2_testutil.
"""
import zlib

import numpy as np
import pytest
import torch

from long_context_decode_full_b200 import synth
import hs2_testutil as U

pytestmark = pytest.mark.gpu


def spec(**kw):
    base = dict(name="parity", batch=3, num_kv_heads=2, group=8, head_dim=128, seq_len=(1500, 5000),
                kv_dtype="bf16", q_dtype="bf16", page_size=64, sparse_layers=2, needles=24)
    base.update(kw)
    return synth.WorkloadSpec(**base)


CASES = {
    "bf16_paged64": spec(),
    "bf16_contiguous": spec(page_size=None),
    "bf16_paged16_nanpad": spec(page_size=16, seq_len=(1100, 3000)),
    "bf16_paged32": spec(page_size=32, batch=2),
    "bf16_paged128": spec(page_size=128, batch=2),
    "bf16_d64_g4": spec(head_dim=64, group=4, num_kv_heads=3),
    "bf16_g1": spec(group=1, num_kv_heads=4, batch=2),
    "bf16_g2": spec(group=2, num_kv_heads=2, batch=2),
    "e4m3_paged64": spec(kv_dtype="e4m3", seq_len=(1500, 4000)),
    "e4m3_paged32_nanpad": spec(kv_dtype="e4m3", page_size=32, batch=2, seq_len=(1200, 2600)),
    "e4m3_paged16": spec(kv_dtype="e4m3", page_size=16, batch=2, seq_len=(1100, 2700)),
    "e4m3_contiguous_g4": spec(kv_dtype="e4m3", page_size=None, group=4, num_kv_heads=3, batch=2),
    "bf16_g16": spec(group=16, num_kv_heads=2, batch=2),
    "bf16_mqa_g32": spec(group=32, num_kv_heads=1, batch=3),
    "bf16_mqa_g32_d64_contiguous": spec(group=32, num_kv_heads=1, batch=2, head_dim=64, page_size=None),
    "e4m3_mqa_g32": spec(kv_dtype="e4m3", group=32, num_kv_heads=1, batch=2, seq_len=(1500, 4000)),
    "f32_tiny": synth.WORKLOADS["tiny_fp32_t2048"],
    "f32_paged_ragged": spec(kv_dtype="f32", q_dtype="f32", head_dim=64, group=4, page_size=16,
                             seq_len=(1200, 2500)),
    # fp32 sparse layers run as clusters of min(16, SMs / units, tiles) CTAs:
    # d 128 with two heads per warp (16 CTAs of 75 KB), and 20 units (7 CTAs each)
    "f32_d128_g8": spec(kv_dtype="f32", q_dtype="f32", batch=2, seq_len=(1300, 3000)),
    "f32_g2_b10_contiguous": spec(kv_dtype="f32", q_dtype="f32", head_dim=64, group=2, batch=10, page_size=None,
                                  seq_len=(100, 2000)),
    "short_window_only": spec(seq_len=(1, 127), batch=4),
    "exactly_window_plus_k": spec(batch=2, seq_len=1152),
    "one_more_than_fits": spec(batch=2, seq_len=1153),
}


@pytest.fixture(scope="module")
def lib():
    from long_context_decode_full_b200 import hs2
    hs2.lib()
    return hs2


@pytest.mark.parametrize("name", list(CASES))
def test_full_and_sparse_match_oracle(oracle, lib, name):
    sp = CASES[name]
    pad = "nan" if "nanpad" in name else None
    w = synth.generate(sp, seed=zlib.crc32(name.encode()) % 1000, pad_fill=pad)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out, idx = U.run_gpu(wd)
    torch.cuda.synchronize()
    err, ndiff = U.check_full(wd, out, idx, ora)
    # sparse layers: oracle's index list into both sides, each layer's own query
    ora_idx = torch.from_numpy(ora["idx"]).cuda()
    for layer in range(sp.sparse_layers):
        g = U.run_gpu_sparse(wd, wd.q_sparse[layer], ora_idx)
        ref = U.run_oracle_sparse(oracle, w, w.q_sparse[layer], ora["idx"])
        U.check_out(g, ref, sp.kv_dtype, f"sparse layer {layer}")
    # and the GPU's own list drives the GPU sparse layer like the oracle's does
    if ndiff == 0:
        g2 = U.run_gpu_sparse(wd, wd.q_sparse[0], idx)
        ref = U.run_oracle_sparse(oracle, w, w.q_sparse[0], ora["idx"])
        U.check_out(g2, ref, sp.kv_dtype, "sparse layer with GPU indices")
    lib_status = lib.workspace_status(torch.zeros(256, dtype=torch.uint8, device="cuda"))
    assert lib_status == 0


def test_sparse_equals_full_when_everything_fits(oracle, lib):
    sp = spec(seq_len=(300, 1152), batch=3)
    w = U.to_device(synth.generate(sp, seed=5))
    out, idx = U.run_gpu(w)
    s = U.run_gpu_sparse(w, w.q_full, idx)
    torch.cuda.synchronize()
    assert (out.float() - s.float()).abs().max().item() <= 2e-2


def test_zero_query_ties_pick_lowest_positions(oracle, lib):
    """q = 0: every score ties, so the global part is exactly the lowest
    k_global positions (bit-exact), and out = mean of V."""
    sp = spec(seq_len=3000, batch=2)
    w = synth.generate(sp, seed=8)
    w.q_full.zero_()
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out, idx = U.run_gpu(wd)
    gi = idx.cpu().numpy()
    assert np.array_equal(gi, ora["idx"])
    U.check_out(out, ora["out"], "bf16")


def test_constant_keys_ties_and_planted_order(oracle, lib):
    """All keys equal except a planted descending ladder: the ladder wins in
    order, the rest tie and fall to the lowest positions."""
    sp = spec(seq_len=2500, batch=1, num_kv_heads=1, page_size=None)
    w = synth.generate(sp, seed=9)
    w.k[:] = w.k[0:1].clone()
    ladder = torch.arange(300, 100, -1)
    base = w.k[0, 0].float()
    for r, t in enumerate(ladder.tolist()):
        w.k[t, 0] = (base * (1.0 + 0.02 * (300 - r) / 300.0)).to(w.k.dtype)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out, idx = U.run_gpu(wd)
    err, ndiff = U.check_full(wd, out, idx, ora)
    assert ndiff == 0


def test_empty_sequence_gives_zeros_and_no_indices(lib):
    sp = spec(batch=3)
    w = U.to_device(synth.generate(sp, seed=2, seq_lens=[2000, 0, 700]))
    out, idx = U.run_gpu(w)
    torch.cuda.synchronize()
    assert torch.all(out[1] == 0)
    assert torch.all(idx[1] == -1)
    assert torch.all(idx[0, :, :1152] >= 0)


def test_window_and_budget_variants(oracle, lib):
    sp = spec(batch=2, seq_len=(2000, 3000))
    w = synth.generate(sp, seed=12)
    wd = U.to_device(w)
    for W, K in [(0, 1), (1, 0), (128, 1), (64, 2048), (512, 1024), (5, 7)]:
        ora = U.run_oracle(oracle, w, window=W, k_global=K)
        out, idx = U.run_gpu(wd, window=W, k_global=K)
        U.check_full(wd, out, idx, ora, window=W, k_global=K)


@pytest.mark.parametrize("kv_dtype", ["f32", "bf16", "e4m3"])
def test_sparse_ragged_lists(oracle, lib, kv_dtype):
    """Sparse layers over index lists of 12, 364 and 1,100 rows (W + K for
    three budgets): shorter than one 64-row tile, and ragged last tiles, with
    the oracle's list as input.  The fp32 clusters' merge is repeatable bit
    for bit."""
    kw = dict(kv_dtype=kv_dtype, q_dtype="f32" if kv_dtype == "f32" else "bf16", batch=3, seq_len=(700, 2600))
    if kv_dtype == "f32":
        kw.update(head_dim=64, group=4)
    w = synth.generate(spec(**kw), seed=31)
    wd = U.to_device(w)
    for W, K in [(5, 7), (64, 300), (100, 1000)]:
        ora = U.run_oracle(oracle, w, window=W, k_global=K)
        ora_idx = torch.from_numpy(ora["idx"]).cuda()
        assert ora_idx.shape[-1] == W + K
        g = U.run_gpu_sparse(wd, wd.q_sparse[0], ora_idx)
        g2 = U.run_gpu_sparse(wd, wd.q_sparse[0], ora_idx)
        torch.cuda.synchronize()
        ref = U.run_oracle_sparse(oracle, w, w.q_sparse[0], ora["idx"])
        U.check_out(g, ref, kv_dtype, f"sparse layer, list of {W + K}")
        assert torch.equal(g, g2)


def test_repeatable_bitwise(lib):
    sp = spec(kv_dtype="bf16")
    w = U.to_device(synth.generate(sp, seed=4))
    a = U.run_gpu(w)
    b = U.run_gpu(w)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    s1 = U.run_gpu_sparse(w, w.q_sparse[0], a[1])
    s2 = U.run_gpu_sparse(w, w.q_sparse[0], a[1])
    assert torch.equal(s1, s2)


def test_paged_and_contiguous_agree_bitwise(lib):
    sp = spec(batch=2, seq_len=3000)
    wp = U.to_device(synth.generate(sp, seed=6))
    wc = U.to_device(synth.generate(sp.replace(page_size=None), seed=6))
    for b in range(2):
        T = int(wp.seq_lens[b])
        spp = synth.slots_of(wp, b, torch.arange(T, device="cuda"))
        scc = synth.slots_of(wc, b, torch.arange(T, device="cuda"))
        wc.k[scc] = wp.k[spp]
        wc.v[scc] = wp.v[spp]
    wc.q_full.copy_(wp.q_full)
    op, ip = U.run_gpu(wp)
    oc, ic = U.run_gpu(wc)
    torch.cuda.synchronize()
    assert torch.equal(op, oc)
    for b in range(2):
        m = {int(c): int(p) for c, p in zip(
            synth.slots_of(wc, b, torch.arange(3000)).tolist(),
            synth.slots_of(wp, b, torch.arange(3000, device="cuda")).tolist())}
        got = [[m[int(x)] for x in row] for row in ic[b].tolist()]
        assert got == ip[b].tolist()


def test_hybrid_block_step_runs_all_layers(oracle, lib):
    from long_context_decode_full_b200 import hs2
    sp = spec(batch=2, sparse_layers=3)
    w = synth.generate(sp, seed=21)
    wd = U.to_device(w)
    outs, idx = hs2.hybrid_block_step(wd.q_full, list(wd.q_sparse), wd.k, wd.v, wd.seq_lens, wd.page_table,
                                      wd.page_size)
    ora = U.run_oracle(oracle, w)
    U.check_full(wd, outs[0], idx, ora)
    for layer in range(3):
        ref = U.run_oracle_sparse(oracle, w, w.q_sparse[layer], ora["idx"])
        U.check_out(outs[1 + layer], ref, "bf16", f"layer {layer}")


def _scale_heads(q, G):
    """Multiply query head h of every group by 2^(h - 3): exact in bf16, and the
    heads of one group then need different power-of-two prescales."""
    f = torch.tensor([2.0 ** (h % G - 3) for h in range(q.shape[-2])], dtype=torch.float32)
    return (q.float() * f[:, None]).to(q.dtype)


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_heads_of_unequal_magnitude(oracle, lib, kv_dtype):
    sp = spec(kv_dtype=kv_dtype, batch=2, seq_len=(2000, 3000))
    w = synth.generate(sp, seed=41)
    w.q_full = _scale_heads(w.q_full, sp.group)
    w.q_sparse = _scale_heads(w.q_sparse, sp.group)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out, idx = U.run_gpu(wd)
    torch.cuda.synchronize()
    U.check_full(wd, out, idx, ora)
    g = U.run_gpu_sparse(wd, wd.q_sparse[0], torch.from_numpy(ora["idx"]).cuda())
    U.check_out(g, U.run_oracle_sparse(oracle, w, w.q_sparse[0], ora["idx"]), kv_dtype, "sparse layer")


# every built tensor-core configuration of the attention kernel: (ncw, nstage, nsl)
FULL_CONFIGS = {
    "bf16": ["8,3,1", "4,6,1", "4,3,2"],
    "e4m3": ["8,3,2", "6,4,2", "4,6,2", "16,3,1", "12,4,1", "8,6,1", "4,8,1"],
}


@pytest.mark.parametrize("kv_dtype,cfg", [(d, c) for d, cs in FULL_CONFIGS.items() for c in cs])
def test_every_attention_config(oracle, lib, monkeypatch, kv_dtype, cfg):
    sp = spec(kv_dtype=kv_dtype, batch=2, seq_len=(2500, 4100), page_size=None, sparse_layers=1)
    w = synth.generate(sp, seed=7)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    monkeypatch.setenv("HS2_FULL_CFG", cfg)
    out, idx = U.run_gpu(wd)
    torch.cuda.synchronize()
    U.check_full(wd, out, idx, ora)


# configurations for groups of 16 and more heads (ncw, nstage, nsl, nt[, tc]): nt = 2
# gives each warp 16 heads; the nt = 1 entries are the 8-head fallbacks
WIDE_CONFIGS = {
    "bf16": ["4,3,2,2,1", "4,3,2,2", "8,3,1,2", "8,3,1,1", "4,3,2,1"],
    "e4m3": ["4,3,2,2,1", "4,6,2,2", "8,3,2,1"],
}
WIDE_SHAPES = {  # (spec fields, sequence lengths)
    "mqa_g32": (dict(group=32, num_kv_heads=1, batch=3), [90, 4100, 1300]),
    "g16": (dict(group=16, num_kv_heads=2, batch=2), [2500, 700]),
}


@pytest.mark.parametrize("shape", list(WIDE_SHAPES))
@pytest.mark.parametrize("kv_dtype,cfg", [(d, c) for d, cs in WIDE_CONFIGS.items() for c in cs])
def test_every_wide_attention_config(oracle, lib, monkeypatch, kv_dtype, cfg, shape):
    """Every configuration built for groups above 8 heads, on short and
    ragged sequences (warps whose row blocks lie past the end merge empty
    states)."""
    fields, lens = WIDE_SHAPES[shape]
    sp = spec(kv_dtype=kv_dtype, sparse_layers=1, seq_len=max(lens), **fields)
    w = synth.generate(sp, seed=11, seq_lens=lens)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    monkeypatch.setenv("HS2_FULL_CFG", cfg)
    out, idx = U.run_gpu(wd)
    torch.cuda.synchronize()
    U.check_full(wd, out, idx, ora)


def test_wide_d64_config(oracle, lib, monkeypatch):
    sp = spec(group=32, num_kv_heads=1, batch=2, head_dim=64, page_size=None, sparse_layers=1, seq_len=3000)
    w = synth.generate(sp, seed=12, seq_lens=[3000, 333])
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    monkeypatch.setenv("HS2_FULL_CFG", "8,6,1,2")
    out, idx = U.run_gpu(wd)
    torch.cuda.synchronize()
    U.check_full(wd, out, idx, ora)


def test_bounded_wait_expires_and_context_stays_usable(oracle, lib):
    """A device wait that nothing completes gives up, flags the workspace,
    and the next status read reports it once; the context keeps working."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    lib.selftest_bounded_wait(ws)
    assert lib.workspace_status(ws) == lib.ERR_TIMEOUT
    assert lib.workspace_status(ws) == 0  # the flag was cleared by the read
    sp = spec(batch=1, seq_len=2000)
    w = synth.generate(sp, seed=3)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out, idx = U.run_gpu(wd)
    torch.cuda.synchronize()
    U.check_full(wd, out, idx, ora)


def planted_margins(kv_dtype, lo, hi, T=6000, seed=0):
    """Keys along one axis so that every query head's logit is set exactly:
    the window's keys are 0 (logit 0) and each selectable key sits lo..hi nats
    (uniform) below it for head 0; head h has 1 + h/8 times that margin.
    With margins beyond ~87 nats the group probabilities fall under fp32's
    normal range, and the k-th score with them."""
    sp = spec(batch=2, seq_len=T, kv_dtype=kv_dtype, sparse_layers=1, needles=0)
    w = synth.generate(sp, seed=seed)
    g = torch.Generator().manual_seed(seed)
    c = 1.0 / np.sqrt(sp.head_dim)
    w.q_full.zero_()
    for h in range(sp.num_q_heads):
        w.q_full[:, h, 0] = 8.0 + (h % sp.group)
    rows = torch.zeros(w.num_slots, sp.num_kv_heads, sp.head_dim)
    for b in range(sp.batch):
        slots = synth.slots_of(w, b, torch.arange(T))
        for kvh in range(sp.num_kv_heads):
            margin = lo + (hi - lo) * torch.rand(T, generator=g)
            x = margin / (8.0 * c)
            x[T - sp.window:] = 0.0
            rows[slots, kvh, 0] = x
    if kv_dtype == "e4m3":
        codes, scale = synth._quantize_e4m3(rows)
        w.k.copy_(codes)
        w.k_scale.copy_(scale)
    else:
        w.k.copy_(rows.to(w.k.dtype))
    return w


@pytest.mark.parametrize("kv_dtype,lo,hi", [
    ("bf16", -200.0, -70.0),   # the k-th group probability underflows fp32 (the top ones do not)
    ("bf16", -90.0, -60.0),    # it sits just above 2^-126, where single heads flush
    ("bf16", -420.0, -260.0),  # two common factors are needed
    ("e4m3", -200.0, -70.0),
])
def test_selection_below_fp32_range(oracle, lib, kv_dtype, lo, hi):
    """Logit margins of 60-420 nats put the k-th score far below fp32's
    normal range; the selection must still rank exactly like the fp64 oracle."""
    w = planted_margins(kv_dtype, lo, hi, seed=int(-lo))
    ora = U.run_oracle(oracle, w)
    nC = int(w.seq_lens[0]) - w.spec.window
    kth = np.sort(ora["score"][0, 0, :nC])[::-1][w.spec.k_global - 1]
    assert kth < 2.0 ** -96, kth  # the case this test is about
    wd = U.to_device(w)
    out, idx = U.run_gpu(wd)
    torch.cuda.synchronize()
    U.check_full(wd, out, idx, ora)


BLOCK_CASES = {
    "bf16_paged64_b16": (spec(), 16, 128, 1024),
    "bf16_contiguous_b1": (spec(page_size=None, batch=2), 1, 128, 1024),
    "e4m3_paged32_b8": (spec(kv_dtype="e4m3", page_size=32, batch=2, seq_len=(1500, 4000)), 8, 128, 1024),
    "f32_tiny_b64": (synth.WORKLOADS["tiny_fp32_t2048"], 64, 128, 1024),
    "mqa_g32_b32": (spec(group=32, num_kv_heads=1, batch=2), 32, 128, 1024),
    "short_contexts_b16": (spec(seq_len=(1, 1400), batch=4), 16, 128, 1024),
    "one_block_of_k": (spec(batch=2), 1024, 128, 1024),
    "odd_budget_b5": (spec(batch=2, seq_len=(900, 2500)), 5, 64, 300),
    "no_global_budget": (spec(batch=2), 4, 128, 0),
}


@pytest.mark.parametrize("name", list(BLOCK_CASES))
def test_block_selection_matches_oracle(oracle, lib, name):
    """Block-level selection (the first-generation comparator) against the
    oracle's block ranking of its own group scores, every unit."""
    sp, block, W, K = BLOCK_CASES[name]
    w = synth.generate(sp, seed=zlib.crc32(name.encode()) % 1000)
    s = w.spec
    code = U.DTYPE_CODE
    ora = oracle.full_attn_select_blocks(synth.raw(w.q_full), code[s.q_dtype], synth.raw(w.k), synth.raw(w.v),
                                         code[s.kv_dtype], synth.raw(w.seq_lens), synth.raw(w.page_table),
                                         w.page_size, window=W, k_global=K, block=block,
                                         k_scale=synth.raw(w.k_scale), v_scale=synth.raw(w.v_scale))
    wd = U.to_device(w)
    out, idx = lib.full_attn_select_blocks(wd.q_full, wd.k, wd.v, wd.seq_lens, wd.page_table, wd.page_size, W, K,
                                           block, wd.k_scale, wd.v_scale, workspace=U.garbage_workspace(wd))
    torch.cuda.synchronize()
    U.check_out(out, ora["out"], s.kv_dtype)
    gi = idx.cpu().numpy()
    for b in range(s.batch):
        T = int(w.seq_lens[b])
        s2p = U.slot_to_pos(w, b)
        for h in range(s.num_kv_heads):
            gpos = np.array([s2p[int(x)] if x >= 0 else -1 for x in gi[b, h]])
            opos = np.array([s2p[int(x)] if x >= 0 else -1 for x in ora["idx"][b, h]])
            U.check_block_positions(gpos, opos, ora["score"][b, h], T, W, K, block)


def test_block_selection_with_zero_query_takes_the_lowest_blocks(oracle, lib):
    """q = 0: every position scores alike, every full block ties, so the
    lowest k_global / block blocks are taken (bit-exact)."""
    sp = spec(seq_len=3000, batch=2)
    w = synth.generate(sp, seed=8)
    w.q_full.zero_()
    ora = oracle.full_attn_select_blocks(synth.raw(w.q_full), 1, synth.raw(w.k), synth.raw(w.v), 1,
                                         synth.raw(w.seq_lens), synth.raw(w.page_table), w.page_size,
                                         window=128, k_global=1024, block=16)
    wd = U.to_device(w)
    _, idx = lib.full_attn_select_blocks(wd.q_full, wd.k, wd.v, wd.seq_lens, wd.page_table, wd.page_size, 128,
                                         1024, 16)
    assert np.array_equal(idx.cpu().numpy(), ora["idx"])

"""Pins for the CPU oracle: it is checked here against things other than
itself -- brute force in 50-digit arithmetic without max-shift, closed forms,
invariants the method fixes, exhaustive ranking, and library decoders.

The method (HySparse2 announcement, "KV Reuse" section and the token-level
selection / forced-window paragraphs): the full layer attends over all T
positions and selects positions from its attention scores; the most recent
W=128 tokens are always kept plus the top 1,024 of the rest; the sparse
layers attend over exactly that list.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

from long_context_decode_full_b200 import synth

mpmath.mp.dps = 50
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers --

def decode_bf16(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_e4m3_torch(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def dequant(w, which):
    """Exact stored values of a workload's cache as float64 (library decoders)."""
    t = getattr(w, which)
    if w.spec.kv_dtype == "f32":
        return t.double().numpy()
    if w.spec.kv_dtype == "bf16":
        return decode_bf16(synth.raw(t))
    sc = getattr(w, which + "_scale").double().numpy()
    return decode_e4m3_torch(synth.raw(t)) * sc[..., None]


def qvals(q, dtype):
    return q.double().numpy() if dtype == "f32" else decode_bf16(synth.raw(q))


def dtype_code(s):
    return {"f32": 0, "bf16": 1, "e4m3": 2}[s]


def run_full(oracle, w, q=None, window=None, k_global=None):
    s = w.spec
    q = w.q_full if q is None else q
    return oracle.full_attn_select(
        synth.raw(q), dtype_code(s.q_dtype), synth.raw(w.k), synth.raw(w.v), dtype_code(s.kv_dtype),
        synth.raw(w.seq_lens), synth.raw(w.page_table), w.page_size,
        window=s.window if window is None else window,
        k_global=s.k_global if k_global is None else k_global,
        k_scale=synth.raw(w.k_scale), v_scale=synth.raw(w.v_scale))


def run_sparse(oracle, w, q, idx):
    s = w.spec
    return oracle.sparse_attn(synth.raw(q), dtype_code(s.q_dtype), synth.raw(w.k), synth.raw(w.v),
                              dtype_code(s.kv_dtype), idx, k_scale=synth.raw(w.k_scale),
                              v_scale=synth.raw(w.v_scale))


def brute_full(w, q=None):
    """50-digit brute force: logits, softmax WITHOUT max-shift, out, lse,
    group score; address rule applied by hand."""
    s = w.spec
    q = qvals(w.q_full if q is None else q, s.q_dtype)
    K, V = dequant(w, "k"), dequant(w, "v")
    B, Hq, d = q.shape
    G = s.group
    res = {"out": np.zeros((B, Hq, d)), "lse": np.zeros((B, Hq)), "score": {}}
    pt = None if w.page_table is None else w.page_table.numpy()
    for b in range(B):
        T = int(w.seq_lens[b])
        slots = [(b * w.page_size + t) if pt is None else
                 (int(pt[b, t // w.page_size]) * w.page_size + t % w.page_size) for t in range(T)]
        probs = {}
        for h in range(Hq):
            kvh = h // G
            logits = [mpmath.fsum(mpmath.mpf(q[b, h, i]) * mpmath.mpf(K[sl, kvh, i]) for i in range(d))
                      / mpmath.sqrt(d) for sl in slots]
            e = [mpmath.exp(x) for x in logits]
            Z = mpmath.fsum(e)
            p = [x / Z for x in e]
            probs[h] = p
            res["lse"][b, h] = float(mpmath.log(Z))
            for i in range(d):
                res["out"][b, h, i] = float(mpmath.fsum(p[t] * mpmath.mpf(V[slots[t], kvh, i])
                                                        for t in range(T)))
        for kvh in range(s.num_kv_heads):
            res["score"][(b, kvh)] = np.array(
                [float(mpmath.fsum(probs[kvh * G + g][t] for g in range(G))) for t in range(T)])
    return res


def small_spec(**kw):
    base = dict(name="pin", batch=2, num_kv_heads=2, group=2, head_dim=8, seq_len=37,
                kv_dtype="bf16", q_dtype="bf16", page_size=4, sparse_layers=1, needles=3,
                window=5, k_global=6)
    base.update(kw)
    return synth.WorkloadSpec(**base)


# ---------------------------------------------------------------- pins ----

def test_golden_hyperparameters_match_pages():
    """window=128 and k_global=1024 are the numbers the pages state."""
    with open(os.path.join(GOLDEN, "hybrid_block_params.json")) as f:
        g = json.load(f)
    for spec in synth.WORKLOADS.values():
        assert spec.window == g["window"] and spec.k_global == g["k_global"]


def test_e4m3_decode_matches_torch_for_all_codes(oracle):
    codes = np.arange(256, dtype=np.uint8)
    ref = decode_e4m3_torch(codes)
    got = np.array([oracle.e4m3_value(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("kv_dtype,q_dtype,page", [("bf16", "bf16", 4), ("f32", "f32", None),
                                                   ("e4m3", "bf16", 8)])
def test_full_layer_matches_50_digit_brute_force(oracle, kv_dtype, q_dtype, page):
    spec = small_spec(kv_dtype=kv_dtype, q_dtype=q_dtype, page_size=page, seq_len=(9, 23))
    w = synth.generate(spec, seed=11)
    got = run_full(oracle, w)
    ref = brute_full(w)
    np.testing.assert_allclose(got["out"], ref["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["lse"], ref["lse"], rtol=0, atol=1e-12)
    for (b, kvh), sc in ref["score"].items():
        T = int(w.seq_lens[b])
        np.testing.assert_allclose(got["score"][b, kvh, :T], sc, rtol=1e-12, atol=0)


def test_two_position_closed_form(oracle):
    """T=2, d=2: logits (x, 0) -> p0 = 1/(1+e^-x), out = p0 v0 + p1 v1."""
    spec = synth.WorkloadSpec("cf", 1, 1, 1, 2, 2, "f32", "f32", None, 1, window=1, k_global=1)
    w = synth.generate(spec, seed=0)
    a, bk, c = 1.5, 2.0, -0.75
    w.q_full[:] = torch.tensor([[[a, 0.0]]])
    w.k[0, 0] = torch.tensor([bk, 0.0])
    w.k[1, 0] = torch.tensor([0.0, c])
    w.v[0, 0] = torch.tensor([1.0, -2.0])
    w.v[1, 0] = torch.tensor([0.5, 4.0])
    r = run_full(oracle, w)
    x = a * bk / math.sqrt(2)
    p0 = 1 / (1 + math.exp(-x))
    np.testing.assert_allclose(r["out"][0, 0], [p0 * 1.0 + (1 - p0) * 0.5, p0 * -2.0 + (1 - p0) * 4.0],
                               atol=1e-14)
    np.testing.assert_allclose(r["lse"][0, 0], math.log(math.exp(x) + 1), atol=1e-14)
    np.testing.assert_allclose(r["score"][0, 0, :2], [p0, 1 - p0], atol=1e-14)
    # window = 1 keeps position 1; the single candidate (position 0) fits k_global = 1
    assert list(r["idx"][0, 0]) == [0, 1]


def test_zero_query_gives_uniform_mean_and_lowest_index_ties(oracle):
    """q = 0: p = 1/T, out = mean of V, every score G/T, so the tie-break
    (lower index first) decides the whole global selection."""
    spec = small_spec(seq_len=40, page_size=8)
    w = synth.generate(spec, seed=3)
    w.q_full.zero_()
    r = run_full(oracle, w)
    V = dequant(w, "v")
    for b in range(spec.batch):
        T = int(w.seq_lens[b])
        sl = synth.slots_of(w, b, torch.arange(T)).numpy()
        for h in range(spec.num_q_heads):
            np.testing.assert_allclose(r["out"][b, h], V[sl, h // spec.group].mean(0), atol=1e-14)
        for kvh in range(spec.num_kv_heads):
            np.testing.assert_allclose(r["score"][b, kvh, :T], spec.group / T, rtol=1e-14)
            want = list(range(spec.k_global)) + list(range(T - spec.window, T))
            assert list(r["idx"][b, kvh]) == [int(x) for x in sl[want]]


def test_constant_values_give_that_value(oracle):
    spec = small_spec(kv_dtype="f32", q_dtype="f32", page_size=None, seq_len=25)
    w = synth.generate(spec, seed=5)
    row = torch.linspace(-1, 1, spec.head_dim)
    w.v[:] = row
    r = run_full(oracle, w)
    np.testing.assert_allclose(r["out"], np.broadcast_to(row.double().numpy(), r["out"].shape),
                               atol=1e-14)


def test_scores_sum_to_group_size_and_selection_invariants(oracle):
    spec = small_spec(seq_len=(1, 60), batch=6, page_size=4)
    w = synth.generate(spec, seed=7)
    r = run_full(oracle, w)
    W, K = spec.window, spec.k_global
    for b in range(spec.batch):
        T = int(w.seq_lens[b])
        sl = synth.slots_of(w, b, torch.arange(T)).numpy()
        pos_of = {int(s): t for t, s in enumerate(sl)}
        for kvh in range(spec.num_kv_heads):
            np.testing.assert_allclose(r["score"][b, kvh, :T].sum(), spec.group, rtol=1e-13)
            n = int(r["n_sel"][b, kvh])
            assert n == min(T, W + K)
            idx = r["idx"][b, kvh]
            assert all(x == -1 for x in idx[n:])
            pos = [pos_of[int(x)] for x in idx[:n]]
            assert pos == sorted(pos) and len(set(pos)) == n
            assert set(range(max(0, T - W), T)) <= set(pos)


def test_selection_matches_exhaustive_ranking(oracle):
    """Each candidate's rank = #candidates with a higher score, or an equal
    score at a lower index; the oracle must keep exactly the ranks < K."""
    spec = small_spec(seq_len=(20, 60), batch=4, page_size=4, window=5, k_global=7)
    for seed in range(4):
        w = synth.generate(spec, seed=seed)
        r = run_full(oracle, w)
        for b in range(spec.batch):
            T = int(w.seq_lens[b])
            sl = synth.slots_of(w, b, torch.arange(T)).numpy()
            C = max(0, T - spec.window)
            for kvh in range(spec.num_kv_heads):
                s = r["score"][b, kvh, :C]
                keep = [t for t in range(C)
                        if sum(1 for u in range(C) if s[u] > s[t] or (s[u] == s[t] and u < t))
                        < spec.k_global]
                want = sorted(set(keep) | set(range(C, T)))
                n = int(r["n_sel"][b, kvh])
                assert list(r["idx"][b, kvh, :n]) == [int(sl[t]) for t in want]


def test_planted_key_order_and_ties_decide_selection(oracle):
    """One head, q = e0: score order follows the planted first key component.
    Three levels with ties: all of the top level, then the lowest indices of
    the next level."""
    T, W, K = 50, 4, 10
    spec = synth.WorkloadSpec("plant", 1, 1, 1, 4, T, "f32", "f32", None, 1, window=W, k_global=K)
    w = synth.generate(spec, seed=1)
    w.q_full[:] = torch.tensor([[[1.0, 0, 0, 0]]])
    rng = np.random.default_rng(0)
    level = rng.choice([0, 1, 2], size=T, p=[0.5, 0.42, 0.08])
    level[:6] = [2, 0, 1, 2, 1, 1]
    w.k[:, 0, :] = 0.0
    w.k[:T, 0, 0] = torch.tensor(level, dtype=torch.float32)
    r = run_full(oracle, w)
    C = T - W
    top = [t for t in range(C) if level[t] == 2]
    assert len(top) < K
    nxt = [t for t in range(C) if level[t] == 1][:K - len(top)]
    want = sorted(set(top) | set(nxt) | set(range(C, T)))
    assert list(r["idx"][0, 0, :len(want)]) == want


def test_short_sequences_take_everything(oracle):
    spec = small_spec(window=8, k_global=5, page_size=4, batch=4)
    w = synth.generate(spec, seed=2, seq_lens=[1, 8, 13, 14])
    r = run_full(oracle, w)
    for b, T in enumerate([1, 8, 13, 14]):
        sl = synth.slots_of(w, b, torch.arange(T)).numpy()
        n = min(T, 13)
        for kvh in range(spec.num_kv_heads):
            assert int(r["n_sel"][b, kvh]) == n
            if T <= 13:
                assert list(r["idx"][b, kvh, :n]) == [int(x) for x in sl]


def test_paged_equals_contiguous(oracle):
    spec = small_spec(page_size=4, seq_len=30, batch=2)
    wp = synth.generate(spec, seed=9)
    wc = synth.generate(spec.replace(page_size=None), seed=9)
    for b in range(2):  # copy the paged data into the contiguous layout
        sp = synth.slots_of(wp, b, torch.arange(30))
        sc = synth.slots_of(wc, b, torch.arange(30))
        wc.k[sc] = wp.k[sp]
        wc.v[sc] = wp.v[sp]
    wc.q_full.copy_(wp.q_full)
    rp, rc = run_full(oracle, wp), run_full(oracle, wc)
    assert np.array_equal(rp["out"], rc["out"]) and np.array_equal(rp["lse"], rc["lse"])
    for b in range(2):
        sp = synth.slots_of(wp, b, torch.arange(30)).numpy()
        sc = synth.slots_of(wc, b, torch.arange(30)).numpy()
        m = {int(c): int(p) for c, p in zip(sc, sp)}
        for kvh in range(2):
            n = int(rc["n_sel"][b, kvh])
            assert [m[int(x)] for x in rc["idx"][b, kvh, :n]] == list(rp["idx"][b, kvh, :n])


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3", "f32"])
def test_sparse_matches_brute_force_and_full_when_everything_fits(oracle, kv_dtype):
    q_dtype = "f32" if kv_dtype == "f32" else "bf16"
    spec = small_spec(kv_dtype=kv_dtype, q_dtype=q_dtype, seq_len=(5, 11), window=4, k_global=8)
    w = synth.generate(spec, seed=4)
    full = run_full(oracle, w)
    # T <= W + K: the index list holds every position, so sparse == full
    sp = run_sparse(oracle, w, w.q_full, full["idx"])
    np.testing.assert_allclose(sp, full["out"], atol=1e-12, rtol=0)
    # own query, shuffled list with holes: brute force over the listed rows
    rng = np.random.default_rng(1)
    idx = full["idx"].copy()
    for b in range(spec.batch):
        for kvh in range(spec.num_kv_heads):
            n = int(full["n_sel"][b, kvh])
            row = idx[b, kvh, :n].copy()
            rng.shuffle(row)
            row[::3] = -1
            idx[b, kvh, :n] = row
    q = w.q_sparse[0]
    got = run_sparse(oracle, w, q, idx)
    qv, K, V = qvals(q, q_dtype), dequant(w, "k"), dequant(w, "v")
    for b in range(spec.batch):
        for h in range(spec.num_q_heads):
            kvh = h // spec.group
            rows = [int(x) for x in idx[b, kvh] if x >= 0]
            lg = [mpmath.fsum(mpmath.mpf(qv[b, h, i]) * mpmath.mpf(K[r, kvh, i])
                              for i in range(spec.head_dim)) / mpmath.sqrt(spec.head_dim) for r in rows]
            e = [mpmath.exp(x) for x in lg]
            Z = mpmath.fsum(e)
            ref = [float(mpmath.fsum(e[j] / Z * mpmath.mpf(V[rows[j], kvh, i]) for j in range(len(rows))))
                   for i in range(spec.head_dim)]
            np.testing.assert_allclose(got[b, h], ref, atol=1e-12, rtol=0)


def test_sparse_single_row_and_order_independence(oracle):
    spec = small_spec(seq_len=20)
    w = synth.generate(spec, seed=6)
    V = dequant(w, "v")
    idx = np.full((spec.batch, spec.num_kv_heads, 6), -1, np.int32)
    idx[:, :, 2] = 17
    got = run_sparse(oracle, w, w.q_sparse[0], idx)
    for h in range(spec.num_q_heads):
        np.testing.assert_allclose(got[:, h], V[17, h // spec.group][None].repeat(2, 0), atol=1e-15)
    idx2 = np.tile(np.array([3, 9, 4, 12, 0, 7], np.int32), (spec.batch, spec.num_kv_heads, 1))
    a = run_sparse(oracle, w, w.q_sparse[0], idx2)
    b = run_sparse(oracle, w, w.q_sparse[0], idx2[:, :, ::-1].copy())
    np.testing.assert_allclose(a, b, atol=1e-15)


# ---- KV Bridging append: encoders and projections --------------------------

def test_e4m3_encode_round_trips_every_finite_code(oracle):
    for c in list(range(0x00, 0x7F)) + list(range(0x80, 0xFF)):
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c or (c == 0x80 and oracle.e4m3_value(c) == 0.0)


def test_e4m3_encode_midpoints_go_to_the_even_code_and_saturate(oracle):
    for c in range(0x00, 0x7E):  # consecutive non-negative codes
        mid = (oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even
        assert oracle.e4m3_encode(-mid) == 0x80 | even
    assert oracle.e4m3_encode(448.0) == 0x7E and oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(-464.0) == 0xFE
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def test_e4m3_encode_matches_torch_cast_of_fp32_values(oracle):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(20000, generator=g) * torch.exp2(torch.randint(-12, 9, (20000,), generator=g).float()))
    x = x.clamp(-448, 448)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x.numpy()], np.uint8)
    assert np.array_equal(got, ref)


def test_bf16_encode_matches_torch_cast_of_fp32_values(oracle):
    g = torch.Generator().manual_seed(6)
    x = torch.randn(20000, generator=g) * torch.exp2(torch.randint(-30, 30, (20000,), generator=g).float())
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.bf16_encode(float(v)) for v in x.numpy()], np.uint16)
    assert np.array_equal(got, ref)


def test_e4m3_row_scale_and_extremes(oracle):
    codes, s = oracle.e4m3_row(np.zeros(16))
    assert s == 1.0 and not codes.any()
    x = np.array([0.3, -2.5, 1.0, 2.5 - 1e-9])
    codes, s = oracle.e4m3_row(x)
    assert s == np.float32(2.5 / 448)
    assert codes[1] == 0xFE  # -max|x| encodes -448
    deq = np.array([oracle.e4m3_value(c) for c in codes]) * s
    assert np.all(np.abs(deq - x) <= 2.5 / 16 + 1e-12)  # half an E4M3 step (2^-4 relative) at the top


def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)


def test_kv_bridge_closed_forms(oracle):
    g = np.random.default_rng(7)
    dm, n = 48, 24
    wk = g.standard_normal((dm, n)).astype(np.float32)
    wv = g.standard_normal((dm, n)).astype(np.float32)
    wkb, wvb = _bf16_bits(wk), _bf16_bits(wv)
    wk_exact = torch.from_numpy(wk).to(torch.bfloat16).double().numpy()
    wv_exact = torch.from_numpy(wv).to(torch.bfloat16).double().numpy()
    # unit hidden states pick rows of the weights
    h = np.zeros((3, dm), np.float32)
    h[0, 5] = 1.0
    h[1, 17] = -2.0
    k, v = oracle.kv_bridge(_bf16_bits(h), wkb, wvb)
    assert np.array_equal(k[0], wk_exact[5]) and np.array_equal(v[1], -2.0 * wv_exact[17])
    assert not k[2].any() and not v[2].any()
    # general inputs: the fp64 matrix product of the stored values
    h = g.standard_normal((4, dm)).astype(np.float32)
    hb = _bf16_bits(h)
    h_exact = torch.from_numpy(h).to(torch.bfloat16).double().numpy()
    k, v = oracle.kv_bridge(hb, wkb, wvb)
    np.testing.assert_allclose(k, h_exact @ wk_exact, rtol=0, atol=1e-12)
    np.testing.assert_allclose(v, h_exact @ wv_exact, rtol=0, atol=1e-12)


# ------------------------------------------------- MQA (one KV head) -----

def test_mqa_layer_matches_50_digit_brute_force(oracle):
    """One KV head shared by 32 query heads: the group score sums all 32
    heads' probabilities."""
    spec = small_spec(num_kv_heads=1, group=32, seq_len=(9, 23))
    w = synth.generate(spec, seed=13)
    got = run_full(oracle, w)
    ref = brute_full(w)
    np.testing.assert_allclose(got["out"], ref["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["lse"], ref["lse"], rtol=0, atol=1e-12)
    for (b, kvh), sc in ref["score"].items():
        T = int(w.seq_lens[b])
        np.testing.assert_allclose(got["score"][b, kvh, :T], sc, rtol=1e-12, atol=0)
        assert abs(sc.sum() - 32) < 1e-12


def test_mqa_equals_gqa_over_copies_of_the_one_kv_head(oracle):
    """MQA over 32 heads against GQA-8 over four identical copies of the KV
    head: the same outputs; the MQA score is the sum of the four group
    scores; the MQA selection is that sum's top-k (ties to the lower
    position) plus the window."""
    W, K = 5, 12
    spec = small_spec(num_kv_heads=1, group=32, seq_len=(40, 90), window=W, k_global=K, page_size=8)
    w = synth.generate(spec, seed=17)
    mqa = run_full(oracle, w)
    code = dtype_code(spec.kv_dtype)
    k4 = np.repeat(synth.raw(w.k), 4, axis=1)
    v4 = np.repeat(synth.raw(w.v), 4, axis=1)
    gqa = oracle.full_attn_select(synth.raw(w.q_full), dtype_code(spec.q_dtype), k4, v4, code,
                                  synth.raw(w.seq_lens), synth.raw(w.page_table), w.page_size, window=W, k_global=K)
    np.testing.assert_allclose(mqa["out"], gqa["out"], rtol=0, atol=1e-14)
    pt = w.page_table.numpy()
    for b in range(spec.batch):
        T = int(w.seq_lens[b])
        summed = gqa["score"][b, :, :T].sum(axis=0)
        np.testing.assert_allclose(mqa["score"][b, 0, :T], summed, rtol=1e-12, atol=0)
        sc = mqa["score"][b, 0, :T - W]
        order = np.lexsort((np.arange(T - W), -sc))
        pos = sorted(order[:K].tolist() + list(range(T - W, T)))
        slots = [int(pt[b, t // w.page_size]) * w.page_size + t % w.page_size for t in pos]
        got = mqa["idx"][b, 0]
        assert got[:len(slots)].tolist() == slots and np.all(got[len(slots):] == -1)
    # a sparse layer over the MQA list equals one over the same list given to each of the four copies
    q_s = synth.raw(w.q_sparse[0])
    s1 = oracle.sparse_attn(q_s, dtype_code(spec.q_dtype), synth.raw(w.k), synth.raw(w.v), code, mqa["idx"])
    s4 = oracle.sparse_attn(q_s, dtype_code(spec.q_dtype), k4, v4, code, np.repeat(mqa["idx"], 4, axis=1))
    np.testing.assert_allclose(s1, s4, rtol=0, atol=1e-14)


# ------------------------------ block-level selection (HySparse v1) -----

def _block_rank_reference(score, T, W, K, block):
    """The definition, by counting: block j is taken when fewer than
    K / block blocks beat it (a higher sum, or an equal sum and a lower
    index).  Scores are dyadic here, so every sum is exact."""
    n_cand = max(T - W, 0)
    blocks = [list(range(j, min(j + block, n_cand))) for j in range(0, n_cand, block)]
    sums = [sum(score[t] for t in blk) for blk in blocks]
    keep = K // block
    taken = set(range(n_cand, T))
    for j, blk in enumerate(blocks):
        beat = sum(1 for i in range(len(blocks)) if sums[i] > sums[j] or (sums[i] == sums[j] and i < j))
        if beat < keep:
            taken.update(blk)
    return sorted(taken)


@pytest.mark.parametrize("block", [1, 2, 3, 4, 6])
def test_block_selection_matches_exhaustive_block_ranking(oracle, block):
    g = np.random.default_rng(100 + block)
    for _ in range(40):
        T = int(g.integers(1, 120))
        W = int(g.integers(0, 10))
        K = block * int(g.integers(1, 6))
        score = g.integers(0, 6, T) / 8.0  # dyadic: exact sums, frequent ties
        got = oracle.select_blocks(score, T, W, K, block)
        assert got.tolist() == _block_rank_reference(score, T, W, K, block), (T, W, K)


def test_blocks_of_one_position_are_token_selection(oracle):
    spec = small_spec(seq_len=(40, 90), window=5, k_global=12, page_size=8)
    for seed, zero_q in ((3, False), (4, True)):
        w = synth.generate(spec, seed=seed)
        if zero_q:  # every score equal: the order is all ties
            w.q_full = torch.zeros_like(w.q_full)
        args = (synth.raw(w.q_full), dtype_code(spec.q_dtype), synth.raw(w.k), synth.raw(w.v),
                dtype_code(spec.kv_dtype), synth.raw(w.seq_lens), synth.raw(w.page_table), w.page_size)
        tok = oracle.full_attn_select(*args, window=5, k_global=12)
        blk = oracle.full_attn_select_blocks(*args, window=5, k_global=12, block=1)
        assert np.array_equal(tok["idx"], blk["idx"]) and np.array_equal(tok["n_sel"], blk["n_sel"])
        assert np.array_equal(tok["out"], blk["out"])


def test_one_needle_brings_its_whole_block(oracle):
    T, W, K, block = 300, 20, 32, 16
    score = np.full(T, 1e-4)
    score[137] = 0.9  # block 8 = [128, 144)
    score[30] = 0.05  # block 1 = [16, 32)
    got = oracle.select_blocks(score, T, W, K, block)
    assert got.tolist() == list(range(16, 32)) + list(range(128, 144)) + list(range(T - W, T))


def test_ragged_last_block_and_short_contexts(oracle):
    W, K, block = 4, 8, 4
    # candidates [0, 10): blocks [0,4) [4,8) [8,10); the short last block wins
    score = np.zeros(14)
    score[8:10] = 1.0
    score[0:4] = 0.25  # block sums: 1.0, 0, 2.0
    got = oracle.select_blocks(score, 14, W, K, block)
    assert got.tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 12, 13]
    # the short block stops at T - W: the window's scores are not part of it
    # (block sums 1.0, 0.9, 0.5; running on into the window would make 1.1)
    score = np.array([0.25] * 4 + [0.225] * 4 + [0.25] * 2 + [0.3] * 4)
    assert oracle.select_blocks(score, 14, W, K, block).tolist() == list(range(8)) + [10, 11, 12, 13]
    # no more candidate blocks than the budget: everything is taken
    assert oracle.select_blocks(np.ones(11), 11, W, K, block).tolist() == list(range(11))
    assert oracle.select_blocks(np.ones(3), 3, W, K, block).tolist() == [0, 1, 2]
    assert oracle.select_blocks(np.ones(1), 0, W, K, block).tolist() == []
    with pytest.raises(ValueError):
        oracle.select_blocks(np.ones(20), 20, W, K, 3)


@pytest.mark.parametrize("kv_dtype,page", [("bf16", 4), ("e4m3", 8), ("f32", None)])
def test_rows_outside_the_sequences_are_never_read(oracle, kv_dtype, page):
    """Every cache row no sequence position maps to is NaN (E4M3: the NaN
    code): the full layer, the selection and a sparse layer over its list
    are unchanged."""
    spec = small_spec(kv_dtype=kv_dtype, q_dtype="f32" if kv_dtype == "f32" else "bf16", page_size=page,
                      seq_len=(9, 30))
    clean = synth.generate(spec, seed=23)
    padded = synth.generate(spec, seed=23, pad_fill="nan")
    assert np.isnan(dequant(padded, "k")).any()  # the fill is really there
    a, b = run_full(oracle, clean), run_full(oracle, padded)
    assert not np.isnan(b["out"]).any()
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["idx"], b["idx"])
    sa = run_sparse(oracle, clean, clean.q_sparse[0], a["idx"])
    sb = run_sparse(oracle, padded, padded.q_sparse[0], b["idx"])
    assert np.array_equal(sa, sb)

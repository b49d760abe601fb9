"""Parity of the KV Bridging append (through the C-ABI) with the oracle: the
new token's K/V rows projected from its hidden state are written at position
T_b - 1 of each sequence (bf16, fp32 or E4M3 with a per-row scale), and no
other row of the cache changes.

The kernel accumulates in fp32, the oracle in fp64.  Each kernel value is a
chain of at most 16 + 8 + d_model / 128 fp32 additions (one warp's rows, the
warps, the splits), so it lies within (that depth + 2) * 2^-24 * sum_i
|h_i w_i| of the exact dot product (the standard bound for recursive
summation).  A stored code may differ from the oracle's only where the exact
value lies within that bound of the midpoint between the two codes, and at
most 1% of a case's codes may differ at all (one row of 64 can hold one such
midpoint: a value 1.3e-8 from a bf16 midpoint, under a bound of 2e-5, has
been seen to round the other way, as it may)."""
import zlib

import numpy as np
import pytest
import torch

from long_context_decode_full_b200 import hs2

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def bf16_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().astype(np.uint16)


def e4m3_values(oracle):
    return np.array([oracle.e4m3_value(c) if c not in (0x7F, 0xFF) else np.nan for c in range(256)])


def bf16_value(u):
    return float(np.array([int(u) << 16], np.uint32).view(np.float32)[0])


def check_rounded(got, ora_codes, exact, tol, decode, what):
    """got / ora_codes: stored codes; exact: the fp64 values they encode; tol:
    the kernel's error bound per value; decode: code -> value.  Codes differ
    only next to a rounding midpoint.  Returns (differing, compared)."""
    bad = got != ora_codes
    for g, o, x, t in zip(got[bad], ora_codes[bad], exact[bad], tol[bad]):
        vg, vo = decode(g), decode(o)
        assert abs(x - (vg + vo) / 2) <= t, f"{what}: {x} stored as {vg}, oracle {vo}"
    return int(bad.sum()), bad.size


CASES = {
    "bf16_paged64": dict(dtype=torch.bfloat16, B=5, Hkv=4, d=128, dm=1024, page=64),
    "bf16_contiguous_d64": dict(dtype=torch.bfloat16, B=4, Hkv=2, d=64, dm=768, page=None),
    "e4m3_paged64": dict(dtype=torch.uint8, B=3, Hkv=4, d=128, dm=512, page=64),
    "e4m3_paged16": dict(dtype=torch.uint8, B=9, Hkv=4, d=128, dm=256, page=16),
    "f32_paged16_d64": dict(dtype=torch.float32, B=2, Hkv=1, d=64, dm=256, page=16),
    # 3 heads of 64: the second 128-column tile is half empty; 11 sequences
    # make two token groups; 3 row splits
    "bf16_ragged_tile_b11": dict(dtype=torch.bfloat16, B=11, Hkv=3, d=64, dm=384, page=32),
    # the projection at the sizes the benchmark times (hidden size 4096): the
    # 256K-context batch, the 1M-token FP8 cache and the 64-sequence batch
    # (8 token groups); the cache itself stays small, the append touches one
    # row per sequence and head
    "bf16_bench_b4": dict(dtype=torch.bfloat16, B=4, Hkv=4, d=128, dm=4096, page=64),
    "e4m3_bench_b1": dict(dtype=torch.uint8, B=1, Hkv=4, d=128, dm=4096, page=64),
    "bf16_bench_b64": dict(dtype=torch.bfloat16, B=64, Hkv=4, d=128, dm=4096, page=64),
}


@pytest.mark.parametrize("name", list(CASES))
def test_kv_bridge_append_matches_oracle(oracle, name):
    c = CASES[name]
    B, Hkv, d, dm, page = c["B"], c["Hkv"], c["d"], c["dm"], c["page"]
    g = torch.Generator().manual_seed(zlib.crc32(name.encode()))  # stable across processes
    cap = 256
    lens = torch.randint(1, cap + 1, (B,), generator=g, dtype=torch.int32)
    if B >= 2:
        lens[B // 2] = 0  # a sequence with no token: nothing is written
    if page is None:
        slots, pt, ps = B * cap, None, cap
    else:
        per = cap // page
        slots, ps = B * per * page, page
        pt = torch.randperm(B * per, generator=g).to(torch.int32).view(B, per)
    N = Hkv * d
    h = torch.randn(B, dm, generator=g).to(torch.bfloat16)
    wk = (torch.randn(dm, N, generator=g) * 0.05).to(torch.bfloat16)
    wv = (torch.randn(dm, N, generator=g) * 0.05).to(torch.bfloat16)
    if c["dtype"] == torch.uint8:
        k0 = torch.randint(0, 0x7E, (slots, Hkv, d), generator=g, dtype=torch.uint8)
        v0 = torch.randint(0, 0x7E, (slots, Hkv, d), generator=g, dtype=torch.uint8)
        ks0, vs0 = torch.rand(slots, Hkv, generator=g), torch.rand(slots, Hkv, generator=g)
    else:
        k0 = torch.randn(slots, Hkv, d, generator=g).to(c["dtype"])
        v0 = torch.randn(slots, Hkv, d, generator=g).to(c["dtype"])
        ks0 = vs0 = None
    dev = lambda t: None if t is None else t.cuda()
    k, v, ks, vs = dev(k0.clone()), dev(v0.clone()), dev(None if ks0 is None else ks0.clone()), \
        dev(None if vs0 is None else vs0.clone())
    # two calls on one workspace: the first (another hidden state) checks that
    # the call leaves its counters ready for the next; the second overwrites
    # the same rows
    ws = torch.zeros(hs2.kv_bridge_workspace_bytes(B, dm, Hkv, d), dtype=torch.uint8, device="cuda")
    h_other = torch.randn(B, dm, generator=g).to(torch.bfloat16)
    for hh in (h_other, h):
        hs2.kv_bridge_append(hh.cuda(), wk.cuda(), wv.cuda(), k, v, lens.cuda(), dev(pt), ps, ks, vs, workspace=ws)
    torch.cuda.synchronize()
    ko, vo = oracle.kv_bridge(bf16_bits(h), bf16_bits(wk), bf16_bits(wv))
    depth = 16 + 8 + dm // 128 + 2
    habs = h.double().abs().numpy()
    eb = {"K": depth * U32 * habs @ wk.double().abs().numpy(), "V": depth * U32 * habs @ wv.double().abs().numpy()}
    k, v = k.cpu(), v.cpu()
    written = set()
    vals = e4m3_values(oracle)
    differ = compared = 0
    for b in range(B):
        T = int(lens[b])
        if T < 1:
            continue
        pos = T - 1
        slot = b * cap + pos if pt is None else int(pt[b, pos // ps]) * ps + pos % ps
        for kvh in range(Hkv):
            written.add((slot, kvh))
            for cache, scales, ref, tag in ((k, ks, ko, "K"), (v, vs, vo, "V")):
                x = ref[b, kvh * d:(kvh + 1) * d]
                tol = eb[tag][b, kvh * d:(kvh + 1) * d]
                what = f"{name} {tag} b{b} h{kvh}"
                if c["dtype"] == torch.bfloat16:
                    got = bf16_bits(cache[slot, kvh])
                    ora = np.array([oracle.bf16_encode(e) for e in x], np.uint16)
                    n, m = check_rounded(got, ora, x, tol, bf16_value, what)
                    differ, compared = differ + n, compared + m
                elif c["dtype"] == torch.float32:
                    err = np.abs(cache[slot, kvh].double().numpy() - x)
                    assert np.all(err <= tol), f"{what}: error {err.max()} above the bound"
                else:
                    codes_o, s_o = oracle.e4m3_row(x)
                    s_g = float(scales.cpu()[slot, kvh])
                    # max|x| moves by at most max(tol); the division and the
                    # two roundings to fp32 add a few units of 2^-24
                    s_tol = tol.max() / 448 + 4 * U32 * s_o
                    assert abs(s_g - s_o) <= s_tol, f"{what}: scale {s_g} vs {s_o}"
                    # x / scale on the device: the value's own error, the
                    # scale's, and one fp32 rounding of the quotient
                    y = x / s_o
                    ytol = tol / s_o + np.abs(y) * (s_tol / s_o + 2 * U32)
                    got = cache[slot, kvh].numpy()
                    n, m = check_rounded(got, codes_o, y, ytol, lambda u: vals[int(u)], what)
                    differ, compared = differ + n, compared + m
    assert differ <= 0.01 * max(compared, 1), f"{name}: {differ} of {compared} codes differ"
    # every other row (and scale) is untouched
    for cache, orig in ((k, k0), (v, v0)):
        diff = (cache.view(torch.uint8) != orig.view(torch.uint8)).reshape(slots, Hkv, -1).any(-1)
        changed = {(int(s), int(hh)) for s, hh in diff.nonzero().tolist()}
        assert changed <= written
    if ks is not None:
        for sc, orig in ((ks.cpu(), ks0), (vs.cpu(), vs0)):
            changed = {(int(s), int(hh)) for s, hh in (sc != orig).nonzero().tolist()}
            assert changed <= written


def test_kv_bridge_zero_hidden_gives_zero_rows_unit_scale(oracle):
    B, Hkv, d, dm, ps = 2, 4, 128, 256, 64
    k = torch.full((B * 4 * ps, Hkv, d), 0x33, dtype=torch.uint8, device="cuda")
    v = k.clone()
    ks = torch.full((B * 4 * ps, Hkv), 7.0, device="cuda")
    vs = ks.clone()
    pt = torch.arange(B * 4, dtype=torch.int32, device="cuda").view(B, 4)
    lens = torch.tensor([5, 200], dtype=torch.int32, device="cuda")
    h = torch.zeros(B, dm, dtype=torch.bfloat16, device="cuda")
    w = torch.randn(dm, Hkv * d, device="cuda").to(torch.bfloat16)
    hs2.kv_bridge_append(h, w, w, k, v, lens, pt, ps, ks, vs)
    torch.cuda.synchronize()
    for b, T in enumerate([5, 200]):
        slot = int(pt[b, (T - 1) // ps]) * ps + (T - 1) % ps
        assert not k[slot].any() and not v[slot].any()
        assert torch.all(ks[slot] == 1.0) and torch.all(vs[slot] == 1.0)

"""The fused full-layer call (hs2_full_attn_select_fused): attention and the
selection's score pass in one cooperative persistent kernel, then the filter
and final kernels.  Its output and index list equal the separate kernels'
bit for bit (the same arithmetic on the same values), and match the oracle."""
import numpy as np
import pytest
import torch

from long_context_decode_full_b200 import hs2, synth
import hs2_testutil as U
from test_gpu_parity import lib, planted_margins, spec  # noqa: F401 (lib is a fixture)

pytestmark = pytest.mark.gpu

CASES = {
    "bf16_paged64": (spec(), None),
    "bf16_contiguous": (spec(page_size=None), None),
    "bf16_paged16": (spec(page_size=16, seq_len=(1100, 3000)), None),
    "bf16_d64_g4": (spec(head_dim=64, group=4, num_kv_heads=3), None),
    "bf16_g1": (spec(group=1, num_kv_heads=4, batch=2), None),
    "bf16_g2": (spec(group=2, num_kv_heads=2, batch=2), None),
    "bf16_g16": (spec(group=16, num_kv_heads=2, batch=2), None),
    "bf16_mqa_g32": (spec(group=32, num_kv_heads=1, batch=3), None),
    "e4m3": (spec(kv_dtype="e4m3", seq_len=(1500, 4000)), None),
    "e4m3_mqa_g32": (spec(kv_dtype="e4m3", group=32, num_kv_heads=1, batch=2, seq_len=(1500, 4000)), None),
    "short_and_empty": (spec(batch=4, seq_len=3000), [3000, 0, 100, 1152]),
    "all_empty": (spec(batch=2, seq_len=64), [0, 0]),
    "many_units": (spec(batch=24, num_kv_heads=4, seq_len=(200, 2600), sparse_layers=1), None),
}


def _both(wd, **kw):
    out_u, idx_u = U.run_gpu(wd, **kw)
    out_f, idx_f = U.run_gpu(wd, fused=True, **kw)
    torch.cuda.synchronize()
    return out_u, idx_u, out_f, idx_f


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_separate_and_oracle(oracle, lib, name):
    sp, lens = CASES[name]
    w = synth.generate(sp, seed=5, seq_lens=lens)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out_u, idx_u, out_f, idx_f = _both(wd)
    assert torch.equal(idx_f, idx_u)
    assert torch.equal(out_f.view(torch.uint8) if out_f.dtype != torch.float32 else out_f,
                       out_u.view(torch.uint8) if out_u.dtype != torch.float32 else out_u)
    U.check_full(wd, out_f, idx_f, ora)


def test_fused_window_and_budget_variants(oracle, lib):
    w = synth.generate(spec(batch=2, seq_len=(2000, 3000)), seed=8)
    wd = U.to_device(w)
    for W, K in [(0, 1024), (128, 0), (64, 200), (512, 3000)]:
        ora = U.run_oracle(oracle, w, window=W, k_global=K)
        out_u, idx_u, out_f, idx_f = _both(wd, window=W, k_global=K)
        assert torch.equal(idx_f, idx_u), (W, K)
        U.check_full(wd, out_f, idx_f, ora, window=W, k_global=K)


def test_fused_repeated_calls_and_garbage_counter(lib):
    """The barrier counter is cleared by each call and returns to zero: calls
    on one workspace repeat, and garbage in the counter word does not matter."""
    w = U.to_device(synth.generate(spec(batch=3, seq_len=(2500, 5000)), seed=9))
    ws = U.garbage_workspace(w)
    ref_out, ref_idx = U.run_gpu(w, workspace=ws)
    ws[64:68] = 0x7F  # the arrival counter
    for _ in range(3):
        out, idx = U.run_gpu(w, workspace=ws, fused=True)
        torch.cuda.synchronize()
        assert hs2.workspace_status(ws) == 0
        assert torch.equal(idx, ref_idx)
        assert torch.equal(out, ref_out)


@pytest.mark.parametrize("kv_dtype,lo,hi", [("bf16", -200.0, -70.0), ("bf16", -420.0, -260.0),
                                             ("e4m3", -200.0, -70.0)])
def test_fused_selection_below_fp32_range(oracle, lib, kv_dtype, lo, hi):
    """Logit margins of 70-420 nats: the k-th score lies below fp32's range
    and the score pass takes the common 2^E factor (the unit's last CTA)."""
    w = planted_margins(kv_dtype, lo, hi, seed=int(-lo))
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out_u, idx_u, out_f, idx_f = _both(wd)
    assert torch.equal(idx_f, idx_u)
    U.check_full(wd, out_f, idx_f, ora)


def test_fused_fp32_cache_runs_separate_kernels(oracle, lib):
    w = synth.generate(spec(kv_dtype="f32", q_dtype="f32", head_dim=64, group=4, num_kv_heads=1, batch=1,
                            seq_len=2048), seed=4)
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out, idx = U.run_gpu(wd, fused=True)
    torch.cuda.synchronize()
    U.check_full(wd, out, idx, ora)


def test_grid_barrier_expires_and_next_fused_call_works(lib):
    """A grid barrier that cannot complete gives up, the status reports it
    once, and the next fused call on the same workspace (which clears the
    barrier's counter) still gives the separate kernels' results."""
    w = U.to_device(synth.generate(spec(batch=2, seq_len=(2000, 3000)), seed=10))
    ws = U.garbage_workspace(w)
    ref_out, ref_idx = U.run_gpu(w, workspace=ws)
    hs2.selftest_grid_barrier(ws)
    assert hs2.workspace_status(ws) == hs2.ERR_TIMEOUT
    assert hs2.workspace_status(ws) == 0
    out, idx = U.run_gpu(w, workspace=ws, fused=True)
    torch.cuda.synchronize()
    assert hs2.workspace_status(ws) == 0
    assert torch.equal(idx, ref_idx)
    assert torch.equal(out, ref_out)


def test_fused_call_with_tcgen05_attention(oracle, lib, monkeypatch):
    """The tcgen05 attention configuration (groups of 32 heads, bf16) through
    the fused call equals its separate kernels and the oracle."""
    monkeypatch.setenv("HS2_FULL_CFG", "4,3,2,2,1")
    sp = spec(group=32, num_kv_heads=1, batch=3)
    w = synth.generate(sp, seed=6, seq_lens=[4100, 90, 2600])
    ora = U.run_oracle(oracle, w)
    wd = U.to_device(w)
    out_u, idx_u, out_f, idx_f = _both(wd)
    assert torch.equal(idx_f, idx_u)
    assert torch.equal(out_f, out_u)
    U.check_full(wd, out_f, idx_f, ora)

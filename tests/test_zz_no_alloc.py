"""hs2_full_attn_select_static: the full-attention + selection call for
callers that may not allocate device memory -- for instance a plugin inside a
serving engine that has reserved nearly all HBM for its own KV-cache pool, or
an extension of a runtime that plans every buffer before execution and gives
its kernels no scratch.  It runs on the library's own fixed 32 MiB device
scratch instead of a caller workspace.  This file runs last, so a failure here
cannot hide the results of the other tests."""
import ctypes

import pytest
import torch

from long_context_decode_full_b200 import hs2, synth
import hs2_testutil as U

pytestmark = pytest.mark.gpu


def _static_call(w, out, idx):
    s = w.spec
    kc = hs2.cache_desc(w.k, w.k_scale, w.page_size)
    vc = hs2.cache_desc(w.v, w.v_scale, w.page_size)
    qd, od = hs2.heads_desc(w.q_full), hs2.heads_desc(out)
    max_pages = 1 if w.page_table is None else w.page_table.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return hs2.lib().hs2_full_attn_select_static(
        ctypes.byref(qd), ctypes.byref(kc), ctypes.byref(vc), ctypes.c_void_p(w.seq_lens.data_ptr()),
        None if w.page_table is None else ctypes.c_void_p(w.page_table.data_ptr()), max_pages, s.window,
        s.k_global, ctypes.byref(od), ctypes.c_void_p(idx.data_ptr()), stream)


def _status():
    return hs2.lib().hs2_full_attn_select_static_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_static_scratch_matches_workspace_call_twice_in_a_row(kv_dtype):
    spec = synth.WorkloadSpec("noalloc", batch=2, num_kv_heads=2, group=8, head_dim=128, seq_len=(2000, 6000),
                              kv_dtype=kv_dtype, q_dtype="bf16", page_size=64, sparse_layers=1, needles=16)
    w = U.to_device(synth.generate(spec, seed=17))
    ref_out, ref_idx = U.run_gpu(w)
    torch.cuda.synchronize()
    for _ in range(2):  # the second call finds the first call's leftovers in the scratch
        out = torch.full_like(ref_out, float("nan"))
        idx = torch.full_like(ref_idx, -7)
        assert _static_call(w, out, idx) == hs2.OK, hs2.last_error()
        assert _status() == hs2.OK, hs2.last_error()  # synchronises; no device wait expired
        err = (out.float() - ref_out.float()).abs().max().item()
        assert err <= U.TOL[kv_dtype]
        assert torch.equal(idx, ref_idx)


def test_static_status_reports_an_expired_wait_once():
    assert _status() == hs2.OK
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert hs2.lib().hs2_selftest_bounded_wait_static(stream) == hs2.OK
    assert _status() == hs2.ERR_TIMEOUT
    assert "flag" in hs2.last_error()
    assert _status() == hs2.OK  # read and cleared


def test_static_scratch_rejects_shapes_beyond_its_size():
    spec = synth.WorkloadSpec("noalloc_big", batch=8, num_kv_heads=4, group=8, head_dim=128, seq_len=4096,
                              kv_dtype="bf16", q_dtype="bf16", page_size=64, sparse_layers=1)
    w = U.to_device(synth.generate(spec, seed=3))
    w.page_table = torch.zeros(8, 512, dtype=torch.int32, device="cuda")  # 32K capacity per sequence
    out = torch.empty_like(w.q_full)
    idx = torch.empty(8, 4, 1152, dtype=torch.int32, device="cuda")
    assert _static_call(w, out, idx) == hs2.ERR_WORKSPACE
    assert "static scratch" in hs2.last_error()

"""The C-ABI boundary without a GPU: the library builds for sm_100a, loads,
exports every entry point that include/hs2.h declares, and rejects bad
arguments on the host with the documented status codes (nothing launches)."""
import ctypes
import os
import re

import pytest
import torch

from long_context_decode_full_b200 import hs2

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "hs2.h")
FAKE = 0x10000  # 16-byte aligned, never dereferenced on the host


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(hs2_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(libhs2):
    names = declared_functions()
    assert "hs2_full_attn_select" in names and "hs2_sparse_attn" in names
    for n in names:
        assert hasattr(libhs2, n), n
    assert set(hs2.EXPORTS) == set(names)
    assert hs2.version() >= 100


def cache(dtype=1, heads=2, dim=128, page=64, slots=1 << 16, scale=None, data=FAKE):
    return hs2.Cache(data, scale, dtype, heads, dim, page, slots)


def heads(dtype=1, b=2, h=16, dim=128, data=FAKE):
    return hs2.Heads(data, dtype, b, h, dim)


def full(q=None, k=None, v=None, seq=FAKE, pt=FAKE, max_pages=64, W=128, K=1024, out=None, idx=FAKE,
         ws=FAKE * 16, ws_bytes=1 << 40):
    q = q or heads()
    k = k or cache()
    v = v or cache()
    out = out or heads()
    return hs2.lib().hs2_full_attn_select(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), seq, pt, max_pages,
                                          W, K, ctypes.byref(out), idx, ws, ws_bytes, None)


def sparse(q=None, k=None, v=None, idx=FAKE, stride=1152, out=None):
    q = q or heads()
    k = k or cache()
    v = v or cache()
    out = out or heads()
    return hs2.lib().hs2_sparse_attn(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), idx, stride,
                                     ctypes.byref(out), None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=heads(data=0)), hs2.ERR_INVALID_ARG),
    (dict(q=heads(data=FAKE + 8)), hs2.ERR_INVALID_ARG),
    (dict(k=cache(dim=96), v=cache(dim=96)), hs2.ERR_UNSUPPORTED),
    (dict(k=cache(heads=4)), hs2.ERR_INVALID_ARG),
    (dict(q=heads(h=6), out=heads(h=6)), hs2.ERR_UNSUPPORTED),
    (dict(q=heads(h=128), out=heads(h=128)), hs2.ERR_UNSUPPORTED),  # G = 64
    (dict(q=heads(h=24), out=heads(h=24)), hs2.ERR_UNSUPPORTED),    # G = 12
    (dict(k=cache(dtype=0, dim=64), v=cache(dtype=0, dim=64), q=heads(dtype=0, h=32, dim=64),
          out=heads(dtype=0, h=32, dim=64)), hs2.ERR_UNSUPPORTED),  # fp32 cache, G = 16
    (dict(q=heads(dtype=0), out=heads(dtype=0)), hs2.ERR_UNSUPPORTED),
    (dict(out=heads(b=3)), hs2.ERR_INVALID_ARG),
    (dict(seq=0), hs2.ERR_INVALID_ARG),
    (dict(idx=0), hs2.ERR_INVALID_ARG),
    (dict(W=-1), hs2.ERR_INVALID_ARG),
    (dict(W=0, K=0), hs2.ERR_INVALID_ARG),
    (dict(max_pages=0), hs2.ERR_INVALID_ARG),
    (dict(pt=0, max_pages=4), hs2.ERR_INVALID_ARG),
    (dict(k=cache(page=48), v=cache(page=48)), hs2.ERR_UNSUPPORTED),
    (dict(k=cache(dtype=2), v=cache(dtype=2)), hs2.ERR_INVALID_ARG),
    (dict(k=cache(dtype=2, dim=64, scale=FAKE), v=cache(dtype=2, dim=64, scale=FAKE),
          q=heads(dim=64), out=heads(dim=64)), hs2.ERR_UNSUPPORTED),
    (dict(k=cache(scale=FAKE), v=cache(scale=FAKE)), hs2.ERR_INVALID_ARG),
    (dict(k=cache(slots=1 << 31), v=cache(slots=1 << 31)), hs2.ERR_INVALID_ARG),
    (dict(ws=0), hs2.ERR_WORKSPACE),
    (dict(ws=FAKE * 16 + 16), hs2.ERR_WORKSPACE),
    (dict(ws_bytes=1024), hs2.ERR_WORKSPACE),
])
def test_full_call_rejects_bad_arguments(libhs2, kw, code):
    assert full(**kw) == code
    assert hs2.last_error()


@pytest.mark.parametrize("kw,code", [
    (dict(idx=0), hs2.ERR_INVALID_ARG),
    (dict(stride=0), hs2.ERR_UNSUPPORTED),
    (dict(stride=5000), hs2.ERR_UNSUPPORTED),
    (dict(q=heads(dim=64)), hs2.ERR_INVALID_ARG),
    (dict(out=heads(h=8)), hs2.ERR_INVALID_ARG),
    (dict(k=cache(dtype=7), v=cache(dtype=7)), hs2.ERR_UNSUPPORTED),
])
def test_sparse_call_rejects_bad_arguments(libhs2, kw, code):
    assert sparse(**kw) == code


def test_workspace_size_rules(libhs2):
    f = hs2.full_workspace_bytes
    a = f(4, 4, 8, 128, 262144)
    assert a > 4 * 4 * 262144 * (8 * 4 + 4)  # at least the logits and the scores
    assert f(4, 4, 8, 128, 2 * 262144) > a
    assert f(0, 4, 8, 128, 1024) == 0 and f(1, 4, 3, 128, 1024) == 0 and f(1, 4, 8, 96, 1024) == 0
    assert a % 256 == 0


def test_copy_rejects_misaligned(libhs2):
    assert hs2.lib().hs2_copy_peak(FAKE, FAKE + 4, 64, None) == hs2.ERR_INVALID_ARG
    assert hs2.lib().hs2_copy_peak(FAKE, FAKE, 60, None) == hs2.ERR_INVALID_ARG


def test_selftest_rejects_bad_workspace(libhs2):
    assert hs2.lib().hs2_selftest_bounded_wait(None, 256, None) == hs2.ERR_WORKSPACE
    assert hs2.lib().hs2_selftest_bounded_wait(FAKE, 16, None) == hs2.ERR_WORKSPACE
    assert hs2.lib().hs2_selftest_bounded_wait(FAKE + 8, 4096, None) == hs2.ERR_WORKSPACE


def test_traffic_hash_ignores_comments_only():
    import bench
    a = 'int f() { // note\n  return 1; /* x */ }\nasm("mov.u64 %0, %%globaltimer; // kept");\n'
    b = 'int f() {\n  return 1; }\nasm("mov.u64 %0, %%globaltimer; // kept");\n'
    c = 'int f() {\n  return 2; }\nasm("mov.u64 %0, %%globaltimer; // kept");\n'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(b) != bench._code_only(c)
    assert "// kept" in bench._code_only(a)  # string literals (inline PTX) are code


def bridge(hidden=FAKE, B=4, dm=4096, wk=FAKE, wv=FAKE, seq=FAKE, pt=FAKE, max_pages=64, k=None, v=None,
           ws=FAKE * 16, ws_bytes=1 << 40):
    k = k or cache()
    v = v or cache()
    return hs2.lib().hs2_kv_bridge_append(hidden, B, dm, wk, wv, seq, pt, max_pages, ctypes.byref(k),
                                          ctypes.byref(v), ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(hidden=0), hs2.ERR_INVALID_ARG),
    (dict(wk=0), hs2.ERR_INVALID_ARG),
    (dict(seq=0), hs2.ERR_INVALID_ARG),
    (dict(wv=FAKE + 4), hs2.ERR_INVALID_ARG),
    (dict(B=0), hs2.ERR_INVALID_ARG),
    (dict(dm=1000), hs2.ERR_UNSUPPORTED),
    (dict(pt=FAKE, max_pages=0), hs2.ERR_INVALID_ARG),
    (dict(pt=0, max_pages=2), hs2.ERR_INVALID_ARG),
    (dict(ws_bytes=1024), hs2.ERR_WORKSPACE),
    (dict(ws=FAKE * 16 + 64), hs2.ERR_WORKSPACE),
    (dict(k=cache(dtype=2), v=cache(dtype=2)), hs2.ERR_INVALID_ARG),  # E4M3 without scales
    (dict(k=cache(heads=4), v=cache(heads=2)), hs2.ERR_INVALID_ARG),
])
def test_kv_bridge_rejects_bad_arguments(libhs2, kw, code):
    assert bridge(**kw) == code


def test_kv_bridge_workspace_size_rule(libhs2):
    f = hs2.kv_bridge_workspace_bytes
    # 256 bytes of tickets (2 x 4 column tiles x 1 token group), then the
    # partial sums [2][d_model / 128][batch][Hkv * d] fp32
    assert f(4, 4096, 4, 128) == 256 + 2 * (4096 // 128) * 4 * 4 * 128 * 4
    assert f(9, 128, 1, 64) == 256 + 2 * 1 * 9 * 64 * 4
    assert f(4, 4000, 4, 128) == 0 and f(0, 4096, 4, 128) == 0 and f(4, 4096, 4, 96) == 0


def _bridge_args(**over):
    B, dm, Hkv, d, slots = 2, 256, 2, 128, 64
    a = dict(hidden=torch.zeros(B, dm, dtype=torch.bfloat16), w_k=torch.zeros(dm, Hkv * d, dtype=torch.bfloat16),
             w_v=torch.zeros(dm, Hkv * d, dtype=torch.bfloat16), k=torch.zeros(slots, Hkv, d, dtype=torch.bfloat16),
             v=torch.zeros(slots, Hkv, d, dtype=torch.bfloat16), seq_lens=torch.ones(B, dtype=torch.int32),
             page_table=torch.zeros(B, 2, dtype=torch.int32), page_size=16)
    a.update(over)
    return a


@pytest.mark.parametrize("over,text", [
    (dict(hidden=torch.zeros(2, 256)), "hidden: dtype"),
    (dict(w_k=torch.zeros(256, 128, dtype=torch.bfloat16)), "w_k: shape"),
    (dict(w_v=torch.zeros(256, 256, dtype=torch.float16)), "w_v: dtype"),
    (dict(seq_lens=torch.ones(2, dtype=torch.int64)), "seq_lens: dtype"),
    (dict(seq_lens=torch.ones(3, dtype=torch.int32)), "seq_lens: shape"),
    (dict(page_table=torch.zeros(3, 2, dtype=torch.int32)), "page_table: 3 rows"),
    (dict(k_scale=torch.zeros(64, 2, dtype=torch.float64)), "k_scale: dtype"),
    (dict(), "not on a CUDA device"),
])
def test_binding_checks_what_pointers_cannot_carry(over, text):
    """Element type, shape and device are checked in the binding, before the
    C call (which only sees bare pointers)."""
    with pytest.raises(hs2.HS2Error, match=text):
        hs2.kv_bridge_append(**_bridge_args(**over))


def test_binding_rejects_int64_lengths_and_lists():
    q = torch.zeros(2, 16, 128, dtype=torch.bfloat16)
    kv = torch.zeros(64, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(hs2.HS2Error, match="seq_lens: dtype"):
        hs2.full_attn_select(q, kv, kv, torch.ones(2, dtype=torch.int64), torch.zeros(2, 2, dtype=torch.int32), 16)
    with pytest.raises(hs2.HS2Error, match="idx: dtype"):
        hs2.sparse_attn(q, kv, kv, torch.zeros(2, 2, 8, dtype=torch.int64), page_size=16)


def test_header_is_plain_c_and_links(libhs2, tmp_path):
    """include/hs2.h compiles as C99 and every entry point it declares links
    against libhs2.so from a C program, which then makes the calls that need
    no GPU (sizes, version, a rejected argument and its message)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    names = declared_functions()
    src = tmp_path / "use_hs2.c"
    src.write_text(
        "#include <stdio.h>\n#include \"hs2.h\"\n"
        "static void *const entry[] = {" + ", ".join(f"(void *){n}" for n in names) + "};\n"
        "int main(void) {\n"
        "  size_t ws = hs2_kv_bridge_workspace(4, 4096, 4, 128);\n"
        "  int rc = hs2_copy_peak(NULL, NULL, 16, NULL);\n"
        "  printf(\"%d %zu %d %d %s\\n\", hs2_version(), ws, rc, (int)(sizeof entry / sizeof entry[0]),\n"
        "         hs2_last_error());\n"
        "  return 0;\n}\n")
    exe = tmp_path / "use_hs2"
    libdir = os.path.dirname(hs2.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                    "-L", libdir, "-lhs2", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split(maxsplit=4)
    assert int(out[0]) == hs2.version()
    assert int(out[1]) == hs2.kv_bridge_workspace_bytes(4, 4096, 4, 128)
    assert int(out[2]) == hs2.ERR_INVALID_ARG and int(out[3]) == len(names) and out[4].strip()


def test_block_selection_rejects_a_block_that_does_not_divide_the_budget(libhs2):
    q, k, v, out = heads(), cache(), cache(), heads()
    call = lambda K, blk: hs2.lib().hs2_full_attn_select_blocks(
        ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), FAKE, FAKE, 64, 128, K, blk, ctypes.byref(out), FAKE,
        FAKE * 16, 1 << 40, None)
    assert call(1024, 3) == hs2.ERR_INVALID_ARG
    assert call(1024, 0) == hs2.ERR_INVALID_ARG
    assert call(1024, -4) == hs2.ERR_INVALID_ARG
    assert "divide" in hs2.last_error()

"""The C-ABI library loads on a CPU-only host, exports every declared symbol, and its host-side
validation rejects bad arguments before touching a GPU."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(helix_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def hx():
    import long_context_decode_helix_b200 as m

    return m


def test_every_declared_symbol_is_exported(hx):
    names = _declared()
    assert {"helix_kv_append", "helix_attn_partial", "helix_attn_combine"} <= set(names)
    for n in names:
        assert hasattr(hx.lib, n), f"libhelix.so does not export {n}"


def test_header_is_plain_c():
    """include/helix.h compiles as C (no C++ in the ABI) and as C++."""
    import shutil
    import subprocess

    inc = os.path.join(ROOT, "include")
    for cc, lang in (("gcc", "c"), ("g++", "c++")):
        exe = shutil.which(cc)
        if exe is None:
            pytest.skip(f"{cc} not found")
        # no CUDA header is needed: the ABI uses only standard C types and opaque handles
        r = subprocess.run([exe, "-fsyntax-only", "-Wall", "-Wextra", "-Werror", "-x", lang,
                            os.path.join(inc, "helix.h")], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_status_strings(hx):
    for code, name in hx.STATUS_NAMES.items():
        assert hx.lib.helix_status_string(code).decode() == name
    assert hx.lib.helix_version() >= 100


def test_combine_rejects_bad_arguments(hx):
    f = hx.lib.helix_attn_combine
    buf = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    assert f(0, 1, 1, 4, buf, buf, buf, 0, None, None) == 1  # kvp = 0
    assert f(1, 1, 1, 6, buf, buf, buf, 0, None, None) == 1  # v_dim not a multiple of 4
    assert f(1, 1, 1, 4, None, buf, buf, 0, None, None) == 1  # null o_partial
    assert f(1, 1, 1, 4, buf, buf, buf, 7, None, None) == 1  # bad o_dtype
    assert f(1, 1, 1, 4, ctypes.c_void_p(8), buf, buf, 0, None, None) == 1  # misaligned


def test_combine_sources_rejects_bad_arguments(hx):
    f = hx.lib.helix_attn_combine_sources
    buf = ctypes.c_void_p(16)  # never dereferenced: validation fails first

    def arr(*p):
        return (ctypes.c_void_p * len(p))(*p)

    o1, l1 = arr(16), arr(16)
    assert f(0, o1, l1, 1, 4, 8, 0, 4, buf, 0, None, None) == 1  # no source
    assert f(17, arr(*([16] * 17)), arr(*([16] * 17)), 1, 4, 8, 0, 4, buf, 0, None, None) == 1
    assert f(1, o1, l1, 1, 4, 8, 2, 2, buf, 0, None, None) == 1  # empty head range
    assert f(1, o1, l1, 1, 4, 8, 0, 5, buf, 0, None, None) == 1  # past the last head
    assert f(1, o1, l1, 1, 4, 6, 0, 4, buf, 0, None, None) == 1  # v_dim not a multiple of 4
    assert f(1, arr(8), l1, 1, 4, 8, 0, 4, buf, 0, None, None) == 1  # misaligned source O
    assert f(1, arr(None), l1, 1, 4, 8, 0, 4, buf, 0, None, None) == 1  # null source
    assert f(1, o1, l1, 1, 4, 8, 0, 4, buf, 3, None, None) == 1  # bad o_dtype
    assert f(1, None, l1, 1, 4, 8, 0, 4, buf, 0, None, None) == 1  # no source array


def _struct(hx, **kw):
    base = dict(kind=0, kv_dtype=0, layout=0, kvp=8, batch=8, num_kv_heads=8, head_dim=128,
                v_dim=128, page_tokens=64, rr_block=16, contig_chunk=0, num_pages=16,
                max_pages_per_shard=2, reserved_=0, k_pool=4096, v_pool=8192, k_scale=None,
                v_scale=None, page_table=256, shard_lens=512, seq_lens=768, err_word=None)
    base.update(kw)
    return hx.CacheStruct(**base)


@pytest.mark.parametrize("bad", [
    dict(kvp=0), dict(batch=0), dict(num_kv_heads=0), dict(layout=5), dict(kind=9),
    dict(rr_block=0), dict(layout=1, contig_chunk=0), dict(k_pool=None), dict(v_pool=None),
    dict(k_pool=4100), dict(page_table=None), dict(seq_lens=None), dict(v_dim=64),
    dict(kv_dtype=1), dict(kind=1, num_kv_heads=1, head_dim=576, v_dim=512),  # MLA needs v_pool NULL
])
def test_append_rejects_bad_cache(hx, bad):
    s = _struct(hx, **bad)
    k = ctypes.c_void_p(1 << 20)
    assert hx.lib.helix_kv_append(ctypes.byref(s), k, k, None, None, 1, None, None) == 1


def test_append_capacity_check(hx):
    s = _struct(hx, num_pages=1 << 24, num_kv_heads=64, page_tokens=64, batch=1, kvp=1)
    k = ctypes.c_void_p(1 << 20)
    assert hx.lib.helix_kv_append(ctypes.byref(s), k, k, None, None, 1, None, None) == 3


def test_null_cache_and_negative_n(hx):
    assert hx.lib.helix_kv_append(None, None, None, None, None, 1, None, None) == 1
    s = _struct(hx)
    k = ctypes.c_void_p(1 << 20)
    assert hx.lib.helix_kv_append(ctypes.byref(s), k, k, None, None, -1, None, None) == 1
    assert hx.lib.helix_kv_append(ctypes.byref(s), k, k, None, None, 0, None, None) == 0  # no-op
    n = ctypes.c_size_t()
    assert hx.lib.helix_attn_workspace_size(None, 128, ctypes.byref(n)) == 1
    assert hx.lib.helix_attn_workspace_size(ctypes.byref(s), 100, ctypes.byref(n)) == 1  # Hq % Hkv
    assert hx.lib.helix_attn_workspace_size(ctypes.byref(s), 256, ctypes.byref(n)) == 2  # G = 32


def test_range_calls_reject_bad_ranges(hx):
    buf = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    f = hx.lib.helix_attn_combine_range
    assert f(2, 4, 8, 128, -1, 2, buf, buf, buf, 0, None, None) == 1  # negative begin
    assert f(2, 4, 8, 128, 3, 2, buf, buf, buf, 0, None, None) == 1  # end < begin
    assert f(2, 4, 8, 128, 0, 5, buf, buf, buf, 0, None, None) == 1  # end > batch
    s = _struct(hx)
    g = hx.lib.helix_attn_partial_range
    assert g(ctypes.byref(s), buf, 128, 0.1, 0, 9, buf, buf, buf, 1 << 20, None) == 1
    assert g(ctypes.byref(s), buf, 128, 0.1, 5, 4, buf, buf, buf, 1 << 20, None) == 1
    assert g(None, buf, 128, 0.1, 0, 1, buf, buf, buf, 1 << 20, None) == 1


def test_overlapped_rejects_missing_events_and_one_stream(hx):
    s = _struct(hx)
    buf = ctypes.c_void_p(16)
    h = hx.lib.helix_attn_overlapped
    ev = (ctypes.c_void_p * 3)(32, 64, 96)
    args = lambda n, sa, sb, evs: (ctypes.byref(s), buf, 128, 0.1, n, buf, buf, buf, 0, None, buf,
                                   1 << 20, sa, sb, evs)
    assert h(*args(2, None, ctypes.c_void_p(8), None)) == 1  # no events
    assert h(*args(2, ctypes.c_void_p(8), ctypes.c_void_p(8), ev)) == 1  # the same stream twice
    assert h(*args(0, None, ctypes.c_void_p(8), ev)) == 1  # no groups
    ev_null = (ctypes.c_void_p * 3)(32, None, 96)
    assert h(*args(2, None, ctypes.c_void_p(8), ev_null)) == 1  # a null event handle


def test_partial_combine_rejects_a_missing_cache(hx):
    buf = ctypes.c_void_p(16)
    f = hx.lib.helix_attn_partial_combine
    assert f(None, buf, 128, 0.1, buf, buf, buf, 0, None, buf, 1 << 20, None) == 1

"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_b200.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", txt)) - {"defined"})


@pytest.fixture(scope="module")
def lib():
    from attention_causal_gqa_b200.build import build
    build()
    from attention_causal_gqa_b200 import binding
    return binding.lib


def test_header_declares_the_three_entry_points():
    names = _declared()
    for n in ("attn_prefill", "attn_decode_paged", "mla_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared():
        assert hasattr(lib, n), n


FAKE = 1 << 20  # non-null, 256-byte aligned; never dereferenced because validation fails first


def _err(lib):
    return lib.attn_last_error().decode()


def test_prefill_chunk_validation_codes(lib):
    f = lib.attn_prefill_chunk
    P = ctypes.c_void_p(FAKE)
    #          q  k  v  kp vp bt cl out lse  B Hq Hkv S_new D  ps maxp np  maxc theta scale ws bytes stream
    args = [P, P, P, P, P, P, P, P, P, 2, 8, 2, 64, 128, 16, 8, 20, 64, 1e4, 0.0, P, 1 << 30, None]

    def call(**over):
        a = list(args)
        for k, v in over.items():
            a[int(k[1:])] = v
        return f(*a)

    assert call(_0=None) == 1 and "null" in _err(lib)
    assert call(_10=6, _11=4) == 1                 # Hq % Hkv
    assert call(_12=0) == 1                        # S_new = 0
    assert call(_13=96) == 2                       # D = 96
    assert call(_14=32) == 2                       # page size 32
    assert call(_17=65) == 1 and "block table" in _err(lib)   # max_cache_len + S_new > 8 pages * 16
    need = lib.attn_prefill_chunk_workspace_size(2, 2, 64, 64, 128)
    assert call(_21=need - 1) == 3
    assert call(_0=ctypes.c_void_p(FAKE + 8), _21=need) == 1  # misaligned q


def test_prefill_validation_codes(lib):
    f = lib.attn_prefill
    P = ctypes.c_void_p(FAKE)
    assert f(None, P, P, P, P, 1, 4, 2, 64, 128, 1, 1e4, 0.0, 1, P, 1 << 30, None) == 1
    assert "null" in _err(lib)
    assert f(P, P, P, P, P, 1, 6, 4, 64, 128, 1, 1e4, 0.0, 1, P, 1 << 30, None) == 1  # Hq % Hkv
    assert f(P, P, P, P, P, 0, 4, 2, 64, 128, 1, 1e4, 0.0, 1, P, 1 << 30, None) == 1  # B = 0
    assert f(P, P, P, P, P, 1, 4, 2, 64, 96, 1, 1e4, 0.0, 1, P, 1 << 30, None) == 2   # D = 96
    assert f(P, P, P, P, P, 1, 4, 2, 64, 128, 1, 1e4, 0.0, 0, P, 1 << 30, None) == 2  # fp32 with D = 128
    assert f(P, P, P, P, P, 1, 4, 2, 64, 128, 1, 1e4, 0.0, 7, P, 1 << 30, None) == 2  # unknown dtype
    need = lib.attn_prefill_workspace_size(1, 2, 64, 128, 1)
    assert f(P, P, P, P, P, 1, 4, 2, 64, 128, 1, 1e4, 0.0, 1, P, need - 1, None) == 3
    Q = ctypes.c_void_p(FAKE + 8)  # misaligned q
    assert f(Q, P, P, P, P, 1, 4, 2, 64, 128, 1, 1e4, 0.0, 1, P, need, None) == 1


def test_decode_validation_codes(lib):
    f = lib.attn_decode_paged
    P = ctypes.c_void_p(FAKE)
    need = lib.attn_decode_paged_workspace_size(2, 32, 128, 64, 16)
    args = lambda **kw: dict(dict(B=2, Hq=32, Hkv=8, D=128, ps=16, maxp=64, npg=100, dt=1, ws=need), **kw)

    def call(**kw):
        a = args(**kw)
        return f(P, P, P, P, P, P, P, a["B"], a["Hq"], a["Hkv"], a["D"], a["ps"], a["maxp"], a["npg"], 0.0, a["dt"],
                 P, a["ws"], None)
    assert call(Hq=30) == 1
    assert call(ps=32) == 2
    assert call(D=256) == 2
    assert call(Hkv=8, Hq=8192) == 2               # beyond 4096 query heads
    assert call(dt=0) == 2
    assert call(ws=need - 1) == 3
    assert call(npg=0) == 1
    assert f(None, P, P, P, P, P, P, 2, 32, 8, 128, 16, 64, 100, 0.0, 1, P, need, None) == 1


def test_mla_validation_codes(lib):
    f = lib.mla_decode
    P = ctypes.c_void_p(FAKE)
    need = lib.mla_decode_workspace_size(2, 128, 512, 64, 4096)
    assert f(P, P, P, P, P, 0.07, P, P, 2, 64, 512, 64, 4096, P, need, None) == 2   # H = 64
    assert f(P, P, P, P, P, 0.07, P, P, 2, 128, 256, 64, 4096, P, need, None) == 2  # Dc = 256
    assert f(P, P, P, P, P, 0.0, P, P, 2, 128, 512, 64, 4096, P, need, None) == 1   # scale
    assert f(P, P, P, P, P, 0.07, P, P, 2, 128, 512, 64, 4096, P, need - 1, None) == 3
    assert f(P, None, P, P, P, 0.07, P, P, 2, 128, 512, 64, 4096, P, need, None) == 1


def test_workspace_sizes_grow_with_problem(lib):
    a = lib.attn_prefill_workspace_size(1, 8, 4096, 128, 1)
    b = lib.attn_prefill_workspace_size(2, 8, 4096, 128, 1)
    assert b > a > 256
    assert lib.mla_decode_workspace_size(32, 128, 512, 64, 32768) > lib.mla_decode_workspace_size(1, 128, 512, 64, 512)
    assert lib.attn_selftest_wait_timeout(ctypes.c_void_p(FAKE), 100, 10 ** 6, None) == 3
    assert lib.attn_selftest_wait_timeout(ctypes.c_void_p(FAKE), 256, 10, None) == 1


def test_prefill_ex_validation_codes(lib):
    f = lib.attn_prefill_ex
    P = ctypes.c_void_p(FAKE)
    need = lib.attn_prefill_workspace_size(1, 2, 256, 128, 1)

    def call(layout=0, fscale=1.0, ws=need, D=128, dt=1):
        return f(P, P, P, P, P, 1, 8, 2, 256, D, 1, 1e4, fscale, layout, 0.0, dt, P, ws, None)
    assert call(layout=2) == 1
    assert call(fscale=0.0) == 1
    assert call(fscale=-1.0) == 1
    assert call(fscale=float("inf")) == 1
    assert call(dt=0) == 2
    assert call(ws=need - 1) == 3
    assert call(layout=1, ws=need - 1) == 3  # the half-split layout itself is accepted


def test_decode_fp8_validation_codes(lib):
    f = lib.attn_decode_paged_fp8
    P = ctypes.c_void_p(FAKE)
    need = lib.attn_decode_paged_fp8_workspace_size(2, 32, 128, 64, 16)

    def call(D=128, Hkv=8, Hq=32, ps=16, ws=need, ks=P):
        return f(P, P, P, ks, P, P, P, P, P, 2, Hq, Hkv, D, ps, 64, 100, 0.0, P, ws, None)
    assert call(D=96) == 2
    assert call(D=256) == 2
    assert call(Hkv=16, Hq=32) == 2
    assert call(ps=32) == 2
    assert call(Hq=30) == 1
    assert call(ws=need - 1) == 3
    assert call(ks=None) == 1
    # one partial per (page range, sequence): independent of the longest sequence
    assert need == lib.attn_decode_paged_fp8_workspace_size(2, 32, 128, 4096, 16)


def test_dsa_validation_codes(lib):
    P = ctypes.c_void_p(FAKE)
    f = lib.dsa_index_topk
    wsi = lib.dsa_index_topk_workspace_size(2, 64, 128, 4096, 2048)

    def idx(HI=64, dI=128, k=2048, ws=wsi, w=P):
        return f(P, w, P, P, P, P, 2, HI, dI, 4096, k, P, ws, None)
    assert idx(dI=64) == 2
    assert idx(HI=24) == 2
    assert idx(HI=128) == 2
    assert idx(k=0) == 1
    assert idx(w=None) == 1
    assert idx(ws=wsi - 1) == 3
    g = lib.dsa_mla_decode
    need = lib.dsa_mla_decode_workspace_size(2, 128, 512, 64, 2048)
    assert need > lib.mla_decode_workspace_size(2, 128, 512, 64, 2048)  # plus the gathered rows

    def mla(H=128, k=2048, scale=0.07, ws=need, ix=P):
        return g(P, P, P, P, P, ix, k, scale, P, P, 2, H, 512, 64, 4096, P, ws, None)
    assert mla(H=64) == 2
    assert mla(k=0) == 1
    assert mla(scale=0.0) == 1
    assert mla(ix=None) == 1
    assert mla(ws=need - 1) == 3


def test_prefill_chunk_ex_validation_codes(lib):
    f = lib.attn_prefill_chunk_ex
    P = ctypes.c_void_p(FAKE)
    need = lib.attn_prefill_chunk_workspace_size(2, 2, 64, 64, 128)

    def call(layout=0, fscale=1.0, ws=need):
        return f(P, P, P, P, P, P, P, P, P, 2, 8, 2, 64, 128, 16, 8, 20, 64, 1e4, fscale, layout, 0.0, P, ws, None)
    assert call(layout=5) == 1
    assert call(fscale=0.0) == 1
    assert call(ws=need - 1) == 3
    assert call(layout=1, ws=need - 1) == 3  # the half-split layout itself is accepted


def test_dsa_fp8_validation_codes(lib):
    P = ctypes.c_void_p(FAKE)
    g = lib.dsa_mla_decode_fp8
    need = lib.dsa_mla_decode_workspace_size(2, 128, 512, 64, 2048)

    def call(Dc=512, k=2048, sc=P, ws=need):
        return g(P, P, P, sc, P, P, P, k, 0.07, P, P, 2, 128, Dc, 64, 4096, P, ws, None)
    assert call(Dc=256) == 2
    assert call(k=0) == 1
    assert call(sc=None) == 1
    assert call(ws=need - 1) == 3


def test_dsa_gather_grid_limit(lib):
    """B * top_k selected rows beyond 2^30 would not fit the gather's grid: rejected up front."""
    P = ctypes.c_void_p(FAKE)
    g = lib.dsa_mla_decode
    assert g(P, P, P, P, P, P, 1 << 21, 0.07, P, P, 1024, 128, 512, 64, 1 << 22, P, 1 << 62, None) == 2


def test_noalloc_array_holds_the_stated_example_and_rejects_past_it(lib):
    """The fixed array of attn_decode_paged_noalloc holds 8 sequences of 32K tokens at
    Hq = 32, D = 128 (2048 pages of 16 tokens); with that table width 31 sequences fit
    and 32 do not. The size check runs before any CUDA call, so the rejection is
    visible without a GPU."""
    cap = 32 << 20
    ws = lib.attn_decode_paged_workspace_size
    ws.restype = ctypes.c_size_t
    assert ws(8, 32, 128, 2048, 16) <= cap
    assert ws(31, 32, 128, 2048, 16) <= cap < ws(32, 32, 128, 2048, 16)
    f = lib.attn_decode_paged_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 7 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
    P = ctypes.c_void_p(FAKE)
    assert f(P, P, P, P, P, P, P, 32, 32, 8, 128, 16, 2048, 100, 0.0, 1, None) == 3
    assert "scratch" in _err(lib)
    g = lib.attn_decode_paged_noalloc_status
    g.restype = ctypes.c_int
    assert g(None, None) == 1 and "null" in _err(lib)


def test_rope_base_helpers_match_the_oracle(lib):
    """The library's NTK-aware and length-scaled RoPE bases (host functions, no GPU)
    against the oracle's, and their argument checks."""
    from oracle import length_scaled_theta_ref, ntk_aware_theta_ref
    from attention_causal_gqa_b200.binding import length_scaled_theta, ntk_aware_theta
    for D, s, th in ((64, 8.0, 1e4), (128, 4.0, 5e5), (128, 1.0, 1e4), (192, 32.0, 1e6)):
        assert abs(ntk_aware_theta(th, s, D) - ntk_aware_theta_ref(th, s, D)) <= 1e-12 * ntk_aware_theta_ref(th, s, D)
    for L, L0, a in ((4096, 4096, 0.2), (131072, 4096, 0.5), (8192, 4096, 1.0), (1024, 4096, 0.3)):
        r = length_scaled_theta_ref(1e4, L, L0, a)
        assert abs(length_scaled_theta(1e4, L, L0, a) - r) <= 1e-12 * r
    lib.attn_rope_ntk_theta.restype = ctypes.c_double
    lib.attn_rope_ntk_theta.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_int]
    assert lib.attn_rope_ntk_theta(1e4, 0.5, 128) == 0.0 and "scale" in _err(lib)   # shrinking is not a stretch
    assert lib.attn_rope_ntk_theta(1e4, 2.0, 3) == 0.0                               # odd head dim
    assert lib.attn_rope_ntk_theta(-1.0, 2.0, 128) == 0.0


def test_lse_merge_validation_codes(lib):
    f = lib.attn_lse_merge
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    P = ctypes.c_void_p(FAKE)
    assert f(None, P, 2, 64, 128, P, P, None) == 1 and "null" in _err(lib)
    assert f(P, P, 0, 64, 128, P, P, None) == 1       # no parts
    assert f(P, P, 2, 0, 128, P, P, None) == 1        # no rows
    assert f(P, P, 2, 64, 96, P, P, None) == 2        # D = 96
    assert f(ctypes.c_void_p(FAKE + 2), P, 2, 64, 128, P, P, None) == 1  # misaligned


def test_prefill_chunk_varlen_validation_codes(lib):
    f = lib.attn_prefill_chunk_varlen
    f.restype = ctypes.c_int
    P = ctypes.c_void_p(FAKE)
    need = lib.attn_prefill_chunk_workspace_size(2, 2, 64, 64, 128)
    #     q  k  v  kp vp bt cl nl out lse  B Hq Hkv S_new D ps maxp np maxc theta fscale layout scale ws bytes stream
    args = [P, P, P, P, P, P, P, P, P, P, 2, 8, 2, 64, 128, 16, 8, 20, 64, 1e4, 1.0, 0, 0.0, P, need, None]
    f.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_int] * 9 + [ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                                                 ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t,
                                                                 ctypes.c_void_p]

    def call(**over):
        a = list(args)
        for k, v in over.items():
            a[int(k[1:])] = v
        return f(*a)

    assert call(_0=None) == 1 and "null" in _err(lib)
    assert call(_7=ctypes.c_void_p(FAKE + 2)) == 1 and "new_lens" in _err(lib)   # misaligned lengths
    assert call(_14=96) == 2                                                       # D = 96
    assert call(_24=need - 1) == 3

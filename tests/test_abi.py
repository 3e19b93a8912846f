"""The C ABI without a GPU: the library builds, loads and exports every declared
entry point; arguments are validated before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "la.h")


@pytest.fixture(scope="module")
def lib():
    from tests.conftest import load_build_module
    return ctypes.CDLL(load_build_module().build())


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(la_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ("la_bidir_fwd", "la_bidir_bwd", "la_simple_fwd", "la_simple_bwd", "la_chunk_decay_fwd",
              "la_chunk_decay_bwd", "la_chunk_decay_step", "la_chunk_decay_fwd_state", "la_chunk_decay_bwd_state",
              "la_chunk_decay_scan", "la_causal_norm_fwd", "la_causal_norm_bwd", "la_gated_fwd", "la_gated_bwd",
              "la_feature_map_fwd", "la_feature_map_bwd",
              "la_workspace_size", "la_status_string", "la_last_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, "not exported: %s" % missing


def _binding():
    import linear_attention_attn_b200 as la
    return la


def test_binding_names_match_abi():
    la = _binding()
    for n in declared_functions():
        if n == "la_prof_collect" or n == "la_prof_enable" or n.startswith("la_"):
            assert hasattr(la, n), "binding lacks %s" % n


def test_workspace_size_is_deterministic():
    la = _binding()
    a = la.la_workspace_size("bidir_bwd", 8, 16, 4096, 64, la.LA_F16)
    b = la.la_workspace_size("bidir_bwd", 8, 16, 4096, 64, la.LA_F16)
    assert a == b and a > 0 and a % 256 == 0
    assert la.la_workspace_size("bidir_fwd", 8, 16, 4096, 65, la.LA_F16) == 0
    assert la.la_workspace_size("bidir_fwd", 0, 16, 4096, 64, la.LA_F16) == 0


def _call_fwd(lib, q=0x1000, k=0x1000, v=0x1000, o=0x1000, B=1, H=1, T=16, D=64, dt=1, eps=1e-6,
              ws=0x100000, wsb=1 << 30):
    P = ctypes.c_void_p
    f = lib.la_bidir_fwd
    f.restype = ctypes.c_int
    return f(P(q), P(k), P(v), P(o), P(0), B, H, T, D, dt, ctypes.c_float(eps), P(ws), ctypes.c_size_t(wsb), P(0))


def test_validation_codes(lib):
    # status codes as in include/la.h; none of these reach a CUDA call
    assert _call_fwd(lib, D=65) == 2            # LA_ERR_UNSUPPORTED
    assert _call_fwd(lib, dt=7) == 2
    assert _call_fwd(lib, q=0) == 1             # LA_ERR_INVALID_ARG
    assert _call_fwd(lib, B=0) == 1
    assert _call_fwd(lib, T=-1) == 1
    assert _call_fwd(lib, eps=-1.0) == 1
    assert _call_fwd(lib, eps=float("nan")) == 1
    assert _call_fwd(lib, k=0x1001) == 3        # LA_ERR_ALIGNMENT
    assert _call_fwd(lib, ws=0) == 4            # LA_ERR_WORKSPACE
    assert _call_fwd(lib, wsb=16) == 4
    assert _call_fwd(lib, ws=0x100010) == 3     # workspace must be 256-byte aligned
    lib.la_last_error.restype = ctypes.c_char_p
    assert b"workspace" in lib.la_last_error()


def test_decay_validation(lib):
    P = ctypes.c_void_p
    f = lib.la_chunk_decay_fwd
    f.restype = ctypes.c_int
    bad = (ctypes.c_float * 2)(0.5, 1.5)
    assert f(P(0x1000), P(0x1000), P(0x1000), P(0x1000), ctypes.cast(bad, P), 1, 2, 16, 64, 2, P(0x100000),
             ctypes.c_size_t(1 << 30), P(0)) == 1
    assert f(P(0x1000), P(0x1000), P(0x1000), P(0x1000), P(0), 1, 2, 16, 64, 2, P(0x100000),
             ctypes.c_size_t(1 << 30), P(0)) == 1
    many = (ctypes.c_float * 600)(*([0.5] * 600))
    assert f(P(0x1000), P(0x1000), P(0x1000), P(0x1000), ctypes.cast(many, P), 1, 600, 16, 64, 2, P(0x100000),
             ctypes.c_size_t(1 << 30), P(0)) == 2


def test_decay_bwd_state_validation(lib):
    # dstate_out is written while other CTAs still read state_in and dstate_in: overlap is refused
    P = ctypes.c_void_p
    f = lib.la_chunk_decay_bwd_state
    f.restype = ctypes.c_int
    gam = (ctypes.c_float * 2)(0.5, 0.9)
    nbytes = 1 * 2 * 64 * 64 * 4

    def call(sin, rin, rout):
        return f(P(0x1000), P(0x1000), P(0x1000), P(0x1000), P(sin), P(rin), P(rout), ctypes.cast(gam, P),
                 P(0x1000), P(0x1000), P(0x1000), 1, 2, 16, 64, 2, P(0x100000), ctypes.c_size_t(1 << 30), P(0))
    assert call(0x200000, 0x400000, 0x400000) == 1
    assert call(0x200000, 0x400000, 0x400000 + nbytes - 16) == 1
    assert call(0x200000 + nbytes - 16, 0x800000, 0x200000) == 1
    assert call(0x200000, 0x400000, 0x400008) == 3     # 16-byte alignment
    lib.la_last_error.restype = ctypes.c_char_p
    assert call(0x200000, 0x400000, 0x400000 + nbytes - 16) == 1 and b"overlaps" in lib.la_last_error()


def test_decay_scan_validation(lib):
    P = ctypes.c_void_p
    f = lib.la_chunk_decay_scan
    f.restype = ctypes.c_int
    gam = (ctypes.c_float * 2)(0.5, 0.9)
    gaps = (ctypes.c_longlong * 200)(*([0] * 200))

    def call(n=2, st=0x200000, gp=True, out=0x400000, D=128, dec=gam):
        return f(P(st), ctypes.cast(gaps, P) if gp else P(0), n, ctypes.cast(dec, P), P(out), 1, 2, D, P(0))
    assert call(n=0) == 2
    assert call(n=129) == 2
    assert call(D=96) == 2
    assert call(gp=False) == 1
    assert call(st=0) == 1
    assert call(out=0x400004) == 3
    bad = (ctypes.c_float * 2)(0.5, 0.0)
    assert call(dec=bad) == 1


def test_causal_norm_validation(lib):
    P = ctypes.c_void_p
    f = lib.la_causal_norm_fwd
    f.restype = ctypes.c_int
    b = lib.la_causal_norm_bwd
    b.restype = ctypes.c_int

    def fwd(feature=1, eps=1e-6, q=0x1000, dec=None, D=64, T=16, ws=0, ws_bytes=0):
        return f(P(q), P(0x1000), P(0x1000), P(0x1000), dec, feature, ctypes.c_float(eps), 1, 2, T, D, 1, P(ws),
                 ctypes.c_size_t(ws_bytes), P(0))
    assert fwd(feature=5) == 2
    assert fwd(eps=-1.0) == 1
    assert fwd(q=0) == 1
    assert fwd(q=0x1008) == 3
    assert fwd(D=32) == 2
    bad = (ctypes.c_float * 2)(0.5, 2.0)
    assert fwd(dec=ctypes.cast(bad, P)) == 1
    # CUDA-core path (bf16): (n, dn) per row, then the chunk states
    need = lib.la_workspace_size(11, 1, 2, 16, 64, 2)
    assert need == 256            # 2 x 16 rows x 8 bytes, rounded up to 256
    # one chunk of 256 tokens needs no chunk states; 257 tokens make two chunks of [64][65] fp32 states
    assert lib.la_workspace_size(10, 1, 2, 256, 64, 2) == 0
    assert lib.la_workspace_size(10, 1, 2, 257, 64, 2) == 2 * 2 * 64 * 65 * 4
    assert lib.la_workspace_size(11, 1, 2, 257, 64, 2) == 4352 + 2 * 2 * 64 * 65 * 4
    # tensor-core path (fp16, D = 64), each part rounded up to 256 bytes: f(q), f(k) for both;
    # the backward adds du (16-bit), dn (fp32 per row), the per-chunk sums ([2 heads][1 chunk]
    # [2][64] fp32) and dq, dk in fp32
    t16, t32 = 2 * 16 * 64 * 2, 2 * 16 * 64 * 4
    assert lib.la_workspace_size(10, 1, 2, 16, 64, 1) == 2 * t16
    assert lib.la_workspace_size(11, 1, 2, 16, 64, 1) == 3 * t16 + 256 + 2 * 128 * 4 + 2 * t32
    assert fwd(T=257) == 4        # no workspace for two chunks
    assert fwd(T=257, ws=0x1080, ws_bytes=1 << 20) == 3     # not 256-byte aligned
    assert fwd(T=257, ws=0x1000, ws_bytes=100) == 4
    assert b(P(0x1000), P(0x1000), P(0x1000), P(0x1000), None, 1, ctypes.c_float(1e-6), P(0x1000), P(0x1000),
             P(0x1000), 1, 2, 16, 64, 1, P(0), ctypes.c_size_t(0), P(0)) == 4


def test_gated_workspace(lib):
    P = ctypes.c_void_p
    f = lib.la_gated_fwd
    f.restype = ctypes.c_int
    lib.la_workspace_size.restype = ctypes.c_size_t
    # one chunk (T <= 256): no forward workspace, the backward holds dq in fp32
    assert lib.la_workspace_size(12, 1, 2, 256, 64, 1) == 0
    assert lib.la_workspace_size(13, 1, 2, 256, 64, 1) == 2 * 256 * 64 * 4
    # two chunks: [2 heads][2 chunks][64][64] states and [2][2][64] gate products (and dg totals)
    states, per_dim = 2 * 2 * 64 * 64 * 4, 2 * 2 * 64 * 4
    assert lib.la_workspace_size(12, 1, 2, 257, 64, 1) == states + per_dim
    assert lib.la_workspace_size(13, 1, 2, 257, 64, 1) == 2 * 257 * 64 * 4 + states + 2 * per_dim

    def fwd(T, ws=0, ws_bytes=0):
        return f(P(0x1000), P(0x1000), P(0x1000), P(0x1000), P(0x1000), 1, 2, T, 64, 1, P(ws),
                 ctypes.c_size_t(ws_bytes), P(0))
    assert fwd(257) == 4
    assert fwd(257, ws=0x1010, ws_bytes=1 << 20) == 3
    assert fwd(257, ws=0x1000, ws_bytes=states) == 4


def test_status_strings(lib):
    lib.la_status_string.restype = ctypes.c_char_p
    assert lib.la_status_string(0) == b"LA_OK"
    assert lib.la_status_string(5) == b"LA_ERR_CUDA"


def test_fail_launch_hook_validates_without_a_gpu(lib):
    assert lib.la_debug_fail_launch(-2) == 1           # LA_ERR_INVALID_ARG
    assert lib.la_debug_fail_launch(-1) == 0           # disarm

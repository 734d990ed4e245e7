"""The C-ABI library without a GPU: it loads, exports every symbol include/la_state.h
declares, its pure host functions return the sizes the pages print, and invalid
arguments are rejected on the host before anything is launched (no call in this file
reaches a kernel launch)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from gated_deltanet_recurrent_la_b200 import lastate as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "la_state.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "page_sizes.txt")


def golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            out[k] = int(v)
    return out


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(L.LIB_PATH):
        from gated_deltanet_recurrent_la_b200 import build
        build.build()
    return L.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(la_[a-z_]+)\s*\(", text)))


def test_header_is_plain_c():
    """The boundary header compiles as C99 and as C++11 on its own (no torch or CUDA types)."""
    import shutil
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "la_state.h")
    for cc, std, lang in (("gcc", "-std=c99", "c"), ("g++", "-std=c++11", "c++")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not installed")
        r = subprocess.run([cc, std, "-fsyntax-only", "-Wall", "-Werror", "-x", lang, hdr], capture_output=True,
                           text=True)
        assert r.returncode == 0, r.stderr


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(L.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (la_[a-z_]+)\b", out))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(lib, f)
    header = open(os.path.join(ROOT, "include", "la_state.h")).read()
    assert lib.la_abi_version() == int(re.search(r"#define LA_ABI_VERSION (\d+)", header).group(1))


def test_state_bytes_match_page_figures(lib):
    G = golden()
    # 64 heads x 128 x 128 at 2 bytes (BF16 has the page's 2 bytes per value)
    assert L.la_state_bytes(64, 64, 128, 128, torch.bfloat16) == G["onnx_64heads_128x128_2byte_state_bytes"]
    # Nemotron-H-8B layer: 128 heads x (N=128) x (head dim 64)
    nb = L.la_state_bytes(1, 128, 128, 64, torch.bfloat16)
    assert nb == G["nemotron_layer_state_bytes_bf16"]
    assert nb // 2 == G["nemotron_layer_state_elements"]
    assert 48 * nb == G["nemotron_48_layer_state_bytes_bf16"]
    assert L.la_state_bytes(16, 32, 128, 128, torch.float32) == 2 * L.la_state_bytes(16, 32, 128, 128, torch.bfloat16)
    s = L.la_shape(16, 33, 128, 128)  # H_v not a multiple of H_qk
    assert lib.la_state_bytes(ctypes.byref(s), 1) == 0
    s = L.la_shape(1, 1, 128, 128)
    assert lib.la_state_bytes(ctypes.byref(s), 7) == 0


def test_byte_model_matches_page(lib):
    from bench import step_bytes_and_flops
    G = golden()
    b, f = step_bytes_and_flops(B=1, n_qk_heads=1, n_v_heads=128, d_k=128, d_v=64, state_bytes=2, io_bytes=2,
                                rule="gated", state_only=True)
    assert b == G["nemotron_layer_step_state_bytes"]
    assert f == G["nemotron_layer_step_flops"]


def test_supported_shapes(lib):
    for dk, dv in [(16, 16), (64, 64), (128, 64), (128, 128)]:
        assert L.la_shape_supported(dk, dv)
    for dk, dv in [(32, 32), (128, 256), (0, 0), (64, 128)]:
        assert not L.la_shape_supported(dk, dv)


# ---- host-side validation (fake, never dereferenced device addresses) ------------------

A = 0x7f0000000000  # 16-byte aligned fake address


def pool(dtype=1, n=8, shape=(2, 4, 128, 128), data=A):
    return L.la_pool(ctypes.c_void_p(data), dtype, n, L.la_shape(*shape))


def step(lib, rule=3, src=None, dst=None, rs=None, ws=None, B=4, q=A, k=A, v=A, io=1, g=A, beta=A, o=A, err=A):
    src = src or pool()
    dst = dst or src
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.la_state_step(rule, ctypes.byref(src), P(rs), ctypes.byref(dst), P(ws), B, P(q), P(k), P(v), io, P(g),
                             P(beta), 1.0, P(o), P(err), None)


def test_step_host_errors(lib):
    assert step(lib, rule=9) == L.LA_ERR_UNSUPPORTED
    assert step(lib, err=None) == L.LA_ERR_NULL
    assert step(lib, B=-1) == L.LA_ERR_SHAPE
    assert step(lib, B=0) == L.LA_OK  # empty batch: no-op, nothing launched
    assert step(lib, q=None) == L.LA_ERR_NULL
    assert step(lib, rule=1, g=None) == L.LA_ERR_NULL
    assert step(lib, rule=2, beta=None) == L.LA_ERR_NULL
    assert step(lib, rule=3, g=None) == L.LA_ERR_NULL
    assert step(lib, src=pool(data=0)) == L.LA_ERR_NULL
    assert step(lib, src=pool(shape=(3, 4, 128, 128))) == L.LA_ERR_SHAPE      # H_v % H_qk != 0
    assert step(lib, src=pool(), dst=pool(shape=(2, 4, 128, 64))) == L.LA_ERR_SHAPE
    assert step(lib, src=pool(dtype=0), dst=pool(dtype=1)) == L.LA_ERR_UNSUPPORTED
    assert step(lib, src=pool(dtype=5)) == L.LA_ERR_UNSUPPORTED
    assert step(lib, io=3) == L.LA_ERR_UNSUPPORTED
    assert step(lib, src=pool(shape=(2, 4, 32, 32))) == L.LA_ERR_UNSUPPORTED
    assert step(lib, q=A + 8) == L.LA_ERR_ALIGN
    assert step(lib, o=A + 2) == L.LA_ERR_ALIGN
    assert step(lib, src=pool(data=A + 4)) == L.LA_ERR_ALIGN
    assert step(lib, g=A + 2) == L.LA_ERR_ALIGN
    assert step(lib, B=9) == L.LA_ERR_SHAPE  # dense mode: B > n_slots
    assert step(lib, rule=4, g=None) == L.LA_ERR_NULL      # kda needs its channel decays
    assert step(lib, rule=4, beta=None) == L.LA_ERR_NULL
    assert step(lib, rule=4, g=A + 4) == L.LA_ERR_ALIGN    # kda decays move in 16-byte pieces
    # a scalar gate needs 4 bytes only: the call gets past the alignment checks and stops
    # at the next one (nothing is launched on these fake addresses)
    assert step(lib, rule=3, g=A + 4, B=9) == L.LA_ERR_SHAPE
    assert step(lib, rule=5) == L.LA_ERR_UNSUPPORTED


def scan(lib, rule=3, src=None, rs=None, dst=None, ws=None, n=2, cu=A, T=10, order=None, q=A, io=1, g=A, err=A):
    dst = dst or pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.la_state_scan(rule, None if src is None else ctypes.byref(src), P(rs), ctypes.byref(dst), P(ws), n,
                             P(cu), T, P(order), P(q), P(A), P(A), io, P(g), P(A), 1.0, P(A), P(err), None)


def test_scan_host_errors(lib):
    assert scan(lib, rule=-1) == L.LA_ERR_UNSUPPORTED
    assert scan(lib, err=None) == L.LA_ERR_NULL
    assert scan(lib, n=-1) == L.LA_ERR_SHAPE
    assert scan(lib, T=-1) == L.LA_ERR_SHAPE
    assert scan(lib, n=0) == L.LA_OK
    assert scan(lib, cu=None) == L.LA_ERR_NULL
    assert scan(lib, q=None) == L.LA_ERR_NULL
    assert scan(lib, rs=A, src=None) == L.LA_ERR_NULL
    assert scan(lib, rs=A, src=pool(shape=(2, 4, 64, 64))) == L.LA_ERR_SHAPE
    assert scan(lib, dst=pool(shape=(2, 4, 128, 96))) == L.LA_ERR_UNSUPPORTED
    assert scan(lib, cu=A + 2) == L.LA_ERR_ALIGN
    assert scan(lib, order=A + 1) == L.LA_ERR_ALIGN
    assert scan(lib, n=9) == L.LA_ERR_SHAPE
    assert scan(lib, rule=4, g=None) == L.LA_ERR_NULL
    assert scan(lib, rule=4, g=A + 8) == L.LA_ERR_ALIGN


def test_chunked_scan_supported_set(lib):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def call(shape=(2, 4, 128, 128), io=1, rule=3):
        dst = pool(shape=shape)
        return lib.la_state_scan_chunked(rule, None, None, ctypes.byref(dst), None, 2, P(A), 10, None, P(A), P(A),
                                         P(A), io, P(A), P(A), 1.0, P(A), P(A), None)
    assert call(rule=4) == L.LA_ERR_UNSUPPORTED  # kda: the two-launch form only
    assert call(shape=(2, 4, 64, 64)) == L.LA_ERR_UNSUPPORTED
    assert call(shape=(2, 4, 128, 64)) == L.LA_ERR_UNSUPPORTED
    assert call(io=0) == L.LA_ERR_UNSUPPORTED


def test_chunked_workspace_size(lib):
    """The two-launch prefill's workspace: a fixed header plus one tile per (chunk, head),
    chunks counted per sequence (a ragged tail is a whole tile); every tile starts on a
    16-byte boundary, as the bulk copies that read it require."""
    b = L.la_scan_chunked_workspace_bytes
    head = b(0, 1, 1) - (b(0, 1, 2) - b(0, 1, 1))  # size = head + tiles * H * tile
    tile = (b(0, 1, 2) - b(0, 1, 1)) // 2               # (0 tokens, 1 sequence: 2 tiles per head)
    assert head >= 16 and head % 16 == 0 and tile % 16 == 0 and tile > 2 * 64 * 64 * 2
    for T, n, H in [(1, 1, 1), (64, 1, 32), (65, 2, 4), (172058, 32, 32), (1 << 20, 1, 32)]:
        tiles = (T + 63) // 64 + n + 1
        assert b(T, n, H) == head + tiles * H * tile
    assert b(10, 0, 4) == head + 2 * 4 * tile and b(-1, 1, 1) == 0


def test_chunked_workspace_size_per_rule(lib):
    """The workspace of the two-launch prefill per rule: the delta rules' tiles as above,
    kda's 65 KB tiles (the decay-scaled Q, K twice, K, P, Tw and Gamma_C of one chunk and
    head, 1024 bytes apart), none for the linear and gated rules or an unknown rule."""
    b = L.la_scan_chunked_workspace_bytes
    r = L.la_scan_chunked_workspace_bytes_rule
    for T, n, H in [(1, 1, 1), (65, 2, 4), (172058, 32, 32)]:
        assert r("delta", T, n, H) == r("gated_delta", T, n, H) == b(T, n, H)
        assert r("linear", T, n, H) == r("gated", T, n, H) == 0
        assert r(7, T, n, H) == 0 and r(-1, T, n, H) == 0
    head = r("kda", 0, 1, 1) - (r("kda", 0, 1, 2) - r("kda", 0, 1, 1))
    tile = (r("kda", 0, 1, 2) - r("kda", 0, 1, 1)) // 2
    assert head >= 16 and head % 16 == 0 and tile % 1024 == 0
    assert tile >= 3 * 64 * 128 * 2 + 2 * 64 * 64 * 2 + 128 * 4
    for T, n, H in [(1, 1, 1), (64, 1, 32), (65, 2, 4), (172058, 32, 32)]:
        assert r("kda", T, n, H) == head + ((T + 63) // 64 + n + 1) * H * tile
    assert r("kda", -1, 1, 1) == 0


def test_chunked_kda_host_errors(lib):
    """kda on the chunked path: the two-launch entry point requires a workspace of kda's
    size; the one-launch and checkpointed chunked entry points have no kda form."""
    dst = pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    need = L.la_scan_chunked_workspace_bytes_rule("kda", 10, 2, 4)

    def ws_call(ws, nbytes):
        return lib.la_state_scan_chunked_ws(4, None, None, ctypes.byref(dst), None, 2, P(A), 10, None, P(A), P(A),
                                            P(A), 1, P(A), P(A), 1.0, P(A), P(ws), nbytes, P(A), None)
    assert ws_call(None, 0) == L.LA_ERR_NULL
    assert ws_call(A, need - 1) == L.LA_ERR_SHAPE
    assert ws_call(A, L.la_scan_chunked_workspace_bytes(10, 2, 4)) == L.LA_ERR_SHAPE  # the delta size is too small
    assert lib.la_state_scan_chunked(4, None, None, ctypes.byref(dst), None, 2, P(A), 10, None, P(A), P(A), P(A), 1,
                                     P(A), P(A), 1.0, P(A), P(A), None) == L.LA_ERR_UNSUPPORTED
    ck = (ctypes.c_int32 * 3)(0, 0, 0)
    assert lib.la_state_scan_chunked_checkpointed(4, None, None, ctypes.byref(dst), None, 2, P(A), 10, None, P(A),
                                                  P(A), P(A), 1, P(A), P(A), 1.0, P(A), 64, ck, ck, P(A),
                                                  None) == L.LA_ERR_UNSUPPORTED


def test_chunked_conv_host_errors(lib):
    """The convolution on the chunked path: a conv description is required, kda and FP32 io
    are not supported there, and a bad width is refused before any launch."""
    dst = pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    conv = L.la_conv(4, 1, 1, A, A, A, A, A)

    def call(rule=3, io=1, c=conv):
        return lib.la_state_scan_chunked_conv(rule, None, None, ctypes.byref(dst), None, 2, P(A), 10, None,
                                              None if c is None else ctypes.byref(c), P(A), P(A), P(A), io, P(A),
                                              P(A), 1.0, P(A), P(A), None)
    assert call(c=None) == L.LA_ERR_NULL
    assert call(rule=4) == L.LA_ERR_UNSUPPORTED
    assert call(io=0) == L.LA_ERR_UNSUPPORTED
    assert call(c=L.la_conv(5, 1, 1, A, A, A, A, A)) == L.LA_ERR_UNSUPPORTED
    # the two-launch form: a workspace of the convolved q, k, v (header + 3 T H_v 128 BF16)
    need = L.la_scan_chunked_conv_workspace_bytes(10, 4)
    assert need == L.la_scan_chunked_conv_workspace_bytes(0, 4) + 3 * 10 * 4 * 128 * 2
    assert L.la_scan_chunked_conv_workspace_bytes(-1, 4) == 0

    def ws_call(ws, nbytes, rule=3):
        return lib.la_state_scan_chunked_conv_ws(rule, None, None, ctypes.byref(dst), None, 2, P(A), 10, None,
                                                 ctypes.byref(conv), P(A), P(A), P(A), 1, P(A), P(A), 1.0, P(A),
                                                 P(ws), nbytes, P(A), None)
    assert ws_call(None, 0) == L.LA_ERR_NULL
    assert ws_call(A, need - 16) == L.LA_ERR_SHAPE
    assert ws_call(A + 8, need) == L.LA_ERR_ALIGN
    assert ws_call(A, need, rule=4) == L.LA_ERR_UNSUPPORTED


def test_chunked_qgroups_host_errors(lib):
    """The chunked prefill in the query-group direction: the one-launch form of the
    scalar-gate rules at d_k = d_v = 128 with BF16 io; the group as for the token-serial
    scan (a multiple of H_v, at most 8 queries per state head, n_qk_heads == n_v_heads)."""
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def call(rule=3, nq=16, io=1, shape=(4, 4, 128, 128), dst=None):
        d = dst or pool(shape=shape)
        return lib.la_state_scan_chunked_qgroups(rule, None, None, ctypes.byref(d), None, 2, P(A), 10, None, nq,
                                                 P(A), P(A), P(A), io, P(A), P(A), 1.0, P(A), P(A), None)
    assert call(nq=0) == L.LA_ERR_SHAPE
    assert call(nq=6) == L.LA_ERR_SHAPE                                  # not a multiple of H_v
    assert call(shape=(2, 4, 128, 128)) == L.LA_ERR_SHAPE                # n_qk_heads != n_v_heads
    assert call(nq=36) == L.LA_ERR_UNSUPPORTED                           # 9 queries per state head
    assert call(rule=4) == L.LA_ERR_UNSUPPORTED                          # kda
    assert call(io=0) == L.LA_ERR_UNSUPPORTED                            # FP32 io
    assert call(shape=(4, 4, 64, 64)) == L.LA_ERR_UNSUPPORTED
    assert call(dst=pool(shape=(4, 4, 128, 128), data=0)) == L.LA_ERR_NULL


def test_noalloc_lookup_failure_is_an_error(lib):
    """The no-alloc prefill looks up the address of the library's own workspace before
    anything else; where that lookup fails (here: no CUDA device at all), the call reports
    LA_ERR_CUDA with the runtime's error code -- never LA_OK with nothing launched."""
    if torch.cuda.is_available():
        pytest.skip("the lookup succeeds on a GPU host")
    dst = pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    st = lib.la_state_scan_chunked_noalloc(3, None, None, ctypes.byref(dst), None, 2, P(A), 10, None, P(A), P(A),
                                           P(A), 1, P(A), P(A), 1.0, P(A), P(A), None)
    assert st == L.LA_ERR_CUDA
    assert lib.la_last_cuda_error() != 0
    # a second call fails the same way (nothing half-initialised is cached)
    assert lib.la_state_scan_chunked_noalloc(3, None, None, ctypes.byref(dst), None, 2, P(A), 10, None, P(A), P(A),
                                             P(A), 1, P(A), P(A), 1.0, P(A), P(A), None) == L.LA_ERR_CUDA


def test_chunked_ws_linear_and_gated_ignore_the_workspace(lib):
    """The linear and gated rules have no intra-chunk inverse: the two-launch entry point
    neither needs nor checks a workspace for them (a NULL workspace of size 0 passes the
    host checks, which end here at an unsupported io type before any launch), while the
    delta rules still require one."""
    dst = pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def call(rule, ws, nbytes, io=0):
        return lib.la_state_scan_chunked_ws(rule, None, None, ctypes.byref(dst), None, 2, P(A), 10, None, P(A),
                                            P(A), P(A), io, P(A), P(A), 1.0, P(A), P(ws), nbytes, P(A), None)
    assert call(0, None, 0) == L.LA_ERR_UNSUPPORTED       # linear: no workspace needed
    assert call(1, None, 0) == L.LA_ERR_UNSUPPORTED       # gated
    assert call(3, None, 0) == L.LA_ERR_NULL              # gated_delta: required
    assert call(3, A, 16, io=1) == L.LA_ERR_SHAPE         # and sized


def test_failure_hooks_are_plain_host_calls(lib):
    """The failure-path test hooks only set host state (no device work): callable here."""
    L.la_debug_set_wait_limit_us(1500)
    L.la_debug_withhold_step_tile(3)
    L.la_debug_withhold_step_tile(-1)
    L.la_debug_set_wait_limit_us(0)


def test_chunked_checkpointed_host_errors(lib):
    """The chunked checkpointed prefill: checkpoints on the 64-token chunk grid only, and the
    checkpointed scan's own host checks."""
    dst = pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def call(every=128, ccu=A, cs=A, n=2, rule=3):
        return lib.la_state_scan_chunked_checkpointed(rule, None, None, ctypes.byref(dst), None, n, P(A), 10, None,
                                                      P(A), P(A), P(A), 1, P(A), P(A), 1.0, P(A), every, P(ccu),
                                                      P(cs), P(A), None)
    assert call(every=0) == L.LA_ERR_SHAPE
    assert call(ccu=None) == L.LA_ERR_NULL
    assert call(cs=A + 2) == L.LA_ERR_ALIGN
    assert call(every=100) == L.LA_ERR_UNSUPPORTED
    assert call(rule=4) == L.LA_ERR_UNSUPPORTED  # kda
    assert call(n=0) == L.LA_OK


def test_checkpointed_scan_host_errors(lib):
    dst = pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def call(every=8, ccu=A, cs=A, n=2):
        return lib.la_state_scan_checkpointed(3, None, None, ctypes.byref(dst), None, n, P(A), 10, None, P(A), P(A),
                                              P(A), 1, P(A), P(A), 1.0, P(A), every, P(ccu), P(cs), P(A), None)
    assert call(every=0) == L.LA_ERR_SHAPE
    assert call(ccu=None) == L.LA_ERR_NULL
    assert call(cs=A + 2) == L.LA_ERR_ALIGN
    assert call(n=0) == L.LA_OK


def test_pool_host_errors(lib):
    p = pool()
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    assert lib.la_state_pool_copy(ctypes.byref(p), 2, P(A), None, P(A), None) == L.LA_ERR_NULL
    assert lib.la_state_pool_copy(ctypes.byref(p), 0, None, None, P(A), None) == L.LA_OK
    assert lib.la_state_pool_gather(ctypes.byref(p), 2, P(A), P(A + 8), P(A), None) == L.LA_ERR_ALIGN
    assert lib.la_state_pool_scatter(ctypes.byref(p), -1, P(A), P(A), P(A), None) == L.LA_ERR_SHAPE
    assert lib.la_state_pool_zero(ctypes.byref(p), 1, P(A), None, None) == L.LA_ERR_NULL
    bad = pool(dtype=9)
    assert lib.la_state_pool_zero(ctypes.byref(bad), 1, P(A), P(A), None) == L.LA_ERR_UNSUPPORTED


def test_q8_pools_host_side(lib):
    """q8 pools: slot sizes of the layout (9.875 bits per value at 1/8 BF16 channels) and
    the host-side errors of the entry points that take or refuse them."""
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def q8(shape=(2, 4, 128, 128), n_hp=16, mask=A, data=A, n=8):
        return L.la_pool(ctypes.c_void_p(data), L.LA_Q8, n, L.la_shape(*shape), n_hp, P(mask))
    assert lib.la_pool_slot_bytes(ctypes.byref(q8())) == 4 * (112 * 128 + 112 * 4 * 4 + 16 * 128 * 2)
    assert lib.la_pool_slot_bytes(ctypes.byref(q8())) * 8 / (4 * 128 * 128) == 9.875
    assert lib.la_pool_slot_bytes(ctypes.byref(q8(shape=(2, 4, 128, 64), n_hp=0))) == 4 * (128 * 64 + 128 * 2 * 4)
    assert lib.la_pool_slot_bytes(ctypes.byref(pool(dtype=1))) == 4 * 128 * 128 * 2
    assert lib.la_pool_slot_bytes(ctypes.byref(q8(shape=(2, 4, 16, 16)))) == 0     # no q8 tile of 16 x 16
    assert lib.la_pool_slot_bytes(ctypes.byref(q8(n_hp=3))) == 0                   # odd
    assert lib.la_pool_slot_bytes(ctypes.byref(q8(n_hp=34))) == 0                  # above d_k / 4
    assert L.q8_tile_bytes(128, 128, 16) * 4 == lib.la_pool_slot_bytes(ctypes.byref(q8()))
    assert step(lib, src=q8(mask=None), dst=q8(mask=None)) == L.LA_ERR_NULL
    assert step(lib, src=q8(mask=A + 2), dst=q8(mask=A + 2)) == L.LA_ERR_ALIGN
    assert step(lib, src=q8(shape=(2, 4, 16, 16)), dst=q8(shape=(2, 4, 16, 16))) == L.LA_ERR_UNSUPPORTED
    assert step(lib, src=q8(n_hp=3), dst=q8(n_hp=3)) == L.LA_ERR_SHAPE
    assert step(lib, src=q8(), dst=pool(dtype=1)) == L.LA_ERR_UNSUPPORTED        # formats differ
    assert step(lib, src=q8(n_hp=16), dst=q8(n_hp=8)) == L.LA_ERR_SHAPE          # tile sizes differ
    assert lib.la_state_step_qgroups(3, ctypes.byref(q8(shape=(4, 4, 128, 128))), None,
                                     ctypes.byref(q8(shape=(4, 4, 128, 128))), None, 2, 8, P(A), P(A), P(A), 1,
                                     P(A), P(A), 1.0, P(A), P(A), None) == L.LA_ERR_UNSUPPORTED
    # the chunked path takes q8 pools in its one-launch form only (not through a workspace)
    assert lib.la_state_scan_chunked_ws(3, None, None, ctypes.byref(q8()), None, 2, P(A), 10, None, P(A), P(A),
                                        P(A), 1, P(A), P(A), 1.0, P(A), P(A), 1 << 30, P(A),
                                        None) == L.LA_ERR_UNSUPPORTED
    assert lib.la_state_scan_chunked_ws(4, None, None, ctypes.byref(q8()), None, 2, P(A), 10, None, P(A), P(A),
                                        P(A), 1, P(A), P(A), 1.0, P(A), P(A), 1 << 30, P(A),
                                        None) == L.LA_ERR_UNSUPPORTED
    assert lib.la_state_pool_encode(ctypes.byref(pool(dtype=1)), 2, P(A), P(A), P(A), None) == L.LA_ERR_UNSUPPORTED
    assert lib.la_state_pool_decode(ctypes.byref(q8()), 2, None, P(A), P(A), None) == L.LA_ERR_NULL
    assert lib.la_state_pool_decode(ctypes.byref(q8()), 2, P(A), P(A + 4), P(A), None) == L.LA_ERR_ALIGN
    assert lib.la_state_pool_encode(ctypes.byref(q8()), 0, None, None, P(A), None) == L.LA_OK


def test_conv_step_host_errors(lib):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def call(width=4, wq=A, hist=A, src=None, B=4):
        conv = L.la_conv(width, 1, 1, P(wq), P(A), P(A), P(hist), P(hist))
        src = src or pool()
        return lib.la_state_step_conv(3, ctypes.byref(src), None, ctypes.byref(src), None, B, ctypes.byref(conv),
                                      P(A), P(A), P(A), 1, P(A), P(A), 1.0, P(A), P(A), None)
    assert call(width=1) == L.LA_ERR_UNSUPPORTED
    assert call(width=5) == L.LA_ERR_UNSUPPORTED
    assert call(wq=None) == L.LA_ERR_NULL
    assert call(hist=A + 8) == L.LA_ERR_ALIGN
    assert call(B=0) == L.LA_OK
    assert lib.la_state_step_conv(3, ctypes.byref(pool()), None, ctypes.byref(pool()), None, 4, None, P(A), P(A),
                                  P(A), 1, P(A), P(A), 1.0, P(A), P(A), None) == L.LA_ERR_NULL
    q8 = L.la_pool(ctypes.c_void_p(A), L.LA_Q8, 8, L.la_shape(2, 4, 128, 128), 16, P(A))
    assert call(src=q8) == L.LA_ERR_UNSUPPORTED


def test_conv_scan_host_errors(lib):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731

    def call(width=4, rs=None, hist_src=A, dst=None):
        conv = L.la_conv(width, 1, 1, P(A), P(A), P(A), P(hist_src), P(A))
        dst = dst or pool()
        return lib.la_state_scan_conv(3, ctypes.byref(pool()), P(rs), ctypes.byref(dst), None, 2, P(A), 10, None,
                                      ctypes.byref(conv), P(A), P(A), P(A), 1, P(A), P(A), 1.0, P(A), P(A), None)
    assert call(width=9) == L.LA_ERR_UNSUPPORTED
    assert call(rs=A, hist_src=None) == L.LA_ERR_NULL
    assert call(hist_src=A + 4) == L.LA_ERR_ALIGN
    q8 = L.la_pool(ctypes.c_void_p(A), L.LA_Q8, 8, L.la_shape(2, 4, 128, 128), 16, P(A))
    assert call(dst=q8) == L.LA_ERR_UNSUPPORTED
    assert lib.la_state_scan_conv(3, None, None, ctypes.byref(pool()), None, 2, P(A), 10, None, None, P(A), P(A),
                                  P(A), 1, P(A), P(A), 1.0, P(A), P(A), None) == L.LA_ERR_NULL


def test_check_slots(lib):
    t = lambda x: torch.tensor(x, dtype=torch.int32)  # noqa: E731
    assert L.la_state_check_slots(t([0, 1, 2]), t([0, 1, 2]), 4) == L.LA_OK
    assert L.la_state_check_slots(t([5, 5, 6]), t([0, 1, 2]), 8) == L.LA_OK          # shared checkpoint reads
    assert L.la_state_check_slots(t([0, 1]), t([2, 2]), 4) == L.LA_ERR_ALIAS          # duplicate write
    assert L.la_state_check_slots(t([0, 1]), t([1, 3]), 4) == L.LA_ERR_ALIAS          # reads a slot another writes
    assert L.la_state_check_slots(t([0, 4]), t([0, 1]), 4) == L.LA_ERR_SHAPE
    assert L.la_state_check_slots(None, None, 4, B=3) == L.LA_OK


def test_status_strings(lib):
    for code, name in L.STATUS.items():
        assert lib.la_status_str(code).decode().startswith(name)

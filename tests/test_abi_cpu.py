"""C ABI checks that need no GPU: the library loads, exports every symbol
the header declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

from tree_masked_verification_b200 import build, hta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "longspec_hta.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return hta.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LONGSPEC_HTA_API\s+[\w\s\*]+?\b(longspec_hta_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_symbols()
    assert "longspec_hta_verify" in names and len(names) >= 10


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", hta.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\b(longspec_hta_\w+)\b", out))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    assert sorted(exported) == sorted(set(hta.EXPORTED)), "binding list out of date"


def test_header_is_plain_c():
    subprocess.run(["gcc", "-fsyntax-only", "-std=c99", "-x", "c", "-I/usr/local/cuda/include",
                    HEADER], check=True)


def test_abi_version_and_strerror(lib):
    assert lib.longspec_hta_abi_version() == 1
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -16, -17, -18, -19, 12345):
        assert lib.longspec_hta_strerror(code)


def _dims(**kw):
    d = dict(B=1, Hq=32, Hkv=8, D=128, T=68, L_cap=32768, scale=0.0)
    d.update(kw)
    return hta.Dims(d["B"], d["Hq"], d["Hkv"], d["D"], d["T"], d["L_cap"], d["scale"])


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=30), hta.ERR_INVALID_DIMS),
    (dict(D=96), hta.ERR_UNSUPPORTED_D),
    (dict(T=257), hta.ERR_T_TOO_LARGE),
    (dict(T=0), hta.ERR_INVALID_DIMS),
    (dict(scale=-1.0), hta.ERR_INVALID_DIMS),
    (dict(L_cap=-1), hta.ERR_INVALID_DIMS),
    (dict(B=1 << 20, Hkv=8, Hq=8), hta.ERR_INVALID_DIMS),
])
def test_verify_rejects_bad_dims_on_host(lib, kw, code):
    d = _dims(**kw)
    rc = lib.longspec_hta_verify(ctypes.byref(d), *([16] * 9), 16, 1 << 30, None)
    assert rc == code


def test_verify_rejects_null_and_misaligned_on_host(lib):
    d = _dims()
    ptrs = [4096 * (i + 1) for i in range(9)]
    for i in range(9):
        bad = list(ptrs)
        bad[i] = 0
        assert lib.longspec_hta_verify(ctypes.byref(d), *bad, 4096 * 20, 1 << 30, None) == hta.ERR_NULL_POINTER
        bad[i] = ptrs[i] + 8
        assert lib.longspec_hta_verify(ctypes.byref(d), *bad, 4096 * 20, 1 << 30, None) == hta.ERR_MISALIGNED


def test_verify_ex_rejects_bad_options(lib):
    d = _dims()
    for opts in (hta.Options(-1, 0, None, None), hta.Options(0, 7, None, None)):
        rc = lib.longspec_hta_verify_ex(ctypes.byref(d), *[4096 * (i + 1) for i in range(9)],
                                        4096 * 20, 1 << 30, ctypes.byref(opts), None)
        assert rc == hta.ERR_INVALID_OPTION


@pytest.mark.parametrize("L_cap,req,S,chunk", [
    (32768, 6, 6, 43 * 128),
    (32768, 1, 1, 32768),
    (256, 6, 2, 128),
    (1000, 3, 3, 384),
    (0, 4, 1, 128),
    (262144, 64, 64, 4096),
    (262144, 100, 64, 4096),
])
def test_chunking_arithmetic(lib, L_cap, req, S, chunk):
    got = hta.chunking(_dims(L_cap=L_cap), req)
    assert got == (S, chunk)
    # chunks cover [0, L_cap) exactly once
    assert (S - 1) * chunk < max(L_cap, 1) <= S * chunk


def test_workspace_bytes_formula(lib):
    d = _dims()
    n = hta.workspace_bytes(d, 6)
    rows = 1 * 32 * 68
    assert n >= 256 + rows * 6 * 129 * 4
    assert n - (256 + rows * 6 * 129 * 4) < 1024


def test_prefix_attention_rejects_bad_arguments_on_host(lib):
    """Prefix-only attention: q, k_prefix, v_prefix, prefix_len, out, lse and
    the workspace are checked (NULL, 16-byte alignment, dims, options)
    before any device work."""
    d = _dims()
    ptrs = [4096 * (i + 1) for i in range(6)]
    ws = 4096 * 20
    for i in range(6):
        bad = list(ptrs)
        bad[i] = 0
        assert lib.longspec_hta_prefix_attention(ctypes.byref(d), *bad, ws, 1 << 30, None,
                                                 None) == hta.ERR_NULL_POINTER
        bad[i] = ptrs[i] + 8
        assert lib.longspec_hta_prefix_attention(ctypes.byref(d), *bad, ws, 1 << 30, None,
                                                 None) == hta.ERR_MISALIGNED
    assert lib.longspec_hta_prefix_attention(ctypes.byref(d), *ptrs, 0, 1 << 30, None,
                                             None) == hta.ERR_NULL_POINTER
    bad_dims = _dims(D=96)
    assert lib.longspec_hta_prefix_attention(ctypes.byref(bad_dims), *ptrs, ws, 1 << 30, None,
                                             None) != hta.OK
    opts = hta.Options(-1, 0, None, None)
    assert lib.longspec_hta_prefix_attention(ctypes.byref(d), *ptrs, ws, 1 << 30, ctypes.byref(opts),
                                             None) == hta.ERR_INVALID_OPTION


def test_paged_calls_reject_bad_arguments_on_host(lib):
    """Paged cache descriptor checks: NULL descriptor or table, block sizes
    outside {16, 32, 64, 128}, a table too short for L_cap, and the SIMT
    prefix kernel (which reads contiguous K/V only)."""
    d = _dims(L_cap=1024)
    base = dict(k_cache=4096 * 30, v_cache=4096 * 31, block_table=4096 * 32, num_blocks=64,
                block_size=16, max_blocks=64)

    def call(kv, opts=None):
        ptrs = [4096 * (i + 1) for i in range(6)]   # q, prefix_len, k_tree, v_tree, parent, out
        return lib.longspec_hta_verify_paged(ctypes.byref(d), ptrs[0],
                                             None if kv is None else ctypes.byref(kv), *ptrs[1:],
                                             4096 * 20, 4096 * 21, 1 << 30,
                                             None if opts is None else ctypes.byref(opts), None)

    assert call(None) == hta.ERR_NULL_POINTER
    assert call(hta.PagedKV(**{**base, "block_table": 0})) == hta.ERR_NULL_POINTER
    assert call(hta.PagedKV(**{**base, "k_cache": 0})) == hta.ERR_NULL_POINTER
    assert call(hta.PagedKV(**{**base, "v_cache": base["v_cache"] + 8})) == hta.ERR_MISALIGNED
    for bs in (8, 24, 256):
        assert call(hta.PagedKV(**{**base, "block_size": bs})) == hta.ERR_INVALID_DIMS
    assert call(hta.PagedKV(**{**base, "max_blocks": 63})) == hta.ERR_INVALID_DIMS
    assert call(hta.PagedKV(**{**base, "num_blocks": 0})) == hta.ERR_INVALID_DIMS
    simt = hta.Options(0, hta.PREFIX_SIMT, None, None)
    assert call(hta.PagedKV(**base), simt) == hta.ERR_INVALID_OPTION


def test_accept_rejects_bad_arguments_on_host(lib):
    """Greedy acceptance: workspace size formula (status word + 32 slice
    partials of 8 bytes per logits row), dims, NULL, alignment and
    workspace checks, all taken before any device call."""
    B, T, V = 4, 68, 128256
    need = lib.longspec_hta_accept_workspace_bytes(B, T, V)
    assert need == 256 + B * (T + 1) * 32 * 8
    assert lib.longspec_hta_accept_workspace_bytes(0, T, V) == 0
    assert lib.longspec_hta_accept_workspace_bytes(B, 257, V) == 0

    def call(B=B, T=T, V=V, ptrs=None, ws_bytes=need):
        p = ptrs or [4096 * (i + 1) for i in range(7)]   # logits, tok, parent, len, path, bonus, ws
        return lib.longspec_hta_accept_greedy(B, T, V, *p, ws_bytes, None)

    assert call(B=0) == hta.ERR_INVALID_DIMS
    assert call(V=0) == hta.ERR_INVALID_DIMS
    assert call(B=1000, T=100) == hta.ERR_INVALID_DIMS     # more than 65535 logits rows
    assert call(T=257) == hta.ERR_T_TOO_LARGE
    for k in range(7):
        p = [4096 * (i + 1) for i in range(7)]
        p[k] = None
        assert call(ptrs=p) == hta.ERR_NULL_POINTER
    p = [4096 * (i + 1) for i in range(7)]
    p[0] += 8                                             # logits need 16 bytes
    assert call(ptrs=p) == hta.ERR_MISALIGNED
    p = [4096 * (i + 1) for i in range(7)]
    p[3] += 2                                             # int32 arrays need 4 bytes
    assert call(ptrs=p) == hta.ERR_MISALIGNED
    assert call(ws_bytes=need - 1) == hta.ERR_WORKSPACE_TOO_SMALL


def test_commit_rejects_bad_arguments_on_host(lib):
    """KV commit: dims, NULL, alignment, paged descriptor and workspace
    checks, all taken before any device call."""
    d = _dims(L_cap=1024)
    good = [4096 * (i + 1) for i in range(7)]   # k_prefix, v_prefix, prefix_len, k_tree, v_tree, len, path

    def call(p=None, ws=4096 * 20, ws_bytes=256, dims=d):
        p = good if p is None else p
        return lib.longspec_hta_commit(ctypes.byref(dims), *p, ws, ws_bytes, None)

    for k in range(7):
        p = list(good)
        p[k] = None
        assert call(p) == hta.ERR_NULL_POINTER
    p = list(good)
    p[0] += 8                                   # the cache needs 16 bytes
    assert call(p) == hta.ERR_MISALIGNED
    p = list(good)
    p[2] += 2                                   # int32 arrays need 4 bytes
    assert call(p) == hta.ERR_MISALIGNED
    assert call(ws=None) == hta.ERR_NULL_POINTER
    assert call(ws_bytes=255) == hta.ERR_WORKSPACE_TOO_SMALL
    assert call(dims=_dims(D=96)) == hta.ERR_UNSUPPORTED_D
    assert call(dims=_dims(T=300)) == hta.ERR_T_TOO_LARGE

    base = dict(k_cache=4096 * 30, v_cache=4096 * 31, block_table=4096 * 32, num_blocks=64,
                block_size=16, max_blocks=64)

    def paged(kv):
        return lib.longspec_hta_commit_paged(ctypes.byref(d), None if kv is None else ctypes.byref(kv),
                                             *good[2:], 4096 * 20, 256, None)

    assert paged(None) == hta.ERR_NULL_POINTER
    assert paged(hta.PagedKV(**{**base, "block_table": 0})) == hta.ERR_NULL_POINTER
    assert paged(hta.PagedKV(**{**base, "block_size": 24})) == hta.ERR_INVALID_DIMS
    assert paged(hta.PagedKV(**{**base, "max_blocks": 63})) == hta.ERR_INVALID_DIMS


def _ws_bytes(d, S):
    """Workspace bytes of S splits, written out from the layout the header
    documents: 256-byte status region, O partials fp32 [rows][S][D], lse
    partials fp32 [rows][S], each 256-byte aligned."""
    a = lambda x: (x + 255) // 256 * 256
    rows = d.B * d.Hq * d.T
    return a(a(256 + rows * S * d.D * 4) + rows * S * 4)


NOALLOC_SCRATCH = 16 << 20


def test_noalloc_chunking_keeps_the_usual_split_when_it_fits(lib):
    # Llama-3-8B shapes on 148 SMs: 6 splits of 43 tiles, 6.7 MB of partials
    d = _dims()
    assert hta.noalloc_chunking(d, 148) == (6, 43 * 128)
    assert _ws_bytes(d, 6) <= NOALLOC_SCRATCH


def test_noalloc_chunking_lowers_the_split_until_it_fits(lib):
    # on a (hypothetical) 1024-SM part the usual choice would be 42 splits,
    # 47 MB of partials: the call lowers it to the largest count that fits
    d = _dims()
    S, chunk = hta.noalloc_chunking(d, 1024)
    assert _ws_bytes(d, S) <= NOALLOC_SCRATCH
    tiles = 32768 // 128
    assert (S - 1) * chunk < 32768 <= S * chunk
    # every larger split count the chunking can produce does not fit
    larger = {-(-tiles // -(-tiles // s)) for s in range(S + 1, 65)}
    assert all(_ws_bytes(d, s) > NOALLOC_SCRATCH for s in larger if s > S)
    assert S >= 10


def test_noalloc_chunking_rejects_what_one_split_cannot_hold(lib):
    # B*Hq*T*(D+1)*4 bytes of partials with one split: 67 MB > 16 MiB
    d = _dims(B=8, Hq=64, T=256, L_cap=1024)
    S, C = ctypes.c_int(0), ctypes.c_int(0)
    rc = lib.longspec_hta_noalloc_chunking(ctypes.byref(d), 148, ctypes.byref(S), ctypes.byref(C))
    assert rc == hta.ERR_WORKSPACE_TOO_SMALL
    assert lib.longspec_hta_noalloc_chunking(ctypes.byref(_dims()), 0, None, None) == hta.ERR_INVALID_OPTION


def test_build_info_reports_the_tuning_knobs(lib):
    """The in-tree build carries the default knobs of csrc/hta_kernels.h."""
    lib.longspec_hta_build_info.restype = ctypes.c_char_p
    text = lib.longspec_hta_build_info().decode()
    assert dict(kv.split("=") for kv in text.split()) == {"kv_stages_d128": "3", "exp2_poly_every": "4"}

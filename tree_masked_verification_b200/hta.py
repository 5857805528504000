"""ctypes binding of liblongspec_hta.so (Hybrid Tree Attention on B200).

Argument marshalling only: every step of the verification attention runs in
the library's CUDA kernels.  Tensors are torch tensors on the current CUDA
device; the library launches on torch's current stream unless a stream is
given.  The library must have been built (``tree_masked_verification_b200.build``):
there is no fallback of any kind, and a missing library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

# The in-tree build; LONGSPEC_HTA_LIB names another build of the same
# library instead (a build with other tuning knobs, for A/B timing).
_LIB_PATH = os.environ.get("LONGSPEC_HTA_LIB") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "liblongspec_hta.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_INVALID_DIMS = -1
ERR_NULL_POINTER = -2
ERR_MISALIGNED = -3
ERR_T_TOO_LARGE = -4
ERR_UNSUPPORTED_D = -5
ERR_WORKSPACE_TOO_SMALL = -6
ERR_CUDA = -7
ERR_UNSUPPORTED_DEVICE = -8
ERR_INVALID_OPTION = -9
ERR_BAD_PARENT = -16
ERR_PREFIX_LEN_RANGE = -17
ERR_PIPELINE_TIMEOUT = -18
ERR_INTERNAL = -19
ERR_BAD_BLOCK = -20
ERR_BAD_PATH = -21

PREFIX_TCGEN05 = 0
PREFIX_SIMT = 1
T_MAX = 256

EXPORTED = [
    "longspec_hta_abi_version", "longspec_hta_build_info", "longspec_hta_strerror", "longspec_hta_default_splits",
    "longspec_hta_chunking",
    "longspec_hta_workspace_bytes", "longspec_hta_workspace_init", "longspec_hta_verify",
    "longspec_hta_verify_ex", "longspec_hta_host_arena_bytes", "longspec_hta_verify_host",
    "longspec_hta_tree_mask", "longspec_hta_tree_partial", "longspec_hta_prefix_partial",
    "longspec_hta_get_status", "longspec_hta_verify_noalloc", "longspec_hta_noalloc_chunking",
    "longspec_hta_selftest_wait_timeout", "longspec_hta_prefix_attention",
    "longspec_hta_verify_paged", "longspec_hta_prefix_attention_paged",
    "longspec_hta_accept_workspace_bytes", "longspec_hta_accept_greedy",
    "longspec_hta_commit", "longspec_hta_commit_paged", "longspec_hta_window_verify",
    "longspec_hta_window_workspace_bytes",
]


class HtaError(RuntimeError):
    def __init__(self, code: int):
        msg = load().longspec_hta_strerror(code).decode()
        super().__init__(f"longspec_hta error {code}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("T", ctypes.c_int), ("L_cap", ctypes.c_int),
                ("scale", ctypes.c_float)]


class Options(ctypes.Structure):
    _fields_ = [("num_splits", ctypes.c_int), ("prefix_kernel", ctypes.c_int),
                ("prefix_begin", ctypes.c_void_p), ("prefix_end", ctypes.c_void_p)]


class PagedKV(ctypes.Structure):
    """longspec_hta_paged_kv: caches [num_blocks][Hkv][block_size][D] bf16,
    block_table [B][max_blocks] int32 (device pointers)."""
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("num_blocks", ctypes.c_int),
                ("block_size", ctypes.c_int), ("max_blocks", ctypes.c_int)]


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load the library (once).  Raises if it was not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m tree_masked_verification_b200.build` (no fallback exists)")
            lib = ctypes.CDLL(_LIB_PATH)
            vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            pd = ctypes.POINTER(Dims)
            lib.longspec_hta_abi_version.restype = ci
            lib.longspec_hta_build_info.restype = ctypes.c_char_p
            lib.longspec_hta_strerror.argtypes = [ci]
            lib.longspec_hta_strerror.restype = ctypes.c_char_p
            lib.longspec_hta_default_splits.argtypes = [pd]
            lib.longspec_hta_workspace_bytes.argtypes = [pd, ci]
            lib.longspec_hta_workspace_bytes.restype = sz
            lib.longspec_hta_workspace_init.argtypes = [vp, sz, vp]
            lib.longspec_hta_verify.argtypes = [pd] + [vp] * 9 + [vp, sz, vp]
            lib.longspec_hta_verify_ex.argtypes = [pd] + [vp] * 9 + [vp, sz, ctypes.POINTER(Options), vp]
            lib.longspec_hta_prefix_attention.argtypes = [pd] + [vp] * 6 + [vp, sz, ctypes.POINTER(Options), vp]
            pk = ctypes.POINTER(PagedKV)
            lib.longspec_hta_verify_paged.argtypes = [pd, vp, pk] + [vp] * 6 + [vp, sz, ctypes.POINTER(Options), vp]
            lib.longspec_hta_prefix_attention_paged.argtypes = [pd, vp, pk] + [vp] * 3 + [vp, sz, ctypes.POINTER(Options), vp]
            lib.longspec_hta_host_arena_bytes.argtypes = [pd]
            lib.longspec_hta_host_arena_bytes.restype = sz
            lib.longspec_hta_verify_host.argtypes = [pd] + [vp] * 9 + [vp, sz, vp]
            lib.longspec_hta_tree_mask.argtypes = [vp, ci, ci, vp, vp, sz, vp]
            lib.longspec_hta_tree_partial.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.longspec_hta_prefix_partial.argtypes = [pd, vp, vp, vp, vp, vp, vp, ci, ci,
                                                        ctypes.POINTER(ci), vp, sz, vp]
            lib.longspec_hta_get_status.argtypes = [vp, vp]
            lib.longspec_hta_selftest_wait_timeout.argtypes = [vp, vp]
            lib.longspec_hta_chunking.argtypes = [pd, ci, ctypes.POINTER(ci), ctypes.POINTER(ci)]
            lib.longspec_hta_noalloc_chunking.argtypes = [pd, ci, ctypes.POINTER(ci), ctypes.POINTER(ci)]
            lib.longspec_hta_accept_workspace_bytes.argtypes = [ci, ci, ci]
            lib.longspec_hta_accept_workspace_bytes.restype = sz
            lib.longspec_hta_accept_greedy.argtypes = [ci, ci, ci] + [vp] * 6 + [vp, sz, vp]
            lib.longspec_hta_commit.argtypes = [pd] + [vp] * 7 + [vp, sz, vp]
            lib.longspec_hta_window_verify.argtypes = [pd] + [vp] * 9 + [vp, sz, vp]
            lib.longspec_hta_window_workspace_bytes.argtypes = [pd]
            lib.longspec_hta_window_workspace_bytes.restype = sz
            lib.longspec_hta_commit_paged.argtypes = [pd, pk] + [vp] * 5 + [vp, sz, vp]
            _lib = lib
    return _lib


def _check(rc: int):
    if rc != OK:
        raise HtaError(rc)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def dims_of(q: torch.Tensor, k_prefix: torch.Tensor, scale: float = 0.0) -> Dims:
    B, Hq, T, D = q.shape
    return Dims(B, Hq, k_prefix.shape[1], D, T, k_prefix.shape[2], float(scale))


def _need(t: torch.Tensor, name: str, dtype, device=None):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}")


def default_splits(dims: Dims) -> int:
    rc = load().longspec_hta_default_splits(ctypes.byref(dims))
    if rc < 0:
        raise HtaError(rc)
    return rc


def chunking(dims: Dims, num_splits: int = 0):
    """(S, chunk_keys) the library uses for a requested split count."""
    S, C = ctypes.c_int(0), ctypes.c_int(0)
    _check(load().longspec_hta_chunking(ctypes.byref(dims), int(num_splits), ctypes.byref(S),
                                        ctypes.byref(C)))
    return S.value, C.value


def noalloc_chunking(dims: Dims, num_sms: int):
    """(S, chunk_keys) longspec_hta_verify_noalloc uses on a GPU with
    num_sms SMs (host only)."""
    S, C = ctypes.c_int(0), ctypes.c_int(0)
    _check(load().longspec_hta_noalloc_chunking(ctypes.byref(dims), int(num_sms), ctypes.byref(S),
                                                ctypes.byref(C)))
    return S.value, C.value


def workspace_bytes(dims: Dims, num_splits: int = 0) -> int:
    n = load().longspec_hta_workspace_bytes(ctypes.byref(dims), int(num_splits))
    if n == 0:
        raise HtaError(ERR_INVALID_DIMS)
    return n


def new_workspace(dims: Dims, num_splits: int = 0, device=None) -> torch.Tensor:
    """A zeroed device workspace for verify (status word cleared)."""
    return torch.zeros(workspace_bytes(dims, num_splits), dtype=torch.uint8,
                       device=device or torch.device("cuda"))


def verify(q, k_prefix, v_prefix, prefix_len, k_tree, v_tree, parent, *, out=None,
           lse=None, workspace=None, scale: float = 0.0, num_splits: int = 0,
           prefix_kernel: int = PREFIX_TCGEN05, prefix_events=None, stream=None):
    """Hybrid Tree Attention of one layer.  Returns (out bf16, lse fp32)."""
    dev = q.device
    for t, n in ((q, "q"), (k_prefix, "k_prefix"), (v_prefix, "v_prefix"),
                 (k_tree, "k_tree"), (v_tree, "v_tree")):
        _need(t, n, torch.bfloat16, dev)
    _need(prefix_len, "prefix_len", torch.int32, dev)
    _need(parent, "parent", torch.int32, dev)
    dims = dims_of(q, k_prefix, scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(dims, num_splits, dev)
    opts = Options(int(num_splits), int(prefix_kernel),
                   prefix_events[0].cuda_event if prefix_events else None,
                   prefix_events[1].cuda_event if prefix_events else None)
    rc = load().longspec_hta_verify_ex(
        ctypes.byref(dims), _ptr(q), _ptr(k_prefix), _ptr(v_prefix), _ptr(prefix_len),
        _ptr(k_tree), _ptr(v_tree), _ptr(parent), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.byref(opts), _stream(stream))
    _check(rc)
    return out, lse


def prefix_attention(q, k_prefix, v_prefix, prefix_len, *, out=None, lse=None, workspace=None,
                     scale: float = 0.0, num_splits: int = 0, prefix_kernel: int = PREFIX_TCGEN05,
                     prefix_events=None, stream=None):
    """Attention of q's rows to the prefix alone (no tree keys, no mask):
    the draft model's cross-attention into the target's KV cache.  q is
    [B][Hq][T][D] with T query tokens per head.  Returns (out bf16, lse fp32);
    rows of a sequence with L_b = 0 get out 0 and lse -inf."""
    dev = q.device
    for t, n in ((q, "q"), (k_prefix, "k_prefix"), (v_prefix, "v_prefix")):
        _need(t, n, torch.bfloat16, dev)
    _need(prefix_len, "prefix_len", torch.int32, dev)
    dims = dims_of(q, k_prefix, scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(dims, num_splits, dev)
    opts = Options(int(num_splits), int(prefix_kernel),
                   prefix_events[0].cuda_event if prefix_events else None,
                   prefix_events[1].cuda_event if prefix_events else None)
    rc = load().longspec_hta_prefix_attention(
        ctypes.byref(dims), _ptr(q), _ptr(k_prefix), _ptr(v_prefix), _ptr(prefix_len),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
        ctypes.byref(opts), _stream(stream))
    _check(rc)
    return out, lse


def _paged(k_cache, v_cache, block_table, dev):
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    _need(block_table, "block_table", torch.int32, dev)
    if k_cache.dim() != 4 or k_cache.shape != v_cache.shape or block_table.dim() != 2:
        raise ValueError("k/v_cache must be [num_blocks][Hkv][block_size][D], block_table [B][max_blocks]")
    return PagedKV(_ptr(k_cache), _ptr(v_cache), _ptr(block_table), int(k_cache.shape[0]),
                   int(k_cache.shape[2]), int(block_table.shape[1]))


def _paged_dims(q, k_cache, L_cap, scale):
    B, Hq, T, D = q.shape
    return Dims(B, Hq, int(k_cache.shape[1]), D, T, int(L_cap), float(scale))


def verify_paged(q, k_cache, v_cache, block_table, prefix_len, k_tree, v_tree, parent, *, L_cap,
                 out=None, lse=None, workspace=None, scale: float = 0.0, num_splits: int = 0,
                 prefix_events=None, stream=None):
    """verify() with the prefix K/V in a paged cache: k/v_cache
    [num_blocks][Hkv][block_size][D], block_table [B][max_blocks] (block ids
    of each sequence in key order), L_cap the longest prefix allowed."""
    dev = q.device
    for t, n in ((q, "q"), (k_tree, "k_tree"), (v_tree, "v_tree")):
        _need(t, n, torch.bfloat16, dev)
    _need(prefix_len, "prefix_len", torch.int32, dev)
    _need(parent, "parent", torch.int32, dev)
    kv = _paged(k_cache, v_cache, block_table, dev)
    dims = _paged_dims(q, k_cache, L_cap, scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev) if lse is None else lse
    workspace = new_workspace(dims, num_splits, dev) if workspace is None else workspace
    opts = Options(int(num_splits), PREFIX_TCGEN05,
                   prefix_events[0].cuda_event if prefix_events else None,
                   prefix_events[1].cuda_event if prefix_events else None)
    rc = load().longspec_hta_verify_paged(
        ctypes.byref(dims), _ptr(q), ctypes.byref(kv), _ptr(prefix_len), _ptr(k_tree), _ptr(v_tree),
        _ptr(parent), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.byref(opts), _stream(stream))
    _check(rc)
    return out, lse


def prefix_attention_paged(q, k_cache, v_cache, block_table, prefix_len, *, L_cap, out=None,
                           lse=None, workspace=None, scale: float = 0.0, num_splits: int = 0,
                           prefix_events=None, stream=None):
    """prefix_attention() with the prefix K/V in a paged cache."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(prefix_len, "prefix_len", torch.int32, dev)
    kv = _paged(k_cache, v_cache, block_table, dev)
    dims = _paged_dims(q, k_cache, L_cap, scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev) if lse is None else lse
    workspace = new_workspace(dims, num_splits, dev) if workspace is None else workspace
    opts = Options(int(num_splits), PREFIX_TCGEN05,
                   prefix_events[0].cuda_event if prefix_events else None,
                   prefix_events[1].cuda_event if prefix_events else None)
    rc = load().longspec_hta_prefix_attention_paged(
        ctypes.byref(dims), _ptr(q), ctypes.byref(kv), _ptr(prefix_len), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), ctypes.byref(opts),
        _stream(stream))
    _check(rc)
    return out, lse


def host_arena_bytes(dims: Dims) -> int:
    n = load().longspec_hta_host_arena_bytes(ctypes.byref(dims))
    if n == 0:
        raise HtaError(ERR_INVALID_DIMS)
    return n


def verify_host(q, k_prefix, v_prefix, prefix_len, k_tree, v_tree, parent, out, lse,
                arena, *, scale: float = 0.0, stream=None):
    """End-to-end call on host tensors (pinned for asynchronous copies): the
    library copies inputs into the device `arena`, runs, and copies out/lse
    back on `stream`.  Synchronise the stream before reading out/lse."""
    for t, n in ((q, "q"), (k_prefix, "k_prefix"), (v_prefix, "v_prefix"),
                 (k_tree, "k_tree"), (v_tree, "v_tree"), (out, "out")):
        _need(t, n, torch.bfloat16, torch.device("cpu"))
    _need(prefix_len, "prefix_len", torch.int32, torch.device("cpu"))
    _need(parent, "parent", torch.int32, torch.device("cpu"))
    _need(lse, "lse", torch.float32, torch.device("cpu"))
    dims = dims_of(q, k_prefix, scale)
    rc = load().longspec_hta_verify_host(
        ctypes.byref(dims), _ptr(q), _ptr(k_prefix), _ptr(v_prefix), _ptr(prefix_len),
        _ptr(k_tree), _ptr(v_tree), _ptr(parent), _ptr(out), _ptr(lse), _ptr(arena),
        arena.numel() * arena.element_size(), _stream(stream))
    _check(rc)


def tree_mask(parent: torch.Tensor, workspace=None, stream=None) -> torch.Tensor:
    """Ancestor-or-self bits uint32-as-int32 [B][T][ceil(T/32)] (debug export)."""
    _need(parent, "parent", torch.int32)
    B, T = parent.shape
    W = (T + 31) // 32
    bits = torch.empty(B, T, W, dtype=torch.int32, device=parent.device)
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=parent.device)
    _check(load().longspec_hta_tree_mask(_ptr(parent), B, T, _ptr(bits), _ptr(workspace),
                                         workspace.numel(), _stream(stream)))
    return bits


def tree_partial(q, k_tree, v_tree, parent, *, scale: float = 0.0, workspace=None, stream=None):
    """Tree-only partial (debug export): (o_tree fp32 [B][Hq][T][D], lse_tree fp32)."""
    B, Hq, T, D = q.shape
    dims = Dims(B, Hq, k_tree.shape[1], D, T, 0, float(scale))
    o = torch.empty(B, Hq, T, D, dtype=torch.float32, device=q.device)
    l = torch.empty(B, Hq, T, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q.device)
    _check(load().longspec_hta_tree_partial(ctypes.byref(dims), _ptr(q), _ptr(k_tree),
                                            _ptr(v_tree), _ptr(parent), _ptr(o), _ptr(l),
                                            _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, l


def prefix_partial(q, k_prefix, v_prefix, prefix_len, *, scale: float = 0.0,
                   num_splits: int = 0, prefix_kernel: int = PREFIX_TCGEN05,
                   workspace=None, stream=None):
    """Split-KV prefix partials (debug export):
    (o_part fp32 [B][Hq][T][S][D], lse_part fp32 [B][Hq][T][S], chunk keys)."""
    dims = dims_of(q, k_prefix, scale)
    lib = load()
    # the default call's split count, passed on explicitly so that every
    # prefix kernel cuts the keys the same way
    S, chunk_keys = chunking(dims, num_splits)
    S_out = ctypes.c_int(0)
    B, Hq, T, D = q.shape
    o = torch.empty(B, Hq, T, S, D, dtype=torch.float32, device=q.device)
    l = torch.empty(B, Hq, T, S, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q.device)
    _check(lib.longspec_hta_prefix_partial(ctypes.byref(dims), _ptr(q), _ptr(k_prefix),
                                           _ptr(v_prefix), _ptr(prefix_len), _ptr(o), _ptr(l),
                                           int(S), int(prefix_kernel), ctypes.byref(S_out),
                                           _ptr(workspace), workspace.numel(), _stream(stream)))
    if S_out.value != S:
        raise RuntimeError(f"split count mismatch: library {S_out.value}, binding {S}")
    return o, l, chunk_keys


def accept_workspace_bytes(B: int, T: int, V: int) -> int:
    return int(load().longspec_hta_accept_workspace_bytes(int(B), int(T), int(V)))


def new_accept_workspace(B: int, T: int, V: int, device=None) -> torch.Tensor:
    n = accept_workspace_bytes(B, T, V)
    if n == 0:
        raise HtaError(ERR_INVALID_DIMS)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def accept_greedy(logits, draft_tokens, parent, *, accept_len=None, path=None, bonus=None,
                  workspace=None, stream=None):
    """Greedy (temperature 0) acceptance of the draft tree.

    logits bf16 [B][T+1][V] (row 0: the prefix end, row 1+i: after node i),
    draft_tokens and parent int32 [B][T].  Returns (accept_len int32 [B],
    path int32 [B][T] padded with -1, bonus int32 [B])."""
    _need(logits, "logits", torch.bfloat16)
    dev = logits.device
    _need(draft_tokens, "draft_tokens", torch.int32, dev)
    _need(parent, "parent", torch.int32, dev)
    B, T1, V = logits.shape
    T = T1 - 1
    if tuple(draft_tokens.shape) != (B, T) or tuple(parent.shape) != (B, T):
        raise ValueError(f"draft_tokens/parent must be [{B}][{T}]")
    if accept_len is None:
        accept_len = torch.empty(B, dtype=torch.int32, device=dev)
    if path is None:
        path = torch.empty(B, T, dtype=torch.int32, device=dev)
    if bonus is None:
        bonus = torch.empty(B, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_accept_workspace(B, T, V, dev)
    _check(load().longspec_hta_accept_greedy(
        B, T, V, _ptr(logits), _ptr(draft_tokens), _ptr(parent), _ptr(accept_len), _ptr(path),
        _ptr(bonus), _ptr(workspace), workspace.numel(), _stream(stream)))
    return accept_len, path, bonus


def new_window_workspace(dims: Dims, device=None) -> torch.Tensor:
    n = int(load().longspec_hta_window_workspace_bytes(ctypes.byref(dims)))
    if n == 0:
        raise HtaError(ERR_INVALID_DIMS)
    return torch.zeros(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def window_verify(q, k_ring, v_ring, prefix_len, k_tree, v_tree, parent, *, out=None, lse=None,
                  workspace=None, scale: float = 0.0, stream=None):
    """Sliding-window tree attention (the draft model's self-attention): the
    ring k/v_ring [B][Hkv][W][D] holds context position p at slot p mod W;
    a node at depth d sees its root path and positions [L_b + d - W, L_b)."""
    _need(q, "q", torch.bfloat16)
    dev = q.device
    for t, n in ((k_ring, "k_ring"), (v_ring, "v_ring"), (k_tree, "k_tree"), (v_tree, "v_tree")):
        _need(t, n, torch.bfloat16, dev)
    _need(prefix_len, "prefix_len", torch.int32, dev)
    _need(parent, "parent", torch.int32, dev)
    dims = dims_of(q, k_ring, scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_window_workspace(dims, dev)
    _check(load().longspec_hta_window_verify(
        ctypes.byref(dims), _ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(prefix_len), _ptr(k_tree),
        _ptr(v_tree), _ptr(parent), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return out, lse


def _commit_dims(k_tree, L_cap):
    B, Hkv, T, D = k_tree.shape
    return Dims(B, Hkv, Hkv, D, T, int(L_cap), 0.0)


def commit(k_prefix, v_prefix, prefix_len, k_tree, v_tree, accept_len, path, *, workspace=None,
           stream=None):
    """Append the accepted path's tree K/V rows to the contiguous cache
    [B][Hkv][L_cap][D] after each prefix and advance prefix_len in place."""
    for t, n in ((k_prefix, "k_prefix"), (v_prefix, "v_prefix"), (k_tree, "k_tree"), (v_tree, "v_tree")):
        _need(t, n, torch.bfloat16, k_tree.device)
    for t, n in ((prefix_len, "prefix_len"), (accept_len, "accept_len"), (path, "path")):
        _need(t, n, torch.int32, k_tree.device)
    dims = _commit_dims(k_tree, k_prefix.shape[2])
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=k_tree.device)
    _check(load().longspec_hta_commit(ctypes.byref(dims), _ptr(k_prefix), _ptr(v_prefix),
                                      _ptr(prefix_len), _ptr(k_tree), _ptr(v_tree),
                                      _ptr(accept_len), _ptr(path), _ptr(workspace),
                                      workspace.numel(), _stream(stream)))


def commit_paged(k_cache, v_cache, block_table, prefix_len, k_tree, v_tree, accept_len, path, *,
                 L_cap, workspace=None, stream=None):
    """commit() into a paged cache [num_blocks][Hkv][block_size][D]."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache"), (k_tree, "k_tree"), (v_tree, "v_tree")):
        _need(t, n, torch.bfloat16, k_tree.device)
    for t, n in ((block_table, "block_table"), (prefix_len, "prefix_len"), (accept_len, "accept_len"),
                 (path, "path")):
        _need(t, n, torch.int32, k_tree.device)
    dims = _commit_dims(k_tree, L_cap)
    kv = _paged(k_cache, v_cache, block_table, k_tree.device)
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=k_tree.device)
    _check(load().longspec_hta_commit_paged(ctypes.byref(dims), ctypes.byref(kv), _ptr(prefix_len),
                                            _ptr(k_tree), _ptr(v_tree), _ptr(accept_len), _ptr(path),
                                            _ptr(workspace), workspace.numel(), _stream(stream)))


def selftest_wait_timeout(workspace: torch.Tensor, stream=None) -> int:
    """Launch the failure-detection self-test on `workspace`'s status word:
    one bounded in-kernel wait that nothing completes (about 2 s); a later
    get_status() returns ERR_PIPELINE_TIMEOUT."""
    return int(load().longspec_hta_selftest_wait_timeout(_ptr(workspace), _stream(stream)))


def build_info() -> dict:
    """The loaded library's build-time tuning knobs, e.g.
    {"kv_stages_d128": 3, "exp2_poly_every": 4}."""
    text = load().longspec_hta_build_info().decode()
    return {k: int(v) for k, v in (kv.split("=") for kv in text.split())}


def get_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the device status word; returns the code."""
    return int(load().longspec_hta_get_status(_ptr(workspace), _stream(stream)))

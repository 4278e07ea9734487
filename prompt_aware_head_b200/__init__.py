"""Python binding of the sm_100a block-sparse attention library (libsa_b200.so).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Functions keep the C names (sa_build_layout, sa_select_blocks,
sa_pattern_mask, sa_block_sparse_attention, sa_dense_attention, sa_density,
...).  Tensor arguments may be torch CUDA tensors or raw device addresses
(int); PyTorch is used only to hold device memory and streams.

Importing this module raises if the compiled library is missing: there is no
fallback path.  Build it with ``python prompt_aware_head_b200/build.py`` (or
``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import logging
import os
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libsa_b200.so not found at %s: build the CUDA library first "
                      "(python prompt_aware_head_b200/build.py)" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

# ---- status codes (include/sa.h) ----
SA_OK, SA_ERR_INVALID_ARG, SA_ERR_SHAPE, SA_ERR_LAYOUT, SA_ERR_HEAD_MASK, SA_ERR_WORKSPACE, \
    SA_ERR_BAD_INDEX, SA_ERR_TIMEOUT, SA_ERR_UNSUPPORTED, SA_ERR_CUDA = range(10)
SA_SEG_TEXT, SA_SEG_PAD, SA_SEG_IMAGE, SA_SEG_OTHER = range(4)
SA_BLOCK_PIN, SA_BLOCK_SPARSE, SA_BLOCK_DROP = range(3)
SA_PAT_RADIAL, SA_PAT_WINDOW_GLOBAL, SA_PAT_DILATED, SA_PAT_RANDOM = range(4)

# Constants of the haagenti_sparse crate (lib.rs): minimum heads kept active
# per layer and the default fraction of heads to skip.
MIN_ACTIVE_HEADS = 4
DEFAULT_SPARSITY = 0.5
MAX_QUALITY_LOSS = 0.02  # the crate's quality-loss bound; its gate needs trained models and is not built here
DEFAULT_MIN_SEQ_LEN = 8192  # SA_DEFAULT_MIN_SEQ_LEN


class sa_segment(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("start", ctypes.c_int32), ("len", ctypes.c_int32)]


class sa_pattern(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("window_tokens", ctypes.c_int32),
                ("n_global_blocks", ctypes.c_int32), ("dilation", ctypes.c_int32), ("seed", ctypes.c_uint64)]


class sa_stats(ctypes.Structure):
    _fields_ = [("density_over_active", ctypes.c_double), ("density_over_all", ctypes.c_double),
                ("tiles", ctypes.c_int64), ("heads_active", ctypes.c_int32)]


_P, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "sa_build_layout": ([ctypes.POINTER(sa_segment), _I, _I, _I, ctypes.POINTER(_P)], _I),
    "sa_layout_info": ([_P] + [ctypes.POINTER(_I)] * 5, _I),
    "sa_layout_classes": ([_P, _P, _I], _I),
    "sa_layout_release": ([_P], _I),
    "sa_budget": ([_F, _I], _I),
    "sa_budget_schedule": ([_P, _I, _I, _P, _P], _I),
    "sa_sparse_stage_gate": ([_I, _I, _I, _I, _I], _I),
    "sa_sparse_stage_decline": ([_I, _I, _I, _I, _I], _I),
    "sa_select_blocks": ([_P, _P, _P, _I, _I, _I, _F, _P, _I, _P, _P, _P, _P, _SZ, _P], _I),
    "sa_select_blocks_noalloc": ([_P, _P, _P, _I, _I, _I, _F, _P, _I, _P, _P, _P, _P], _I),
    "sa_pattern_mask": ([_P, ctypes.POINTER(sa_pattern), _I, _I, _F, _P, _I, _P, _P, _P], _I),
    "sa_block_sparse_attention": ([_P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _I, _F, _P, _P, _SZ, _P], _I),
    "sa_attention_plan": ([_P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _SZ, _P], _I),
    "sa_attention_run": ([_P, _P, _P, _I, _I, _I, _I, _P, _I, _F, _P, _P, _SZ, _P], _I),
    "sa_dense_attention": ([_P, _P, _P, _I, _I, _I, _I, _F, _P, _P, _SZ, _P], _I),
    "sa_select_blocks_gqa": ([_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _P, _P, _P, _SZ, _P], _I),
    "sa_select_blocks_noalloc_gqa": ([_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _P, _P, _P], _I),
    "sa_block_sparse_attention_gqa": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _I, _F, _P, _P, _SZ, _P], _I),
    "sa_attention_run_gqa": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _F, _P, _P, _SZ, _P], _I),
    "sa_dense_attention_gqa": ([_P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _SZ, _P], _I),
    "sa_block_sparse_attention_masked": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _I, _F, _P, _P, _SZ, _P],
                                         _I),
    "sa_attention_run_masked": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _F, _P, _P, _SZ, _P], _I),
    "sa_density": ([_P, _I, _I, _I, _P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                    ctypes.POINTER(sa_stats), _P, _SZ, _P], _I),
    "sa_workspace_size": ([_I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "sa_workspace_init": ([_P, _SZ, _P], _I),
    "sa_check": ([_P, _P], _I),
    "sa_check_noalloc": ([_P], _I),
    "sa_debug_noalloc_error": ([_I, _P], _I),
    "sa_debug_exp2": ([_P, _P, _I, _P], _I),
    "sa_debug_wait_timeout": ([_P, _SZ, _P], _I),
    "sa_status_string": ([_I], ctypes.c_char_p),
    "sa_version": ([], ctypes.c_char_p),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class SAError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__("%s: %s (status %d)" % (where, _lib.sa_status_string(status).decode(), status))
        self.status = status


def _check(status: int, where: str) -> None:
    if status != SA_OK:
        raise SAError(status, where)


def _addr(x) -> Optional[int]:
    """Device address of a torch tensor (or an int / None passed through)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _host_mask(head_mask) -> Tuple[Optional[ctypes.Array], Optional[np.ndarray]]:
    if head_mask is None:
        return None, None
    m = np.ascontiguousarray(np.asarray(head_mask, dtype=np.uint8))
    return m.ctypes.data_as(ctypes.c_void_p), m


# ------------------------------------------------------------------ layouts
class Layout:
    """Refcounted handle of a cached layout (sa_build_layout)."""

    def __init__(self, segments: Sequence[Tuple[int, int, int]], N: int, block: int = 64):
        segs = (sa_segment * max(len(segments), 1))(*[sa_segment(int(k), int(s), int(l)) for k, s, l in segments])
        h = ctypes.c_void_p()
        _check(_lib.sa_build_layout(segs, len(segments), int(N), int(block), ctypes.byref(h)), "sa_build_layout")
        self.handle = h
        self.N = int(N)
        vals = [ctypes.c_int() for _ in range(5)]
        _check(_lib.sa_layout_info(h, *[ctypes.byref(v) for v in vals]), "sa_layout_info")
        self.nB, self.n_pin, self.n_drop, self.n_cand, self.cap = (v.value for v in vals)

    def classes(self) -> np.ndarray:
        out = np.zeros(self.nB, dtype=np.uint8)
        _check(_lib.sa_layout_classes(self.handle, out.ctypes.data_as(ctypes.c_void_p), self.nB), "sa_layout_classes")
        return out

    def release(self) -> None:
        if self.handle:
            _check(_lib.sa_layout_release(self.handle), "sa_layout_release")
            self.handle = None

    def __del__(self):
        try:
            self.release()
        except Exception:
            pass


def sa_build_layout(segments, N: int, block: int = 64) -> Layout:
    return Layout(segments, N, block)


def sa_budget(density: float, n_cand: int) -> int:
    return int(_lib.sa_budget(ctypes.c_float(density), int(n_cand)))


def sa_budget_schedule(densities, n_cand: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per-step budgets k and dense flags of a schedule with at most two
    distinct densities (host only)."""
    d = np.ascontiguousarray(densities, dtype=np.float32).reshape(-1)
    k = np.zeros(d.size, dtype=np.int32)
    dense = np.zeros(d.size, dtype=np.uint8)
    _check(_lib.sa_budget_schedule(d.ctypes.data_as(ctypes.c_void_p), int(d.size), int(n_cand),
                                   k.ctypes.data_as(ctypes.c_void_p), dense.ctypes.data_as(ctypes.c_void_p)),
           "sa_budget_schedule")
    return k, dense.astype(bool)


SA_DECLINE_NOT_SELF_ATTENTION, SA_DECLINE_TOKEN_MASK, SA_DECLINE_CAUSAL, SA_DECLINE_SHORT = 1, 2, 4, 8
# Token mask kinds the gate tells apart: a general (query-dependent) mask declines; a key padding
# mask [B, N] is served by the _masked attention calls.
SA_TOKEN_MASK_NONE, SA_TOKEN_MASK_GENERAL, SA_TOKEN_MASK_KEY_PADDING = 0, 1, 2


def _mask_kind(token_mask) -> int:
    """None / False: no mask; "keys": a key padding mask; True or "general": any other token mask;
    an int is passed through."""
    if token_mask is None or token_mask is False:
        return SA_TOKEN_MASK_NONE
    if token_mask is True or token_mask == "general":
        return SA_TOKEN_MASK_GENERAL
    if token_mask == "keys":
        return SA_TOKEN_MASK_KEY_PADDING
    return int(token_mask)
_DECLINE_NAMES = ((SA_DECLINE_NOT_SELF_ATTENTION, "not self attention"), (SA_DECLINE_TOKEN_MASK, "token mask"),
                  (SA_DECLINE_CAUSAL, "causal"), (SA_DECLINE_SHORT, "below the minimum length"))
_declines_logged = set()
_log = logging.getLogger("prompt_aware_head_b200")


def sa_sparse_stage_decline(N: int, min_seq_len: int = DEFAULT_MIN_SEQ_LEN, self_attention: bool = True,
                            token_mask=None, causal: bool = False) -> int:
    """Bit set of the reasons the sparse stage declines a call (0: it does not).
    token_mask: None, "keys" (a key padding mask: served) or True / "general" (declined)."""
    return int(_lib.sa_sparse_stage_decline(int(N), int(min_seq_len), int(bool(self_attention)),
                                            _mask_kind(token_mask), int(bool(causal))))


def sa_sparse_stage_gate(N: int, min_seq_len: int = DEFAULT_MIN_SEQ_LEN, self_attention: bool = True,
                         token_mask=None, causal: bool = False) -> bool:
    """True when a call should take the block-sparse path (host only).  A
    decline is logged once per (reasons, N), so a setting that cannot act is
    visible without repeating every call."""
    why = sa_sparse_stage_decline(N, min_seq_len, self_attention, token_mask, causal)
    if why and (why, int(N)) not in _declines_logged:
        _declines_logged.add((why, int(N)))
        _log.info("sparse attention declined at N=%d: %s", int(N),
                  ", ".join(name for bit, name in _DECLINE_NAMES if why & bit))
    return why == 0


def sa_workspace_size(B: int, H: int, N: int, d: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.sa_workspace_size(B, H, N, d, ctypes.byref(n)), "sa_workspace_size")
    return n.value


def sa_workspace_init(ws, ws_bytes: int, stream=None) -> None:
    _check(_lib.sa_workspace_init(_addr(ws), ws_bytes, _stream(stream)), "sa_workspace_init")


def sa_check(ws, stream=None) -> int:
    """Synchronises the stream and returns the device-side status (SA_OK, ...)."""
    return int(_lib.sa_check(_addr(ws), _stream(stream)))


def sa_check_noalloc(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device-side status
    of sa_select_blocks_noalloc calls on the current device."""
    return int(_lib.sa_check_noalloc(_stream(stream)))


def sa_select_blocks(L: Layout, Q, K, B: int, H: int, d: int, density: float, head_mask, min_active: int,
                     idx, counts, scores_out, ws, ws_bytes: int, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_select_blocks(L.handle, _addr(Q), _addr(K), B, H, d, ctypes.c_float(density), mptr, min_active,
                                 _addr(idx), _addr(counts), _addr(scores_out), _addr(ws), ws_bytes, _stream(stream)),
           "sa_select_blocks")


def sa_select_blocks_noalloc(L: Layout, Q, K, B: int, H: int, d: int, density: float, head_mask, min_active: int,
                             idx, counts, scores_out, stream=None) -> None:
    """sa_select_blocks without a workspace, for callers that cannot allocate
    device memory (its scratch is a fixed 16 MiB array inside the library)."""
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_select_blocks_noalloc(L.handle, _addr(Q), _addr(K), B, H, d, ctypes.c_float(density), mptr,
                                         min_active, _addr(idx), _addr(counts), _addr(scores_out), _stream(stream)),
           "sa_select_blocks_noalloc")


def sa_pattern_mask(L: Layout, kind: int, B: int, H: int, density: float = 1.0, head_mask=None,
                    min_active: int = 0, idx=None, counts=None, window_tokens: int = 0, n_global_blocks: int = 0,
                    dilation: int = 1, stream=None, seed: int = 0) -> None:
    p = sa_pattern(kind, window_tokens, n_global_blocks, dilation, seed)
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_pattern_mask(L.handle, ctypes.byref(p), B, H, ctypes.c_float(density), mptr, min_active,
                                _addr(idx), _addr(counts), _stream(stream)), "sa_pattern_mask")


def sa_block_sparse_attention(Q, K, V, B: int, H: int, N: int, d: int, idx, counts, cap: int, head_mask,
                              min_active: int, softmax_scale: float, O, ws, ws_bytes: int, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_block_sparse_attention(_addr(Q), _addr(K), _addr(V), B, H, N, d, _addr(idx), _addr(counts), cap,
                                          mptr, min_active, ctypes.c_float(softmax_scale), _addr(O), _addr(ws),
                                          ws_bytes, _stream(stream)), "sa_block_sparse_attention")


def sa_attention_plan(idx, counts, B: int, H: int, N: int, d: int, cap: int, head_mask, min_active: int, ws,
                      ws_bytes: int, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_attention_plan(_addr(idx), _addr(counts), B, H, N, d, cap, mptr, min_active, _addr(ws), ws_bytes,
                                  _stream(stream)), "sa_attention_plan")


def sa_attention_run(Q, K, V, B: int, H: int, N: int, d: int, head_mask, min_active: int, softmax_scale: float, O,
                     ws, ws_bytes: int, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_attention_run(_addr(Q), _addr(K), _addr(V), B, H, N, d, mptr, min_active,
                                 ctypes.c_float(softmax_scale), _addr(O), _addr(ws), ws_bytes, _stream(stream)),
           "sa_attention_run")


def sa_dense_attention(Q, K, V, B: int, H: int, N: int, d: int, softmax_scale: float, O, ws, ws_bytes: int,
                       stream=None) -> None:
    _check(_lib.sa_dense_attention(_addr(Q), _addr(K), _addr(V), B, H, N, d, ctypes.c_float(softmax_scale),
                                   _addr(O), _addr(ws), ws_bytes, _stream(stream)), "sa_dense_attention")


# Grouped key/value heads: K and V hold H_kv heads, query head h reads h // (H // H_kv).

def sa_select_blocks_gqa(L: Layout, Q, K, B: int, H: int, H_kv: int, d: int, density: float, head_mask,
                         min_active: int, idx, counts, scores_out, ws, ws_bytes: int, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_select_blocks_gqa(L.handle, _addr(Q), _addr(K), B, H, H_kv, d, ctypes.c_float(density), mptr,
                                     min_active, _addr(idx), _addr(counts), _addr(scores_out), _addr(ws), ws_bytes,
                                     _stream(stream)), "sa_select_blocks_gqa")


def sa_select_blocks_noalloc_gqa(L: Layout, Q, K, B: int, H: int, H_kv: int, d: int, density: float, head_mask,
                                 min_active: int, idx, counts, scores_out, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_select_blocks_noalloc_gqa(L.handle, _addr(Q), _addr(K), B, H, H_kv, d, ctypes.c_float(density),
                                             mptr, min_active, _addr(idx), _addr(counts), _addr(scores_out),
                                             _stream(stream)), "sa_select_blocks_noalloc_gqa")


def sa_block_sparse_attention_gqa(Q, K, V, B: int, H: int, H_kv: int, N: int, d: int, idx, counts, cap: int,
                                  head_mask, min_active: int, softmax_scale: float, O, ws, ws_bytes: int,
                                  stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_block_sparse_attention_gqa(_addr(Q), _addr(K), _addr(V), B, H, H_kv, N, d, _addr(idx),
                                              _addr(counts), cap, mptr, min_active, ctypes.c_float(softmax_scale),
                                              _addr(O), _addr(ws), ws_bytes, _stream(stream)),
           "sa_block_sparse_attention_gqa")


def sa_attention_run_gqa(Q, K, V, B: int, H: int, H_kv: int, N: int, d: int, head_mask, min_active: int,
                         softmax_scale: float, O, ws, ws_bytes: int, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_attention_run_gqa(_addr(Q), _addr(K), _addr(V), B, H, H_kv, N, d, mptr, min_active,
                                     ctypes.c_float(softmax_scale), _addr(O), _addr(ws), ws_bytes, _stream(stream)),
           "sa_attention_run_gqa")


def sa_dense_attention_gqa(Q, K, V, B: int, H: int, H_kv: int, N: int, d: int, softmax_scale: float, O, ws,
                           ws_bytes: int, stream=None) -> None:
    _check(_lib.sa_dense_attention_gqa(_addr(Q), _addr(K), _addr(V), B, H, H_kv, N, d,
                                       ctypes.c_float(softmax_scale), _addr(O), _addr(ws), ws_bytes,
                                       _stream(stream)), "sa_dense_attention_gqa")


# Token-level key mask inside the kept tiles: key_mask is a device uint8 [B, N] (nonzero = may be attended).

def sa_block_sparse_attention_masked(Q, K, V, B: int, H: int, H_kv: int, N: int, d: int, idx, counts, cap: int,
                                     key_mask, head_mask, min_active: int, softmax_scale: float, O, ws, ws_bytes: int,
                                     stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_block_sparse_attention_masked(_addr(Q), _addr(K), _addr(V), B, H, H_kv, N, d, _addr(idx),
                                                 _addr(counts), cap, _addr(key_mask), mptr, min_active,
                                                 ctypes.c_float(softmax_scale), _addr(O), _addr(ws), ws_bytes,
                                                 _stream(stream)), "sa_block_sparse_attention_masked")


def sa_attention_run_masked(Q, K, V, B: int, H: int, H_kv: int, N: int, d: int, key_mask, head_mask,
                            min_active: int, softmax_scale: float, O, ws, ws_bytes: int, stream=None) -> None:
    mptr, _keep = _host_mask(head_mask)
    _check(_lib.sa_attention_run_masked(_addr(Q), _addr(K), _addr(V), B, H, H_kv, N, d, _addr(key_mask), mptr,
                                        min_active, ctypes.c_float(softmax_scale), _addr(O), _addr(ws), ws_bytes,
                                        _stream(stream)), "sa_attention_run_masked")


def sa_density(counts, B: int, H: int, nB: int, head_mask, ws, ws_bytes: int, stream=None):
    """Returns (density over active heads, density over all heads, sa_stats)."""
    mptr, _keep = _host_mask(head_mask)
    a, b, st = ctypes.c_double(), ctypes.c_double(), sa_stats()
    _check(_lib.sa_density(_addr(counts), B, H, nB, mptr, ctypes.byref(a), ctypes.byref(b), ctypes.byref(st),
                           _addr(ws), ws_bytes, _stream(stream)), "sa_density")
    return a.value, b.value, st


def sa_debug_wait_timeout(ws, ws_bytes: int, stream=None) -> None:
    """Runs one kernel whose bounded wait runs out (about 2 s); the next
    sa_check reports SA_ERR_TIMEOUT."""
    _check(_lib.sa_debug_wait_timeout(_addr(ws), ws_bytes, _stream(stream)), "sa_debug_wait_timeout")


def sa_debug_noalloc_error(status: int, stream=None) -> None:
    """Records status in the no-allocation path's error word (test hook); the
    next sa_check_noalloc reports it."""
    _check(_lib.sa_debug_noalloc_error(int(status), _stream(stream)), "sa_debug_noalloc_error")


def sa_debug_exp2(y, out, n: int, stream=None) -> None:
    _check(_lib.sa_debug_exp2(_addr(y), _addr(out), n, _stream(stream)), "sa_debug_exp2")


def sa_status_string(status: int) -> str:
    return _lib.sa_status_string(status).decode()


def sa_version() -> str:
    return _lib.sa_version().decode()

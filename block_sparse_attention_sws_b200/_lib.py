"""ctypes binding of libsws (include/sws.h): argument marshalling only.

Every entry point here forwards to the C function of the same name with raw
pointers taken from torch tensors; no step of the computation happens in
Python. If the shared library is missing, loading fails loudly: there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsws.so")

SWS_OK, SWS_ERR_INVALID_ARG, SWS_ERR_UNSUPPORTED, SWS_ERR_WORKSPACE, SWS_ERR_CUDA, SWS_ERR_DEVICE_CHECK = range(6)
SWS_BF16, SWS_FP32 = 0, 1
SWS_WALK_MATRIX_POWER, SWS_WALK_ELEMENTWISE = 0, 1
SWS_OP_SKETCH, SWS_OP_WALK_SELECT, SWS_OP_PREFILL_ATTN, SWS_OP_DECODE_ATTN = range(4)

# Every exported symbol of include/sws.h (the CPU test checks the header and this list agree).
EXPORTS = [
    "sws_status_string", "sws_config_check", "sws_num_blocks", "sws_csr_nnz", "sws_build_projection_host",
    "sws_workspace_size", "sws_create", "sws_destroy", "sws_projection_device", "sws_launch_count",
    "sws_sync_check", "sws_layout_check", "sws_sketch",
    "sws_walk_select", "sws_walk_select_sketch", "sws_sparse_attn_prefill", "sws_sparse_attn_prefill_varlen_ws_bytes",
    "sws_sparse_attn_prefill_varlen", "sws_decode_init_cache", "sws_decode_advance", "sws_decode_step",
    "sws_sparse_attn_decode", "sws_sparse_attn_decode_noalloc", "sws_decode_init_cache_paged", "sws_decode_step_paged",
    "sws_sparse_attn_decode_paged", "sws_decode_step_exact", "sws_decode_exact_rows_entries",
    "sws_decode_exact_rows_init", "sws_decode_step_exact_rows",
]
NOALLOC_SCRATCH_BYTES = 32 << 20  # SWS_NOALLOC_SCRATCH_BYTES


class SwsConfig(ctypes.Structure):
    _fields_ = [
        ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("sketch_dim", ctypes.c_int32),
        ("walk_power", ctypes.c_int32), ("walk_mode", ctypes.c_int32), ("density_num", ctypes.c_int32),
        ("density_den", ctypes.c_int32), ("select_group", ctypes.c_int32), ("seed", ctypes.c_uint64),
    ]


class SwsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libsws.so is not built ({LIB_PATH}); run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, U64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    CFG = ctypes.POINTER(SwsConfig)
    sig = {
        "sws_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "sws_config_check": (ctypes.c_int, [CFG]),
        "sws_num_blocks": (I64, [CFG, I64]),
        "sws_csr_nnz": (I64, [CFG, I64]),
        "sws_build_projection_host": (ctypes.c_int, [CFG, P]),
        "sws_workspace_size": (ctypes.c_int, [CFG, ctypes.c_int, I64, I32, I32, I32, ctypes.POINTER(SZ)]),
        "sws_create": (ctypes.c_int, [CFG, ctypes.POINTER(P)]),
        "sws_destroy": (ctypes.c_int, [P]),
        "sws_projection_device": (P, [P]),
        "sws_launch_count": (U64, []),
        "sws_sync_check": (ctypes.c_int, [P, P, ctypes.POINTER(I32)]),
        "sws_sketch": (ctypes.c_int, [P, P, P, ctypes.c_int, I64, I32, I32, P, P, P, P, P, P, SZ, P]),
        "sws_layout_check": (ctypes.c_int, [CFG, ctypes.c_int, I64, P]),
        "sws_walk_select": (ctypes.c_int, [P, P, I64, I32, ctypes.c_int, P, P, P, P, SZ, P]),
        "sws_walk_select_sketch": (ctypes.c_int, [P, P, P, I64, I32, I32, ctypes.c_int, P, P, P, P, SZ, P]),
        "sws_sparse_attn_prefill": (ctypes.c_int, [P, P, P, P, ctypes.c_int, I64, I32, I32, P, P, P, P, P, P, P, P,
                                                   SZ, P]),
        "sws_sparse_attn_prefill_varlen_ws_bytes": (SZ, [I32, P]),
        "sws_sparse_attn_prefill_varlen": (ctypes.c_int, [P, P, P, P, ctypes.c_int, I32, P, I32, I32, P, P, P, P, P, P,
                                                          P, P, SZ, P]),
        "sws_decode_init_cache": (ctypes.c_int, [P, P, I32, I32, I64, P, P, P, P]),
        "sws_decode_advance": (ctypes.c_int, [P, P, I32, P]),
        "sws_decode_step": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I64, P, P, P, P, P, ctypes.c_int, P, P, P, P,
                                           P, P, P]),
        "sws_sparse_attn_decode": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I64, P, P, P, P, P, P, SZ, P]),
        "sws_sparse_attn_decode_noalloc": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I64, P, P, P, P, P, P]),
        "sws_decode_init_cache_paged": (ctypes.c_int, [P, P, I64, P, I64, I32, I32, P, P, P, P]),
        "sws_decode_step_exact": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I64, P, P, P, P, P, P, P, ctypes.c_int,
                                                 P, P, P, P, P, P, P]),
        "sws_decode_exact_rows_entries": (I64, [CFG, I64]),
        "sws_decode_exact_rows_init": (ctypes.c_int, [P, P, P, I32, I32, I32, I64, P, P, P]),
        "sws_decode_step_exact_rows": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I64, P, P, P, P, P, P, P, P,
                                                      ctypes.c_int, P, P, P, P, P, P, P]),
        "sws_decode_step_paged": (ctypes.c_int, [P, P, P, P, I32, I32, I32, P, P, I64, P, I64, P, P, P, ctypes.c_int,
                                                 P, P, P, P, P, P, P]),
        "sws_sparse_attn_decode_paged": (ctypes.c_int, [P, P, P, P, I64, P, I64, I32, I32, I32, P, P, P, P, P, P, SZ,
                                                        P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load().sws_status_string(int(s)).decode()


def _check(s: int, where: str) -> None:
    if s != SWS_OK:
        raise SwsError(s, where)


def make_config(head_dim=128, block_size=64, sketch_dim=32, walk_power=8, walk_mode=SWS_WALK_MATRIX_POWER,
                density=(1, 5), seed=0, select_group=0) -> SwsConfig:
    return SwsConfig(head_dim, block_size, sketch_dim, walk_power, walk_mode, density[0], density[1], select_group,
                     seed)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _head_tok(t: torch.Tensor):
    """(pointer, strides) of a [heads, n, d] operand: strides None when it is
    dense, else the (head, token) element strides of a view whose rows are
    contiguous (e.g. x.transpose(0, 1) of a [n, heads, d] activation)."""
    if t.dim() != 3 or t.stride(-1) != 1:
        raise ValueError("operands are [heads, n, d] with contiguous rows")
    if t.is_contiguous():
        return t.data_ptr(), None
    return t.data_ptr(), (ctypes.c_int64 * 2)(t.stride(0), t.stride(1))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SWS_BF16
    if t.dtype == torch.float32:
        return SWS_FP32
    raise ValueError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------ host ----

def sws_config_check(cfg: SwsConfig) -> int:
    return load().sws_config_check(ctypes.byref(cfg))


def sws_num_blocks(cfg: SwsConfig, n: int) -> int:
    return load().sws_num_blocks(ctypes.byref(cfg), n)


def sws_csr_nnz(cfg: SwsConfig, n: int) -> int:
    return load().sws_csr_nnz(ctypes.byref(cfg), n)


def sws_build_projection_host(cfg: SwsConfig) -> torch.Tensor:
    out = torch.empty(cfg.head_dim, cfg.sketch_dim, dtype=torch.float64)
    _check(load().sws_build_projection_host(ctypes.byref(cfg), out.data_ptr()), "sws_build_projection_host")
    return out


def sws_workspace_size(cfg: SwsConfig, op: int, n: int, hq: int, hkv: int, batch: int = 1) -> int:
    v = ctypes.c_size_t(0)
    _check(load().sws_workspace_size(ctypes.byref(cfg), op, n, hq, hkv, batch, ctypes.byref(v)), "sws_workspace_size")
    return v.value


# ---------------------------------------------------------------- handle ----

class Handle:
    """Owns an sws_handle (H_d on the current CUDA device)."""

    def __init__(self, cfg: SwsConfig):
        self.cfg = cfg
        self._lib = load()
        p = ctypes.c_void_p()
        _check(self._lib.sws_create(ctypes.byref(cfg), ctypes.byref(p)), "sws_create")
        self.ptr = p

    def close(self):
        if getattr(self, "ptr", None):
            self._lib.sws_destroy(self.ptr)
            self.ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def as_parameter(self):
        return self.ptr


def sws_create(cfg: SwsConfig) -> Handle:
    return Handle(cfg)


def sws_destroy(h: Handle) -> None:
    h.close()


def sws_launch_count() -> int:
    return int(load().sws_launch_count())


def sws_sync_check(h: Handle, stream=None) -> int:
    code = ctypes.c_int32(0)
    s = load().sws_sync_check(h.ptr, _stream(stream), ctypes.byref(code))
    if s not in (SWS_OK, SWS_ERR_DEVICE_CHECK):
        _check(s, "sws_sync_check")
    return code.value


# --------------------------------------------------------------- prefill ----

def sws_sketch(h: Handle, q, k, q_sk, k_sk, scores, ws, stream=None) -> None:
    """q [hq, n, d], k [hkv, n, d]: dense or strided views with contiguous rows;
    scores None skips the score matrix (see sws_walk_select_sketch)."""
    hq, n, _ = q.shape
    hkv = k.shape[0]
    (qp, qs), (kp, ks) = _head_tok(q), _head_tok(k)
    _check(load().sws_sketch(h.ptr, qp, kp, _dtype_code(q), n, hq, hkv, qs, ks, _ptr(q_sk), _ptr(k_sk),
                             _ptr(scores), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "sws_sketch")


def sws_walk_select(h: Handle, scores, n: int, first_layer: bool, walk_state, row_ptr, col_idx, ws,
                    stream=None) -> None:
    hq = scores.shape[0]
    _check(load().sws_walk_select(h.ptr, _ptr(scores), n, hq, int(bool(first_layer)), _ptr(walk_state),
                                  _ptr(row_ptr), _ptr(col_idx), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "sws_walk_select")


def sws_walk_select_sketch(h: Handle, q_sk, k_sk, n: int, first_layer: bool, walk_state, row_ptr, col_idx, ws,
                           stream=None) -> None:
    hq, hkv = q_sk.shape[0], k_sk.shape[0]
    _check(load().sws_walk_select_sketch(h.ptr, _ptr(q_sk), _ptr(k_sk), n, hq, hkv, int(bool(first_layer)),
                                         _ptr(walk_state), _ptr(row_ptr), _ptr(col_idx), _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)), "sws_walk_select_sketch")


def sws_sparse_attn_prefill(h: Handle, q, k, v, row_ptr, col_idx, o, ws=None, stream=None) -> None:
    """q, o [hq, n, d], k, v [hkv, n, d]: dense or strided views with contiguous rows."""
    hq, n, _ = q.shape
    hkv = k.shape[0]
    wsp = _ptr(ws) if ws is not None else None
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    (qp, qs), (kp, ks), (vp, vs), (op, os_) = _head_tok(q), _head_tok(k), _head_tok(v), _head_tok(o)
    _check(load().sws_sparse_attn_prefill(h.ptr, qp, kp, vp, _dtype_code(q), n, hq, hkv, qs, ks, vs, os_,
                                          _ptr(row_ptr), _ptr(col_idx), op, wsp, wsb, _stream(stream)),
           "sws_sparse_attn_prefill")


def _cu_array(cu_seqlens):
    return (ctypes.c_int64 * len(cu_seqlens))(*[int(x) for x in cu_seqlens])


def sws_sparse_attn_prefill_varlen_ws_bytes(cu_seqlens) -> int:
    """Workspace bytes of a packed launch over the sequences cu_seqlens describes
    (0 for an invalid list)."""
    return int(load().sws_sparse_attn_prefill_varlen_ws_bytes(len(cu_seqlens) - 1, _cu_array(cu_seqlens)))


def sws_sparse_attn_prefill_varlen(h: Handle, q, k, v, cu_seqlens, row_ptrs, col_idxs, o, ws, stream=None) -> None:
    """q, o [hq, N, d], k, v [hkv, N, d] bf16 (dense or strided views with contiguous
    rows), the sequences end to end along N; cu_seqlens: nseq + 1 token offsets
    (host); row_ptrs, col_idxs: each sequence's CSR tensors."""
    nseq = len(cu_seqlens) - 1
    hq = q.shape[0]
    hkv = k.shape[0]
    if len(row_ptrs) != nseq or len(col_idxs) != nseq:
        raise ValueError("one CSR per sequence")
    rp = (ctypes.c_void_p * nseq)(*[_ptr(t) for t in row_ptrs])
    ci = (ctypes.c_void_p * nseq)(*[_ptr(t) for t in col_idxs])
    (qp, qs), (kp, ks), (vp, vs), (op, os_) = _head_tok(q), _head_tok(k), _head_tok(v), _head_tok(o)
    _check(load().sws_sparse_attn_prefill_varlen(h.ptr, qp, kp, vp, _dtype_code(q), nseq, _cu_array(cu_seqlens), hq,
                                                 hkv, qs, ks, vs, os_, rp, ci, op, _ptr(ws),
                                                 ws.numel() * ws.element_size(), _stream(stream)),
           "sws_sparse_attn_prefill_varlen")


# ---------------------------------------------------------------- decode ----

def sws_decode_init_cache(h: Handle, k_cache, seq_lens, k_psum, k_sketch, stream=None) -> None:
    batch, hkv, max_len, _ = k_cache.shape
    _check(load().sws_decode_init_cache(h.ptr, _ptr(k_cache), batch, hkv, max_len, _ptr(seq_lens), _ptr(k_psum),
                                        _ptr(k_sketch), _stream(stream)), "sws_decode_init_cache")


def sws_decode_advance(h: Handle, seq_lens, stream=None) -> None:
    _check(load().sws_decode_advance(h.ptr, _ptr(seq_lens), seq_lens.numel(), _stream(stream)), "sws_decode_advance")


def sws_decode_step(h: Handle, q_tok, k_tok, v_tok, seq_lens, k_cache, v_cache, k_psum, k_sketch, first_layer: bool,
                    walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt, stream=None) -> None:
    batch, hq, _ = q_tok.shape
    hkv, max_len = k_cache.shape[1], k_cache.shape[2]
    _check(load().sws_decode_step(h.ptr, _ptr(q_tok), _ptr(k_tok), _ptr(v_tok), batch, hq, hkv, max_len,
                                  _ptr(seq_lens), _ptr(k_cache), _ptr(v_cache), _ptr(k_psum), _ptr(k_sketch),
                                  int(bool(first_layer)), _ptr(walk_state), _ptr(head_sel), _ptr(head_cnt), _ptr(sel),
                                  _ptr(sel_mask), _ptr(sel_cnt), _stream(stream)), "sws_decode_step")


def sws_sparse_attn_decode(h: Handle, q_tok, k_cache, v_cache, seq_lens, sel, sel_mask, sel_cnt, o, ws,
                           stream=None) -> None:
    batch, hq, _ = q_tok.shape
    hkv, max_len = k_cache.shape[1], k_cache.shape[2]
    _check(load().sws_sparse_attn_decode(h.ptr, _ptr(q_tok), _ptr(k_cache), _ptr(v_cache), batch, hq, hkv, max_len,
                                         _ptr(seq_lens), _ptr(sel), _ptr(sel_mask), _ptr(sel_cnt), _ptr(o), _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)), "sws_sparse_attn_decode")


def sws_sparse_attn_decode_noalloc(h: Handle, q_tok, k_cache, v_cache, seq_lens, sel, sel_mask, sel_cnt, o,
                                   stream=None) -> None:
    """sws_sparse_attn_decode without a workspace, for callers that cannot allocate:
    the partials live in the library's built-in scratch array (see include/sws.h)."""
    batch, hq, _ = q_tok.shape
    hkv, max_len = k_cache.shape[1], k_cache.shape[2]
    _check(load().sws_sparse_attn_decode_noalloc(h.ptr, _ptr(q_tok), _ptr(k_cache), _ptr(v_cache), batch, hq, hkv,
                                                 max_len, _ptr(seq_lens), _ptr(sel), _ptr(sel_mask), _ptr(sel_cnt),
                                                 _ptr(o), _stream(stream)), "sws_sparse_attn_decode_noalloc")


# ------------------------------------------------------ paged KV cache ----

def sws_decode_init_cache_paged(h: Handle, k_pages, block_table, seq_lens, k_psum, k_sketch, stream=None) -> None:
    """k_pages [num_pages, hkv, B, d]; block_table [batch, max_blocks] int32."""
    num_pages, hkv = k_pages.shape[0], k_pages.shape[1]
    batch, max_blocks = block_table.shape
    _check(load().sws_decode_init_cache_paged(h.ptr, _ptr(k_pages), num_pages, _ptr(block_table), max_blocks, batch,
                                              hkv, _ptr(seq_lens), _ptr(k_psum), _ptr(k_sketch), _stream(stream)),
           "sws_decode_init_cache_paged")


def sws_decode_step_paged(h: Handle, q_tok, k_tok, v_tok, k_pages, v_pages, block_table, seq_lens, k_psum, k_sketch,
                          first_layer: bool, walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt,
                          stream=None) -> None:
    batch, hq, _ = q_tok.shape
    num_pages, hkv = k_pages.shape[0], k_pages.shape[1]
    max_blocks = block_table.shape[1]
    _check(load().sws_decode_step_paged(h.ptr, _ptr(q_tok), _ptr(k_tok), _ptr(v_tok), batch, hq, hkv, _ptr(k_pages),
                                        _ptr(v_pages), num_pages, _ptr(block_table), max_blocks, _ptr(seq_lens),
                                        _ptr(k_psum), _ptr(k_sketch), int(bool(first_layer)), _ptr(walk_state),
                                        _ptr(head_sel), _ptr(head_cnt), _ptr(sel), _ptr(sel_mask), _ptr(sel_cnt),
                                        _stream(stream)), "sws_decode_step_paged")


def sws_sparse_attn_decode_paged(h: Handle, q_tok, k_pages, v_pages, block_table, seq_lens, sel, sel_mask, sel_cnt, o,
                                 ws, stream=None) -> None:
    batch, hq, _ = q_tok.shape
    num_pages, hkv = k_pages.shape[0], k_pages.shape[1]
    max_blocks = block_table.shape[1]
    _check(load().sws_sparse_attn_decode_paged(h.ptr, _ptr(q_tok), _ptr(k_pages), _ptr(v_pages), num_pages,
                                               _ptr(block_table), max_blocks, batch, hq, hkv, _ptr(seq_lens),
                                               _ptr(sel), _ptr(sel_mask), _ptr(sel_cnt), _ptr(o), _ptr(ws),
                                               ws.numel() * ws.element_size(), _stream(stream)),
           "sws_sparse_attn_decode_paged")


# ------------------------------------------------------ exact decode walk ----

def sws_decode_step_exact(h: Handle, q_tok, k_tok, v_tok, seq_lens, k_cache, v_cache, k_psum, k_sketch, q_psum,
                          q_sketch, first_layer: bool, walk_state, head_sel, head_cnt, sel, sel_mask, sel_cnt,
                          stream=None) -> None:
    batch, hq, _ = q_tok.shape
    hkv, max_len = k_cache.shape[1], k_cache.shape[2]
    _check(load().sws_decode_step_exact(h.ptr, _ptr(q_tok), _ptr(k_tok), _ptr(v_tok), batch, hq, hkv, max_len,
                                        _ptr(seq_lens), _ptr(k_cache), _ptr(v_cache), _ptr(k_psum), _ptr(k_sketch),
                                        _ptr(q_psum), _ptr(q_sketch), int(bool(first_layer)), _ptr(walk_state),
                                        _ptr(head_sel), _ptr(head_cnt), _ptr(sel), _ptr(sel_mask), _ptr(sel_cnt),
                                        _stream(stream)), "sws_decode_step_exact")


def sws_decode_exact_rows_entries(cfg: SwsConfig, max_len: int) -> int:
    n = load().sws_decode_exact_rows_entries(ctypes.byref(cfg), max_len)
    if n < 0:
        raise SwsError(SWS_ERR_INVALID_ARG, "sws_decode_exact_rows_entries")
    return n


def sws_decode_exact_rows_init(h: Handle, q_sketch, k_sketch, seq_lens, rows, stream=None) -> None:
    """q_sketch [batch, hq, max_blocks, k], k_sketch [batch, hkv, max_blocks, k] (fp64);
    rows [batch, hq, E] int32 (uint32 entries), E = sws_decode_exact_rows_entries."""
    batch, hq, mb, _ = q_sketch.shape
    hkv = k_sketch.shape[1]
    max_len = mb * h.cfg.block_size
    _check(load().sws_decode_exact_rows_init(h.ptr, _ptr(q_sketch), _ptr(k_sketch), batch, hq, hkv, max_len,
                                             _ptr(seq_lens), _ptr(rows), _stream(stream)), "sws_decode_exact_rows_init")


def sws_decode_step_exact_rows(h: Handle, q_tok, k_tok, v_tok, seq_lens, k_cache, v_cache, k_psum, k_sketch, q_psum,
                               q_sketch, rows, first_layer: bool, walk_state, head_sel, head_cnt, sel, sel_mask,
                               sel_cnt, stream=None) -> None:
    batch, hq, _ = q_tok.shape
    hkv, max_len = k_cache.shape[1], k_cache.shape[2]
    _check(load().sws_decode_step_exact_rows(h.ptr, _ptr(q_tok), _ptr(k_tok), _ptr(v_tok), batch, hq, hkv, max_len,
                                             _ptr(seq_lens), _ptr(k_cache), _ptr(v_cache), _ptr(k_psum),
                                             _ptr(k_sketch), _ptr(q_psum), _ptr(q_sketch), _ptr(rows),
                                             int(bool(first_layer)), _ptr(walk_state), _ptr(head_sel),
                                             _ptr(head_cnt), _ptr(sel), _ptr(sel_mask), _ptr(sel_cnt),
                                             _stream(stream)), "sws_decode_step_exact_rows")

"""Buffer set-up and call order for the prefill and decode paths.

torch allocates the device buffers and provides the stream; every step runs
in libsws through the C ABI (see ``_lib``).
"""
from __future__ import annotations

import torch

from . import _lib as L


class PrefillPath:
    """Per-layer prefill: sws_sketch -> sws_walk_select -> sws_sparse_attn_prefill.

    The walk state R [hq, b, b] (fp64) is carried from layer to layer.

    ``dense_layers`` is the caller policy of "Scout Before You Attend" §7 (the
    first layers attend densely): layers below it select every causal block,
    through a second handle with density 1/1 and the same projection, while
    the walk state still runs through them."""

    def __init__(self, handle: L.Handle, n: int, hq: int, hkv: int, dtype=torch.bfloat16, device="cuda",
                 dense_layers: int = 0):
        cfg = handle.cfg
        self.dense_layers = dense_layers
        self.h, self.n, self.hq, self.hkv = handle, n, hq, hkv
        self.b = L.sws_num_blocks(cfg, n)
        self.nnz = L.sws_csr_nnz(cfg, n)
        k, d = cfg.sketch_dim, cfg.head_dim
        f64 = dict(dtype=torch.float64, device=device)
        self.q_sk = torch.empty(hq, self.b, k, **f64)
        self.k_sk = torch.empty(hkv, self.b, k, **f64)
        self.scores = torch.empty(hq, self.b, self.b, **f64)
        self.walk_state = torch.zeros(hq, self.b, self.b, **f64)
        self.row_ptr = torch.empty(hq, self.b + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(hq, self.nnz, dtype=torch.int32, device=device)
        ws = L.sws_workspace_size(cfg, L.SWS_OP_WALK_SELECT, n, hq, hkv)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
        wss = L.sws_workspace_size(cfg, L.SWS_OP_SKETCH, n, hq, hkv)
        self.ws_sketch = torch.empty(max(wss, 16), dtype=torch.uint8, device=device)
        self.o = torch.empty(hq, n, d, dtype=dtype, device=device)
        self.h_dense = None
        if dense_layers > 0:
            self.h_dense = L.Handle(L.make_config(cfg.head_dim, cfg.block_size, cfg.sketch_dim, cfg.walk_power,
                                                  cfg.walk_mode, (1, 1), cfg.seed, cfg.select_group))
            nnz_dense = L.sws_csr_nnz(self.h_dense.cfg, n)
            self.row_ptr_dense = torch.empty(hq, self.b + 1, dtype=torch.int32, device=device)
            self.col_idx_dense = torch.empty(hq, nnz_dense, dtype=torch.int32, device=device)

    def _dense(self, layer) -> bool:
        return self.h_dense is not None and layer is not None and layer < self.dense_layers

    def csr(self, layer=None):
        """(row_ptr, col_idx) that the given layer uses."""
        if self._dense(layer):
            return self.row_ptr_dense, self.col_idx_dense
        return self.row_ptr, self.col_idx

    def sketch(self, q, k, stream=None):
        L.sws_sketch(self.h, q, k, self.q_sk, self.k_sk, self.scores, self.ws_sketch, stream)

    def walk_select(self, first_layer: bool, stream=None, layer=None):
        h = self.h_dense if self._dense(layer) else self.h
        rp, ci = self.csr(layer)
        L.sws_walk_select(h, self.scores, self.n, first_layer, self.walk_state, rp, ci, self.ws, stream)

    def attention(self, q, k, v, out=None, stream=None, layer=None):
        o = self.o if out is None else out
        h = self.h_dense if self._dense(layer) else self.h
        rp, ci = self.csr(layer)
        L.sws_sparse_attn_prefill(h, q, k, v, rp, ci, o, None, stream)
        return o

    def layer(self, q, k, v, first_layer: bool, out=None, stream=None, layer=None):
        """One layer; ``layer`` (its index) is needed only with dense_layers > 0."""
        self.sketch(q, k, stream)
        self.walk_select(first_layer, stream, layer)
        return self.attention(q, k, v, out, stream, layer)


class DecodePath:
    """Per-layer decode state and the per-step call order:
    sws_decode_step -> sws_sparse_attn_decode for each layer, then
    sws_decode_advance once the step's layers are done."""

    def __init__(self, handle: L.Handle, batch: int, hq: int, hkv: int, max_len: int, layers: int, device="cuda"):
        cfg = handle.cfg
        self.h, self.batch, self.hq, self.hkv, self.max_len, self.layers = handle, batch, hq, hkv, max_len, layers
        d, k = cfg.head_dim, cfg.sketch_dim
        self.mb = L.sws_num_blocks(cfg, max_len)
        bf = dict(dtype=torch.bfloat16, device=device)
        f64 = dict(dtype=torch.float64, device=device)
        i32 = dict(dtype=torch.int32, device=device)
        self.k_cache = [torch.empty(batch, hkv, max_len, d, **bf) for _ in range(layers)]
        self.v_cache = [torch.empty(batch, hkv, max_len, d, **bf) for _ in range(layers)]
        self.k_psum = [torch.zeros(batch, hkv, d, **f64) for _ in range(layers)]
        self.k_sketch = [torch.zeros(batch, hkv, self.mb, k, **f64) for _ in range(layers)]
        self.seq_lens = torch.zeros(batch, **i32)
        self.walk_state = torch.zeros(batch, hq, self.mb, **f64)
        self.head_sel = torch.zeros(batch, hq, self.mb, **i32)
        self.head_cnt = torch.zeros(batch, hq, **i32)
        self.sel = torch.zeros(batch, hkv, self.mb, **i32)
        self.sel_mask = torch.zeros(batch, hkv, self.mb, dtype=torch.uint8, device=device)
        self.sel_cnt = torch.zeros(batch, hkv, **i32)
        ws = L.sws_workspace_size(cfg, L.SWS_OP_DECODE_ATTN, max_len, hq, hkv, batch)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.o = torch.empty(batch, hq, d, **bf)

    def init_cache(self, lens: torch.Tensor, stream=None):
        """Caches already hold lens[i] tokens per sequence: build their sketches."""
        self.seq_lens.copy_(lens)
        for layer in range(self.layers):
            L.sws_decode_init_cache(self.h, self.k_cache[layer], self.seq_lens, self.k_psum[layer],
                                    self.k_sketch[layer], stream)

    def begin_step(self, stream=None):
        L.sws_decode_advance(self.h, self.seq_lens, stream)

    def layer(self, layer: int, q_tok, k_tok, v_tok, out=None, stream=None):
        L.sws_decode_step(self.h, q_tok, k_tok, v_tok, self.seq_lens, self.k_cache[layer], self.v_cache[layer],
                          self.k_psum[layer], self.k_sketch[layer], layer == 0, self.walk_state, self.head_sel,
                          self.head_cnt, self.sel, self.sel_mask, self.sel_cnt, stream)
        o = self.o if out is None else out
        L.sws_sparse_attn_decode(self.h, q_tok, self.k_cache[layer], self.v_cache[layer], self.seq_lens, self.sel,
                                 self.sel_mask, self.sel_cnt, o, self.ws, stream)
        return o

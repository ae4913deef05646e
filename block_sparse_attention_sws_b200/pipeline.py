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
    the walk state still runs through them.

    ``scores_in_memory`` = True (the default) has sws_sketch write the
    [hq, b, b] score matrix (``self.scores``) and sws_walk_select walk on it:
    the faster route at every measured size. False skips the matrix (and its
    memory): sws_sketch writes only the sketches and sws_walk_select_sketch
    forms the scores on chip."""

    def __init__(self, handle: L.Handle, n: int, hq: int, hkv: int, dtype=torch.bfloat16, device="cuda",
                 dense_layers: int = 0, scores_in_memory: bool = True):
        cfg = handle.cfg
        self.dense_layers = dense_layers
        self.scores_in_memory = scores_in_memory
        self.h, self.n, self.hq, self.hkv = handle, n, hq, hkv
        self.b = L.sws_num_blocks(cfg, n)
        self.nnz = L.sws_csr_nnz(cfg, n)
        k, d = cfg.sketch_dim, cfg.head_dim
        f64 = dict(dtype=torch.float64, device=device)
        self.q_sk = torch.empty(hq, self.b, k, **f64)
        self.k_sk = torch.empty(hkv, self.b, k, **f64)
        self.scores = torch.empty(hq, self.b, self.b, **f64) if scores_in_memory else None
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
        if self.scores_in_memory:
            L.sws_walk_select(h, self.scores, self.n, first_layer, self.walk_state, rp, ci, self.ws, stream)
        else:
            L.sws_walk_select_sketch(h, self.q_sk, self.k_sk, self.n, first_layer, self.walk_state, rp, ci, self.ws,
                                     stream)

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


class PrefillBatch:
    """Prefill of several sequences of different lengths through one handle.

    Each sequence keeps its own PrefillPath (its own walk state and CSR).
    ``layer`` issues every sequence's sketch, walk and attention on a stream of
    its own, all ordered after the caller's stream and joined back into it, so
    the kernels of short sequences overlap on the GPU. ``layer_packed`` takes
    the sequences end to end along the token axis: the sketches and walks run
    per sequence on those streams, then one attention launch covers them all
    (sws_sparse_attn_prefill_varlen). Results equal those of the sequences run
    one by one, bit for bit (tests/test_gpu_prefill.py)."""

    def __init__(self, handle: L.Handle, lengths, hq: int, hkv: int, dtype=torch.bfloat16, device="cuda",
                 dense_layers: int = 0):
        self.paths = [PrefillPath(handle, int(n), hq, hkv, dtype, device, dense_layers) for n in lengths]
        self.streams = [torch.cuda.Stream(device=device) for _ in lengths]
        self.cu_seqlens = [0]
        for n in lengths:
            self.cu_seqlens.append(self.cu_seqlens[-1] + int(n))
        self.hq, self.dtype, self.device = hq, dtype, device
        self.ws_var = None
        self.o_packed = None

    def layer_packed(self, q, k, v, first_layer: bool, out=None, layer=None):
        """q [hq, N, d], k, v [hkv, N, d]: sequence i on tokens cu_seqlens[i] ..
        cu_seqlens[i + 1] - 1. Returns the packed output [hq, N, d] (a buffer of
        the batch unless ``out``)."""
        cu = self.cu_seqlens
        cur = torch.cuda.current_stream()
        ready = torch.cuda.Event()
        ready.record(cur)
        for i, (p, st) in enumerate(zip(self.paths, self.streams)):
            st.wait_event(ready)
            a, z = cu[i], cu[i + 1]
            p.sketch(q[:, a:z], k[:, a:z], st)
            p.walk_select(first_layer, st, layer)
        for st in self.streams:
            cur.wait_stream(st)
        if self.ws_var is None:
            nb = L.sws_sparse_attn_prefill_varlen_ws_bytes(cu)
            self.ws_var = torch.empty(max(nb, 16), dtype=torch.uint8, device=self.device)
        o = out
        if o is None:
            if self.o_packed is None:
                self.o_packed = torch.empty(self.hq, cu[-1], q.shape[2], dtype=self.dtype, device=self.device)
            o = self.o_packed
        p0 = self.paths[0]
        h = p0.h_dense if p0._dense(layer) else p0.h
        csrs = [p.csr(layer) for p in self.paths]
        L.sws_sparse_attn_prefill_varlen(h, q, k, v, cu, [c[0] for c in csrs], [c[1] for c in csrs], o, self.ws_var,
                                         cur)
        return o

    def layer(self, qs, ks, vs, first_layer: bool, outs=None, layer=None):
        """qs[i] [hq, n_i, d], ks[i], vs[i] [hkv, n_i, d]: layer inputs of sequence i.
        Returns the outputs [hq, n_i, d] (the paths' buffers unless ``outs``)."""
        cur = torch.cuda.current_stream()
        ready = torch.cuda.Event()
        ready.record(cur)
        res = []
        for i, (p, st) in enumerate(zip(self.paths, self.streams)):
            st.wait_event(ready)
            o = None if outs is None else outs[i]
            res.append(p.layer(qs[i], ks[i], vs[i], first_layer, out=o, stream=st, layer=layer))
        for st in self.streams:
            cur.wait_stream(st)
        return res


class DecodePath:
    """Per-layer decode state and the per-step call order:
    sws_decode_step -> sws_sparse_attn_decode for each layer, then
    sws_decode_advance once the step's layers are done.

    exact=True selects with the exact decode walk (sws_decode_step_exact): the
    row of the new token's block in the prefill recurrence, which needs the
    prompt's query sketches (init_queries) next to the key sketches.
    exact="rows" is the same walk for contexts of any length: each layer's
    block attention rows are kept in device memory (init_rows builds them once
    the key and query sketches are in place) and the steps call
    sws_decode_step_exact_rows.

    paged=True keeps each layer's keys and values in a pool of pages
    [num_pages, hkv, B, d] addressed through block_table [batch, max_blocks]
    (shared by the layers) and calls the *_paged entry points. The default
    table gives sequence i the pages i * max_blocks .. (i + 1) * max_blocks - 1;
    a caller may overwrite self.block_table with any assignment of distinct
    pages before writing the caches."""

    def __init__(self, handle: L.Handle, batch: int, hq: int, hkv: int, max_len: int, layers: int, device="cuda",
                 paged=False, num_pages=None, exact=False):
        cfg = handle.cfg
        self.h, self.batch, self.hq, self.hkv, self.max_len, self.layers = handle, batch, hq, hkv, max_len, layers
        d, k, B = cfg.head_dim, cfg.sketch_dim, cfg.block_size
        self.mb = L.sws_num_blocks(cfg, max_len)
        self.paged = paged
        bf = dict(dtype=torch.bfloat16, device=device)
        f64 = dict(dtype=torch.float64, device=device)
        i32 = dict(dtype=torch.int32, device=device)
        if paged:
            self.num_pages = batch * self.mb if num_pages is None else num_pages
            self.block_table = torch.arange(batch * self.mb, **i32).reshape(batch, self.mb) % self.num_pages
            self.k_cache = [torch.empty(self.num_pages, hkv, B, d, **bf) for _ in range(layers)]
            self.v_cache = [torch.empty(self.num_pages, hkv, B, d, **bf) for _ in range(layers)]
            self.max_len = self.mb * B
        else:
            self.k_cache = [torch.empty(batch, hkv, max_len, d, **bf) for _ in range(layers)]
            self.v_cache = [torch.empty(batch, hkv, max_len, d, **bf) for _ in range(layers)]
        self.k_psum = [torch.zeros(batch, hkv, d, **f64) for _ in range(layers)]
        self.k_sketch = [torch.zeros(batch, hkv, self.mb, k, **f64) for _ in range(layers)]
        self.exact = exact
        if exact:  # the exact walk's cached query sketches (see init_queries)
            assert not paged, "the exact walk runs on the contiguous cache"
            self.q_psum = [torch.zeros(batch, hq, d, **f64) for _ in range(layers)]
            self.q_sketch = [torch.zeros(batch, hq, self.mb, k, **f64) for _ in range(layers)]
        self.rows = None
        if exact == "rows":
            e = L.sws_decode_exact_rows_entries(cfg, max_len)
            self.rows = [torch.zeros(batch, hq, e, dtype=torch.int32, device=device) for _ in range(layers)]
        self.seq_lens = torch.zeros(batch, **i32)
        self.walk_state = torch.zeros(batch, hq, self.mb, **f64)
        self.head_sel = torch.zeros(batch, hq, self.mb, **i32)
        self.head_cnt = torch.zeros(batch, hq, **i32)
        self.sel = torch.zeros(batch, hkv, self.mb, **i32)
        self.sel_mask = torch.zeros(batch, hkv, self.mb, dtype=torch.uint8, device=device)
        self.sel_cnt = torch.zeros(batch, hkv, **i32)
        ws = L.sws_workspace_size(cfg, L.SWS_OP_DECODE_ATTN, self.max_len, hq, hkv, batch)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.o = torch.empty(batch, hq, d, **bf)

    @staticmethod
    def _scatter_pages(pool, pages, src, n: int, B: int):
        # tokens [0, n) of src [hkv, >= n, d] to the pages of their blocks
        nf, r = divmod(n, B)
        if nf:
            pool[pages[:nf]] = src[:, :nf * B].reshape(src.shape[0], nf, B, -1).transpose(0, 1)
        if r:
            pool[pages[nf], :, :r] = src[:, nf * B:n]

    def write_cache(self, layer: int, seq: int, k, v, n: int):
        """Store the first n tokens of k, v [hkv, >= n, d] as sequence seq's cache."""
        if not self.paged:
            self.k_cache[layer][seq, :, :n] = k[:, :n]
            self.v_cache[layer][seq, :, :n] = v[:, :n]
            return
        pages = self.block_table[seq].long()
        B = self.h.cfg.block_size
        self._scatter_pages(self.k_cache[layer], pages, k, n, B)
        self._scatter_pages(self.v_cache[layer], pages, v, n, B)

    def to_paged(self, block_table: torch.Tensor, num_pages: int):
        """Move contiguous caches into page pools (every token slot, one layer
        and one of K, V at a time, so that about one layer's cache is the extra
        memory); block_table [batch, max_blocks] int32 on the device, distinct
        pages in [0, num_pages). Sketches and lengths are kept."""
        assert not self.paged and tuple(block_table.shape) == (self.batch, self.mb)
        B, d = self.h.cfg.block_size, self.h.cfg.head_dim
        pages = block_table.long()
        for caches in (self.k_cache, self.v_cache):
            for layer in range(self.layers):
                src = caches[layer]
                pool = torch.empty(num_pages, self.hkv, B, d, dtype=src.dtype, device=src.device)
                for i in range(self.batch):
                    self._scatter_pages(pool, pages[i], src[i], self.max_len, B)
                caches[layer] = pool
                del src
        self.paged, self.block_table, self.num_pages = True, block_table, num_pages
        self.max_len = self.mb * B

    def init_cache(self, lens: torch.Tensor, stream=None):
        """Caches already hold lens[i] tokens per sequence: build their sketches."""
        self.seq_lens.copy_(lens)
        for layer in range(self.layers):
            if self.paged:
                L.sws_decode_init_cache_paged(self.h, self.k_cache[layer], self.block_table, self.seq_lens,
                                              self.k_psum[layer], self.k_sketch[layer], stream)
            else:
                L.sws_decode_init_cache(self.h, self.k_cache[layer], self.seq_lens, self.k_psum[layer],
                                        self.k_sketch[layer], stream)

    def init_queries(self, layer: int, q_prompt, stream=None):
        """Exact walk: the prompt's queries q_prompt [batch, hq, max_len, d] bf16
        (rows below the lengths given to init_cache are read) give every cached
        block's q~ and the last block's query sum, as a prefill would."""
        assert self.exact and tuple(q_prompt.shape[:3]) == (self.batch, self.hq, self.max_len)
        L.sws_decode_init_cache(self.h, q_prompt, self.seq_lens, self.q_psum[layer], self.q_sketch[layer], stream)

    def init_rows(self, stream=None):
        """Exact walk with stored rows: every layer's block attention rows from
        the key sketches (init_cache) and query sketches (init_queries)."""
        assert self.rows is not None
        for layer in range(self.layers):
            L.sws_decode_exact_rows_init(self.h, self.q_sketch[layer], self.k_sketch[layer], self.seq_lens,
                                         self.rows[layer], stream)

    def begin_step(self, stream=None):
        L.sws_decode_advance(self.h, self.seq_lens, stream)

    def layer(self, layer: int, q_tok, k_tok, v_tok, out=None, stream=None):
        o = self.o if out is None else out
        if self.exact == "rows":
            L.sws_decode_step_exact_rows(self.h, q_tok, k_tok, v_tok, self.seq_lens, self.k_cache[layer],
                                         self.v_cache[layer], self.k_psum[layer], self.k_sketch[layer],
                                         self.q_psum[layer], self.q_sketch[layer], self.rows[layer], layer == 0,
                                         self.walk_state, self.head_sel, self.head_cnt, self.sel, self.sel_mask,
                                         self.sel_cnt, stream)
            L.sws_sparse_attn_decode(self.h, q_tok, self.k_cache[layer], self.v_cache[layer], self.seq_lens,
                                     self.sel, self.sel_mask, self.sel_cnt, o, self.ws, stream)
            return o
        if self.exact:
            L.sws_decode_step_exact(self.h, q_tok, k_tok, v_tok, self.seq_lens, self.k_cache[layer],
                                    self.v_cache[layer], self.k_psum[layer], self.k_sketch[layer], self.q_psum[layer],
                                    self.q_sketch[layer], layer == 0, self.walk_state, self.head_sel, self.head_cnt,
                                    self.sel, self.sel_mask, self.sel_cnt, stream)
            L.sws_sparse_attn_decode(self.h, q_tok, self.k_cache[layer], self.v_cache[layer], self.seq_lens,
                                     self.sel, self.sel_mask, self.sel_cnt, o, self.ws, stream)
            return o
        if self.paged:
            L.sws_decode_step_paged(self.h, q_tok, k_tok, v_tok, self.k_cache[layer], self.v_cache[layer],
                                    self.block_table, self.seq_lens, self.k_psum[layer], self.k_sketch[layer],
                                    layer == 0, self.walk_state, self.head_sel, self.head_cnt, self.sel,
                                    self.sel_mask, self.sel_cnt, stream)
            L.sws_sparse_attn_decode_paged(self.h, q_tok, self.k_cache[layer], self.v_cache[layer], self.block_table,
                                           self.seq_lens, self.sel, self.sel_mask, self.sel_cnt, o, self.ws, stream)
            return o
        L.sws_decode_step(self.h, q_tok, k_tok, v_tok, self.seq_lens, self.k_cache[layer], self.v_cache[layer],
                          self.k_psum[layer], self.k_sketch[layer], layer == 0, self.walk_state, self.head_sel,
                          self.head_cnt, self.sel, self.sel_mask, self.sel_cnt, stream)
        L.sws_sparse_attn_decode(self.h, q_tok, self.k_cache[layer], self.v_cache[layer], self.seq_lens, self.sel,
                                 self.sel_mask, self.sel_cnt, o, self.ws, stream)
        return o

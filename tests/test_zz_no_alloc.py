"""The decode attention call that allocates nothing.

Some callers cannot allocate device memory where they run decode attention: a
plug-in whose host framework owns every device allocation, a serving loop that
may not pay an allocation's latency and synchronisation on each token, code
held to a memory budget fixed in advance. sws_sparse_attn_decode_noalloc serves
them: it keeps its split-KV partial results in a scratch array built into the
library instead of a workspace the caller passes. These checks run it through
the C ABI and compare it with the workspace form on the same inputs, on two
calls in a row. Both forms run the same kernels with the same split count, so
their outputs are equal bit for bit (which is stricter than the attention
tolerances the other tests use).

This file sorts last so that a run stopping at its first failure has already
run every other test; it needs nothing from them and also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_sws_b200 as S
import sws_inputs as W
from parity import ATTN_MAX_ABS, ATTN_MEAN_ABS

pytestmark = pytest.mark.gpu


def _decode_state(layers=2):
    """A small ragged decode batch, stepped once, with each layer's selection made."""
    w = W.DECODE_128K.scaled(layers=layers, hq=8, hkv=2, hubs=4)
    n0s = [1000, 1500, 638]
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    max_len = max(n0s) + 1
    path = S.DecodePath(h, len(n0s), w.hq, w.hkv, max_len, layers)
    toks = []
    for layer in range(layers):
        qs, ks, vs = [], [], []
        for i, n0 in enumerate(n0s):
            wi = w.scaled(n0=n0, steps=1)
            K, V = W.decode_cache_inputs(wi, i, layer, "cuda")
            path.k_cache[layer][i, :, :n0] = K[:, :n0]
            path.v_cache[layer][i, :, :n0] = V[:, :n0]
            qs.append(W.decode_queries(wi, i, layer, "cuda")[:, 0])
            ks.append(K[:, n0])
            vs.append(V[:, n0])
        toks.append((torch.stack(qs).contiguous(), torch.stack(ks).contiguous(), torch.stack(vs).contiguous()))
    path.init_cache(torch.tensor(n0s, dtype=torch.int32, device="cuda"))
    path.begin_step()
    return h, path, toks


def _same(a, b):
    assert torch.isfinite(a.float()).all()
    d = (a.float() - b.float()).abs()
    assert d.max().item() <= ATTN_MAX_ABS and d.mean().item() <= ATTN_MEAN_ABS
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_noalloc_matches_workspace_form_on_consecutive_calls():
    h, path, toks = _decode_state()
    outs = []
    for layer, (q, k, v) in enumerate(toks):
        S.sws_decode_step(h, q, k, v, path.seq_lens, path.k_cache[layer], path.v_cache[layer], path.k_psum[layer],
                          path.k_sketch[layer], layer == 0, path.walk_state, path.head_sel, path.head_cnt, path.sel,
                          path.sel_mask, path.sel_cnt)
        o_ws = torch.empty_like(path.o)
        S.sws_sparse_attn_decode(h, q, path.k_cache[layer], path.v_cache[layer], path.seq_lens, path.sel,
                                 path.sel_mask, path.sel_cnt, o_ws, path.ws)
        o_na = torch.full_like(path.o, float("nan"))
        S.sws_sparse_attn_decode_noalloc(h, q, path.k_cache[layer], path.v_cache[layer], path.seq_lens, path.sel,
                                         path.sel_mask, path.sel_cnt, o_na)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        _same(o_na, o_ws)
        outs.append((o_ws, o_na))
    # the two calls saw different selections and queries
    assert not torch.equal(outs[0][1], outs[1][1])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Partials beyond SWS_NOALLOC_SCRATCH_BYTES are refused on the host, before any launch."""
    cfg = S.make_config(128, 64, 32, 8, 0, (1, 5), 4)
    h = S.Handle(cfg)
    batch, hq, hkv, max_len = 64, 32, 8, 131136
    need = S.sws_workspace_size(cfg, S.SWS_OP_DECODE_ATTN, max_len, hq, hkv, batch)
    assert need > S.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(64, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    lib = S.load()
    s = lib.sws_sparse_attn_decode_noalloc(h.ptr, p, p, p, batch, hq, hkv, max_len, p, p, p, p, p, None)
    assert s == S.SWS_ERR_WORKSPACE


def test_noalloc_at_its_largest_batch():
    """A real call whose partials fill the built-in scratch as far as whole
    sequences can: 8 query heads on one KV head, d = 64, 1024-token caches at
    density 1/1 (one split per head), so each sequence takes 8 x (64 + 2) x 4
    bytes and 15887 sequences leave less than one sequence's worth unused. The
    next larger batch is refused; the call that fits matches the workspace form
    bit for bit, twice in a row."""
    hq, hkv, d, B, max_len = 8, 1, 64, 64, 1024
    cfg = S.make_config(d, B, 16, 8, 0, (1, 1), 4)
    h = S.Handle(cfg)
    per_seq = S.sws_workspace_size(cfg, S.SWS_OP_DECODE_ATTN, max_len, hq, hkv, 1)
    assert per_seq == hq * 1 * (d + 2) * 4
    batch = S.NOALLOC_SCRATCH_BYTES // per_seq
    assert S.NOALLOC_SCRATCH_BYTES - batch * per_seq < per_seq
    assert S.sws_workspace_size(cfg, S.SWS_OP_DECODE_ATTN, max_len, hq, hkv, batch) == batch * per_seq
    dev = "cuda"
    g = torch.Generator(device=dev)
    g.manual_seed(31)
    kc = torch.randn(batch, hkv, max_len, d, generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn(batch, hkv, max_len, d, generator=g, device=dev).to(torch.bfloat16)
    lens = torch.randint(1, max_len + 1, (batch,), generator=g, device=dev, dtype=torch.int32)
    mb = max_len // B
    # density 1/1: every head takes every block below its length; the union is the same
    nb = (lens + B - 1) // B
    sel = torch.arange(mb, device=dev, dtype=torch.int32).repeat(batch, hkv, 1).contiguous()
    sel_mask = torch.where(sel < nb[:, None, None], 255, 0).to(torch.uint8).contiguous()
    sel_cnt = nb[:, None].repeat(1, hkv).to(torch.int32).contiguous()
    ws = torch.empty(batch * per_seq, dtype=torch.uint8, device=dev)
    for call in range(2):
        q = torch.randn(batch, hq, d, generator=g, device=dev).to(torch.bfloat16)
        o_ws = torch.empty(batch, hq, d, dtype=torch.bfloat16, device=dev)
        o_na = torch.full_like(o_ws, float("nan"))
        S.sws_sparse_attn_decode(h, q, kc, vc, lens, sel, sel_mask, sel_cnt, o_ws, ws)
        S.sws_sparse_attn_decode_noalloc(h, q, kc, vc, lens, sel, sel_mask, sel_cnt, o_na)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        _same(o_na, o_ws)
    lib = S.load()
    p = ctypes.c_void_p(q.data_ptr())
    s = lib.sws_sparse_attn_decode_noalloc(h.ptr, p, p, p, batch + 1, hq, hkv, max_len, p, p, p, p, p, None)
    assert s == S.SWS_ERR_WORKSPACE
    h.close()

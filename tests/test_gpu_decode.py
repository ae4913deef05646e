"""Parity of the decode path (sws_decode_step, sws_sparse_attn_decode) against
the oracle, through the C ABI, on seeded synthetic caches.

Every step appends one token per sequence; every layer's selection (each
head's blocks, the log-domain walk state, the GQA union and its head mask)
and its attention output are compared with the oracle for the checked
sequences. Cache slots beyond a sequence's length hold NaN, so any read of a
token that should be masked shows up in the output.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_sws_b200 as S
import oracle
import sws_inputs as W
from oracle import sws_oracle as so
from parity import compare_attention, compare_selection, record_ties

pytestmark = pytest.mark.gpu


def make_path(h, w, batch, max_len, paged, dev="cuda"):
    """A decode path; paged: the pool has a few spare pages and each sequence's
    blocks sit on pages in a seeded random order."""
    if not paged:
        return S.DecodePath(h, batch, w.hq, w.hkv, max_len, w.layers, dev)
    mb = -(-max_len // w.B)
    path = S.DecodePath(h, batch, w.hq, w.hkv, max_len, w.layers, dev, paged=True, num_pages=batch * mb + 5)
    perm = torch.randperm(batch * mb + 5, generator=torch.Generator().manual_seed(w.seed + 77))[:batch * mb]
    path.block_table.copy_(perm.reshape(batch, mb).to(torch.int32))
    return path


def run_decode(w: W.DecodeWorkload, n0s, steps, check_seqs=None, shared=False, paged=False, path_out=None):
    dev = "cuda"
    batch = len(n0s)
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed, select_group=(w.hq // w.hkv) if shared else 0)
    h = S.Handle(cfg)
    max_len = max(n0s) + steps
    path = make_path(h, w, batch, max_len, paged, dev)
    group = w.hq // w.hkv
    check_seqs = list(range(batch)) if check_seqs is None else list(check_seqs)
    KV, Qs = {}, {}
    for layer in range(w.layers):
        path.k_cache[layer].fill_(float("nan"))
        path.v_cache[layer].fill_(float("nan"))
        for s_, n0 in enumerate(n0s):
            ws_ = w.scaled(n0=n0, steps=steps)
            K, V = W.decode_cache_inputs(ws_, s_, layer, dev)
            path.write_cache(layer, s_, K, V, n0)
            KV[(s_, layer)] = (K, V)
            Qs[(s_, layer)] = W.decode_queries(ws_, s_, layer, dev)
    path.init_cache(torch.tensor(n0s, dtype=torch.int32, device=dev))
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)
    host = {key: (K.double().cpu().numpy(), V.double().cpu().numpy()) for key, (K, V) in KV.items()
            if key[0] in check_seqs}
    swaps = []
    outputs = []
    for t in range(steps):
        path.begin_step()
        rho_prev = {s_: None for s_ in check_seqs}
        for layer in range(w.layers):
            q_tok = torch.stack([Qs[(s_, layer)][:, t] for s_ in range(batch)]).contiguous()
            k_tok = torch.stack([KV[(s_, layer)][0][:, n0s[s_] + t] for s_ in range(batch)]).contiguous()
            v_tok = torch.stack([KV[(s_, layer)][1][:, n0s[s_] + t] for s_ in range(batch)]).contiguous()
            o = path.layer(layer, q_tok, k_tok, v_tok)
            torch.cuda.synchronize()
            assert S.sws_sync_check(h) == 0
            hs = path.head_sel.cpu().numpy()
            hc = path.head_cnt.cpu().numpy()
            rho_gpu = path.walk_state.cpu().numpy()
            sel = path.sel.cpu().numpy()
            msk = path.sel_mask.cpu().numpy()
            cnt = path.sel_cnt.cpu().numpy()
            og = o.float().cpu().numpy()
            outputs.append((hs.copy(), hc.copy(), rho_gpu.copy(), sel.copy(), msk.copy(), cnt.copy(),
                            o.view(torch.int16).cpu().numpy()))
            for s_ in check_seqs:
                length = n0s[s_] + t + 1
                nb = -(-length // w.B)
                Kh, Vh = host[(s_, layer)]
                q = Qs[(s_, layer)][:, t].double().cpu().numpy()
                rho, z, osel = so.decode_layer_select(q, Kh, length, Hd, w.B, w.s, w.density, rho_prev[s_],
                                                      select="group_shared" if shared else "per_head")
                rho_prev[s_] = rho
                assert np.allclose(rho_gpu[s_, :, :nb], rho, rtol=1e-9, atol=1e-9 * np.abs(rho).max())
                union = {}
                for hh in range(w.hq):
                    tau = hc[s_, hh]
                    gsel = hs[s_, hh, :tau]
                    assert tau == so.tau_of_row(nb - 1, *w.density)
                    assert np.all(np.diff(gsel) > 0) and gsel.max() < nb
                    g0 = (hh // group) * group
                    score = so.group_shared_log_rows(rho[g0:g0 + group]) if shared else rho[hh]
                    swaps += [(t, layer, s_, hh) + x for x in compare_selection(gsel, osel[hh], score,
                                                                                 log_domain=True)]
                    for j in gsel:
                        union[int(j)] = union.get(int(j), 0) | (1 << (hh % group))
                    g = hh // group
                    want = so.decode_attention(q[hh], Kh[g], Vh[g], length, gsel, w.B)
                    compare_attention(og[s_, hh], want)
                for g in range(w.hkv):
                    u = {j: m >> 0 for j, m in union.items()}
                    # union of this KV head's group only
                    ug = {}
                    for hh in range(g * group, (g + 1) * group):
                        for j in hs[s_, hh, :hc[s_, hh]]:
                            ug[int(j)] = ug.get(int(j), 0) | (1 << (hh - g * group))
                    n = cnt[s_, g]
                    assert n == len(ug)
                    assert list(sel[s_, g, :n]) == sorted(ug)
                    assert [int(m) for m in msk[s_, g, :n]] == [ug[j] for j in sorted(ug)]
    if path_out is not None:
        path_out.extend(outputs)
    record_ties(swaps, compared=steps * w.layers * len(check_seqs) * w.hq)
    h.close()
    return swaps


def test_decode_small_ragged():
    """Three sequences of different lengths with partial blocks, crossing a block boundary."""
    w = W.DECODE_128K.scaled(layers=3, hq=8, hkv=2, hubs=4)
    swaps = run_decode(w, [1000, 1500, 638], steps=5)


def test_decode_group_sizes():
    for hq, hkv in ((4, 4), (4, 2), (8, 1)):
        w = W.DECODE_128K.scaled(layers=2, hq=hq, hkv=hkv, hubs=3)
        run_decode(w, [700, 333], steps=3)


def test_decode_dense_density():
    w = W.DECODE_128K.scaled(layers=2, hq=4, hkv=1, hubs=2, density=(1, 1))
    run_decode(w, [500], steps=2)


def test_decode_first_token_of_block():
    """n0 a multiple of B: the first decode token opens a new block holding only itself."""
    w = W.DECODE_128K.scaled(layers=2, hq=4, hkv=1, hubs=2)
    run_decode(w, [1024, 64], steps=2)


@pytest.mark.parametrize("d,B,k", [(64, 64, 16), (128, 128, 32), (64, 128, 16)])
@pytest.mark.parametrize("paged", [False, True])
def test_decode_head_dim_and_block_size(d, B, k, paged):
    """The other instantiations of the decode kernels: head dim 64 and block
    size 128, contiguous and paged. The first sequence's steps cross a block
    boundary of either size (766 + 3 > 768); the last holds one full block of
    64 and a partial one, or a partial second block of 128."""
    w = W.DECODE_128K.scaled(layers=2, hq=8, hkv=2, hubs=3, d=d, B=B, k=k)
    swaps = run_decode(w, [766, 1200, 130], steps=3, paged=paged)


def test_decode_full_size_sampled():
    """The full decode workload (16 sequences, 131072 cached tokens, 8 layers)
    for a few steps; the oracle recomputes two sampled sequences."""
    w = W.DECODE_128K
    swaps = run_decode(w, [w.n0] * w.batch, steps=2, check_seqs=[0, w.batch - 1])


def test_decode_bad_length_guard():
    """A sequence length beyond the cache is rejected by the kernel's own check
    and reported through the device error word."""
    w = W.DECODE_128K.scaled(layers=1, hq=4, hkv=1)
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    path = S.DecodePath(h, 1, 4, 1, 256, 1)
    path.k_cache[0].zero_()
    path.v_cache[0].zero_()
    path.init_cache(torch.tensor([10], dtype=torch.int32, device="cuda"))
    assert S.sws_sync_check(h) == 0
    path.seq_lens.fill_(999)
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 1, 128, dtype=torch.bfloat16, device="cuda")
    L = S
    L.sws_decode_step(h, q, kv, kv, path.seq_lens, path.k_cache[0], path.v_cache[0], path.k_psum[0],
                      path.k_sketch[0], True, path.walk_state, path.head_sel, path.head_cnt, path.sel, path.sel_mask,
                      path.sel_cnt)
    assert S.sws_sync_check(h) == 4  # GUARD_BAD_LEN


def test_decode_group_shared_selection():
    """Group-shared selection: the group's heads get one set of blocks (the
    top-tau of the log-sum-exp of their rho rows), the union is that set with
    every head's bit, and attention matches the oracle on it."""
    w = W.DECODE_128K.scaled(layers=3, hq=8, hkv=2, hubs=4)
    swaps = run_decode(w, [1000, 1500, 638], steps=4, shared=True)


def test_decode_paged_cache():
    """The paged pool (blocks on shuffled pages, spare pages, NaN in every
    unwritten slot) against the oracle, ragged lengths crossing block ends."""
    w = W.DECODE_128K.scaled(layers=3, hq=8, hkv=2, hubs=4)
    swaps = run_decode(w, [1000, 1500, 638], steps=5, paged=True)


def test_decode_paged_equals_contiguous_bitwise():
    """The same caches and tokens through the contiguous and the paged calls:
    every selection, walk state and attention output is bit-identical."""
    w = W.DECODE_128K.scaled(layers=2, hq=8, hkv=2, hubs=4)
    outs = {}
    for paged in (False, True):
        outs[paged] = []
        run_decode(w, [900, 1300, 64], steps=3, check_seqs=[], paged=paged, path_out=outs[paged])
    assert len(outs[False]) == len(outs[True]) == 6
    for a, b in zip(outs[False], outs[True]):
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_decode_paged_bad_page_guard():
    """A block table entry outside the pool is not dereferenced: the kernels
    record guard code 6 and the context stays usable."""
    w = W.DECODE_128K.scaled(layers=1, hq=4, hkv=1)
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    path = S.DecodePath(h, 1, 4, 1, 256, 1, paged=True)
    path.k_cache[0].zero_()
    path.v_cache[0].zero_()
    path.init_cache(torch.tensor([100], dtype=torch.int32, device="cuda"))
    assert S.sws_sync_check(h) == 0
    path.block_table[0, 1] = path.num_pages  # one past the pool
    path.init_cache(torch.tensor([100], dtype=torch.int32, device="cuda"))
    assert S.sws_sync_check(h) == 6  # GUARD_BAD_PAGE
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 1, 128, dtype=torch.bfloat16, device="cuda")
    path.begin_step()
    path.layer(0, q, kv, kv)  # the token goes to block 1: not appended
    assert S.sws_sync_check(h) == 6
    path.block_table[0, 1] = -3
    path.sel[0, 0, 0] = 1
    path.sel_mask[0, 0, 0] = 1
    path.sel_cnt[0, 0] = 1
    S.sws_sparse_attn_decode_paged(h, q, path.k_cache[0], path.v_cache[0], path.block_table, path.seq_lens,
                                   path.sel, path.sel_mask, path.sel_cnt, path.o, path.ws)
    assert S.sws_sync_check(h) == 6
    path.block_table[0, 1] = 1
    path.init_cache(torch.tensor([100], dtype=torch.int32, device="cuda"))
    assert S.sws_sync_check(h) == 0  # usable again
    # host validation: an empty pool, an empty table, a misaligned table queue nothing
    lib, P = S.load(), S._lib._ptr
    for num_pages, bt, mb in ((0, P(path.block_table), 4), (4, P(path.block_table), 0),
                              (4, P(path.block_table) + 4, 4)):
        assert lib.sws_decode_init_cache_paged(h.ptr, P(path.k_cache[0]), num_pages, bt, mb, 1, 1,
                                               P(path.seq_lens), P(path.k_psum[0]), P(path.k_sketch[0]),
                                               None) == S.SWS_ERR_INVALID_ARG
    h.close()

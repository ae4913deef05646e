"""Parity of the exact decode walk (sws_decode_step_exact) against the oracle.

The oracle runs the prefill recurrence of §4 on each sequence as it stands
after every step (prompt and decoded tokens, fresh walk state per step,
carried over the step's layers) and takes the newest block's row and its
top-tau (oracle.decode_exact_layer). The GPU carries that row across the
layers in walk_state, starting from the prompt's query sketches. Cache slots
beyond a sequence's length, and query rows beyond the prompt, hold NaN.

The GPU computes the block attention in fp32 (scores on fp32 FMA, exp, a
row sum in fp64) and the products in fp64. Every entry of A then carries a
relative error of about 1e-6 (the fp32 rounding of scores up to ~20), and
the row, a sum of positive terms, at most that much per product: s = 8
products over three layers stay below 3e-5. So the row is compared at a
relative 1e-4 (plus 1e-9 of its largest entry), its sum at 1e-5, and
selections must agree up to the near-ties of the shared tolerance.
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


def run_exact(w: W.DecodeWorkload, n0s, steps, shared=False, check_seqs=None):
    dev = "cuda"
    batch = len(n0s)
    group = w.hq // w.hkv
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed, select_group=group if shared else 0)
    h = S.Handle(cfg)
    max_len = max(n0s) + steps
    path = S.DecodePath(h, batch, w.hq, w.hkv, max_len, w.layers, dev, exact=True)
    check_seqs = list(range(batch)) if check_seqs is None else list(check_seqs)
    KV, Qs = {}, {}
    lens = torch.tensor(n0s, dtype=torch.int32, device=dev)
    for layer in range(w.layers):
        path.k_cache[layer].fill_(float("nan"))
        path.v_cache[layer].fill_(float("nan"))
        qp = torch.full((batch, w.hq, max_len, w.d), float("nan"), dtype=torch.bfloat16, device=dev)
        for s_, n0 in enumerate(n0s):
            ws_ = w.scaled(n0=n0, steps=steps)
            K, V = W.decode_cache_inputs(ws_, s_, layer, dev)
            Q = W.decode_sequence_queries(ws_, s_, layer, dev)
            path.write_cache(layer, s_, K, V, n0)
            qp[s_, :, :n0] = Q[:, :n0]
            KV[(s_, layer)] = (K, V)
            Qs[(s_, layer)] = Q
        path.seq_lens.copy_(lens)
        path.init_queries(layer, qp)
        del qp
    path.init_cache(lens)
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)
    host = {key: (K.double().cpu().numpy(), V.double().cpu().numpy(), Qs[key].double().cpu().numpy())
            for key, (K, V) in KV.items() if key[0] in check_seqs}
    swaps = []
    for t in range(steps):
        path.begin_step()
        states = {s_: so.PrefillState() for s_ in check_seqs}
        for layer in range(w.layers):
            q_tok = torch.stack([Qs[(s_, layer)][:, n0s[s_] + t] for s_ in range(batch)]).contiguous()
            k_tok = torch.stack([KV[(s_, layer)][0][:, n0s[s_] + t] for s_ in range(batch)]).contiguous()
            v_tok = torch.stack([KV[(s_, layer)][1][:, n0s[s_] + t] for s_ in range(batch)]).contiguous()
            o = path.layer(layer, q_tok, k_tok, v_tok)
            torch.cuda.synchronize()
            assert S.sws_sync_check(h) == 0
            hs = path.head_sel.cpu().numpy()
            hc = path.head_cnt.cpu().numpy()
            u_gpu = path.walk_state.cpu().numpy()
            sel = path.sel.cpu().numpy()
            msk = path.sel_mask.cpu().numpy()
            cnt = path.sel_cnt.cpu().numpy()
            og = o.float().cpu().numpy()
            for s_ in check_seqs:
                length = n0s[s_] + t + 1
                nb = -(-length // w.B)
                Kh, Vh, Qh = host[(s_, layer)]
                ref = so.decode_exact_layer(Qh[:, :length], Kh[:, :length], Hd, w.B, w.s, w.density, states[s_],
                                            select="group_shared" if shared else "per_head")
                ug = {}
                for hh in range(w.hq):
                    r = ref[hh]
                    row = u_gpu[s_, hh, :nb]
                    assert np.allclose(row, r["row"], rtol=1e-4, atol=1e-9 * np.abs(r["row"]).max()), (t, layer, hh)
                    assert abs(row.sum() - 1.0) < 1e-5
                    tau = hc[s_, hh]
                    gsel = hs[s_, hh, :tau]
                    assert tau == so.tau_of_row(nb - 1, *w.density)
                    assert np.all(np.diff(gsel) > 0) and gsel.max() < nb
                    swaps += [(t, layer, s_, hh) + x for x in compare_selection(gsel, r["blocks"], r["score"])]
                    g = hh // group
                    q = Qh[hh, length - 1]
                    compare_attention(og[s_, hh], so.decode_attention(q, Kh[g], Vh[g], length, gsel, w.B))
                    for j in gsel:
                        ug.setdefault((g, int(j)), 0)
                        ug[(g, int(j))] |= 1 << (hh % group)
                for g in range(w.hkv):
                    blocks = sorted(j for (gg, j) in ug if gg == g)
                    n = cnt[s_, g]
                    assert n == len(blocks)
                    assert list(sel[s_, g, :n]) == blocks
                    assert [int(m) for m in msk[s_, g, :n]] == [ug[(g, j)] for j in blocks]
    record_ties(swaps, compared=steps * w.layers * len(check_seqs) * w.hq)
    h.close()
    return swaps


def test_decode_exact_small_ragged():
    """Three sequences of different lengths, steps crossing a block boundary,
    three layers: the walk row, the selection, the union and attention."""
    w = W.DECODE_128K.scaled(layers=3, hq=8, hkv=2, hubs=4)
    swaps = run_exact(w, [1000, 1500, 638], steps=5)


def test_decode_exact_first_token_of_block():
    """n0 a multiple of B: the first decoded token opens a block of its own,
    whose query sketch is that token's projection."""
    w = W.DECODE_128K.scaled(layers=2, hq=4, hkv=1, hubs=2)
    run_exact(w, [1024, 64], steps=2)


def test_decode_exact_group_shared():
    """Exact walk with group-shared selection: the top-tau of the group's summed rows."""
    w = W.DECODE_128K.scaled(layers=2, hq=8, hkv=2, hubs=3)
    swaps = run_exact(w, [900, 1300], steps=3, shared=True)


@pytest.mark.parametrize("d,B,k", [(64, 64, 16), (64, 128, 16), (128, 128, 32)])
def test_decode_exact_head_dim_and_block_size(d, B, k):
    """The exact walk's other instantiation (head dim 64) and block size 128,
    with steps crossing a block boundary of either size."""
    w = W.DECODE_128K.scaled(layers=2, hq=8, hkv=2, hubs=3, d=d, B=B, k=k)
    swaps = run_exact(w, [766, 1200, 130], steps=3)


def test_decode_exact_16k_sampled():
    """The exact walk at a 16K context (257 blocks, the size its shared-memory
    triangle is built for), batch 4, two layers; one sequence checked."""
    w = W.DECODE_128K.scaled(layers=2, batch=4, hubs=8)
    run_exact(w, [16384, 16000, 9000, 12345], steps=2, check_seqs=[1])


def test_decode_exact_rejects_beyond_shared_memory():
    """Host validation: a cache whose block triangle does not fit is refused
    before any launch."""
    w = W.DECODE_128K.scaled(layers=1, hq=4, hkv=1)
    h = S.Handle(S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed))
    path = S.DecodePath(h, 1, 4, 1, 64 * 400, 1, exact=True)
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SwsError):
        path.layer(0, q, kv, kv)
    h.close()

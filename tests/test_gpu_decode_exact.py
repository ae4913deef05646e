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


class _Heads:
    """[heads, n, d] device tensor seen by the oracle one head at a time (fp64 numpy)."""

    def __init__(self, t):
        self.t, self.shape = t, tuple(t.shape)

    def __getitem__(self, h):
        return self.t[h].double().cpu().numpy()


def run_exact(w: W.DecodeWorkload, n0s, steps, shared=False, check_seqs=None, mode=True, check_heads=None):
    """mode True: sws_decode_step_exact (shared-memory triangle); "rows": the
    stored-rows walk (sws_decode_step_exact_rows). check_heads: the query heads
    compared with the oracle (all by default; a subset for the wide contexts)."""
    dev = "cuda"
    batch = len(n0s)
    group = w.hq // w.hkv
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed, select_group=group if shared else 0)
    h = S.Handle(cfg)
    max_len = max(n0s) + steps
    path = S.DecodePath(h, batch, w.hq, w.hkv, max_len, w.layers, dev, exact=mode)
    check_seqs = list(range(batch)) if check_seqs is None else list(check_seqs)
    heads = list(range(w.hq)) if check_heads is None else list(check_heads)
    if shared:  # a shared choice needs every head of a checked head's group
        heads = sorted({(hh // group) * group + r for hh in heads for r in range(group)})
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
            if s_ in check_seqs:
                KV[(s_, layer)] = (K, V)
                Qs[(s_, layer)] = Q
            else:  # only the tokens the steps append
                KV[(s_, layer)] = (K[:, n0:].clone(), V[:, n0:].clone())
                Qs[(s_, layer)] = Q[:, n0:].clone()
            del K, V, Q
        path.seq_lens.copy_(lens)
        path.init_queries(layer, qp)
        del qp
    path.init_cache(lens)
    if mode == "rows":
        path.init_rows()
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)

    def tok(s_, layer, kind, t):
        x = Qs[(s_, layer)] if kind == "q" else KV[(s_, layer)][0 if kind == "k" else 1]
        return x[:, (n0s[s_] if s_ in check_seqs else 0) + t]

    swaps = []
    for t in range(steps):
        path.begin_step()
        states = {s_: so.PrefillState() for s_ in check_seqs}
        for layer in range(w.layers):
            q_tok = torch.stack([tok(s_, layer, "q", t) for s_ in range(batch)]).contiguous()
            k_tok = torch.stack([tok(s_, layer, "k", t) for s_ in range(batch)]).contiguous()
            v_tok = torch.stack([tok(s_, layer, "v", t) for s_ in range(batch)]).contiguous()
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
                K, V = KV[(s_, layer)]
                Q = Qs[(s_, layer)]
                ref = so.decode_exact_layer(_Heads(Q[:, :length]), _Heads(K[:, :length]), Hd, w.B, w.s, w.density,
                                            states[s_], heads=heads, select="group_shared" if shared else "per_head")
                ug = {}
                for hh in heads:
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
                    q = Q[hh, length - 1].double().cpu().numpy()
                    Kg, Vg = K[g, :length].double().cpu().numpy(), V[g, :length].double().cpu().numpy()
                    compare_attention(og[s_, hh], so.decode_attention(q, Kg, Vg, length, gsel, w.B))
                    for j in gsel:
                        ug.setdefault((g, int(j)), 0)
                        ug[(g, int(j))] |= 1 << (hh % group)
                full_groups = {g for g in range(w.hkv) if all(g * group + r in heads for r in range(group))}
                for g in range(w.hkv):
                    n = cnt[s_, g]
                    got = {int(j): int(m) for j, m in zip(sel[s_, g, :n], msk[s_, g, :n])}
                    assert list(sel[s_, g, :n]) == sorted(got)
                    mine = {j: m for (gg, j), m in ug.items() if gg == g}
                    if g in full_groups:
                        assert got == mine
                    else:  # the checked heads' blocks are in the union with their bits
                        assert all(got.get(j, 0) & m == m for j, m in mine.items())
    record_ties(swaps, compared=steps * w.layers * len(check_seqs) * len(heads))
    h.close()
    return swaps


def test_decode_exact_small_ragged():
    """Three sequences of different lengths, steps crossing a block boundary,
    three layers: the walk row, the selection, the union and attention."""
    w = W.DECODE_128K.scaled(layers=3, hq=8, hkv=2, hubs=4)
    swaps = run_exact(w, [1000, 1500, 638], steps=5)


@pytest.mark.parametrize("shared", [False, True], ids=["per_head", "group_shared"])
def test_decode_exact_rows_small_ragged(shared):
    """The stored-rows walk on the same small ragged case: three sequences,
    steps crossing a block boundary, three layers."""
    w = W.DECODE_128K.scaled(layers=3, hq=8, hkv=2, hubs=4)
    run_exact(w, [1000, 1500, 638], steps=5, shared=shared, mode="rows")


def test_decode_exact_rows_first_token_of_block():
    w = W.DECODE_128K.scaled(layers=2, hq=4, hkv=1, hubs=2)
    run_exact(w, [1024, 64], steps=2, mode="rows")


@pytest.mark.parametrize("d,B,k", [(64, 64, 16), (128, 128, 32)])
def test_decode_exact_rows_head_dim_and_block_size(d, B, k):
    w = W.DECODE_128K.scaled(layers=2, hq=8, hkv=2, hubs=3, d=d, B=B, k=k)
    run_exact(w, [766, 1200, 130], steps=3, mode="rows")


def test_decode_exact_rows_s_beyond_one_sweep():
    """s = 11: the products take two sweeps over the stored rows (8 levels, then 3)."""
    w = W.DECODE_128K.scaled(layers=2, hq=4, hkv=1, hubs=3, s=11)
    run_exact(w, [2000, 700], steps=2, mode="rows")


def test_decode_exact_rows_matches_shared_memory_walk():
    """Where both fit (a 16K context), the stored-rows walk and the shared-memory
    walk give the same rows up to rounding and the same selections."""
    w = W.DECODE_128K.scaled(layers=2, hq=8, hkv=2, hubs=8, batch=2)
    n0s = [16000, 9000]
    outs = {}
    for mode in (True, "rows"):
        h = S.Handle(S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed))
        path = S.DecodePath(h, 2, w.hq, w.hkv, max(n0s) + 1, w.layers, exact=mode)
        lens = torch.tensor(n0s, dtype=torch.int32, device="cuda")
        toks = []
        for layer in range(w.layers):
            qp = torch.zeros(2, w.hq, path.max_len, w.d, dtype=torch.bfloat16, device="cuda")
            tl = []
            for s_, n0 in enumerate(n0s):
                ws_ = w.scaled(n0=n0, steps=1)
                K, V = W.decode_cache_inputs(ws_, s_, layer, "cuda")
                Q = W.decode_sequence_queries(ws_, s_, layer, "cuda")
                path.write_cache(layer, s_, K, V, n0)
                qp[s_, :, :n0] = Q[:, :n0]
                tl.append((Q[:, n0], K[:, n0], V[:, n0]))
            path.seq_lens.copy_(lens)
            path.init_queries(layer, qp)
            toks.append(tuple(torch.stack([x[c] for x in tl]).contiguous() for c in range(3)))
        path.init_cache(lens)
        if mode == "rows":
            path.init_rows()
        path.begin_step()
        res = []
        for layer in range(w.layers):
            path.layer(layer, *toks[layer])
            res.append((path.walk_state.clone(), path.head_sel.clone(), path.sel.clone(), path.sel_cnt.clone()))
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        outs[mode] = res
        h.close()
    for (ua, sa, ua_sel, ca), (ub, sb, ub_sel, cb) in zip(outs[True], outs["rows"]):
        nz = ua > 1e-300
        assert ((ua - ub).abs()[nz] / ua[nz]).max().item() < 1e-9
        assert torch.equal(sa, sb) and torch.equal(ca, cb) and torch.equal(ua_sel, ub_sel)


def test_decode_exact_rows_full_context_sampled():
    """The decode workload's context (131,072 cached tokens, 2049 blocks at
    B = 64, 32 query / 8 KV heads): the stored-rows walk over two layers, one
    step, two sequences; the oracle's exact recurrence checked on one sequence
    for the first and last query head."""
    w = W.DECODE_128K.scaled(layers=2, batch=2)
    run_exact(w, [w.n0, w.n0 - 1000], steps=1, check_seqs=[0], mode="rows", check_heads=[0, w.hq - 1])


def test_decode_exact_rows_at_the_largest_context():
    """The largest context the stored-rows walk takes: 2560 blocks of 64
    (163,840 tokens; the walk's shared memory at its limit), one sequence, four
    query heads of one KV head, two layers; the step's token is the last of
    the 2560th block. The first and last head against the oracle's exact
    recurrence, the union with their bits."""
    w = W.DECODE_128K.scaled(layers=2, batch=1, hq=4, hkv=1, hubs=4)
    n0 = 2560 * 64 - 1
    run_exact(w, [n0], steps=1, mode="rows", check_heads=[0, 3])


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

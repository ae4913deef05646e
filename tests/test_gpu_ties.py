"""Exact ties in the top-tau selection, on the GPU, through the C ABI.

The selection of §4 ("Scout Before You Attend", top-tau key blocks per query
block) keeps the tau largest walk scores of a row; where equal scores straddle
the cut, this library gives the places to the lower block indices (reading R6).
Seeded continuous inputs almost never produce exact ties, so these tests build
them on purpose:

* prefill: sketched scores whose rows repeat a few values along the columns,
  fed straight to sws_walk_select. With s = 1 (or the entrywise walk) the walk
  rows keep those ties exactly.
* decode: caches whose full blocks are copies of one block, so their sketched
  means, row logits and log-domain walk scores are equal bit for bit.

Each test first checks that the GPU's own scores do hold the ties, then that
its selection is the lower-index one (which a higher-index rule fails), and
then compares with the oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_sws_b200 as S
import oracle
import sws_inputs as W
from oracle import sws_oracle as so
from parity import compare_selection, record_ties

pytestmark = pytest.mark.gpu


def _higher_index_choice(row, tau):
    idx = np.arange(row.shape[0])
    return np.sort(np.lexsort((-idx, -row))[:tau])


def _tied_scores(hq, b, classes, seed):
    """Scores [hq, b, b]: column j of every row gets the value of class j % classes
    (one random value per class and head); NaN above the diagonal, which the
    call must not read."""
    r = np.random.default_rng(seed)
    c = r.standard_normal((hq, classes))
    j = np.arange(b)
    S_ = np.broadcast_to(c[:, j % classes][:, None, :], (hq, b, b)).copy()
    S_[:, ~np.tril(np.ones((b, b), dtype=bool))] = np.nan
    return S_


@pytest.mark.parametrize("mode,s,b,classes,density,group", [
    (S.SWS_WALK_MATRIX_POWER, 1, 256, 1, (1, 5), 0),    # constant rows: blocks 0..tau_i-1
    (S.SWS_WALK_MATRIX_POWER, 1, 256, 3, (1, 5), 0),
    (S.SWS_WALK_ELEMENTWISE, 8, 300, 4, (1, 10), 0),
    (S.SWS_WALK_MATRIX_POWER, 1, 1100, 3, (1, 5), 0),   # the general selection kernel (> 1024 blocks)
    (S.SWS_WALK_MATRIX_POWER, 1, 256, 3, (1, 5), 4),    # group-shared selection
], ids=["constant", "three_values", "elementwise_s8", "b1100", "group_shared"])
def test_prefill_selection_ties_go_to_lower_index(mode, s, b, classes, density, group):
    hq, hkv, B = 4, 1, 64
    n = b * B
    cfg = S.make_config(128, B, 32, s, mode, density, 7, select_group=group)
    h = S.Handle(cfg)
    scores = _tied_scores(hq, b, classes, seed=b + classes)
    dev = "cuda"
    sc = torch.from_numpy(scores).to(dev)
    R = torch.zeros(hq, b, b, dtype=torch.float64, device=dev)
    nnz = S.sws_csr_nnz(cfg, n)
    rp = torch.empty(hq, b + 1, dtype=torch.int32, device=dev)
    ci = torch.empty(hq, nnz, dtype=torch.int32, device=dev)
    ws = torch.empty(max(16, S.sws_workspace_size(cfg, S.SWS_OP_WALK_SELECT, n, hq, hkv)), dtype=torch.uint8,
                     device=dev)
    S.sws_walk_select(h, sc, n, True, R, rp, ci, ws)
    torch.cuda.synchronize()
    assert S.sws_sync_check(h) == 0
    Rg, rpg, cig = R.cpu().numpy(), rp.cpu().numpy(), ci.cpu().numpy()
    modename = "elementwise" if mode == S.SWS_WALK_ELEMENTWISE else "matrix_power"
    Ro = []
    for hh in range(hq):
        So = np.where(np.tril(np.ones((b, b), dtype=bool)), scores[hh], -np.inf)
        Ro.append(so.walk_update(None, so.walk_matrix(so.block_attention(So), s, modename)))
    score_rows = [so.group_shared_walk_rows(Ro[(hh // group) * group:(hh // group + 1) * group]) if group > 1
                  else Ro[hh] for hh in range(hq)]
    gpu_rows = [so.group_shared_walk_rows([Rg[x] for x in range((hh // group) * group, (hh // group + 1) * group)])
                if group > 1 else Rg[hh] for hh in range(hq)]
    tied_cut, differs = 0, 0
    for hh in range(hq):
        for i in range(b):
            tau = so.tau_of_row(i, *density)
            g = gpu_rows[hh][i, :i + 1]
            got = cig[hh, rpg[hh, i]:rpg[hh, i + 1]]
            # the GPU's selection is its own scores' top-tau with ties to the lower index
            assert np.array_equal(got, so.top_tau_row(g, tau)), (hh, i)
            srt = np.sort(g)[::-1]
            if tau < i + 1 and srt[tau - 1] == srt[tau]:
                tied_cut += 1
                differs += not np.array_equal(got, _higher_index_choice(g, tau))
            # and the oracle's, from its own fp64 walk rows
            want = so.top_tau_row(score_rows[hh][i, :i + 1], tau)
            assert np.array_equal(got, want), (hh, i, got, want)
    if classes == 1:
        for i in range(b):
            assert np.array_equal(cig[0, rpg[0, i]:rpg[0, i + 1]], np.arange(so.tau_of_row(i, *density)))
    # the case really has exact ties at the cut, and a higher-index rule would choose otherwise
    assert tied_cut > b // 2 and differs > b // 2, (tied_cut, differs)
    record_ties([], compared=hq * b)
    h.close()


def _periodic_caches(w, n0s, layer, dev):
    """K caches whose full blocks are copies of one random block (per sequence,
    KV head); the last, partial block holds its first rows. V, queries random."""
    r = torch.Generator(device=dev)
    r.manual_seed(1000 + layer)
    L = max(n0s) + 4
    K = torch.empty(len(n0s), w.hkv, L, w.d, dtype=torch.bfloat16, device=dev)
    for s_ in range(len(n0s)):
        for g in range(w.hkv):
            pat = torch.randn(w.B, w.d, generator=r, device=dev)
            K[s_, g] = pat.repeat(-(-L // w.B), 1)[:L].to(torch.bfloat16)
    V = torch.randn(len(n0s), w.hkv, L, w.d, generator=r, device=dev).to(torch.bfloat16)
    Q = torch.randn(len(n0s), 4, w.hq, w.d, generator=r, device=dev).to(torch.bfloat16)
    return K, V, Q


@pytest.mark.parametrize("shared", [False, True], ids=["per_head", "group_shared"])
def test_decode_selection_ties_go_to_lower_index(shared):
    w = W.DECODE_128K.scaled(layers=2, hq=8, hkv=2, hubs=0)
    n0s = [10 * w.B + 5, 7 * w.B + 20]
    dev = "cuda"
    group = w.hq // w.hkv
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed, select_group=group if shared else 0)
    h = S.Handle(cfg)
    steps = 2
    max_len = max(n0s) + steps
    path = S.DecodePath(h, len(n0s), w.hq, w.hkv, max_len, w.layers, dev)
    data = [_periodic_caches(w, n0s, layer, dev) for layer in range(w.layers)]
    for layer, (K, V, _) in enumerate(data):
        for s_, n0 in enumerate(n0s):
            path.write_cache(layer, s_, K[s_], V[s_], n0)
    path.init_cache(torch.tensor(n0s, dtype=torch.int32, device=dev))
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)
    swaps, tied_cut, differs = [], 0, 0
    for t in range(steps):
        path.begin_step()
        rho_prev = [None] * len(n0s)
        for layer, (K, V, Q) in enumerate(data):
            q_tok = Q[:, t].contiguous()
            k_tok = torch.stack([K[s_, :, n0 + t] for s_, n0 in enumerate(n0s)]).contiguous()
            v_tok = torch.stack([V[s_, :, n0 + t] for s_, n0 in enumerate(n0s)]).contiguous()
            path.layer(layer, q_tok, k_tok, v_tok)
            torch.cuda.synchronize()
            assert S.sws_sync_check(h) == 0
            rho = path.walk_state.cpu().numpy()
            hs, hc = path.head_sel.cpu().numpy(), path.head_cnt.cpu().numpy()
            for s_, n0 in enumerate(n0s):
                length = n0 + t + 1
                nb = -(-length // w.B)
                tau = so.tau_of_row(nb - 1, *w.density)
                Kh = K[s_].double().cpu().numpy()
                q = q_tok[s_].double().cpu().numpy()
                rho_o, _, osel = so.decode_layer_select(q, Kh, length, Hd, w.B, w.s, w.density, rho_prev[s_],
                                                        select="group_shared" if shared else "per_head")
                rho_prev[s_] = rho_o
                for hh in range(w.hq):
                    g0 = (hh // group) * group
                    row = (so.group_shared_log_rows(rho[s_, g0:g0 + group, :nb]) if shared else rho[s_, hh, :nb])
                    # the full blocks are copies: their scores are equal bit for bit on the GPU
                    if shared:
                        assert np.all(rho[s_, g0:g0 + group, :nb - 1] == rho[s_, g0:g0 + group, :1]), (s_, hh)
                    else:
                        assert np.all(row[:nb - 1] == row[0]), (s_, hh, row[:nb - 1])
                    got = hs[s_, hh, :hc[s_, hh]]
                    assert np.array_equal(got, so.top_tau_row(row, tau)), (t, layer, s_, hh, got)
                    tied_cut += 1
                    differs += not np.array_equal(got, _higher_index_choice(row, tau))
                    score = so.group_shared_log_rows(rho_o[g0:g0 + group]) if shared else rho_o[hh]
                    swaps += [(t, layer, s_, hh) + x for x in compare_selection(got, osel[hh], score,
                                                                                 log_domain=True)]
    assert differs == tied_cut  # every selection here cuts through the tied copies
    record_ties(swaps, compared=tied_cut)
    h.close()

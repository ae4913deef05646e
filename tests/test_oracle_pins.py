"""Pins for the oracle: checks against what the page and the mathematics fix.

Each pin compares the oracle with something other than itself: a published
test vector, a closed form, an invariant, a textbook or library routine, or
brute force on tiny inputs. The "planted" tests at the end put a plausible
mistake into the oracle (on the CPU, via monkeypatch) and check that the pin
meant to catch it fails.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import sws_oracle as so

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


# ---------------------------------------------------------------- pins ----

def pin_splitmix64():
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as f:
        want = [int(x, 16) for x in f.read().split() if x.startswith("0x")]
    state, got = 0, []
    for _ in want:
        state, z = so.splitmix64(state)
        got.append(z)
    assert got == want


def pin_hadamard():
    for d in (1, 2, 4, 8, 16, 64, 128):
        H = so.sylvester_hadamard(d)
        formula = np.array([[(-1) ** bin(r & c).count("1") for c in range(d)] for r in range(d)], dtype=float)
        assert np.array_equal(H, formula)
        assert np.array_equal(H @ H.T, d * np.eye(d))


def pin_srht_draws():
    for d, k, seed in ((64, 16, 0), (128, 32, 1), (128, 128, 7), (8, 3, 99)):
        signs, cols = so.srht_draws(d, k, seed)
        assert set(signs) <= {1, -1} and len(signs) == d
        assert len(cols) == k and len(set(cols)) == k and all(0 <= c < d for c in cols)
        assert so.srht_draws(d, k, seed) == (signs, cols)
    _, perm = so.srht_draws(32, 32, 5)
    assert sorted(perm) == list(range(32))


def pin_srht_draws_published_stream():
    """The draws follow the published splitmix64 stream: a seed equal to the
    stream tag starts the generator at state 0, whose first three outputs are
    the golden test vector. d = 2 takes exactly those three: the signs come
    from the top bits of outputs 0 and 1, the one shuffle step swaps position
    1 with (output 2 mod 2). H_d is then D H / sqrt(2) in closed form."""
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as f:
        g = [int(x, 16) for x in f.read().split() if x.startswith("0x")]
    tag = so.SRHT_STREAM_TAG
    signs = [1 if (x >> 63) == 0 else -1 for x in g[:2]]
    perm = [0, 1]
    j = g[2] % 2
    perm[1], perm[j] = perm[j], perm[1]
    assert so.srht_draws(2, 2, tag) == (signs, perm)
    assert so.srht_draws(2, 1, tag) == (signs, perm[:1])
    H = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2.0)
    want = (np.diag(signs) @ H)[:, perm]
    assert np.allclose(so.srht_matrix(2, 2, tag), want, rtol=0, atol=1e-15)


def pin_srht_shuffle_uniform():
    """Fisher-Yates draws every permutation equally often: over 4800 seeds
    all 24 orders of d = 4 appear with chi-square well inside its range. A
    shuffle that swaps with (draw mod r) instead (Sattolo's cyclic variant)
    never yields the identity and fails."""
    counts = {}
    for seed in range(4800):
        _, perm = so.srht_draws(4, 4, seed)
        counts[tuple(perm)] = counts.get(tuple(perm), 0) + 1
    assert len(counts) == 24 and (0, 1, 2, 3) in counts
    expected = 4800 / 24
    chi2 = sum((c - expected) ** 2 / expected for c in counts.values())
    assert chi2 < 60.0  # 23 degrees of freedom: p(chi2 > 60) < 1e-4
    signs = np.array([so.srht_draws(8, 1, seed)[0] for seed in range(2000)])
    assert np.all(np.abs(signs.mean(axis=0)) < 0.1)


def pin_srht_orthogonal_when_k_equals_d():
    """k = d: H_d is orthogonal, so the sketch keeps every inner product (Parseval)."""
    for d, seed in ((64, 3), (128, 11)):
        Hd = so.srht_matrix(d, d, seed)
        assert np.allclose(Hd @ Hd.T, np.eye(d), atol=1e-12)
        u, v = rng.standard_normal(d), rng.standard_normal(d)
        assert abs((u @ Hd) @ (v @ Hd) - u @ v) <= 1e-11 * np.linalg.norm(u) * np.linalg.norm(v)


def pin_srht_unbiased():
    """§6.2: the sketch preserves inner products in expectation. Averaging
    (u H_d)(v H_d)^T over every choice of the k columns gives u.v exactly."""
    for d, k in ((16, 1), (8, 3), (8, 8)):
        signs = [1 if x > 0 else -1 for x in rng.standard_normal(d)]
        u, v = rng.standard_normal(d), rng.standard_normal(d)
        vals = [(u @ so.srht_from_draws(signs, c)) @ (v @ so.srht_from_draws(signs, c))
                for c in itertools.combinations(range(d), k)]
        assert abs(np.mean(vals) - u @ v) < 1e-12 * max(1.0, abs(u @ v)) + 1e-12


def pin_srht_concentration():
    """§6.2 bound |(u^T H)(H^T v) - u^T v| <= eps |u||v|: over many seeds the
    error shrinks like 1/sqrt(k) and its mean is ~0 (statistical, loose)."""
    d = 128
    u, v = rng.standard_normal(d), rng.standard_normal(d)
    scale = np.linalg.norm(u) * np.linalg.norm(v)
    rms = {}
    for k in (8, 32, 128):
        errs = np.array([((u @ (H := so.srht_matrix(d, k, s))) @ (v @ H) - u @ v) / scale for s in range(300)])
        assert abs(errs.mean()) < 4 * errs.std() / math.sqrt(len(errs)) + 1e-12
        rms[k] = math.sqrt((errs ** 2).mean())
    assert rms[128] < 1e-12
    assert rms[8] > rms[32] and 1.3 < rms[8] / rms[32] < 3.0  # ~ sqrt(32/8) = 2


def pin_block_means_identity():
    """§2 vs §3.1: the literal double sum of A_true equals q_bar . k_bar / sqrt(d)."""
    n, B, d = 12, 3, 5
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    lit = so.a_true_literal(Q, K, B)
    via = so.a_true(so.block_means(Q, B), so.block_means(K, B))
    assert np.allclose(lit, via, rtol=1e-12, atol=1e-13)


def pin_block_means_partial():
    """A partial last block averages only the rows it holds (reading R1)."""
    X = rng.standard_normal((7, 4))
    m = so.block_means(X, 3)
    assert m.shape == (3, 4)
    assert np.allclose(m[2], X[6])
    assert np.allclose(m[1], (X[3] + X[4] + X[5]) / 3)


def pin_sws_special_case():
    """B = 1 and k = d: the sketched scores are exactly Q K^T / sqrt(d) (causal part)."""
    n, d = 20, 16
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    Hd = so.srht_matrix(d, d, 4)
    S = so.sketch_scores(so.sketch_project(so.block_means(Q, 1), Hd), so.sketch_project(so.block_means(K, 1), Hd))
    ref = np.asarray(torch.from_numpy(Q) @ torch.from_numpy(K).T / math.sqrt(d))
    low = np.tril_indices(n)
    assert np.allclose(S[low], ref[low], rtol=1e-11, atol=1e-11)
    assert np.all(np.isneginf(S[np.triu_indices(n, 1)]))


def pin_block_attention():
    S = so.sketch_scores(rng.standard_normal((9, 4)), rng.standard_normal((9, 4)))
    A = so.block_attention(S)
    assert np.allclose(A.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(A[np.triu_indices(9, 1)] == 0.0)
    assert A[0, 0] == 1.0
    ref = torch.softmax(torch.from_numpy(np.where(np.isneginf(S), -np.inf, S)), dim=1).numpy()
    assert np.allclose(A, ref, atol=1e-14)


def pin_walk_power():
    """(A)^s as a matrix power: numpy's matrix_power and repeated squaring agree."""
    A = so.block_attention(so.sketch_scores(rng.standard_normal((10, 4)), rng.standard_normal((10, 4))))
    for s in (1, 2, 3, 8):
        assert np.allclose(so.walk_matrix(A, s), np.linalg.matrix_power(A, s), rtol=1e-12, atol=1e-15)
    sq = A @ A
    sq = sq @ sq
    sq = sq @ sq
    assert np.allclose(so.walk_matrix(A, 8), sq, rtol=1e-12, atol=1e-15)


def pin_walk_path_sum():
    """§4: R^l[i, j] sums, over every walk i -> ... -> j, the product of the
    per-step block attention weights: s steps with layer 0's matrix, then s
    steps with layer 1's. Enumerated path by path on a tiny case."""
    b, s = 3, 2
    A0 = so.block_attention(so.sketch_scores(rng.standard_normal((b, 3)), rng.standard_normal((b, 3))))
    A1 = so.block_attention(so.sketch_scores(rng.standard_normal((b, 3)), rng.standard_normal((b, 3))))
    R = so.walk_update(so.walk_update(None, so.walk_matrix(A0, s)), so.walk_matrix(A1, s))
    mats = [A0] * s + [A1] * s
    for i in range(b):
        for j in range(b):
            tot = 0.0
            for mid in itertools.product(range(b), repeat=len(mats) - 1):
                path = (i,) + mid + (j,)
                p = 1.0
                for t, M in enumerate(mats):
                    p *= M[path[t], path[t + 1]]
                tot += p
            assert abs(R[i, j] - tot) < 1e-14


def pin_walk_invariants():
    """R^l stays row-stochastic and lower-triangular across layers (real inputs)."""
    import sws_inputs as W
    w = W.TINY
    Hd = so.srht_matrix(w.d, w.k, w.seed)
    st = so.PrefillState()
    for layer in range(w.layers):
        Q, K, V = W.prefill_layer_inputs(w, layer)
        R = so.prefill_layer(Q.numpy(), K.numpy(), V.numpy(), Hd, w.B, w.s, w.density, st, attention_blocks=None)[0]["R"]
        assert np.allclose(R.sum(axis=1), 1.0, atol=1e-12)
        assert np.all(R[np.triu_indices(w.b, 1)] == 0.0)
        assert np.all(R[np.tril_indices(w.b)] > 0.0)


def pin_walk_elementwise():
    """Reading R5's alternative: the entrywise power with rows renormalised is
    row-stochastic and lower-triangular, keeps each row's order, and raises
    every ratio of two entries of a row to the power s."""
    A = so.block_attention(so.sketch_scores(rng.standard_normal((12, 4)), rng.standard_normal((12, 4))))
    for s in (1, 2, 8):
        M = so.walk_matrix(A, s, "elementwise")
        assert np.allclose(M.sum(axis=1), 1.0, atol=1e-14)
        assert np.all(M[np.triu_indices(12, 1)] == 0.0)
        for i in range(1, 12):
            r, a = M[i, :i + 1], A[i, :i + 1]
            assert np.array_equal(np.argsort(-r, kind="stable"), np.argsort(-a, kind="stable"))
            assert np.allclose(r[1:] / r[0], (a[1:] / a[0]) ** s, rtol=1e-11)


def pin_top_tau_bruteforce():
    """Brute force: the chosen set maximises the sum of the row over all sets
    of size tau; among maximisers it takes the lowest indices (tie rule R6)."""
    r = np.random.default_rng(7)
    for trial in range(300):
        m = int(r.integers(1, 10))
        row = r.integers(0, 4, size=m).astype(float)  # small range: many ties
        tau = int(r.integers(1, m + 1))
        got = tuple(int(x) for x in so.top_tau_row(row, tau))
        best = max(sum(row[list(c)]) for c in itertools.combinations(range(m), tau))
        cands = [c for c in itertools.combinations(range(m), tau) if sum(row[list(c)]) == best]
        assert got == min(cands), (row, tau, got)


def pin_tau():
    table = {0: 1, 3: 1, 4: 1, 5: 2, 9: 2, 10: 3, 255: 52, 1023: 205}
    for i, t in table.items():
        assert so.tau_of_row(i, 1, 5) == t
    assert so.tau_of_row(9, 1, 10) == 1 and so.tau_of_row(10, 1, 10) == 2
    assert all(so.tau_of_row(i, 1, 1) == i + 1 for i in range(50))
    assert so.csr_nnz(16, 1, 5) == 34 and so.csr_nnz(1024, 1, 5) == 105370


def _dense_causal_sdpa(Q, K, V):
    q, k, v = (torch.from_numpy(np.asarray(x, dtype=np.float64))[None, None] for x in (Q, K, V))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)[0, 0].numpy()


def pin_attention_dense_limit():
    """Density 100%: every causal block is kept, so the sparse attention equals
    dense causal softmax attention (torch's SDPA in fp64)."""
    n, d, B = 40, 8, 8
    Q, K, V = (rng.standard_normal((n, d)) for _ in range(3))
    b = n // B
    row_ptr, col_idx = so.select_top_tau(np.tril(np.ones((b, b))), 1, 1)
    O = so.sparse_attention(Q, K, V, row_ptr, col_idx, B)
    assert np.allclose(O, _dense_causal_sdpa(Q, K, V), rtol=1e-12, atol=1e-12)
    # ragged n (partial last block)
    n2 = 37
    b2 = -(-n2 // B)
    rp, ci = so.select_top_tau(np.tril(np.ones((b2, b2))), 1, 1)
    O2 = so.sparse_attention(Q[:n2], K[:n2], V[:n2], rp, ci, B)
    assert np.allclose(O2, _dense_causal_sdpa(Q[:n2], K[:n2], V[:n2]), rtol=1e-12, atol=1e-12)


def pin_attention_special_cases():
    n, d, B = 24, 4, 4
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    Vc = np.tile(rng.standard_normal(d), (n, 1))
    b = n // B
    rp, ci = so.select_top_tau(rng.random((b, b)), 1, 3)
    assert np.allclose(so.sparse_attention(Q, K, Vc, rp, ci, B), Vc, atol=1e-13)  # constant V
    V = rng.standard_normal((n, d))
    O = so.sparse_attention(Q, K, V, rp, ci, B)
    assert np.allclose(O[0], V[0])  # the first token only sees itself
    # a query block whose only key block is block 0, strictly below it: plain softmax over block 0
    rp1 = np.array([0, 1, 2])
    ci1 = np.array([0, 0])
    O1 = so.sparse_attention(Q[:8], K[:8], V[:8], rp1, ci1, B)
    w = np.exp(Q[4:8] @ K[:4].T / math.sqrt(d))
    assert np.allclose(O1[4:8], (w / w.sum(axis=1, keepdims=True)) @ V[:4])


def pin_one_hop_when_s1():
    """s = 1 and one layer: the selection is the top-tau of the sketched scores
    themselves (the row softmax is monotone)."""
    S = so.sketch_scores(rng.standard_normal((30, 4)), rng.standard_normal((30, 4)))
    R = so.walk_update(None, so.walk_matrix(so.block_attention(S), 1))
    rp, ci = so.select_top_tau(R, 1, 5)
    for i in range(30):
        raw = S[i, :i + 1]
        want = np.sort(np.argsort(-raw, kind="stable")[:so.tau_of_row(i, 1, 5)])
        assert np.array_equal(ci[rp[i]:rp[i + 1]], want)


def pin_gqa_mapping():
    """Query head h reads KV head h // (hq / hkv)."""
    n, d, B = 32, 8, 8
    Q = rng.standard_normal((4, n, d))
    K, V = rng.standard_normal((2, n, d)), rng.standard_normal((2, n, d))
    Hd = so.srht_matrix(d, 4, 1)
    full = so.prefill_layer(Q, K, V, Hd, B, 2, (1, 2), so.PrefillState())
    for h in range(4):
        one = so.prefill_layer(Q[h:h + 1], K[h // 2:h // 2 + 1], V[h // 2:h // 2 + 1], Hd, B, 2, (1, 2),
                               so.PrefillState())[0]
        assert np.array_equal(one["col_idx"], full[h]["col_idx"])
        assert np.allclose(one["O"], full[h]["O"])


def pin_decode():
    """Decode (readings R7, R8): block means by count; rho^0 / s is the log of a
    softmax; with s = 1 and one layer the choice is the top-tau of the row
    logits; s does not change the ranking; all blocks kept = dense attention."""
    hq, hkv, d, B, L = 2, 1, 8, 4, 19
    Kc, Vc = rng.standard_normal((hkv, 24, d)), rng.standard_normal((hkv, 24, d))
    q = rng.standard_normal((hq, d))
    Hd = so.srht_matrix(d, 4, 2)
    means = so.decode_block_means(Kc[0], L, B)
    assert means.shape == (5, d) and np.allclose(means[4], Kc[0, 16:19].mean(axis=0))
    assert np.allclose(means[1], Kc[0, 4:8].sum(axis=0) / 4)
    rho1, z, sel1 = so.decode_layer_select(q, Kc, L, Hd, B, 1, (2, 5), None)
    assert np.allclose(np.exp(rho1).sum(axis=1), 1.0, atol=1e-13)
    tau = so.tau_of_row(4, 2, 5)
    for h in range(hq):
        assert np.array_equal(sel1[h], np.sort(np.argsort(-z[h], kind="stable")[:tau]))
    rho8, _, sel8 = so.decode_layer_select(q, Kc, L, Hd, B, 8, (2, 5), None)
    assert np.allclose(rho8, 8 * rho1)
    assert all(np.array_equal(a, b) for a, b in zip(sel1, sel8))
    o = so.decode_attention(q[0], Kc[0], Vc[0], L, range(5), B)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0])[None, None, None], torch.from_numpy(Kc[0, :L])[None, None],
        torch.from_numpy(Vc[0, :L])[None, None])[0, 0, 0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)


def _softmax_plain(z):
    """exp(z - max) / sum: a probability row, without any logarithm."""
    e = np.exp(z - z.max())
    return e / e.sum()


def pin_decode_walk_carry():
    """Decode walk over layers (reading R7): the carried log-domain row, taken
    back out of the logs, is the entrywise product over the layers of each
    layer's softmax row raised to s, multiplied out directly (no logarithms):
    exp(rho^L) = prod_l softmax(z^l)^s. A carry that is dropped, or that adds
    s * z instead of s * (z - logsumexp z), changes these values. The
    selection after the last layer is the top-tau of that product."""
    hq, hkv, d, B, k, s, L = 3, 1, 8, 4, 8, 2, 21
    Hd = so.srht_matrix(d, k, 11)
    r = np.random.default_rng(2024)
    rho, prod, zs = None, None, []
    for layer in range(3):
        Kc = r.standard_normal((hkv, 24, d))
        q = r.standard_normal((hq, d))
        rho, z, sel = so.decode_layer_select(q, Kc, L, Hd, B, s, (2, 5), rho)
        zs.append(z)
        f = np.stack([_softmax_plain(z[h]) ** s for h in range(hq)])
        prod = f if prod is None else prod * f
        assert np.allclose(np.exp(rho), prod, rtol=1e-12, atol=0.0)
        tau = so.tau_of_row(-(-L // B) - 1, 2, 5)
        for h in range(hq):
            want = np.sort(np.lexsort((np.arange(prod.shape[1]), -prod[h]))[:tau])
            assert np.array_equal(sel[h], want)
    # the three layers' rows differ, so the carry matters for the values
    assert not np.allclose(zs[0], zs[2])


def pin_decode_logits_literal():
    """With k = d the projection is orthogonal, so the decode row logit of
    block j is the plain mean over the block's cached tokens of q . K[t] /
    sqrt(d) (the partial last block by its count), summed here token by token."""
    d, B, L = 8, 4, 18
    Kc = rng.standard_normal((1, 20, d))
    q = rng.standard_normal((1, d))
    Hd = so.srht_matrix(d, d, 9)
    _, z, _ = so.decode_layer_select(q, Kc, L, Hd, B, 1, (1, 2), None)
    nb = -(-L // B)
    for j in range(nb):
        toks = range(j * B, min(L, (j + 1) * B))
        acc = 0.0
        for t in toks:
            acc += sum(float(q[0, c]) * float(Kc[0, t, c]) for c in range(d))
        assert abs(z[0, j] - acc / (len(toks) * math.sqrt(d))) < 1e-12


def pin_attention_triple_loop():
    """Sparse attention against a naive loop: for every query token, every
    allowed key token (in a selected block, at or before the query), the
    score, the softmax and the weighted sum of V, one scalar at a time.
    A random selection (every row holds tau_i blocks) with a ragged tail."""
    n, d, B = 22, 4, 4
    Q, K, V = (rng.standard_normal((n, d)) for _ in range(3))
    b = -(-n // B)
    rp, ci = so.select_top_tau(rng.random((b, b)), 1, 2)
    O = so.sparse_attention(Q, K, V, rp, ci, B)
    for t in range(n):
        i = t // B
        allowed = [u for j in ci[rp[i]:rp[i + 1]] for u in range(j * B, min(n, (j + 1) * B)) if u <= t]
        sc = []
        for u in allowed:
            acc = 0.0
            for c in range(d):
                acc += Q[t, c] * K[u, c]
            sc.append(acc / math.sqrt(d))
        mx = max(sc)
        w = [math.exp(x - mx) for x in sc]
        tot = sum(w)
        for c in range(d):
            want = sum(w[a] * V[u, c] for a, u in enumerate(allowed)) / tot
            assert abs(O[t, c] - want) < 1e-12


def pin_group_shared_log_rows():
    """The decode group score is log(sum_h exp(rho_h)): scipy's logsumexp on
    rows far below exp's range, and shift invariance."""
    from scipy.special import logsumexp
    rho = rng.uniform(-1500.0, -900.0, size=(4, 37))
    got = so.group_shared_log_rows(rho)
    assert np.all(np.isfinite(got))
    assert np.allclose(got, logsumexp(rho, axis=0), rtol=1e-13, atol=0)
    assert np.allclose(so.group_shared_log_rows(rho + 3.5), got + 3.5, rtol=1e-13, atol=0)
    one = rng.standard_normal((1, 9))
    assert np.array_equal(so.group_shared_log_rows(one), one[0])


def _shared_case(hq, hkv, same_heads=False, perm=None):
    d, B, n = 8, 4, 29
    r = np.random.default_rng(77)
    Q = r.standard_normal((hq, n, d))
    if same_heads:
        Q[:] = Q[0]
    if perm is not None:
        Q = Q[perm]
    K, V = r.standard_normal((hkv, n, d)), r.standard_normal((hkv, n, d))
    Hd = so.srht_matrix(d, 4, 3)
    return Q, K, V, Hd, B


def pin_group_shared_prefill():
    """Group-shared prefill selection: with one head per group it is the
    per-head choice; with identical heads it is each head's own choice; it
    does not depend on the order of the group's heads; every head of a group
    gets the same CSR rows."""
    for hq, hkv in ((2, 2), (4, 2)):
        Q, K, V, Hd, B = _shared_case(hq, hkv, same_heads=(hq != hkv))
        for layers in (1, 2):
            sp, ss = so.PrefillState(), so.PrefillState()
            for _ in range(layers):
                per = so.prefill_layer(Q, K, V, Hd, B, 2, (2, 5), sp, attention_blocks=None)
                sh = so.prefill_layer(Q, K, V, Hd, B, 2, (2, 5), ss, attention_blocks=None, select="group_shared")
            for h in range(hq):
                assert np.array_equal(per[h]["col_idx"], sh[h]["col_idx"])
                assert np.array_equal(per[h]["row_ptr"], sh[h]["row_ptr"])
    Q, K, V, Hd, B = _shared_case(4, 2)
    a = so.prefill_layer(Q, K, V, Hd, B, 2, (2, 5), so.PrefillState(), attention_blocks=None, select="group_shared")
    Qp = Q[[1, 0, 3, 2]]
    b = so.prefill_layer(Qp, K, V, Hd, B, 2, (2, 5), so.PrefillState(), attention_blocks=None, select="group_shared")
    for h in range(4):
        assert np.array_equal(a[h]["col_idx"], b[h]["col_idx"])
        assert np.array_equal(a[h]["col_idx"], a[(h // 2) * 2]["col_idx"])
    per = so.prefill_layer(Q, K, V, Hd, B, 2, (2, 5), so.PrefillState(), attention_blocks=None)
    assert any(not np.array_equal(per[h]["col_idx"], a[h]["col_idx"]) for h in range(4))  # the choice is shared


def pin_group_shared_decode():
    """Group-shared decode selection: per-head choice when a group has one
    head or identical heads, independent of head order, one set per group."""
    d, B, L = 8, 4, 37
    r = np.random.default_rng(5)
    Kc = r.standard_normal((2, 40, d))
    Hd = so.srht_matrix(d, 4, 2)
    q = r.standard_normal((2, d))
    _, _, per = so.decode_layer_select(q, Kc, L, Hd, B, 8, (1, 3), None)
    _, _, sh = so.decode_layer_select(q, Kc, L, Hd, B, 8, (1, 3), None, select="group_shared")
    assert all(np.array_equal(x, y) for x, y in zip(per, sh))
    q4 = np.repeat(q[:1], 4, axis=0)
    _, _, per = so.decode_layer_select(q4, Kc[:1], L, Hd, B, 8, (1, 3), None)
    _, _, sh = so.decode_layer_select(q4, Kc[:1], L, Hd, B, 8, (1, 3), None, select="group_shared")
    assert all(np.array_equal(x, y) for x, y in zip(per, sh))
    q4 = r.standard_normal((4, d))
    rho, _, a = so.decode_layer_select(q4, Kc, L, Hd, B, 8, (1, 3), None, select="group_shared")
    _, _, b = so.decode_layer_select(q4[[1, 0, 3, 2]], Kc, L, Hd, B, 8, (1, 3), None, select="group_shared")
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert np.array_equal(a[0], a[1]) and np.array_equal(a[2], a[3])


def pin_exact_decode():
    """Exact decode walk: the newest block's row of the prefill recurrence.
    (1) With s = 1 and one layer, when the newest block holds only the new
    token, the row is the softmax of the row logits: exp of the log-domain
    decode's rho (a separate route, from the token's own query). (2) Over
    layers the row stays a probability row. (3) Brute force: e_i times
    numpy's matrix_power of each layer's block attention, multiplied out."""
    hq, hkv, d, B, k = 2, 1, 8, 4, 4
    n = 17  # block 4 holds position 16 only
    Hd = so.srht_matrix(d, k, 5)
    Qs = [rng.standard_normal((hq, n, d)) for _ in range(3)]
    Ks = [rng.standard_normal((hkv, n, d)) for _ in range(3)]
    one = so.decode_exact_layer(Qs[0], Ks[0], Hd, B, 1, (2, 5), so.PrefillState())
    rho1, _, sel1 = so.decode_layer_select(Qs[0][:, n - 1], Ks[0], n, Hd, B, 1, (2, 5), None)
    for h in range(hq):
        assert np.allclose(one[h]["row"], np.exp(rho1[h]), rtol=1e-12, atol=1e-15)
        assert np.array_equal(one[h]["blocks"], sel1[h])
    st = so.PrefillState()
    rows = [so.decode_exact_layer(Qs[l], Ks[l], Hd, B, 3, (2, 5), st) for l in range(3)]
    nb = -(-n // B)
    for h in range(hq):
        u = np.eye(nb)[nb - 1]
        for l in range(3):
            A = so.block_attention(so.sketch_scores(so.sketch_project(so.block_means(Qs[l][h], B), Hd),
                                                    so.sketch_project(so.block_means(Ks[l][0], B), Hd)))
            u = u @ np.linalg.matrix_power(A, 3)
            got = rows[l][h]["row"]
            assert np.all(got >= 0) and abs(got.sum() - 1.0) < 1e-12
            assert np.allclose(got, u, rtol=1e-12, atol=1e-15)
            assert np.array_equal(rows[l][h]["blocks"], so.top_tau_row(u, so.tau_of_row(nb - 1, 2, 5)))


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------- planted mistakes ----

PLANTED = {
    "hadamard_scale_dropped": ("srht_from_draws",
                               lambda orig: (lambda signs, cols: orig(signs, cols) / math.sqrt(len(signs) / len(cols))),
                               pin_srht_unbiased),
    "splitmix_constant": ("splitmix64", lambda orig: (lambda s: (orig(s)[0], orig(s)[1] ^ 1)), pin_splitmix64),
    "partial_block_divides_by_B": ("block_means", lambda orig: (
        lambda X, B: np.stack([np.asarray(X, float)[i * B:(i + 1) * B].sum(0) / B for i in range(-(-len(X) // B))])),
        pin_block_means_partial),
    "no_causal_block_mask": ("block_attention", lambda orig: (
        lambda S: (lambda e: e / e.sum(1, keepdims=True))(np.exp(np.where(np.isneginf(S), 0.0, S)))),
        pin_block_attention),
    "walk_power_off_by_one": ("walk_matrix", lambda orig: (lambda A, s, mode="matrix_power": orig(A, s + 1, mode)),
                              pin_walk_power),
    "walk_operands_swapped": ("walk_update", lambda orig: (lambda R, M: M.copy() if R is None else M @ R),
                              pin_walk_path_sum),
    "ties_to_higher_index": ("top_tau_row", lambda orig: (
        lambda row, tau: np.sort(np.lexsort((-np.arange(len(row)), -row))[:tau])), pin_top_tau_bruteforce),
    "tau_floor": ("tau_of_row", lambda orig: (lambda i, num, den: max(1, (i + 1) * num // den)), pin_tau),
    "no_causal_mask_in_diagonal_block": ("sparse_attention_block", lambda orig: (
        lambda Q, K, V, i, blocks, B: orig(Q, K, V, i, blocks, B) if i == 0 else
        (lambda u: (lambda s: (np.exp(s - s.max(1, keepdims=True)) @ V[u]) /
                    np.exp(s - s.max(1, keepdims=True)).sum(1, keepdims=True))(
            Q[i * B:(i + 1) * B] @ K[u].T / math.sqrt(Q.shape[1])))(
            np.concatenate([np.arange(j * B, min(len(Q), (j + 1) * B)) for j in blocks]))),
        pin_attention_dense_limit),
    "group_shared_first_head_only": ("group_shared_walk_rows", lambda orig: (lambda R_heads: orig(R_heads[:1])),
                                     pin_group_shared_prefill),
    "group_shared_lse_without_shift": ("group_shared_log_rows", lambda orig: (
        lambda rho: np.log(np.exp(rho).sum(axis=0))), pin_group_shared_log_rows),
    "attention_scale_1_over_d": ("sparse_attention_block", lambda orig: (
        lambda Q, K, V, i, blocks, B: orig(np.asarray(Q) / math.sqrt(Q.shape[1]), K, V, i, blocks, B)),
        pin_attention_dense_limit),
}


PLANTED["signs_from_set_top_bit"] = (
    "srht_draws", lambda orig: (lambda d, k, seed: ([-x for x in orig(d, k, seed)[0]], orig(d, k, seed)[1])),
    pin_srht_draws_published_stream)


def _sattolo_draws(d, k, seed):
    signs, _ = _ORIG_DRAWS(d, k, seed)
    state = (seed ^ so.SRHT_STREAM_TAG) & ((1 << 64) - 1)
    draws = []
    for _ in range(2 * d - 1):
        state, z = so.splitmix64(state)
        draws.append(z)
    perm, nxt = list(range(d)), d
    for r in range(d - 1, 0, -1):
        j = draws[nxt] % r
        nxt += 1
        perm[r], perm[j] = perm[j], perm[r]
    return signs, perm[:k]


_ORIG_DRAWS = so.srht_draws
PLANTED["shuffle_mod_r"] = ("srht_draws", lambda orig: _sattolo_draws, pin_srht_shuffle_uniform)
PLANTED["elementwise_not_renormalised"] = (
    "walk_matrix", lambda orig: (lambda A, s, mode="matrix_power": A ** s if mode == "elementwise" else orig(A, s, mode)),
    pin_walk_elementwise)

PLANTED["exact_decode_previous_block_row"] = (
    "decode_exact_layer", lambda orig: (lambda Q, K, Hd, B, s, density, state, heads=None, select="per_head": {
        h: dict(r, row=np.append(state.R[h][-2, :-1], 0.0)) for h, r in orig(Q, K, Hd, B, s, density, state, heads,
                                                                             select).items()}),
    pin_exact_decode)



def _decode_carry_wrapped(wrong_rho):
    """A decode_layer_select whose returned rho is replaced by wrong_rho(s, z, rho_prev),
    the selection taken again on it (as the oracle would after that mistake)."""
    orig = _ORIG_DECODE

    def f(q_tok, Kc, length, Hd, B, s, density, rho_prev, select="per_head"):
        _, z, _ = orig(q_tok, Kc, length, Hd, B, s, density, rho_prev, select)
        rho = wrong_rho(s, z, rho_prev)
        tau = so.tau_of_row(-(-length // B) - 1, *density)
        return rho, z, [so.top_tau_row(rho[h], tau) for h in range(rho.shape[0])]
    return f


def _lse(z):
    m = z.max(axis=1, keepdims=True)
    return m + np.log(np.exp(z - m).sum(axis=1, keepdims=True))


_ORIG_DECODE = so.decode_layer_select
PLANTED["decode_carry_dropped"] = (
    "decode_layer_select", lambda orig: _decode_carry_wrapped(lambda s, z, rp: s * (z - _lse(z))),
    pin_decode_walk_carry)
PLANTED["decode_carry_of_raw_logits"] = (
    "decode_layer_select", lambda orig: _decode_carry_wrapped(
        lambda s, z, rp: s * (z - _lse(z)) if rp is None else s * z + rp),
    pin_decode_walk_carry)
PLANTED["decode_carry_scaled_twice"] = (
    "decode_layer_select", lambda orig: _decode_carry_wrapped(
        lambda s, z, rp: s * (z - _lse(z) + (0.0 if rp is None else rp))),
    pin_decode_walk_carry)
PLANTED["decode_logits_scale_sqrt_d"] = (
    "decode_layer_select", lambda orig: (
        lambda q_tok, Kc, length, Hd, B, s, density, rho_prev, select="per_head":
        (lambda r: (r[0], r[1] * 2.0, r[2]))(orig(q_tok, Kc, length, Hd, B, s, density, rho_prev, select))),
    pin_decode_logits_literal)
PLANTED["attention_causal_mask_off_by_one"] = (
    "sparse_attention_block", lambda orig: _attn_mask_lt, pin_attention_triple_loop)


def _attn_mask_lt(Q, K, V, i, blocks, B):
    """sparse_attention_block with the diagonal excluded (u < t instead of u <= t)
    wherever a token has an earlier allowed key."""
    n, d = Q.shape
    t0, t1 = i * B, min(n, (i + 1) * B)
    u = np.concatenate([np.arange(j * B, min(n, (j + 1) * B)) for j in blocks])
    s = Q[t0:t1] @ K[u].T / math.sqrt(d)
    t = np.arange(t0, t1)
    allow = u[None, :] < t[:, None]
    allow[~allow.any(axis=1)] = u[None, :] <= t[~allow.any(axis=1), None]
    s = np.where(allow, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p @ V[u]) / p.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, make, pin = PLANTED[name]
    orig = getattr(so, attr)
    monkeypatch.setattr(so, attr, make(orig))
    with pytest.raises(AssertionError):
        pin()


def test_planted_decode_lse_dropped(monkeypatch):
    """Dropping logsumexp leaves the decode ranking unchanged; the softmax
    normalisation check inside pin_decode still catches it."""
    orig = so.decode_layer_select

    def wrong(q_tok, Kc, length, Hd, B, s, density, rho_prev):
        rho, z, sel = orig(q_tok, Kc, length, Hd, B, s, density, rho_prev)
        return s * z + (0.0 if rho_prev is None else rho_prev), z, sel

    monkeypatch.setattr(so, "decode_layer_select", wrong)
    with pytest.raises(AssertionError):
        pin_decode()

"""fp64 statement of what the Sketch&Walk hot path computes.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Source: "Scout Before You Attend: Sketch-and-Walk Sparse Attention for
Efficient LLM Inference" (blog deep-dive of arXiv 2602.07397):
  §2   true block score A_true (the double sum over a block pair)
  §3.1 token-space sketch: block means of Q and K
  §3.2 feature-space sketch: Hadamard projection H_d (d x k) and the
       sketched block scores  A_SWS = (Q_bar H_d)(K_bar H_d)^T / sqrt(k)
  §4   walk state R^0 = (A_block^0)^s, R^l = R^{l-1} (A_block^l)^s and top-tau
       key blocks per query block from the rows of R^l
  §5   the same selection for decode; exact attention on the original Q/K/V
       restricted to the selected blocks
  §6.2 the inner-product preservation property of the Hadamard sketch
  §7   defaults B=64, k=64, s=8

Readings taken where the page is silent (each one is also listed, with its
reason, in the design notes):
  R1 partial last block: its mean divides by the rows it actually holds.
  R2 H_d = sqrt(d/k) * D * H_n * P: D random signs, H_n the Sylvester
     Hadamard matrix scaled by 1/sqrt(d), P k distinct columns; the signs and
     columns come from a splitmix64 stream (spelled out in ``srht_draws``).
  R3 the sketched scores divide by sqrt(k), as §3.2 writes them.
  R4 the "sketched block attention matrix" of §4 is the row softmax of the
     sketched scores under the causal block mask (j <= i).
  R5 (.)^s is the matrix power; the elementwise power with rows renormalised
     is kept as the alternative reading (mode "elementwise").
  R6 tau_i = ceil((i+1) * num / den) in integers; candidates j <= i; ties go to
     the lower block index; the chosen blocks are listed in ascending order.
  R7 decode: the new query token is a block of one row; key blocks are the
     means of the cached blocks (the partial block by its count); a 1 x b row
     has no matrix power, so the walk over layers is the elementwise product
     of the per-layer rows raised to s, kept in the log domain:
     rho^l = rho^{l-1} + s * (z^l - logsumexp(z^l)).
  R8 the decode token is appended to the cache before it attends.
No blocking, fusion or reordering is done beyond what those definitions state.

Group-shared selection (an extension the pages do not define; §8 row F1 of
the build's scope): the query heads of one GQA group share one set of key
blocks per query block, the top-tau of the sum of the group's walk rows
(their mean up to a positive factor) in prefill, and of the log-sum-exp over
the group's log-domain walk rows rho in decode (the same sum, taken of
exp(rho), in the log domain).
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "splitmix64", "SRHT_STREAM_TAG", "srht_draws", "sylvester_hadamard", "srht_from_draws", "srht_matrix",
    "block_means", "a_true_literal", "a_true", "sketch_project", "sketch_scores", "block_attention",
    "walk_matrix", "walk_update", "tau_of_row", "csr_nnz", "top_tau_row", "select_top_tau",
    "sparse_attention_block", "sparse_attention", "prefill_layer", "PrefillState",
    "decode_block_means", "decode_layer_select", "decode_attention",
    "group_shared_walk_rows", "group_shared_log_rows",
]

_M64 = (1 << 64) - 1
SRHT_STREAM_TAG = 0x5357535F48414431  # "SWS_HAD1": separates the projection's stream from other uses of a seed


# ---------------------------------------------------------------------------
# §3.2 feature-space sketch: the randomized Hadamard projection (reading R2)
# ---------------------------------------------------------------------------

def splitmix64(state: int) -> Tuple[int, int]:
    """One step of the published splitmix64 generator (Steele, Lea and Flood,
    "Fast splittable pseudorandom number generators", OOPSLA 2014): returns the
    advanced state and the 64-bit output."""
    state = (state + 0x9E3779B97F4A7C15) & _M64
    z = state
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return state, z ^ (z >> 31)


def srht_draws(d: int, k: int, seed: int) -> Tuple[List[int], List[int]]:
    """Random signs D (d entries of +-1) and the k sampled columns P.

    The splitmix64 stream starts from ``seed XOR SRHT_STREAM_TAG``. Draws
    0..d-1 give the signs (+1 when the top bit is 0). The next d-1 draws run a
    Fisher-Yates shuffle of [0, d): for r = d-1 down to 1, swap positions r and
    (draw mod (r+1)). P is the first k entries of the shuffled array, in order.
    """
    if not (0 < k <= d):
        raise ValueError("need 0 < k <= d")
    state = (seed ^ SRHT_STREAM_TAG) & _M64
    draws = []
    for _ in range(2 * d - 1):
        state, z = splitmix64(state)
        draws.append(z)
    signs = [1 if (draws[r] >> 63) == 0 else -1 for r in range(d)]
    perm = list(range(d))
    nxt = d
    for r in range(d - 1, 0, -1):
        j = draws[nxt] % (r + 1)
        nxt += 1
        perm[r], perm[j] = perm[j], perm[r]
    return signs, perm[:k]


def sylvester_hadamard(d: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix of order d (a power of two):
    H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]]."""
    if d < 1 or (d & (d - 1)) != 0:
        raise ValueError("Hadamard order must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def srht_from_draws(signs: Sequence[int], cols: Sequence[int]) -> np.ndarray:
    """H_d = sqrt(d/k) * D * (H / sqrt(d)) * P as an explicit d x k matrix."""
    d, k = len(signs), len(cols)
    Hn = sylvester_hadamard(d) / math.sqrt(d)
    D = np.diag(np.asarray(signs, dtype=np.float64))
    P = np.zeros((d, k))
    for c, col in enumerate(cols):
        P[col, c] = 1.0
    return math.sqrt(d / k) * (D @ Hn @ P)


def srht_matrix(d: int, k: int, seed: int) -> np.ndarray:
    signs, cols = srht_draws(d, k, seed)
    return srht_from_draws(signs, cols)


# ---------------------------------------------------------------------------
# §2 true block score and §3.1 token-space sketch
# ---------------------------------------------------------------------------

def block_means(X: np.ndarray, B: int) -> np.ndarray:
    """§3.1 block aggregation: row i is the mean of the rows of block i
    (b = ceil(n/B) blocks; a partial last block divides by its count, R1)."""
    X = np.asarray(X, dtype=np.float64)
    n = X.shape[0]
    b = -(-n // B)
    out = np.empty((b, X.shape[1]))
    for i in range(b):
        out[i] = X[i * B:min(n, (i + 1) * B)].mean(axis=0)
    return out


def a_true_literal(Q: np.ndarray, K: np.ndarray, B: int) -> np.ndarray:
    """§2 true block score, written as the page's double sum over the B x B
    token pairs of blocks i and j, scaled by 1/sqrt(d) and 1/B^2 (full blocks).
    Pure-Python loops: tiny inputs only."""
    n, d = Q.shape
    b = n // B
    A = np.zeros((b, b))
    for i in range(b):
        for j in range(b):
            acc = 0.0
            for s_ in range(B):
                for t in range(B):
                    acc += float(np.dot(Q[i * B + s_], K[j * B + t]))
            A[i, j] = acc / (math.sqrt(d) * B * B)
    return A


def a_true(Qbar: np.ndarray, Kbar: np.ndarray) -> np.ndarray:
    """§2 true block score from the block means: q_bar_i . k_bar_j / sqrt(d)."""
    return Qbar @ Kbar.T / math.sqrt(Qbar.shape[1])


def sketch_project(Xbar: np.ndarray, Hd: np.ndarray) -> np.ndarray:
    """§3.2: q_tilde_i = q_bar_i H_d (and the same for keys)."""
    return Xbar @ Hd


def sketch_scores(Qt: np.ndarray, Kt: np.ndarray) -> np.ndarray:
    """§3.2 sketched block scores Q_tilde K_tilde^T / sqrt(k) (R3), with the
    causal block mask: entries j > i are -inf."""
    k = Qt.shape[1]
    S = Qt @ Kt.T / math.sqrt(k)
    b = S.shape[0]
    S[np.triu_indices(b, 1)] = -np.inf
    return S


# ---------------------------------------------------------------------------
# §4 sketch-determined walk and top-tau selection
# ---------------------------------------------------------------------------

def block_attention(S: np.ndarray) -> np.ndarray:
    """R4: the sketched block attention matrix is the row softmax of the
    sketched scores over the causal blocks j <= i (zero above the diagonal)."""
    b = S.shape[0]
    A = np.zeros_like(S)
    for i in range(b):
        row = S[i, :i + 1]
        e = np.exp(row - row.max())
        A[i, :i + 1] = e / e.sum()
    return A


def walk_matrix(Ahat: np.ndarray, s: int, mode: str = "matrix_power") -> np.ndarray:
    """(A_block)^s of §4. R5: the matrix power, computed as s-1 plain products;
    or, in mode "elementwise", the entrywise power with rows renormalised."""
    if s < 1:
        raise ValueError("s >= 1")
    if mode == "matrix_power":
        M = Ahat.copy()
        for _ in range(s - 1):
            M = M @ Ahat
        return M
    if mode == "elementwise":
        M = Ahat ** s
        return M / M.sum(axis=1, keepdims=True)
    raise ValueError(mode)


def walk_update(R_prev: Optional[np.ndarray], M: np.ndarray) -> np.ndarray:
    """§4: R^0 = M for the first layer, R^l = R^{l-1} M afterwards."""
    return M.copy() if R_prev is None else R_prev @ M


def tau_of_row(i: int, num: int, den: int) -> int:
    """R6: tau_i = ceil((i+1) * num / den) key blocks for query block i."""
    return -(-(i + 1) * num // den)


def csr_nnz(b: int, num: int, den: int) -> int:
    return sum(tau_of_row(i, num, den) for i in range(b))


def top_tau_row(row: np.ndarray, tau: int) -> np.ndarray:
    """R6: the tau largest entries of ``row`` (ties to the lower index), listed
    in ascending index order. A stable sort on (-value, index)."""
    idx = np.arange(row.shape[0])
    order = np.lexsort((idx, -row))
    return np.sort(order[:tau])


def select_top_tau(R: np.ndarray, num: int, den: int) -> Tuple[np.ndarray, np.ndarray]:
    """§4 top-tau key blocks per query block from the rows of R, as CSR."""
    b = R.shape[0]
    row_ptr = np.zeros(b + 1, dtype=np.int64)
    cols = []
    for i in range(b):
        sel = top_tau_row(R[i, :i + 1], tau_of_row(i, num, den))
        cols.append(sel)
        row_ptr[i + 1] = row_ptr[i] + sel.shape[0]
    return row_ptr, np.concatenate(cols).astype(np.int64)


# ---------------------------------------------------------------------------
# §4/§5 exact attention on the original Q, K, V restricted to the selection
# ---------------------------------------------------------------------------

def sparse_attention_block(Q: np.ndarray, K: np.ndarray, V: np.ndarray, i: int, blocks: Sequence[int],
                           B: int) -> np.ndarray:
    """Output rows of query block i: each query token t attends to the tokens u
    of the selected key blocks with u <= t, with the textbook softmax
    (two passes: the row max, then normalised exponentials)."""
    n, d = Q.shape
    t0, t1 = i * B, min(n, (i + 1) * B)
    u = np.concatenate([np.arange(j * B, min(n, (j + 1) * B)) for j in blocks])
    q = np.asarray(Q[t0:t1], dtype=np.float64)
    kk = np.asarray(K[u], dtype=np.float64)
    vv = np.asarray(V[u], dtype=np.float64)
    s = q @ kk.T / math.sqrt(d)
    t = np.arange(t0, t1)
    s = np.where(u[None, :] <= t[:, None], s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p @ vv) / p.sum(axis=1, keepdims=True)


def sparse_attention(Q, K, V, row_ptr, col_idx, B: int, query_blocks: Optional[Sequence[int]] = None):
    """Attention output for all (or the listed) query blocks; rows of query
    blocks that are not listed are left as NaN."""
    n, d = Q.shape
    O = np.full((n, d), np.nan)
    b = len(row_ptr) - 1
    for i in (range(b) if query_blocks is None else query_blocks):
        blocks = col_idx[row_ptr[i]:row_ptr[i + 1]]
        O[i * B:min(n, (i + 1) * B)] = sparse_attention_block(Q, K, V, i, blocks, B)
    return O


class PrefillState:
    """The walk state R per query head, carried from layer to layer (§4)."""

    def __init__(self):
        self.R = {}


def group_shared_walk_rows(R_heads: Sequence[np.ndarray]) -> np.ndarray:
    """Selection scores shared by one GQA group: the sum of its heads' walk
    matrices, added in head order (their mean up to the factor 1/group, which
    does not change the ranking)."""
    acc = np.array(R_heads[0], dtype=np.float64, copy=True)
    for R in R_heads[1:]:
        acc = acc + R
    return acc


def group_shared_log_rows(rho_heads: np.ndarray) -> np.ndarray:
    """Decode counterpart: log(sum_h exp(rho_h)) per key block for the rows
    rho_heads [group, nb], as max + log(sum exp(rho - max))."""
    m = rho_heads.max(axis=0)
    return m + np.log(np.exp(rho_heads - m).sum(axis=0))


def prefill_layer(Q, K, V, Hd, B: int, s: int, density: Tuple[int, int], state: PrefillState,
                  heads: Optional[Sequence[int]] = None, attention_blocks="all", mode: str = "matrix_power",
                  select: str = "per_head"):
    """One layer of the prefill path for the listed query heads.

    Q [hq, n, d], K and V [hkv, n, d] (any float dtype; widened to fp64).
    Query head h reads KV head h // (hq / hkv). ``attention_blocks``: "all",
    None (skip attention), or a list of query blocks to compute.
    ``select``: "per_head" (each head its own top-tau) or "group_shared" (the
    group's heads share the top-tau of ``group_shared_walk_rows``; every head
    of a listed head's group is then computed, since the choice needs them all).
    Returns per head: q_tilde, k_tilde, S, R (the new walk state), CSR and O.
    """
    hq, hkv = Q.shape[0], K.shape[0]
    group = hq // hkv
    num, den = density
    out = {}
    kbar_cache = {}
    heads = list(range(hq) if heads is None else heads)
    if select == "group_shared":
        heads = sorted({g * group + r for h in heads for g in [h // group] for r in range(group)})
    shared = {}
    if select == "group_shared":
        # the walk of every head of the groups first, then one choice per group
        for h in heads:
            g = h // group
            q64 = np.asarray(Q[h], dtype=np.float64)
            if g not in kbar_cache:
                kbar_cache[g] = block_means(np.asarray(K[g], dtype=np.float64), B)
            qt = sketch_project(block_means(q64, B), Hd)
            kt = sketch_project(kbar_cache[g], Hd)
            S = sketch_scores(qt, kt)
            M = walk_matrix(block_attention(S), s, mode)
            R = walk_update(state.R.get(h), M)
            state.R[h] = R
            out[h] = dict(q_tilde=qt, k_tilde=kt, S=S, R=R)
        for g in sorted({h // group for h in heads}):
            shared[g] = select_top_tau(group_shared_walk_rows([out[g * group + r]["R"] for r in range(group)]),
                                       num, den)
        for h in heads:
            g = h // group
            row_ptr, col_idx = shared[g]
            O = None
            if attention_blocks is not None:
                qb = None if attention_blocks == "all" else attention_blocks
                O = sparse_attention(np.asarray(Q[h], dtype=np.float64), np.asarray(K[g], dtype=np.float64),
                                     np.asarray(V[g], dtype=np.float64), row_ptr, col_idx, B, qb)
            out[h].update(row_ptr=row_ptr, col_idx=col_idx, O=O,
                          shared_scores=group_shared_walk_rows([out[g * group + r]["R"] for r in range(group)]))
        return out
    for h in heads:
        g = h // group
        q64 = np.asarray(Q[h], dtype=np.float64)
        if g not in kbar_cache:
            kbar_cache[g] = block_means(np.asarray(K[g], dtype=np.float64), B)
        qt = sketch_project(block_means(q64, B), Hd)
        kt = sketch_project(kbar_cache[g], Hd)
        S = sketch_scores(qt, kt)
        M = walk_matrix(block_attention(S), s, mode)
        R = walk_update(state.R.get(h), M)
        state.R[h] = R
        row_ptr, col_idx = select_top_tau(R, num, den)
        O = None
        if attention_blocks is not None:
            qb = None if attention_blocks == "all" else attention_blocks
            O = sparse_attention(q64, np.asarray(K[g], dtype=np.float64), np.asarray(V[g], dtype=np.float64),
                                 row_ptr, col_idx, B, qb)
        out[h] = dict(q_tilde=qt, k_tilde=kt, S=S, R=R, row_ptr=row_ptr, col_idx=col_idx, O=O)
    return out


# ---------------------------------------------------------------------------
# §5 decode (readings R7, R8)
# ---------------------------------------------------------------------------

def decode_block_means(Kcache: np.ndarray, length: int, B: int) -> np.ndarray:
    """Block means of the first ``length`` cached keys (the partial block by its count)."""
    return block_means(np.asarray(Kcache[:length], dtype=np.float64), B)


def decode_layer_select(q_tok, Kcaches, length: int, Hd, B: int, s: int, density: Tuple[int, int],
                        rho_prev: Optional[np.ndarray], select: str = "per_head"):
    """Selection for one decode token in one layer, all query heads.

    q_tok [hq, d]; Kcaches [hkv, >=length, d] holds the new token at length-1.
    rho_prev [hq, nb] (None in the first layer). Returns (rho [hq, nb],
    z [hq, nb], sel: list of ascending block-index arrays, one per head).
    ``select`` = "group_shared": every head of a GQA group gets the top-tau of
    ``group_shared_log_rows`` of the group's rho rows (the walk state itself
    stays per head).
    """
    hq, hkv = q_tok.shape[0], Kcaches.shape[0]
    group = hq // hkv
    nb = -(-length // B)
    k = Hd.shape[1]
    tau = tau_of_row(nb - 1, *density)
    z = np.empty((hq, nb))
    kt = [sketch_project(decode_block_means(Kcaches[g], length, B), Hd) for g in range(hkv)]
    for h in range(hq):
        qt = np.asarray(q_tok[h], dtype=np.float64) @ Hd
        z[h] = kt[h // group] @ qt / math.sqrt(k)
    m = z.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(z - m).sum(axis=1, keepdims=True))
    rho = s * (z - lse) + (0.0 if rho_prev is None else rho_prev)
    if select == "group_shared":
        gsel = [top_tau_row(group_shared_log_rows(rho[g * group:(g + 1) * group]), tau) for g in range(hkv)]
        sel = [gsel[h // group] for h in range(hq)]
    else:
        sel = [top_tau_row(rho[h], tau) for h in range(hq)]
    return rho, z, sel


def decode_exact_layer(Q, K, Hd, B: int, s: int, density: Tuple[int, int], state: PrefillState,
                       heads: Optional[Sequence[int]] = None, select: str = "per_head"):
    """Exact decode walk, one layer (an extension of §5, the "next" row that
    replaces reading R7's log-domain reduction): the newest token's selection
    is the row of its query block i = ceil(n/B) - 1 in the walk state R^l of
    §4, computed by the prefill recurrence on the sequence as it stands.

    Q [hq, n, d] holds the queries of every position so far (prompt and
    decoded tokens), K [hkv, n, d] the keys. ``state`` carries R over the
    layers of one decode step (a fresh PrefillState per step: the query block
    i changes from step to step). Returns per head: ``row`` = R^l[i, :i+1],
    ``blocks`` = the chosen blocks (ascending) and ``score`` = what they were
    chosen on (R^l[i], or the group's summed rows for a group-shared choice).
    """
    res = prefill_layer(Q, K, K, Hd, B, s, density, state, heads=heads, attention_blocks=None, select=select)
    out = {}
    for h, r in res.items():
        R = r["R"]
        i = R.shape[0] - 1
        rp, ci = r["row_ptr"], r["col_idx"]
        score = r["shared_scores"][i] if select == "group_shared" else R[i]
        out[h] = dict(row=R[i, :i + 1].copy(), blocks=ci[rp[i]:rp[i + 1]].copy(), score=score[:i + 1].copy())
    return out


def decode_attention(q_tok, Kcache, Vcache, length: int, blocks: Sequence[int], B: int) -> np.ndarray:
    """One query row (the token at position length-1) over the tokens of the
    selected blocks that lie below ``length``; textbook two-pass softmax."""
    d = q_tok.shape[0]
    u = np.concatenate([np.arange(j * B, min(length, (j + 1) * B)) for j in blocks])
    kk = np.asarray(Kcache[u], dtype=np.float64)
    vv = np.asarray(Vcache[u], dtype=np.float64)
    sc = kk @ np.asarray(q_tok, dtype=np.float64) / math.sqrt(d)
    p = np.exp(sc - sc.max())
    return (p @ vv) / p.sum()

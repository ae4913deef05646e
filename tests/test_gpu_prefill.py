"""Parity of the prefill path (sws_sketch, sws_walk_select, sws_sparse_attn_prefill)
against the oracle, through the C ABI, on seeded synthetic inputs.

Small cases are compared element by element in full; the full-size workloads
are compared on sampled heads and query blocks (every layer, the whole walk
chain of the sampled heads), in the launch configuration the benchmark uses.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_sws_b200 as S
import oracle
import sws_inputs as W
from oracle import sws_oracle as so
from parity import (LazyHeads, check_csr_valid, compare_attention, compare_csr, compare_scores, compare_walk,
                    record_ties)

pytestmark = pytest.mark.gpu

MODES = {S.SWS_WALK_MATRIX_POWER: "matrix_power", S.SWS_WALK_ELEMENTWISE: "elementwise"}


def run_case(w: W.PrefillWorkload, heads=None, blocks=None, mode=S.SWS_WALK_MATRIX_POWER, report=None,
             shared=False):
    dev = "cuda"
    cfg = S.make_config(w.d, w.B, w.k, w.s, mode, w.density, w.seed,
                        select_group=(w.hq // w.hkv) if shared else 0)
    h = S.Handle(cfg)
    dtype = torch.float32 if w.dtype == "fp32" else torch.bfloat16
    path = S.PrefillPath(h, w.n, w.hq, w.hkv, dtype, dev)
    # the score matrix of the path, or (when the path forms the scores on chip)
    # one that sws_sketch writes on request, is checked against the oracle
    scores = path.scores if path.scores is not None else torch.empty(w.hq, w.b, w.b, dtype=torch.float64, device=dev)
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)
    st = so.PrefillState()
    heads = list(range(w.hq)) if heads is None else list(heads)
    group = w.hq // w.hkv
    swaps = []
    for layer in range(w.layers):
        Q, K, V = W.prefill_layer_inputs(w, layer, dev)
        path.layer(Q, K, V, layer == 0)
        if path.scores is None:
            S.sws_sketch(h, Q, K, path.q_sk, path.k_sk, scores, path.ws_sketch)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        ref = so.prefill_layer(LazyHeads(Q), LazyHeads(K), LazyHeads(V), Hd, w.B, w.s, w.density, st, heads=heads,
                               attention_blocks=None, mode=MODES[mode],
                               select="group_shared" if shared else "per_head")
        rp_all = path.row_ptr.cpu().numpy()
        ci_all = path.col_idx.cpu().numpy()
        for hh in heads:
            r = ref[hh]
            g = hh // group
            qs = path.q_sk[hh].cpu().numpy()
            assert np.allclose(qs, r["q_tilde"], rtol=1e-6, atol=1e-6 * np.abs(r["q_tilde"]).max())
            assert np.allclose(path.k_sk[g].cpu().numpy(), r["k_tilde"], rtol=1e-6,
                               atol=1e-6 * np.abs(r["k_tilde"]).max())
            compare_scores(scores[hh].cpu().numpy(), r["S"])
            compare_walk(path.walk_state[hh].cpu().numpy(), r["R"])
            rp, ci = rp_all[hh], ci_all[hh]
            check_csr_valid(rp, ci, w.b, *w.density)
            swaps += [(layer, hh) + s for s in compare_csr(rp, ci, r["row_ptr"], r["col_idx"],
                                                          r["shared_scores"] if shared else r["R"])]
            qb = range(w.b) if blocks is None else [i for i in blocks if 0 <= i < w.b]
            Qh, Kg, Vg = LazyHeads(Q)[hh], LazyHeads(K)[g], LazyHeads(V)[g]
            o_gpu = path.o[hh].float().cpu().numpy()
            for i in qb:
                cols = ci[rp[i]:rp[i + 1]]
                want = so.sparse_attention_block(Qh, Kg, Vg, i, cols, w.B)
                compare_attention(o_gpu[i * w.B:min(w.n, (i + 1) * w.B)], want)
    if report is not None:
        report.extend(swaps)
    record_ties(swaps, compared=w.layers * len(heads) * w.b)
    h.close()
    return swaps


def test_tiny_workload_in_full():
    """n=1024, d=64, B=64, k=16, fp32, two layers: every output compared."""
    swaps = run_case(W.TINY)
    assert len(swaps) == 0


@pytest.mark.parametrize("w", [
    W.PREFILL_16K.scaled(name="p16k_scaled", hq=8, hkv=2, n=2000),                 # ragged tail, B=64
    W.PREFILL_64K.scaled(name="p64k_scaled", hq=4, hkv=1, n=8292),                 # ragged, B=128, 8 layers
    W.PREFILL_128K_D10.scaled(name="p128k_d10_scaled", hq=4, hkv=1, n=16384),      # density 1/10
], ids=lambda w: w.name)
def test_scaled_workloads_in_full(w):
    swaps = run_case(w)


@pytest.mark.parametrize("w,mode", [
    (W.TINY.scaled(name="dense", density=(1, 1), n=640, hq=2, hkv=1), 0),
    (W.TINY.scaled(name="s1_one_hop", s=1, layers=1), 0),
    (W.TINY.scaled(name="elementwise", layers=3), 1),
    (W.TINY.scaled(name="k_eq_d", k=64), 0),
    (W.TINY.scaled(name="n_below_B", n=50, hubs=0), 0),
    (W.TINY.scaled(name="n_one", n=1, hubs=0), 0),
    (W.TINY.scaled(name="one_row_tail", n=65), 0),
    (W.PREFILL_16K.scaled(name="bf16_d64_B128", d=64, B=128, k=16, n=3000, hq=4, hkv=2, layers=2), 0),
    (W.PREFILL_16K.scaled(name="gqa8", n=1500, hq=8, hkv=1, layers=2), 0),
    (W.PREFILL_16K.scaled(name="odd_blocks_B64", n=1050, hq=2, hkv=1, layers=2), 0),
    (W.PREFILL_16K.scaled(name="bf16_one_block", n=100, hq=2, hkv=1, layers=1, hubs=0), 0),
    (W.PREFILL_64K.scaled(name="bf16_B128_dense", n=700, hq=2, hkv=1, layers=1, density=(1, 1)), 0),
    (W.PREFILL_16K.scaled(name="bf16_d64_B64", d=64, k=16, n=2500, hq=4, hkv=2, layers=2), 0),
    (W.PREFILL_16K.scaled(name="fp32_d128_B64", dtype="fp32", n=1100, hq=2, hkv=1, layers=2), 0),
    (W.PREFILL_64K.scaled(name="fp32_d128_B128", dtype="fp32", n=1500, hq=2, hkv=1, layers=2), 0),
    (W.TINY.scaled(name="fp32_d64_B128", B=128, n=1000, layers=2), 0),
], ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_edge_cases(w, mode):
    run_case(w, mode=mode)


def test_dense_density_equals_dense_attention():
    """Density 100%: the GPU's prefill output equals dense causal attention (torch SDPA, fp64)."""
    w = W.TINY.scaled(density=(1, 1), n=512, layers=1)
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    path = S.PrefillPath(h, w.n, w.hq, w.hkv, torch.float32)
    Q, K, V = W.prefill_layer_inputs(w, 0, "cuda")
    o = path.layer(Q, K, V, True)
    ref = torch.nn.functional.scaled_dot_product_attention(Q.double()[None], K.double()[None], V.double()[None],
                                                           is_causal=True)[0]
    assert (o.double() - ref).abs().max().item() < 1e-4


def test_dense_density_equals_dense_attention_bf16():
    """Density 100% on the tensor-core path: equals dense causal attention (fp64 SDPA) within bf16 tolerance."""
    for w in (W.PREFILL_16K.scaled(density=(1, 1), n=1000, hq=4, hkv=2, layers=1),
              W.PREFILL_64K.scaled(density=(1, 1), n=1000, hq=2, hkv=1, layers=1)):
        cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
        h = S.Handle(cfg)
        path = S.PrefillPath(h, w.n, w.hq, w.hkv, torch.bfloat16)
        Q, K, V = W.prefill_layer_inputs(w, 0, "cuda")
        o = path.layer(Q, K, V, True)
        g = w.hq // w.hkv
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q.double()[None], K.double().repeat_interleave(g, 0)[None], V.double().repeat_interleave(g, 0)[None],
            is_causal=True)[0]
        err = (o.double() - ref).abs()
        assert err.max().item() < 2e-2 and err.mean().item() < 5e-3


FULL = [W.PREFILL_16K, W.PREFILL_64K, W.PREFILL_128K, W.PREFILL_128K_D10]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled(w):
    """Full-size workload on the GPU; the oracle recomputes two sampled heads
    (whole walk chain) and sampled query blocks of their attention."""
    b = w.b
    blocks = sorted({0, 1, b // 3, b // 2, b - 2, b - 1})
    swaps = run_case(w, heads=[0, w.hq - 1], blocks=blocks)


def test_device_guard_reports_bad_csr():
    """A column outside [0, i] is skipped by the kernel and reported through the
    device error word; nothing faults and later calls still work."""
    w = W.TINY.scaled(layers=1)
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    path = S.PrefillPath(h, w.n, w.hq, w.hkv, torch.float32)
    Q, K, V = W.prefill_layer_inputs(w, 0, "cuda")
    path.layer(Q, K, V, True)
    assert S.sws_sync_check(h) == 0
    bad = path.col_idx.clone()
    bad[0, -1] = w.b + 7
    S.sws_sparse_attn_prefill(h, Q, K, V, path.row_ptr, bad, path.o)
    assert S.sws_sync_check(h) == 2  # GUARD_BAD_CSR
    assert S.sws_sync_check(h) == 0  # cleared
    path.layer(Q, K, V, True)
    assert S.sws_sync_check(h) == 0


def test_repeat_runs_bit_identical():
    """Race canary: two runs give the same CSR and the same bits of output."""
    w = W.PREFILL_16K.scaled(n=4096, hq=8, hkv=2, layers=2)
    outs = []
    for _ in range(2):
        cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
        h = S.Handle(cfg)
        path = S.PrefillPath(h, w.n, w.hq, w.hkv)
        res = []
        for layer in range(w.layers):
            Q, K, V = W.prefill_layer_inputs(w, layer, "cuda")
            o = path.layer(Q, K, V, layer == 0)
            res.append((path.col_idx.clone(), o.clone(), path.walk_state.clone()))
        outs.append(res)
    for a, b in zip(*outs):
        for x, y in zip(a, b):
            assert torch.equal(x, y)


@pytest.mark.parametrize("w,mode", [
    (W.PREFILL_16K.scaled(name="p16k", n=3000, hq=8, hkv=2, layers=3), 0),
    (W.PREFILL_64K.scaled(name="p64k", n=9000, hq=4, hkv=1, layers=2), 0),
    (W.PREFILL_16K.scaled(name="elementwise", n=2000, hq=4, hkv=2, layers=2), 1),
    (W.PREFILL_16K.scaled(name="k64_d64", d=64, k=64, n=1500, hq=2, hkv=1, layers=2), 0),
    (W.TINY.scaled(name="tiny_k16", layers=2), 0),
], ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_scores_on_chip_match_scores_in_memory(w, mode):
    """sws_walk_select_sketch (scores formed on chip) against sws_sketch's score
    matrix fed to sws_walk_select: the same walk state to rounding, the same
    selections."""
    dtype = torch.float32 if w.dtype == "fp32" else torch.bfloat16
    cfg = S.make_config(w.d, w.B, w.k, w.s, mode, w.density, w.seed)
    h = S.Handle(cfg)
    a = S.PrefillPath(h, w.n, w.hq, w.hkv, dtype, scores_in_memory=False)
    b = S.PrefillPath(h, w.n, w.hq, w.hkv, dtype, scores_in_memory=True)
    for layer in range(w.layers):
        Q, K, V = W.prefill_layer_inputs(w, layer, "cuda")
        oa = a.layer(Q, K, V, layer == 0)
        ob = b.layer(Q, K, V, layer == 0)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        assert torch.equal(a.q_sk, b.q_sk) and torch.equal(a.k_sk, b.k_sk)
        Ra, Rb = a.walk_state, b.walk_state
        low = Rb > 1e-280
        rel = ((Ra - Rb).abs()[low] / Rb[low]).max().item()
        assert rel < 1e-12, rel
        assert torch.equal(a.row_ptr, b.row_ptr)
        same = (a.col_idx == b.col_idx).all().item()
        if not same:  # only where two walk scores tie to rounding
            ca, cb = a.col_idx.cpu().numpy(), b.col_idx.cpu().numpy()
            rp = b.row_ptr.cpu().numpy()
            Rn = Rb.cpu().numpy()
            for hh in range(w.hq):
                for i in range(w.b):
                    x, y = set(ca[hh, rp[hh, i]:rp[hh, i + 1]]), set(cb[hh, rp[hh, i]:rp[hh, i + 1]])
                    for u, v in zip(sorted(x - y), sorted(y - x)):
                        assert abs(Rn[hh, i, u] - Rn[hh, i, v]) <= 1e-12 * Rn[hh, i, v]
        else:
            assert torch.equal(oa, ob)
    h.close()


@pytest.mark.parametrize("w", [
    W.PREFILL_16K.scaled(name="bf16_B64", n=3000, hq=8, hkv=2, layers=2),
    W.PREFILL_64K.scaled(name="bf16_B128", n=2500, hq=4, hkv=1, layers=2),
    W.PREFILL_16K.scaled(name="fp32_B64", dtype="fp32", n=1100, hq=2, hkv=1, layers=1),
], ids=lambda w: w.name)
def test_strided_operands_read_in_place(w):
    """Q, K, V held as [n, heads, d] activations (the layout a model produces)
    and O written into an [n, hq, d] buffer, through strides: the same
    sketches, selection and output bits as the dense [heads, n, d] layout, and
    the output within tolerance of the oracle."""
    dtype = torch.float32 if w.dtype == "fp32" else torch.bfloat16
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    dense = S.PrefillPath(h, w.n, w.hq, w.hkv, dtype)
    strided = S.PrefillPath(h, w.n, w.hq, w.hkv, dtype)
    for layer in range(w.layers):
        Q, K, V = W.prefill_layer_inputs(w, layer, "cuda")
        Qn, Kn, Vn = (x.transpose(0, 1).contiguous() for x in (Q, K, V))  # [n, heads, d]
        Qv, Kv, Vv = (x.transpose(0, 1) for x in (Qn, Kn, Vn))          # strided [heads, n, d] views
        assert not Qv.is_contiguous() and Qv.stride() == (w.d, w.hq * w.d, 1)
        On = torch.full((w.n, w.hq, w.d), float("nan"), dtype=dtype, device="cuda")
        od = dense.layer(Q, K, V, layer == 0)
        strided.layer(Qv, Kv, Vv, layer == 0, out=On.transpose(0, 1))
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        assert torch.equal(strided.q_sk, dense.q_sk) and torch.equal(strided.k_sk, dense.k_sk)
        assert torch.equal(strided.row_ptr, dense.row_ptr) and torch.equal(strided.col_idx, dense.col_idx)
        assert torch.equal(On.transpose(0, 1), od)
    # one head of the last layer against the oracle's attention on the same selection
    rp, ci = dense.row_ptr[0].cpu().numpy(), dense.col_idx[0].cpu().numpy()
    q64, k64, v64 = (x[0].double().cpu().numpy() for x in (Q, K, V))
    want = so.sparse_attention(q64, k64, v64, rp, ci, w.B)
    compare_attention(On[:, 0].float().cpu().numpy(), want)
    h.close()


def test_invalid_arguments_queue_nothing():
    cfg = S.make_config()
    h = S.Handle(cfg)
    q = torch.zeros(4, 256, 128, dtype=torch.bfloat16, device="cuda")
    kk = torch.zeros(3, 256, 128, dtype=torch.bfloat16, device="cuda")  # 4 % 3 != 0
    out = torch.zeros(4, 4, 32, dtype=torch.float64, device="cuda")
    with pytest.raises(S.SwsError) as e:
        S.sws_sketch(h, q, kk, out, out, out, torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == S.SWS_ERR_INVALID_ARG
    ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(4, 4, 4, dtype=torch.float64, device="cuda")
    with pytest.raises(S.SwsError) as e:
        S.sws_walk_select(h, sc, 256, True, sc, torch.zeros(4, 5, dtype=torch.int32, device="cuda"),
                          torch.zeros(4, 8, dtype=torch.int32, device="cuda"), ws)
    assert e.value.status == S.SWS_ERR_WORKSPACE
    # a head stride of 132 elements (264 bytes) leaves rows off the 16-byte grid
    qpad = torch.zeros(256, 4, 132, dtype=torch.bfloat16, device="cuda")[:, :, :128].transpose(0, 1)
    k1 = torch.zeros(1, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SwsError) as e:
        S.sws_sketch(h, qpad, k1, out, out, None, ws)
    assert e.value.status == S.SWS_ERR_INVALID_ARG
    with pytest.raises(S.SwsError) as e:
        S.sws_sparse_attn_prefill(h, qpad, k1, k1, torch.zeros(4, 5, dtype=torch.int32, device="cuda"),
                                  torch.zeros(4, 8, dtype=torch.int32, device="cuda"), torch.zeros_like(q))
    assert e.value.status == S.SWS_ERR_INVALID_ARG


def test_dense_first_layers_policy():
    """The dense-first-layers policy of §7: layers 0-1 select every causal block
    (the walk still runs through them), later layers the configured density;
    compared with the oracle run with density 1/1 for the first two layers."""
    w = W.PREFILL_16K.scaled(name="dense_first2", n=2000, hq=4, hkv=2, layers=4)
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    path = S.PrefillPath(h, w.n, w.hq, w.hkv, dense_layers=2)
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)
    st = so.PrefillState()
    for layer in range(w.layers):
        Q, K, V = W.prefill_layer_inputs(w, layer, "cuda")
        o = path.layer(Q, K, V, layer == 0, layer=layer)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        dens = (1, 1) if layer < 2 else w.density
        ref = so.prefill_layer(LazyHeads(Q), LazyHeads(K), LazyHeads(V), Hd, w.B, w.s, dens, st, heads=range(w.hq),
                               attention_blocks=None)
        rp_all, ci_all = (x.cpu().numpy() for x in path.csr(layer))
        og = o.float().cpu().numpy()
        for hh in range(w.hq):
            r = ref[hh]
            compare_walk(path.walk_state[hh].cpu().numpy(), r["R"])
            rp, ci = rp_all[hh], ci_all[hh]
            check_csr_valid(rp, ci, w.b, *dens)
            compare_csr(rp, ci, r["row_ptr"], r["col_idx"], r["R"])
            Qh, Kg, Vg = LazyHeads(Q)[hh], LazyHeads(K)[hh // 2], LazyHeads(V)[hh // 2]
            for i in (0, w.b // 2, w.b - 1):
                want = so.sparse_attention_block(Qh, Kg, Vg, i, ci[rp[i]:rp[i + 1]], w.B)
                compare_attention(og[hh, i * w.B:min(w.n, (i + 1) * w.B)], want)


@pytest.mark.parametrize("w", [
    W.PREFILL_16K.scaled(name="shared_p16k", hq=8, hkv=2, n=2000, layers=3),
    W.PREFILL_64K.scaled(name="shared_p64k", hq=4, hkv=1, n=4200, layers=2),
], ids=lambda w: w.name)
def test_group_shared_selection(w):
    """Group-shared selection: every head of a GQA group gets the top-tau of
    the sum of the group's walk rows; the walk state stays per head."""
    swaps = run_case(w, shared=True)


@pytest.mark.parametrize("shared", [False, True])
def test_beyond_1024_blocks(shared):
    """b = 1094 key blocks: past the register-resident row kernels, the walk's
    softmax and the top-tau selection take their general forms (rows staged
    through global and shared memory). Two heads of one KV head, whole walk
    chain over two layers, attention on sampled query blocks."""
    w = W.PREFILL_16K.scaled(name="b1094_B64", n=70000, hq=2, hkv=1, layers=2)
    b = w.b
    assert b > 1024
    swaps = run_case(w, blocks=sorted({0, 1, 511, 1023, 1024, b - 2, b - 1}), shared=shared)


@pytest.mark.parametrize("b", [1025, 1030])
def test_walk_products_on_64_tiles(b):
    """Walks of 1024 blocks and more take the 64 x 64 tiles of the walk product.
    b = 1025 (odd: rows not 16-byte aligned, 8-byte copies) and b = 1030 (a
    ragged last tile row): the whole walk chain of two heads over two layers
    against the oracle, attention on sampled query blocks."""
    w = W.PREFILL_16K.scaled(name=f"b{b}_B64", n=b * 64 - 21, hq=2, hkv=1, layers=2)
    assert w.b == b
    run_case(w, blocks=sorted({0, 1, 63, 64, 511, b - 2, b - 1}))


def test_prefill_batch_matches_single_sequences():
    """PrefillBatch: three sequences of different lengths (ragged tails), their
    layers on concurrent streams, give bit for bit what each sequence gives
    alone through PrefillPath (which the tests above hold to the oracle)."""
    base = W.PREFILL_16K.scaled(hq=8, hkv=2, layers=2)
    ws = [base.scaled(name=f"seq{i}", n=n, seed=base.seed + i) for i, n in enumerate((1000, 2065, 640))]
    cfg = S.make_config(base.d, base.B, base.k, base.s, 0, base.density, base.seed)
    h = S.Handle(cfg)
    batch = S.PrefillBatch(h, [w.n for w in ws], base.hq, base.hkv, torch.bfloat16, "cuda")
    singles = [S.PrefillPath(h, w.n, base.hq, base.hkv, torch.bfloat16, "cuda") for w in ws]
    for layer in range(base.layers):
        ins = [W.prefill_layer_inputs(w, layer, "cuda") for w in ws]
        outs = batch.layer([x[0] for x in ins], [x[1] for x in ins], [x[2] for x in ins], layer == 0)
        for p, (Q, K, V) in zip(singles, ins):
            p.layer(Q, K, V, layer == 0)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        for bp, p, o in zip(batch.paths, singles, outs):
            assert torch.equal(bp.row_ptr, p.row_ptr) and torch.equal(bp.col_idx, p.col_idx)
            assert torch.equal(bp.walk_state, p.walk_state)
            assert torch.equal(o.view(torch.int16), p.o.view(torch.int16))
    h.close()


@pytest.mark.parametrize("w0,strided", [
    (W.PREFILL_16K.scaled(name="packed_B64", hq=8, hkv=2, layers=2), False),
    (W.PREFILL_16K.scaled(name="packed_B64_strided", hq=8, hkv=2, layers=2), True),
    (W.PREFILL_64K.scaled(name="packed_B128_d64", d=64, k=16, hq=4, hkv=2, layers=2), False),
], ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_packed_prefill_matches_single_sequences(w0, strided):
    """sws_sparse_attn_prefill_varlen through PrefillBatch.layer_packed: five
    sequences end to end (ragged tails, one shorter than a block, one of exactly
    two slabs) in one attention launch. Each sequence's rows equal, bit for
    bit, what its own PrefillPath gives (held to the oracle above), its walk and
    CSR too; sampled query blocks of every sequence are also compared with the
    oracle on the packed output. strided: Q, K, V and O are [N, heads, d]
    activations read and written in place."""
    lengths = (1000, 2065, 40, 512, 1537)
    ws = [w0.scaled(name=f"seq{i}", n=n, seed=w0.seed + i) for i, n in enumerate(lengths)]
    cfg = S.make_config(w0.d, w0.B, w0.k, w0.s, 0, w0.density, w0.seed)
    h = S.Handle(cfg)
    batch = S.PrefillBatch(h, lengths, w0.hq, w0.hkv, torch.bfloat16, "cuda")
    singles = [S.PrefillPath(h, n, w0.hq, w0.hkv, torch.bfloat16, "cuda") for n in lengths]
    cu = batch.cu_seqlens
    N = cu[-1]

    def packed(parts):
        x = torch.cat(parts, dim=1)
        return x.transpose(0, 1).contiguous().transpose(0, 1) if strided else x

    out = torch.full((N, w0.hq, w0.d), float("nan"), dtype=torch.bfloat16, device="cuda").transpose(0, 1) \
        if strided else None
    for layer in range(w0.layers):
        ins = [W.prefill_layer_inputs(w, layer, "cuda") for w in ws]
        Q, K, V = (packed([x[j] for x in ins]) for j in range(3))
        o = batch.layer_packed(Q, K, V, layer == 0, out=out)
        for p, (q, k, v) in zip(singles, ins):
            p.layer(q, k, v, layer == 0)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        for i, (bp, p) in enumerate(zip(batch.paths, singles)):
            assert torch.equal(bp.row_ptr, p.row_ptr) and torch.equal(bp.col_idx, p.col_idx)
            assert torch.equal(bp.walk_state, p.walk_state)
            assert torch.equal(o[:, cu[i]:cu[i + 1]].contiguous().view(torch.int16), p.o.view(torch.int16))
    group = w0.hq // w0.hkv
    for i, (w, (q, k, v)) in enumerate(zip(ws, ins)):
        rp = batch.paths[i].row_ptr.cpu().numpy()
        ci = batch.paths[i].col_idx.cpu().numpy()
        for hh in (0, w0.hq - 1):
            Qh, Kg, Vg = LazyHeads(q)[hh], LazyHeads(k)[hh // group], LazyHeads(v)[hh // group]
            o_gpu = o[hh, cu[i]:cu[i + 1]].float().cpu().numpy()
            for qb in sorted({0, w.b // 2, w.b - 1}):
                cols = ci[hh][rp[hh][qb]:rp[hh][qb + 1]]
                compare_attention(o_gpu[qb * w.B:min(w.n, (qb + 1) * w.B)],
                                  so.sparse_attention_block(Qh, Kg, Vg, qb, cols, w.B))
    h.close()


def test_packed_prefill_invalid_arguments():
    """Host validation of the packed launch: nothing is queued."""
    cfg = S.make_config(128, 64, 32)
    h = S.Handle(cfg)
    q = torch.zeros(4, 600, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 600, 128, dtype=torch.bfloat16, device="cuda")
    rp = [torch.zeros(4, 8, dtype=torch.int32, device="cuda") for _ in range(2)]
    ci = [torch.zeros(4, 64, dtype=torch.int32, device="cuda") for _ in range(2)]
    ws = torch.zeros(S.sws_sparse_attn_prefill_varlen_ws_bytes([0, 300, 600]), dtype=torch.uint8, device="cuda")
    cases = [
        ([0, 300, 600], q.float(), kv.float(), ws, S.SWS_ERR_UNSUPPORTED),   # fp32
        ([1, 300, 600], q, kv, ws, S.SWS_ERR_INVALID_ARG),                   # does not start at 0
        ([0, 300, 300], q, kv, ws, S.SWS_ERR_INVALID_ARG),                   # an empty sequence
        ([0, 300, 600], q, kv, ws[:16], S.SWS_ERR_WORKSPACE),                # workspace too small
    ]
    for cu, qq, kk, w, want in cases:
        with pytest.raises(S.SwsError) as e:
            S.sws_sparse_attn_prefill_varlen(h, qq, kk, kk, cu, rp, ci, torch.zeros_like(qq), w)
        assert e.value.status == want, cu
    torch.cuda.synchronize()
    assert S.sws_sync_check(h) == 0
    h.close()


def test_prefill_at_the_largest_walk():
    """The largest walk the library takes: 8192 key blocks (524,288 tokens at
    B = 64), two query heads of one KV head, one layer, in the 64 x 64-tile walk
    products and the general selection kernel.
    - Sketches and sampled score rows against the oracle.
    - The walk: A and R are lower-triangular, so the leading m x m block of
      R = A^s is the s-th power of A's leading m x m block; the oracle's walk on
      the first 512 blocks is compared with the GPU's, and so is the selection
      of those rows. The whole of R is lower-triangular and row-stochastic.
    - Sampled rows past 512: the selection is the top-tau (ties to the lower
      index) of the GPU's own row of R, and the CSR is valid throughout.
    - Attention on sampled query blocks against the oracle fed the GPU's CSR."""
    w = W.PREFILL_16K.scaled(name="b8192_B64", n=8192 * 64, hq=2, hkv=1, layers=1)
    b, m = w.b, 512
    assert b == 8192
    num, den = w.density
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    path = S.PrefillPath(h, w.n, w.hq, w.hkv, torch.bfloat16, "cuda")
    Q, K, V = W.prefill_layer_inputs(w, 0, "cuda")
    path.layer(Q, K, V, True)
    torch.cuda.synchronize()
    assert S.sws_sync_check(h) == 0
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)
    Kt = so.sketch_project(so.block_means(LazyHeads(K)[0], w.B), Hd)
    assert np.allclose(path.k_sk[0].cpu().numpy(), Kt, rtol=1e-6, atol=1e-6 * np.abs(Kt).max())
    rows = sorted({0, 1, 511, 512, 1023, 1024, 4095, b - 2, b - 1})
    rp_all, ci_all = path.row_ptr.cpu().numpy(), path.col_idx.cpu().numpy()
    swaps = []
    for hh in range(w.hq):
        Qt = so.sketch_project(so.block_means(LazyHeads(Q)[hh], w.B), Hd)
        assert np.allclose(path.q_sk[hh].cpu().numpy(), Qt, rtol=1e-6, atol=1e-6 * np.abs(Qt).max())
        S_or = so.sketch_scores(Qt, Kt)
        S_gpu = path.scores[hh].cpu().numpy()
        for i in rows:
            want, got = S_or[i, :i + 1], S_gpu[i, :i + 1]
            bound = 1e-3 * np.maximum(np.abs(want), np.sqrt((want ** 2).mean()))
            assert np.all(np.abs(got - want) <= bound), i
        R = path.walk_state[hh].cpu().numpy()
        assert not np.triu(R, 1).any()
        assert np.allclose(R.sum(axis=1), 1.0, rtol=0, atol=1e-9)
        R_lead = so.walk_matrix(so.block_attention(S_or[:m, :m]), w.s)
        compare_walk(R[:m, :m], R_lead)
        rp, ci = rp_all[hh], ci_all[hh]
        check_csr_valid(rp, ci, b, num, den)
        orp, oci = so.select_top_tau(R_lead, num, den)
        swaps += compare_csr(rp[:m + 1], ci, orp, oci, R_lead)
        for i in rows:
            assert np.array_equal(ci[rp[i]:rp[i + 1]], so.top_tau_row(R[i, :i + 1], so.tau_of_row(i, num, den))), i
        del S_or, S_gpu, R
        Qh, Kg, Vg = LazyHeads(Q)[hh], LazyHeads(K)[0], LazyHeads(V)[0]
        o_gpu = path.o[hh].float().cpu().numpy()
        for i in (0, 4095, b - 1):
            cols = ci[rp[i]:rp[i + 1]]
            compare_attention(o_gpu[i * w.B:(i + 1) * w.B], so.sparse_attention_block(Qh, Kg, Vg, i, cols, w.B))
    record_ties(swaps, compared=w.hq * m)
    h.close()


def test_packed_prefill_with_dense_layers_and_shared_selection():
    """The packed launch under the dense-first-layers policy (layer 0 through a
    density-1/1 handle) and group-shared selection: each sequence's rows equal
    its own PrefillPath's, bit for bit, over three layers."""
    w0 = W.PREFILL_16K.scaled(name="packed_policy", hq=8, hkv=2, layers=3)
    lengths = (1500, 333, 2100)
    ws = [w0.scaled(name=f"seq{i}", n=n, seed=w0.seed + 10 + i) for i, n in enumerate(lengths)]
    cfg = S.make_config(w0.d, w0.B, w0.k, w0.s, 0, w0.density, w0.seed, select_group=w0.hq // w0.hkv)
    h = S.Handle(cfg)
    batch = S.PrefillBatch(h, lengths, w0.hq, w0.hkv, torch.bfloat16, "cuda", dense_layers=1)
    singles = [S.PrefillPath(h, n, w0.hq, w0.hkv, torch.bfloat16, "cuda", dense_layers=1) for n in lengths]
    cu = batch.cu_seqlens
    for layer in range(w0.layers):
        ins = [W.prefill_layer_inputs(w, layer, "cuda") for w in ws]
        Q, K, V = (torch.cat([x[j] for x in ins], dim=1) for j in range(3))
        o = batch.layer_packed(Q, K, V, layer == 0, layer=layer)
        for p, (q, k, v) in zip(singles, ins):
            p.layer(q, k, v, layer == 0, layer=layer)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        for i, (bp, p) in enumerate(zip(batch.paths, singles)):
            rp_b, ci_b = bp.csr(layer)
            rp_s, ci_s = p.csr(layer)
            assert torch.equal(rp_b, rp_s) and torch.equal(ci_b, ci_s)
            assert torch.equal(bp.walk_state, p.walk_state)
            assert torch.equal(o[:, cu[i]:cu[i + 1]].contiguous().view(torch.int16), p.o.view(torch.int16))
    h.close()

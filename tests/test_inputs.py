"""The seeded workload generator: determinism and the recipe's statistics."""
import math

import numpy as np
import torch

import sws_inputs as W


def test_linear_scan_matches_sequential_loop():
    g = torch.Generator().manual_seed(3)
    e = torch.randn(3, 1000, 5, generator=g, dtype=torch.float64)
    a = 0.93
    want = torch.empty_like(e)
    acc = torch.zeros(3, 5, dtype=torch.float64)
    for t in range(e.shape[1]):
        acc = a * acc + e[:, t]
        want[:, t] = acc
    got = W._linear_scan(e, a, chunk=16)
    assert torch.allclose(got, want, atol=1e-11)


def test_ar1_statistics():
    x = W.ar1(200000, 4, 0.9, W._gen("cpu", 11), "cpu").numpy()
    assert abs(x.var() - 1.0) < 0.05
    lag1 = (x[1:] * x[:-1]).mean() / x.var()
    assert abs(lag1 - 0.9) < 0.01


def test_prefill_inputs_deterministic_and_structured():
    w = W.TINY.scaled(hq=4, hkv=2, n=512, d=32)
    Q1, K1, V1 = W.prefill_layer_inputs(w, 0)
    Q2, K2, V2 = W.prefill_layer_inputs(w, 0)
    assert torch.equal(Q1, Q2) and torch.equal(K1, K2) and torch.equal(V1, V2)
    Q3, _, _ = W.prefill_layer_inputs(w, 1)
    assert not torch.equal(Q1, Q3)
    assert Q1.shape == (4, 512, 32) and K1.shape == (2, 512, 32) and Q1.dtype == torch.float32
    # sink: block 0 is shifted by +1 in Q and K
    assert K1[:, :w.B].mean() > 0.7 and abs(K1[:, w.B:].mean()) < 0.3
    pos, off = W.hub_layout(w.b, w.hubs, w.d, w.seed, 0, 0, "cpu")
    assert pos.numel() == w.hubs and len(set(pos.tolist())) == w.hubs and int(pos.min()) >= 1
    assert off.shape == (w.hubs, w.d)


def test_bf16_workload_dtype():
    w = W.PREFILL_16K.scaled(n=256, hq=4, hkv=1, layers=1)
    Q, K, V = W.prefill_layer_inputs(w, 0)
    assert Q.dtype == K.dtype == V.dtype == torch.bfloat16


def test_decode_inputs():
    w = W.DECODE_128K.scaled(batch=2, n0=256, steps=4, hq=4, hkv=1)
    K, V = W.decode_cache_inputs(w, 0, 0)
    assert K.shape == (1, 260, 128) and V.shape == (1, 260, 128)
    Q = W.decode_queries(w, 1, 0)
    assert Q.shape == (4, 4, 128)
    K2, _ = W.decode_cache_inputs(w, 1, 0)
    assert not torch.equal(K, K2)


def test_head_inputs_match_layer_inputs():
    w = W.TINY.scaled(hq=4, hkv=2, n=300, d=16, dtype="fp32")
    Q, K, V = W.prefill_layer_inputs(w, 1)
    for h in range(4):
        q, k, v = W.prefill_head_inputs(w, 1, h)
        assert torch.equal(q, Q[h]) and torch.equal(k, K[h // 2]) and torch.equal(v, V[h // 2])


def test_decode_sequence_queries():
    """The exact decode walk's per-position queries: deterministic, one stream
    per query head (distinct heads differ), the sink on block 0 and the KV
    group's hubs on the same blocks as the keys."""
    w = W.DECODE_128K.scaled(batch=2, layers=1, hq=4, hkv=2, n0=640, steps=3, hubs=2)
    Q = W.decode_sequence_queries(w, 1, 0, "cpu")
    assert Q.shape == (4, 643, 128) and Q.dtype == torch.bfloat16
    assert torch.equal(Q, W.decode_sequence_queries(w, 1, 0, "cpu"))
    assert not torch.equal(Q[0], Q[1])
    assert not torch.equal(Q, W.decode_sequence_queries(w, 0, 0, "cpu"))
    q = Q.double()
    assert abs(q[:, :w.B].mean().item() - 1.0) < 0.15          # sink shift on block 0
    assert abs(q[:, 2 * w.B:].mean().item()) < 0.15
    pos, off = W.hub_layout(-(-w.n0 // w.B), w.hubs, w.d, w.seed, 0, 0, "cpu", 1)
    for j, p in enumerate(pos.tolist()):                       # group 0's hubs move heads 0 and 1 alike
        blk = q[:2, p * w.B:(p + 1) * w.B].mean(dim=(0, 1))
        assert torch.corrcoef(torch.stack([blk, off[j]]))[0, 1] > 0.8

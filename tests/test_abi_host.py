"""Host-side checks of the C ABI: no GPU and no compute kernel needed.

The library loads, exports every function include/sws.h declares, validates
its arguments and computes its host-only quantities (block counts, CSR sizes,
workspace sizes, the projection matrix) as the oracle does.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_attention_sws_b200 as S
from block_sparse_attention_sws_b200 import build as B
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return S.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "sws.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sws_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    decl = declared_functions()
    assert len(decl) >= 15
    assert sorted(S.EXPORTS) == decl
    for name in decl:
        assert hasattr(lib, name), name


def test_nm_lists_symbols_as_c(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True).stdout
    names = set(re.findall(r"\bT (sws_\w+)", out))
    assert set(declared_functions()) <= names


def test_status_strings(lib):
    for s in range(6):
        assert S.status_string(s)
    assert S.status_string(99) == "unknown status"


@pytest.mark.parametrize("field,value,want", [
    ("head_dim", 96, S.SWS_ERR_UNSUPPORTED), ("head_dim", 0, S.SWS_ERR_UNSUPPORTED),
    ("block_size", 32, S.SWS_ERR_UNSUPPORTED), ("sketch_dim", 0, S.SWS_ERR_INVALID_ARG),
    ("sketch_dim", 129, S.SWS_ERR_INVALID_ARG), ("walk_power", 0, S.SWS_ERR_INVALID_ARG),
    ("walk_power", 65, S.SWS_ERR_INVALID_ARG), ("walk_mode", 2, S.SWS_ERR_INVALID_ARG),
    ("density_num", 0, S.SWS_ERR_INVALID_ARG), ("density_num", 6, S.SWS_ERR_INVALID_ARG),
    ("select_group", 9, S.SWS_ERR_INVALID_ARG), ("select_group", -1, S.SWS_ERR_INVALID_ARG),
])
def test_config_rejections(lib, field, value, want):
    cfg = S.make_config()
    setattr(cfg, field, value)
    assert S.sws_config_check(cfg) == want


def test_config_accepts_defaults(lib):
    assert S.sws_config_check(S.make_config()) == S.SWS_OK
    assert S.sws_config_check(S.make_config(64, 128, 64, 1, S.SWS_WALK_ELEMENTWISE, (1, 1), 5)) == S.SWS_OK


@pytest.mark.parametrize("n,B,num,den", [(1024, 64, 1, 5), (16384, 64, 1, 5), (131072, 128, 1, 10),
                                          (1000, 64, 1, 5), (1, 64, 1, 5), (65536, 128, 3, 7)])
def test_blocks_and_nnz_match_oracle(lib, n, B, num, den):
    cfg = S.make_config(128, B, 32, 8, 0, (num, den))
    b = -(-n // B)
    assert S.sws_num_blocks(cfg, n) == b
    assert S.sws_csr_nnz(cfg, n) == oracle.csr_nnz(b, num, den)


def test_invalid_sizes(lib):
    cfg = S.make_config()
    assert S.sws_num_blocks(cfg, 0) == -1 and S.sws_csr_nnz(cfg, -5) == -1


@pytest.mark.parametrize("d,k,seed", [(64, 16, 0), (128, 32, 1), (128, 32, 2), (128, 64, 3), (128, 128, 4),
                                      (64, 1, 12345678901234), (128, 7, 2 ** 63 + 5)])
def test_projection_matches_oracle(lib, d, k, seed):
    cfg = S.make_config(d, 64, k, 8, 0, (1, 5), seed)
    got = S.sws_build_projection_host(cfg).numpy()
    want = oracle.srht_matrix(d, k, seed)
    assert np.array_equal(np.sign(got), np.sign(want))
    assert np.allclose(got, want, rtol=1e-15, atol=0)


def test_workspace_sizes(lib):
    cfg = S.make_config(128, 64, 32)
    assert S.sws_workspace_size(cfg, S.SWS_OP_SKETCH, 16384, 32, 8) == 0  # means stay on chip
    assert S.sws_workspace_size(cfg, S.SWS_OP_PREFILL_ATTN, 16384, 32, 8) == 0
    assert S.sws_workspace_size(cfg, S.SWS_OP_WALK_SELECT, 16384, 32, 8) == 4 * 32 * 256 * 256 * 8
    dec = S.sws_workspace_size(cfg, S.SWS_OP_DECODE_ATTN, 131136, 32, 8, 16)
    assert dec > 0 and dec % (130 * 4) == 0
    with pytest.raises(S.SwsError):
        S.sws_workspace_size(cfg, S.SWS_OP_WALK_SELECT, 0, 32, 8)
    with pytest.raises(S.SwsError):
        S.sws_workspace_size(cfg, S.SWS_OP_WALK_SELECT, 10, 32, 7)  # hq % hkv != 0


def test_packed_prefill_workspace(lib):
    """The packed attention's workspace: a 48-byte entry per sequence (rounded
    up to 16 bytes), then 8 bytes per 256-row slab of every sequence; 0 for a
    list that is not strictly increasing."""
    assert S.sws_sparse_attn_prefill_varlen_ws_bytes([0, 300, 1000]) == 96 + 8 * (2 + 3)
    assert S.sws_sparse_attn_prefill_varlen_ws_bytes([0, 1]) == 48 + 8
    assert S.sws_sparse_attn_prefill_varlen_ws_bytes([0, 256, 512, 513]) == 144 + 8 * (1 + 1 + 1)
    assert S.sws_sparse_attn_prefill_varlen_ws_bytes([0, 300, 300]) == 0
    assert S.sws_sparse_attn_prefill_varlen_ws_bytes([0, 300, 200]) == 0
    assert S.sws_sparse_attn_prefill_varlen_ws_bytes([0]) == 0


def test_null_handle_rejected_without_launch(lib):
    """Host validation fails before any CUDA call, so this runs without a GPU."""
    P = ctypes.c_void_p
    assert lib.sws_sketch(None, P(16), P(16), 0, 64, 1, 1, None, None, P(16), P(16), P(16), P(16), 16,
                          None) == S.SWS_ERR_INVALID_ARG
    assert lib.sws_walk_select(None, P(16), 64, 1, 1, P(16), P(16), P(16), P(16), 16, None) == S.SWS_ERR_INVALID_ARG
    assert lib.sws_walk_select_sketch(None, P(16), P(16), 64, 1, 1, 1, P(16), P(16), P(16), P(16), 16,
                                      None) == S.SWS_ERR_INVALID_ARG
    assert lib.sws_sparse_attn_prefill(None, P(16), P(16), P(16), 0, 64, 1, 1, None, None, None, None, P(16), P(16),
                                       P(16), None, 0, None) == S.SWS_ERR_INVALID_ARG
    cu = (ctypes.c_int64 * 3)(0, 300, 1000)
    ptrs = (ctypes.c_void_p * 2)(16, 32)
    assert lib.sws_sparse_attn_prefill_varlen(None, P(16), P(16), P(16), 0, 2, cu, 1, 1, None, None, None, None,
                                              ptrs, ptrs, P(16), P(16), 1 << 10, None) == S.SWS_ERR_INVALID_ARG
    assert lib.sws_destroy(None) == S.SWS_ERR_INVALID_ARG
    assert lib.sws_projection_device(None) is None
    assert lib.sws_decode_init_cache_paged(None, P(16), 4, P(16), 4, 1, 1, P(16), P(16), P(16),
                                           None) == S.SWS_ERR_INVALID_ARG
    assert lib.sws_decode_step_paged(None, P(16), P(16), P(16), 1, 4, 1, P(16), P(16), 4, P(16), 4, P(16), P(16),
                                     P(16), 1, P(16), P(16), P(16), P(16), P(16), P(16), None) == S.SWS_ERR_INVALID_ARG
    assert lib.sws_sparse_attn_decode_paged(None, P(16), P(16), P(16), 4, P(16), 4, 1, 4, 1, P(16), P(16), P(16),
                                            P(16), P(16), P(16), 1 << 20, None) == S.SWS_ERR_INVALID_ARG


def test_stride_checks(lib):
    """Strided prefill operands: each stride at least d elements and a multiple of
    16 bytes; NULL is the dense layout."""
    cfg = S.make_config(128, 64, 32)
    ok = lambda dt, st: lib.sws_layout_check(ctypes.byref(cfg), dt, 1000,  # noqa: E731
                                             None if st is None else (ctypes.c_int64 * 2)(*st))
    assert ok(S.SWS_BF16, None) == S.SWS_OK
    assert ok(S.SWS_BF16, (128, 32 * 128)) == S.SWS_OK  # [n, 32 heads, d] read in place
    assert ok(S.SWS_BF16, (1000 * 128, 128)) == S.SWS_OK  # dense, spelled out
    assert ok(S.SWS_FP32, (128, 8 * 128)) == S.SWS_OK
    assert ok(S.SWS_BF16, (128, 32 * 128 + 4)) == S.SWS_ERR_INVALID_ARG  # 8 bytes past a 16-byte multiple
    assert ok(S.SWS_BF16, (136, 8 * 128)) == S.SWS_OK  # 272 bytes: padded heads
    assert ok(S.SWS_BF16, (132, 8 * 128)) == S.SWS_ERR_INVALID_ARG  # 264 bytes
    assert ok(S.SWS_FP32, (128, 8 * 128 + 2)) == S.SWS_ERR_INVALID_ARG  # 8 bytes past
    assert ok(S.SWS_BF16, (64, 32 * 128)) == S.SWS_ERR_INVALID_ARG  # heads overlap within a row
    assert ok(S.SWS_BF16, (128, 120)) == S.SWS_ERR_INVALID_ARG  # tokens overlap
    assert ok(S.SWS_BF16, (0, 128)) == S.SWS_ERR_INVALID_ARG


def test_create_reports_error_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p = ctypes.c_void_p(1)
    s = lib.sws_create(ctypes.byref(S.make_config()), ctypes.byref(p))
    assert s == S.SWS_ERR_CUDA and not p.value

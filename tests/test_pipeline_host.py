"""Host-side logic of the pipeline that runs without a GPU: placing tokens on
the pages of a paged KV cache (the layout the *_paged entry points read:
pool [num_pages, hkv, B, d], token t of sequence i on page
block_table[i, t // B], row t % B)."""
import torch

from block_sparse_attention_sws_b200.pipeline import DecodePath


def _check(n, B, hkv=3, d=5, num_pages=11, seed=0):
    g = torch.Generator().manual_seed(seed)
    nb = -(-n // B)
    src = torch.randn(hkv, n + 7, d, generator=g)
    pages = torch.randperm(num_pages, generator=g)[:nb]
    sentinel = -1234.5
    pool = torch.full((num_pages, hkv, B, d), sentinel)
    DecodePath._scatter_pages(pool, pages, src, n, B)
    for t in range(n):
        assert torch.equal(pool[pages[t // B], :, t % B], src[:, t]), t
    written = torch.zeros(num_pages, B, dtype=torch.bool)
    for t in range(n):
        written[pages[t // B], t % B] = True
    assert torch.all(pool.permute(0, 2, 1, 3)[~written] == sentinel)  # nothing else touched


def test_scatter_full_blocks():
    _check(n=24, B=8)


def test_scatter_partial_last_block():
    _check(n=21, B=8)


def test_scatter_single_partial_block():
    _check(n=3, B=8, num_pages=4)


def test_scatter_one_token_per_block_boundary():
    for n in (1, 7, 8, 9, 16, 17):
        _check(n=n, B=8, seed=n)

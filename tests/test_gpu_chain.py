"""GPU parity of the whole hot path (indexer -> Top-K -> sparse MLA) on the
four DSA workloads: the tiny one in full, the full-size ones (32x32K decode,
64 ragged sequences up to 128K in shuffled pages, the 4096-token prefill
chunk) on sampled query rows, launched exactly as the benchmark launches them."""
import numpy as np
import pytest
import torch

import sparse_attention_07_b200 as sa
import workloads as W
from _gpu import check_rows, gpu_step

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_chain_tiny_full():
    inp = W.dsa_inputs(W.TINY, DEV)
    scores, idx, out, lse = gpu_step(inp)
    torch.cuda.synchronize()
    check_rows(inp, [0], scores, idx, out, lse)


def test_chain_small_paged_ragged():
    cfg = W.small_dsa(W.RAGGED, n_seqs=5, rows=5, lens=(3000, 70, 2048, 2049, 4500), topk=512)
    inp = W.dsa_inputs(cfg, DEV, seed=21)
    scores, idx, out, lse = gpu_step(inp)
    torch.cuda.synchronize()
    check_rows(inp, list(range(5)), scores, idx, out, lse)


def test_chain_small_prefill():
    cfg = W.small_dsa(W.PREFILL, lens=(3000,), rows=37, prefill_start=2963, topk=1024)
    inp = W.dsa_inputs(cfg, DEV, seed=22)
    scores, idx, out, lse = gpu_step(inp)
    torch.cuda.synchronize()
    check_rows(inp, [0, 1, 17, 35, 36], scores, idx, out, lse)


def _properties(inp, idx, out):
    """For every row: ascending distinct positions below the visible length,
    -1 after them, finite outputs."""
    nv = inp["n_visible"].cpu().numpy()
    ii = idx.cpu().numpy()
    k = ii.shape[1]
    for r in range(ii.shape[0]):
        m = min(k, nv[r])
        assert (np.diff(ii[r, :m]) > 0).all() and ii[r, 0] >= 0 and ii[r, m - 1] < nv[r]
        assert (ii[r, m:] == -1).all()
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("name", ["long", "ragged"])
def test_chain_full_size_every_row(name):
    """The long (32 x 32K) and ragged (64 rows up to 128K, shuffled pages)
    decode workloads at full size, launched as the benchmark launches them:
    every row's index scores and Top-K set bit for bit, every row's attention
    output and LSE within tolerance (rows checked eight at a time to bound
    the oracle's host memory)."""
    inp = W.dsa_inputs(W.DSA_CONFIGS[name], DEV)
    scores, idx, out, lse = gpu_step(inp)
    torch.cuda.synchronize()
    rows = inp["cfg"].rows
    for r0 in range(0, rows, 8):
        check_rows(inp, list(range(r0, min(rows, r0 + 8))), scores, idx, out, lse)
    _properties(inp, idx, out)
    del inp
    torch.cuda.empty_cache()


def test_chain_full_size_prefill():
    """The 4096-token prefill chunk over a 61440-token history at full size:
    index scores and Top-K sets bit for bit on a seeded subset of 192 query
    rows (both ends of the chunk included; the oracle's indexer over all 4096
    rows would take minutes of host time), attention and LSE on 64 of them;
    properties on every row."""
    inp = W.dsa_inputs(W.PREFILL, DEV)
    scores, idx, out, lse = gpu_step(inp)
    torch.cuda.synchronize()
    T = inp["cfg"].rows
    rng = np.random.default_rng(4096)
    pick = sorted(set([0, 1, 2, T // 2, T - 2, T - 1]) | set(rng.choice(T, 186, replace=False).tolist()))
    for i in range(0, len(pick), 32):
        part = pick[i:i + 32]
        if i < 64:
            check_rows(inp, part, scores, idx, out, lse)
        else:
            check_rows(inp, part, scores, idx, None, None)
    _properties(inp, idx, out)
    del inp
    torch.cuda.empty_cache()

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


@pytest.mark.parametrize("name,rows", [("long", [0, 13, 31]), ("ragged", [0, 21, 63]),
                                       ("prefill", [0, 1, 2047, 4095])])
def test_chain_full_size_sampled(name, rows):
    inp = W.dsa_inputs(W.DSA_CONFIGS[name], DEV)
    scores, idx, out, lse = gpu_step(inp)
    torch.cuda.synchronize()
    check_rows(inp, rows, scores, idx, out, lse)
    # properties for every row: ascending distinct positions below the visible length, -1 after
    nv = inp["n_visible"].cpu().numpy()
    ii = idx.cpu().numpy()
    k = ii.shape[1]
    for r in range(ii.shape[0]):
        m = min(k, nv[r])
        assert (np.diff(ii[r, :m]) > 0).all() and ii[r, 0] >= 0 and ii[r, m - 1] < nv[r]
        assert (ii[r, m:] == -1).all()
    assert torch.isfinite(out).all()
    del inp
    torch.cuda.empty_cache()

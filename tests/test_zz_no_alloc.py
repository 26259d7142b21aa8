"""sa_sparse_mla_decode_static: sparse MLA decode for callers that cannot
allocate device memory (no allocator of their own to hand the library a
workspace, or code running where cudaMalloc is not allowed).  The call keeps
its scratch (the partial-score exchange area and the split-key partial
states) in the library's static device array, so its results must match
sa_sparse_mla_decode given a caller workspace.

This file is named so that pytest collects it last: a run that stops at the
first failure has run every other test before it reaches this one."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_07_b200 as sa
import workloads as W

DEV = "cuda"
FAKE = ctypes.c_void_p(0x1000)  # aligned, never dereferenced: the call rejects the shape first


@pytest.mark.gpu
def test_static_scratch_decode_matches_workspace_decode():
    """Two calls in a row through the static array against the workspace
    call: the same kernels with the same key split and a combine that adds the
    splits in a fixed order, so the outputs and LSEs must be identical bit for
    bit (a tolerance would hide stale scratch contents or a race on the
    array).  The outputs start as NaN so a value not written shows up."""
    cfg = W.small_dsa(W.LONG, n_seqs=3, rows=3, lens=(5000, 2100, 4097), topk=2048)
    inp = W.dsa_inputs(cfg, DEV, seed=31)
    need = sa.sparse_mla_workspace_size(cfg.rows, cfg.H, cfg.topk, cfg.d_c)
    assert 0 < need <= sa.STATIC_SCRATCH_BYTES, "shape must split its keys and fit the static array"

    scores = sa.index_scores(inp["q_idx"], inp["w"], inp["k_idx_cache"], inp["n_visible"], cfg.pages_per_seq)
    idx = sa.topk_select(scores, inp["n_visible"], cfg.topk)
    args = (inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale, cfg.pages_per_seq)

    lse_ref = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=DEV)
    ref = sa.sparse_mla_decode(*args, lse=lse_ref)
    outs = []
    for _ in range(2):  # two calls in a row share (and reuse) the static array
        out = torch.full((cfg.rows, cfg.H, cfg.d_c), float("nan"), dtype=torch.float32, device=DEV)
        lse = torch.full((cfg.rows, cfg.H), float("nan"), dtype=torch.float32, device=DEV)
        sa.sparse_mla_decode_static(*args, out=out, lse=lse)
        outs.append((out, lse))
    torch.cuda.synchronize()
    assert sa.check_device_error() == 0
    assert torch.isfinite(ref).all()
    for out, lse in outs:
        assert torch.equal(out, ref), (out - ref).abs().max().item()
        assert torch.equal(lse, lse_ref)


def test_static_scratch_rejects_shapes_beyond_the_array():
    """Shapes whose scratch (exchange area plus split-key partial states)
    exceeds the static array are refused on the host, before any launch (no
    device pointer is touched)."""
    from sparse_attention_07_b200 import build
    build.build()
    L = sa.lib()
    rejected = 0
    for rows, k in ((1, 2048), (37, 4096), (74, 8192), (100, 8192)):
        need = sa.sparse_mla_workspace_size(rows, 128, k, 512)
        if need <= sa.STATIC_SCRATCH_BYTES:
            continue
        st = L.sa_sparse_mla_decode_static(FAKE, FAKE, FAKE, 512, FAKE, 64, 1024, None, 16, None, FAKE, rows, 128,
                                           k, 512, 64, 0.07, FAKE, None, None)
        assert st == sa.SA_EUNSUPPORTED
        rejected += 1
    assert rejected > 0, "no shape exceeded the static array"

"""GPU parity: block mean pooling and the block-sparse decode against the fp64
oracle.  Block selection of N(0,1) inputs is compared as sets; a block may
differ only when fp32 and fp64 order two near-tied scores differently, i.e.
when its oracle score is within 1e-5 * max|score| of the boundary score; the
output is then compared with the oracle evaluated on the GPU's own choice."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_07_b200 as sa
import workloads as W
from _gpu import assert_attention_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIE_REL = 1e-5


def _check_pairs(cfg, inp, out, sel, pairs):
    for b, h in pairs:
        q = inp["q"][b, h].double().cpu().numpy()
        K = inp["K"][b, :, h].double().cpu().numpy()
        V = inp["V"][b, :, h].double().cpu().numpy()
        ref_out, ref_sel, bs = oracle.block_sparse(q, K, V, cfg.block, cfg.top_blocks, cfg.sink_blocks, cfg.window,
                                                   cfg.scale)
        got_sel = sel[b, h].cpu().numpy()
        if not np.array_equal(got_sel, ref_sel):
            ntop = min(cfg.top_blocks, len(bs))
            boundary = np.sort(bs)[::-1][ntop - 1]
            diff = set(got_sel.tolist()) ^ set(ref_sel.tolist())
            for blk in diff:
                assert abs(bs[blk] - boundary) <= TIE_REL * np.abs(bs).max(), f"({b},{h}) block {blk} not a near tie"
            ref_out = oracle.block_attend(q, K, V, got_sel[got_sel >= 0], cfg.block, cfg.sink_blocks, cfg.window,
                                          cfg.scale)
        assert_attention_close(out[b, h].cpu().numpy(), ref_out, f"block ({b},{h})")


@pytest.mark.parametrize("L,top,sink,win", [(1000, 4, 1, 100), (4096, 16, 1, 512), (700, 64, 2, 0),
                                            (130, 16, 1, 512), (64 * 33, 16, 0, 64),
                                            (50, 4, 1, 100), (64 * 5 + 7, 64, 8, 10), (64 * 9, 3, 0, 1000)])
def test_block_sparse_small(L, top, sink, win):
    cfg = W.BlockConfig(name="t", seed=0, B=2, L=L, H=3, top_blocks=top, sink_blocks=sink, window=win)
    inp = W.block_inputs(cfg, DEV, seed=L + top)
    pooled = sa.block_mean_pool(inp["K"], cfg.block)
    sel = torch.empty(cfg.B, cfg.H, cfg.top_blocks, dtype=torch.int32, device=DEV)
    out = sa.block_sparse_attn(inp["q"], pooled, inp["K"], inp["V"], cfg.block, cfg.top_blocks, cfg.sink_blocks,
                               cfg.window, cfg.scale, sel_blocks=sel)
    torch.cuda.synchronize()
    _check_pairs(cfg, inp, out, sel, [(b, h) for b in range(cfg.B) for h in range(cfg.H)])
    assert sa.check_device_error() == 0


def test_block_mean_pool_vs_oracle():
    cfg = W.BlockConfig(name="t", seed=0, B=2, L=1000, H=3)
    inp = W.block_inputs(cfg, DEV, seed=2)
    pooled = sa.block_mean_pool(inp["K"], 64).cpu().numpy()
    for b in range(2):
        for h in range(3):
            ref = oracle.block_mean_pool(inp["K"][b, :, h].double().cpu().numpy(), 64)
            np.testing.assert_allclose(pooled[b, h, : ref.shape[0]], ref, rtol=0, atol=2e-6)


def test_block_sparse_full_size_sampled():
    """The block workload at full size (B=8, L=131072, H=32); sampled heads."""
    cfg = W.BLOCK
    inp = W.block_inputs(cfg, DEV)
    pooled = sa.block_mean_pool(inp["K"], cfg.block)
    sel = torch.empty(cfg.B, cfg.H, cfg.top_blocks, dtype=torch.int32, device=DEV)
    out = sa.block_sparse_attn(inp["q"], pooled, inp["K"], inp["V"], cfg.block, cfg.top_blocks, cfg.sink_blocks,
                               cfg.window, cfg.scale, sel_blocks=sel)
    torch.cuda.synchronize()
    _check_pairs(cfg, inp, out, sel, [(0, 0), (3, 17), (7, 31)])
    # properties that hold for every head: ascending distinct chosen blocks, finite outputs
    s = sel.cpu().numpy()
    assert (np.diff(s, axis=-1) > 0).all() and (s >= 0).all() and (s < cfg.n_blocks).all()
    assert torch.isfinite(out).all()
    assert sa.check_device_error() == 0


def test_block_sparse_unaligned_fallback():
    """K and V as views 8 bytes past a 16-byte boundary: the tensor-map path
    needs 16-byte alignment, so the per-thread-load kernel serves the call;
    both paths agree with the oracle alike."""
    cfg = W.BlockConfig(name="t", seed=0, B=2, L=1000, H=3, top_blocks=4, sink_blocks=1, window=100)
    inp = W.block_inputs(cfg, DEV, seed=77)
    shape = inp["K"].shape
    kbuf = torch.empty(inp["K"].numel() + 4, dtype=inp["K"].dtype, device=DEV)
    vbuf = torch.empty(inp["V"].numel() + 4, dtype=inp["V"].dtype, device=DEV)
    K = kbuf[4:].view(shape)
    V = vbuf[4:].view(shape)
    K.copy_(inp["K"])
    V.copy_(inp["V"])
    assert K.data_ptr() % 16 == 8
    pooled = sa.block_mean_pool(K, cfg.block)
    sel = torch.empty(cfg.B, cfg.H, cfg.top_blocks, dtype=torch.int32, device=DEV)
    out = sa.block_sparse_attn(inp["q"], pooled, K, V, cfg.block, cfg.top_blocks, cfg.sink_blocks, cfg.window,
                               cfg.scale, sel_blocks=sel)
    torch.cuda.synchronize()
    _check_pairs(cfg, inp, out, sel, [(b, h) for b in range(cfg.B) for h in range(cfg.H)])
    assert sa.check_device_error() == 0


@pytest.mark.parametrize("B,H", [(1, 2), (2, 80)])
def test_block_sparse_all_scores_tied(B, H):
    """A zero query scores every block 0: the choice is the lowest top_blocks
    blocks (ties go to the lower block), taken by the fallback rounds since
    the tied keys outnumber what the choosing warp holds; the output is the
    uniform average over the union.  (1, 2) runs clusters of four CTAs per
    pair, (2, 80) one CTA per pair."""
    cfg = W.BlockConfig(name="t", seed=0, B=B, L=64 * 700, H=H, top_blocks=16, sink_blocks=1, window=512)
    inp = W.block_inputs(cfg, DEV, seed=5)
    q = torch.zeros_like(inp["q"])
    pooled = sa.block_mean_pool(inp["K"], cfg.block)
    sel = torch.empty(cfg.B, cfg.H, cfg.top_blocks, dtype=torch.int32, device=DEV)
    out = sa.block_sparse_attn(q, pooled, inp["K"], inp["V"], cfg.block, cfg.top_blocks, cfg.sink_blocks,
                               cfg.window, cfg.scale, sel_blocks=sel)
    torch.cuda.synchronize()
    assert (sel.cpu().numpy() == np.arange(cfg.top_blocks)).all()
    for b, h in [(0, 0), (B - 1, H - 1)]:
        K = inp["K"][b, :, h].double().cpu().numpy()
        V = inp["V"][b, :, h].double().cpu().numpy()
        ref_out, ref_sel, _ = oracle.block_sparse(np.zeros(128), K, V, cfg.block, cfg.top_blocks, cfg.sink_blocks,
                                                  cfg.window, cfg.scale)
        assert (ref_sel == np.arange(cfg.top_blocks)).all()
        assert_attention_close(out[b, h].cpu().numpy(), ref_out, f"tied ({b},{h})")
    assert sa.check_device_error() == 0

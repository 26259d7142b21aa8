"""GPU parity: CSA compression and the CSA decode chain (indexer over the
compressed keys -> Top-K -> window slots -> sparse attention over the selected
entries and the raw window) against the fp64 oracle.

The compressed indexer keys of the workload are exact integers, so index
scores and Top-K sets must match bit for bit.  The compressed entries are
bf16 roundings of fp32 (GPU) and fp64 (oracle) sums: equal except where the
two sums straddle a rounding boundary, so within half a bf16 step (plus the
fp32 sum's own error) of the exact value."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_07_b200 as sa
import workloads as W
from _gpu import assert_attention_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16_step(x):
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def _compress_all(cfg, inp):
    S = cfg.n_seqs
    lat = inp["lat_pool"].view(S, cfg.lat_pages * 64, cfg.c)
    sa.csa_compress(inp["Ca"], inp["Cb"], inp["Za"], inp["Zb"], inp["Ba"], inp["Bb"], cfg.m, inp["lat_pool"],
                    lat.stride(0), lat.stride(1))
    idx = inp["idx_pool"].view(S, cfg.idx_pages * 64, cfg.d_I)
    sa.csa_compress(inp["CIa"], inp["CIb"], inp["ZIa"], inp["ZIb"], inp["BIa"], inp["BIb"], cfg.m, inp["idx_pool"],
                    idx.stride(0), idx.stride(1))


def _decode(cfg, inp):
    scores = sa.index_scores(inp["q_idx"], inp["w"], inp["idx_pool"], inp["n_visible"], cfg.idx_pages)
    idx = sa.topk_select(scores, inp["n_visible"], cfg.topk)
    slots = sa.csa_window_index(idx, inp["seq_lens"], cfg.window, cfg.n_cap)
    out = sa.sparse_mla_decode(inp["q"], inp["q_rope"], inp["lat_pool"], inp["lat_pool"], slots, cfg.scale,
                               cfg.lat_pages)
    torch.cuda.synchronize()
    return scores, idx, slots, out


@pytest.mark.parametrize("m,c", [(4, 512), (1, 128), (16, 128), (3, 64)])
def test_csa_compress_vs_oracle(m, c):
    g = torch.Generator(device=DEV).manual_seed(7 + m)
    S, L = 2, 64 * m + m // 2 + 5
    Ca, Cb, Za, Zb = (torch.randn(S, L, c, generator=g, device=DEV).to(torch.bfloat16) for _ in range(4))
    Ba, Bb = (torch.randn(m, c, generator=g, device=DEV) for _ in range(2))
    nc = L // m
    out = torch.full((S, nc + 3, c), float("nan"), dtype=torch.bfloat16, device=DEV)
    sa.csa_compress(Ca, Cb, Za, Zb, Ba, Bb, m, out, out.stride(0), out.stride(1))
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    assert np.isnan(got[:, nc:]).all()  # nothing written past the complete entries
    for s in range(S):
        want = oracle.csa_compress(*(x[s].double().cpu().numpy() for x in (Ca, Cb, Za, Zb)),
                                   Ba.double().cpu().numpy(), Bb.double().cpu().numpy(), m)
        d = np.abs(got[s, :nc] - want)
        # half a bf16 step of rounding, plus the fp32 sum's error (eight terms of |x| < 6)
        assert (d <= _bf16_step(want) * 0.5 + 1e-5).all(), d.max()
        rounded = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
        assert (got[s, :nc] == rounded).mean() > 0.99
    assert sa.check_device_error() == 0


def test_csa_compress_group_range_and_e4m3():
    """Only entries g0..g1-1 are written (decode compresses the group that
    completed); e4m3 output rounds like torch's float8 conversion."""
    cfg = W.CSAConfig(name="t", seed=0, n_seqs=2, L=700, H=16, topk=64, window=32)
    inp = W.csa_inputs(cfg, DEV, seed=11)
    idx = inp["idx_pool"].view(cfg.n_seqs, cfg.idx_pages * 64, cfg.d_I)
    sa.csa_compress(inp["CIa"], inp["CIb"], inp["ZIa"], inp["ZIb"], inp["BIa"], inp["BIb"], cfg.m, inp["idx_pool"],
                    idx.stride(0), idx.stride(1), g0=40, g1=60)
    torch.cuda.synchronize()
    got = idx.float().cpu().numpy()
    assert (got[:, :40] == 0).all() and (got[:, 60:] == 0).all()
    for s in range(cfg.n_seqs):
        want = inp["CIa"][s, :: cfg.m].float().cpu().numpy()[40:60]
        np.testing.assert_array_equal(got[s, 40:60], want)


@pytest.mark.parametrize("L,topk,window", [(3000, 256, 64), (700, 256, 32), (20, 8, 64), (4 * 64 * 9 + 2, 64, 1)])
def test_csa_decode_small(L, topk, window):
    cfg = W.CSAConfig(name="t", seed=0, n_seqs=3, L=L, H=32, topk=topk, window=window)
    inp = W.csa_inputs(cfg, DEV, seed=L + window)
    _compress_all(cfg, inp)
    scores, idx, slots, out = _decode(cfg, inp)
    ref = oracle.csa_step(inp, list(range(cfg.n_seqs)))
    got_s = scores[:, : cfg.n_c].double().cpu().numpy()
    assert np.array_equal(got_s, ref["scores"][:, : cfg.n_c]), "index scores must be bit-exact"
    assert np.array_equal(idx.cpu().numpy(), ref["idx"]), "Top-K sets must be bit-exact"
    s = slots.cpu().numpy()
    wl = min(cfg.window, cfg.L)
    assert (s[:, cfg.topk: cfg.topk + wl] == cfg.n_cap + np.arange(wl)).all() and (s[:, cfg.topk + wl:] == -1).all()
    assert_attention_close(out.cpu().numpy(), ref["out"], "csa")
    assert sa.check_device_error() == 0


def test_csa_full_size_sampled():
    """The CSA workload at full size (32 sequences of 131072 tokens, m = 4);
    the chain as bench.py launches it, two sequences against the oracle."""
    cfg = W.CSA
    inp = W.csa_inputs(cfg, DEV)
    _compress_all(cfg, inp)
    scores, idx, slots, out = _decode(cfg, inp)
    rows = [0, cfg.n_seqs - 1]
    ref = oracle.csa_step(inp, rows)
    assert np.array_equal(scores[rows, : cfg.n_c].double().cpu().numpy(), ref["scores"])
    assert np.array_equal(idx[rows].cpu().numpy(), ref["idx"])
    assert_attention_close(out[rows].cpu().numpy(), ref["out"], "csa full size")
    i = idx.cpu().numpy()
    assert (np.diff(i, axis=1) > 0).all() and (i >= 0).all() and (i < cfg.n_c).all()
    assert torch.isfinite(out).all()
    assert sa.check_device_error() == 0

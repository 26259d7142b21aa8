"""GPU parity: the NSA compressed cache and the NSA three-branch decode
against the fp64 oracle.

The compressed cache is the exact block mean rounded once to bf16 on both
sides (the kernel's fp64 block sums are exact for these inputs), so it must
match bit for bit.  The group's block choice of N(0,1) inputs is
compared as a set; a block may differ only where fp32 and fp64 order two
near-tied group probabilities differently (oracle probability within
TIE_REL * max of the boundary one), and the output is then compared with the
oracle evaluated on the GPU's own choice."""
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


def _run(cfg, inp):
    Kc, Vc = sa.nsa_compress(inp["K"], inp["V"], cfg.block)
    sel = torch.full((cfg.B, cfg.H_kv, max(cfg.top_blocks, 1)), -7, dtype=torch.int32, device=DEV)
    out = sa.nsa_decode(inp["q"], inp["K"], inp["V"], Kc, Vc, inp["gates"], cfg.block, cfg.top_blocks, cfg.window,
                        cfg.scale, sel_blocks=sel if cfg.top_blocks > 0 else None)
    torch.cuda.synchronize()
    return Kc, Vc, out, sel


def _check_pairs(cfg, inp, out, sel, pairs):
    G = cfg.G
    ref = oracle.nsa_step(inp, pairs)
    for (b, g) in pairs:
        want, want_sel, p_cmp = ref[(b, g)]
        hs = slice(g * G, (g + 1) * G)
        if cfg.top_blocks > 0:
            got_sel = sel[b, g].cpu().numpy()
            ntop = min(cfg.top_blocks, cfg.n_blocks)
            assert (got_sel[ntop:] == -1).all(), f"({b},{g}) padding of the choice"
            got_sel = got_sel[:ntop]
            if not np.array_equal(got_sel, want_sel):
                P = p_cmp.sum(axis=0)
                boundary = np.sort(P)[::-1][ntop - 1]
                for blk in set(got_sel.tolist()) ^ set(want_sel.tolist()):
                    assert abs(P[blk] - boundary) <= TIE_REL * P.max(), f"({b},{g}) block {blk} is not a near tie"
                assert (np.diff(got_sel) > 0).all()
                K = oracle._host64(inp["K"][b, :, g])
                V = oracle._host64(inp["V"][b, :, g])
                cache = (oracle.nsa_compress(K, cfg.block), oracle.nsa_compress(V, cfg.block))
                want = oracle.nsa_decode_group(oracle._host64(inp["q"][b, hs]), K, V, cfg.block, cfg.top_blocks,
                                               cfg.window, oracle._host64(inp["gates"][b, hs]), cfg.scale,
                                               chosen=got_sel, compressed=cache)[0]
        assert_attention_close(out[b, hs].cpu().numpy(), want, f"nsa ({b},{g})")


def test_nsa_compress_bit_exact():
    cfg = W.NSAConfig(name="t", seed=0, B=2, L=1000, H=6, H_kv=3)
    inp = W.nsa_inputs(cfg, DEV, seed=3)
    for block in (32, 64, 96):
        Kc, Vc = sa.nsa_compress(inp["K"], inp["V"], block)
        torch.cuda.synchronize()
        for b in range(cfg.B):
            for h in range(cfg.H_kv):
                for X, got in ((inp["K"], Kc), (inp["V"], Vc)):
                    want = oracle.nsa_compress(X[b, :, h].double().cpu().numpy(), block)
                    np.testing.assert_array_equal(got[b, h, : want.shape[0]].double().cpu().numpy(), want)
    assert sa.check_device_error() == 0


# (H, H_kv, L, block, top, window): GQA groups of 1..16 heads, ragged tails,
# fewer blocks than the selection, no complete block, no window, no selection,
# a window longer than the history, blocks of 32..256 tokens.
CASES = [
    (8, 2, 4096, 64, 16, 512),
    (16, 2, 3000, 64, 4, 100),
    (16, 1, 5000, 64, 16, 512),
    (3, 1, 1000, 64, 4, 64),
    (4, 4, 700, 64, 16, 512),
    (8, 1, 63, 64, 16, 512),
    (8, 1, 130, 64, 16, 0),
    (8, 2, 2048 + 31, 64, 0, 300),
    (2, 1, 20000, 32, 64, 4096),
    (12, 3, 9000, 128, 7, 1000),
    (8, 1, 6000, 256, 5, 17),
    (8, 1, 64 * 4096, 64, 16, 512),
]


@pytest.mark.parametrize("H,H_kv,L,block,top,window", CASES)
def test_nsa_decode_small(H, H_kv, L, block, top, window):
    cfg = W.NSAConfig(name="t", seed=0, B=2 if L < 100000 else 1, L=L, H=H, H_kv=H_kv, block=block,
                      top_blocks=top, window=window)
    inp = W.nsa_inputs(cfg, DEV, seed=L + top + 7 * H)
    _, _, out, sel = _run(cfg, inp)
    pairs = [(b, g) for b in range(cfg.B) for g in range(cfg.H_kv)]
    if L > 100000:
        pairs = pairs[:1]
    _check_pairs(cfg, inp, out, sel, pairs)
    assert sa.check_device_error() == 0


def test_nsa_equal_blocks_choose_the_lowest():
    """Every block alike: the group probabilities tie exactly on both sides,
    so the choice is the lowest blocks, bit for bit."""
    cfg = W.NSAConfig(name="t", seed=0, B=1, L=64 * 50 + 9, H=8, H_kv=1, top_blocks=16, window=64)
    inp = W.nsa_inputs(cfg, DEV, seed=5)
    row = inp["K"][:, :1].clone()
    inp["K"] = row.expand(-1, cfg.L, -1, -1).contiguous()
    _, _, out, sel = _run(cfg, inp)
    assert sel[0, 0].cpu().tolist() == list(range(16))
    _check_pairs(cfg, inp, out, sel, [(0, 0)])


def test_nsa_decode_repeatable():
    cfg = W.NSAConfig(name="t", seed=0, B=2, L=10000, H=16, H_kv=2)
    inp = W.nsa_inputs(cfg, DEV, seed=9)
    a = _run(cfg, inp)
    b = _run(cfg, inp)
    assert torch.equal(a[2], b[2]) and torch.equal(a[3], b[3])


def test_nsa_full_size_sampled():
    """The NSA workload at full size (B=8, L=131072, 32 heads in 4 groups);
    sampled (sequence, KV head) pairs against the oracle, properties for all."""
    cfg = W.NSA
    inp = W.nsa_inputs(cfg, DEV)
    _, _, out, sel = _run(cfg, inp)
    _check_pairs(cfg, inp, out, sel, [(0, 0), (3, 2), (7, 3)])
    s = sel.cpu().numpy()
    assert (np.diff(s, axis=-1) > 0).all() and (s >= 0).all() and (s < cfg.n_blocks).all()
    assert torch.isfinite(out).all()
    assert sa.check_device_error() == 0

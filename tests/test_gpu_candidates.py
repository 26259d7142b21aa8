"""GPU parity: the decode indexer that keeps only Top-K candidates, and the
Top-K taken from them, against the fp64 oracle (index sets bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_07_b200 as sa
import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _order_key_np(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def _run(inp, k, cand_ld=None):
    cfg = inp["cfg"]
    ld = cand_ld or cfg.pages_per_seq * 64
    cand, cnt, hist = sa.candidate_buffers(cfg.rows, ld, DEV)
    sa.index_candidates(inp["q_idx"], inp["w"], inp["k_idx_cache"], inp["n_visible"], cfg.pages_per_seq, k,
                        cand, cnt, hist, page_table=inp["page_table"])
    torch.cuda.synchronize()
    snap = (cand.cpu().numpy().view(np.uint64), cnt.cpu().numpy().copy(), hist.cpu().numpy().copy())
    idx = sa.topk_from_candidates(cand, cnt, inp["n_visible"], k, hist)
    torch.cuda.synchronize()
    assert int(hist.abs().sum()) == 0 and int(cnt.abs().sum()) == 0  # cleared for the next step
    assert sa.check_device_error() == 0
    return idx.cpu().numpy(), snap


def _check_candidates(snap, ref, k):
    """Every candidate is a real (key, position) pair of its row, positions are
    distinct, every position of the exact Top-K is among them, and the counts
    are the histogram of the row's scores."""
    cand, cnt, hist = snap
    for i in range(len(cnt)):
        n = int(ref["n_visible"][i])
        keys = _order_key_np(ref["scores"][i, :n])
        assert np.array_equal(hist[i], np.bincount(keys >> 20, minlength=4096)), f"row {i}: histogram"
        c = cand[i, : cnt[i]]
        pos = (np.uint64(0xFFFFFFFF) - (c & np.uint64(0xFFFFFFFF))).astype(np.int64)
        key = (c >> np.uint64(32)).astype(np.uint32)
        assert 0 <= cnt[i] <= n
        assert (pos >= 0).all() and (pos < n).all(), f"row {i}: position out of range"
        assert len(np.unique(pos)) == len(pos), f"row {i}: a position emitted twice"
        assert np.array_equal(key, keys[pos]), f"row {i}: key does not match the score"
        top = ref["idx"][i][ref["idx"][i] >= 0]
        assert np.isin(top, pos).all(), f"row {i}: a Top-K position was dropped"
        if n > k:  # nothing below the k-th largest key's digit is needed; the bound never cuts above it
            kth = np.sort(keys)[::-1][k - 1]
            kept_hi = np.isin(np.nonzero((keys >> 20) > (kth >> 20))[0], pos)
            assert kept_hi.all(), f"row {i}: a key above the boundary digit was dropped"


@pytest.mark.parametrize("base,kw", [
    (W.LONG, dict(n_seqs=3, rows=3, lens=(5000, 2100, 4097), topk=2048)),
    (W.RAGGED, dict(n_seqs=5, rows=5, lens=(9000, 700, 3000, 64, 20001), topk=512)),
    (W.LONG, dict(n_seqs=4, rows=4, lens=(3000, 129, 6000, 4096), topk=256, H_I=16)),
    (W.LONG, dict(n_seqs=2, rows=2, lens=(7000, 300), topk=1000, H_I=32, paged=True)),
    (W.LONG, dict(n_seqs=2, rows=2, lens=(4000, 2500), topk=128, H_I=128, H=8)),
])
def test_candidates_match_oracle(base, kw):
    cfg = W.small_dsa(base, **kw)
    inp = W.dsa_inputs(cfg, DEV, seed=41)
    ref = oracle.dsa_step(inp, list(range(cfg.rows)), with_attention=False)
    idx, snap = _run(inp, cfg.topk)
    assert np.array_equal(idx, ref["idx"])
    _check_candidates(snap, ref, cfg.topk)


def test_candidates_short_rows_and_padding():
    """Rows with n <= k (0, 1, k - 1, k) are all selected and padded with -1;
    a row one past k takes the selection."""
    cfg = W.small_dsa(W.LONG, n_seqs=5, rows=5, lens=(1, 255, 256, 257, 64), topk=256)
    inp = W.dsa_inputs(cfg, DEV, seed=43)
    inp["n_visible"] = torch.tensor([0, 255, 256, 257, 64], dtype=torch.int32, device=DEV)
    ref = oracle.dsa_step(inp, list(range(cfg.rows)), with_attention=False)
    idx, _ = _run(inp, cfg.topk)
    assert np.array_equal(idx, ref["idx"])
    assert (idx[0] == -1).all() and (idx[1, :255] == np.arange(255)).all() and idx[1, 255] == -1


def test_candidates_all_scores_equal():
    """Zero weights: every score is +0.0, so every key lies on the boundary
    digit and the bound keeps them all; the boundary list (more keys than the
    Top-K holds in shared memory) overflows and the selection re-reads the
    candidates.  Ties go to the lowest positions."""
    cfg = W.small_dsa(W.LONG, n_seqs=3, rows=3, lens=(20000, 4097, 3000), topk=2048)
    inp = W.dsa_inputs(cfg, DEV, seed=45)
    inp["w"].zero_()
    idx, snap = _run(inp, cfg.topk)
    n = [20000, 4097, 3000]
    for i in range(3):
        assert (idx[i] == np.arange(2048)).all()
        assert snap[1][i] == n[i]  # nothing can be ruled out


def test_candidates_ragged_full_size_sampled():
    """The full-size ragged decode workload (64 rows up to 128K keys, shuffled
    pages) through the candidate path, three steps on one set of buffers: the
    sets equal those of the histogram path on the same scores (all rows), the
    oracle's on sampled rows, and the bound keeps far fewer keys than the
    rows hold."""
    cfg = W.RAGGED
    inp = W.dsa_inputs(cfg, DEV)
    nv = inp["n_visible"]
    hist = sa.topk_histogram(cfg.rows, DEV)
    scores = sa.index_scores(inp["q_idx"], inp["w"], inp["k_idx_cache"], nv, cfg.pages_per_seq,
                             page_table=inp["page_table"], hist=hist)
    want = sa.topk_select(scores, nv, cfg.topk, hist=hist)
    cand, cnt, chist = sa.candidate_buffers(cfg.rows, cfg.pages_per_seq * 64, DEV)
    kept = []
    for _ in range(3):
        sa.index_candidates(inp["q_idx"], inp["w"], inp["k_idx_cache"], nv, cfg.pages_per_seq, cfg.topk,
                            cand, cnt, chist, page_table=inp["page_table"])
        kept.append(cnt.clone())
        idx = sa.topk_from_candidates(cand, cnt, nv, cfg.topk, chist)
        torch.cuda.synchronize()
        assert torch.equal(idx, want)
    assert sa.check_device_error() == 0
    assert int(chist.abs().sum()) == 0 and int(cnt.abs().sum()) == 0
    frac = (kept[-1].double() / nv.double()).median().item()
    assert frac < 0.5, f"median kept fraction {frac:.3f}"
    rows = [0, 17, 63]
    ref = oracle.dsa_step(inp, rows, with_attention=False)
    assert np.array_equal(idx.cpu().numpy()[rows], ref["idx"])

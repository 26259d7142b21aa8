"""Helpers shared by the GPU parity tests: run the library's chain on a
workload and compare with the fp64 oracle at the stated tolerances."""
import numpy as np
import torch

import sparse_attention_07_b200 as sa

# Attention outputs (bf16 inputs, fp32 accumulation) against the fp64 oracle.
MLA_MAX_ABS = 1e-2
MLA_MEAN_ABS = 1e-3
# log-sum-exp: the scores are exact bf16 products summed in fp32 (relative
# error ~576 * 2^-24), so 1e-3 absolute leaves two orders of margin.
LSE_ABS = 1e-3


def gpu_step(inp, lse=True):
    cfg = inp["cfg"]
    scores = sa.index_scores(inp["q_idx"], inp["w"], inp["k_idx_cache"], inp["n_visible"], cfg.pages_per_seq,
                             page_table=inp["page_table"], seq_of_row=inp["seq_of_row"])
    idx = sa.topk_select(scores, inp["n_visible"], cfg.topk)
    lse_t = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=scores.device) if lse else None
    fn = sa.sparse_mla_prefill if cfg.prefill_start >= 0 else sa.sparse_mla_decode
    out = fn(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale, cfg.pages_per_seq,
             page_table=inp["page_table"], seq_of_row=inp["seq_of_row"], lse=lse_t)
    return scores, idx, out, lse_t


def assert_attention_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= MLA_MAX_ABS, f"{what}: max abs error {err.max():.3e}"
    assert err.mean() <= MLA_MEAN_ABS, f"{what}: mean abs error {err.mean():.3e}"


def assert_lse_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    both_inf = np.isneginf(got) & np.isneginf(want)
    assert (np.isneginf(got) == np.isneginf(want)).all(), f"{what}: -inf pattern differs"
    err = np.abs(np.where(both_inf, 0, got - want))
    assert err.max() <= LSE_ABS, f"{what}: max abs error {err.max():.3e}"


def check_rows(inp, rows, scores, idx, out, lse):
    """Compare GPU results of the given query rows with the oracle (scores and
    Top-K sets bit for bit; attention and LSE within tolerance unless `out` /
    `lse` is None)."""
    import oracle
    ref = oracle.dsa_step(inp, rows, with_attention=out is not None)
    for i, r in enumerate(rows):
        n = int(ref["n_visible"][i])
        g = scores[r, :n].double().cpu().numpy()
        assert np.array_equal(g, ref["scores"][i, :n]), f"row {r}: index scores differ (must be bit-exact)"
    got_idx = idx[rows].cpu().numpy()
    assert np.array_equal(got_idx, ref["idx"]), "Top-K index sets differ (must be bit-exact)"
    if out is not None:
        assert_attention_close(out[rows].cpu().numpy(), ref["out"], "sparse MLA")
    if lse is not None:
        assert_lse_close(lse[rows].cpu().numpy(), ref["lse"], "lse")
    assert sa.check_device_error() == 0

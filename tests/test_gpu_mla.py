"""GPU parity: sparse MLA (decode with split keys, prefill) against the fp64
oracle, on selections drawn independently of the indexer (ragged tiles, -1
slots, empty sets, head counts below 128)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_07_b200 as sa
import workloads as W
from _gpu import assert_attention_close, assert_lse_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(rows, H, k, L, seed, paged=True, hole_frac=0.1, empty_rows=()):
    cfg = W.small_dsa(W.RAGGED, n_seqs=rows, rows=rows, lens=(L,) * rows, H_I=16, topk=k, H=H, paged=paged)
    inp = W.dsa_inputs(cfg, DEV, seed=seed)
    rng = np.random.default_rng(seed)
    idx = np.full((rows, k), -1, dtype=np.int32)
    for r in range(rows):
        if r in empty_rows:
            continue
        n = min(k, L)
        pos = np.sort(rng.choice(L, size=n, replace=False))
        pos[rng.random(n) < hole_frac] = -1
        idx[r, :n] = pos
    return cfg, inp, torch.from_numpy(idx).to(DEV)


def _oracle(cfg, inp, idx):
    table = None if inp["page_table"] is None else inp["page_table"].cpu().numpy()
    idx_np = idx.cpu().numpy()
    sel = np.full(idx_np.shape, -1, dtype=np.int64)
    flat = []
    for r in range(cfg.rows):
        v = idx_np[r] >= 0
        pr = oracle.pool_rows(table, cfg.pages_per_seq, r, idx_np[r][v])
        sel[r, v] = np.arange(len(flat), len(flat) + len(pr))
        flat.extend(pr.tolist())
    fr = torch.tensor(flat, dtype=torch.long, device=DEV)
    c = inp["c_cache"][fr].double().cpu().numpy() if flat else np.zeros((0, cfg.d_c))
    kr = inp["kr_cache"][fr].double().cpu().numpy() if flat else np.zeros((0, cfg.d_R))
    return oracle.sparse_mla(inp["q_lat"].double().cpu().numpy(), inp["q_rope"].double().cpu().numpy(), c, kr,
                             sel, cfg.scale)


def _run(fn, cfg, inp, idx):
    lse = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=DEV)
    out = fn(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale, cfg.pages_per_seq,
             page_table=inp["page_table"], lse=lse)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("fn_name", ["decode", "prefill"])
@pytest.mark.parametrize("rows,H,k,L", [(1, 128, 100, 300), (3, 128, 2048, 5000), (2, 16, 128, 2048),
                                        (5, 77, 33, 40)])
def test_sparse_mla_vs_oracle(fn_name, rows, H, k, L):
    fn = sa.sparse_mla_decode if fn_name == "decode" else sa.sparse_mla_prefill
    cfg, inp, idx = _case(rows, H, k, L, seed=rows * 100 + H)
    out, lse = _run(fn, cfg, inp, idx)
    ref_out, ref_lse = _oracle(cfg, inp, idx)
    assert_attention_close(out, ref_out, f"{fn_name} rows={rows} H={H} k={k}")
    assert_lse_close(lse, ref_lse, "lse")
    assert sa.check_device_error() == 0


@pytest.mark.parametrize("fn_name", ["decode", "prefill"])
def test_sparse_mla_empty_selection(fn_name):
    fn = sa.sparse_mla_decode if fn_name == "decode" else sa.sparse_mla_prefill
    cfg, inp, idx = _case(3, 128, 64, 500, seed=4, empty_rows=(1,))
    out, lse = _run(fn, cfg, inp, idx)
    assert (out[1] == 0).all() and np.isneginf(lse[1]).all()
    ref_out, ref_lse = _oracle(cfg, inp, idx)
    assert_attention_close(out, ref_out, "rows around an empty one")
    assert sa.check_device_error() == 0


def test_sparse_mla_contiguous_fused_row_layout():
    """c and k^R interleaved in one 576-wide row (strides instead of two pools)."""
    cfg, inp, idx = _case(2, 128, 256, 1024, seed=8, paged=False)
    fused = torch.cat([inp["c_cache"], inp["kr_cache"]], dim=1).contiguous()
    c_view = fused[:, :512]
    kr_view = fused[:, 512:]
    out = sa.sparse_mla_decode(inp["q_lat"], inp["q_rope"], c_view, kr_view, idx, cfg.scale, cfg.pages_per_seq)
    ref_out, _ = _oracle(cfg, inp, idx)
    assert_attention_close(out.cpu().numpy(), ref_out, "fused rows")
    assert sa.check_device_error() == 0


def test_sparse_mla_large_scores_rescale():
    """Scores growing along the selection force the lazy rescale of O."""
    cfg, inp, idx = _case(1, 128, 512, 600, seed=12, hole_frac=0.0)
    # scale the keys of later positions up so the running maximum keeps rising
    ramp = torch.linspace(0.2, 3.0, inp["c_cache"].shape[0], device=DEV)[:, None]
    inp["c_cache"] = (inp["c_cache"].float() * ramp).to(torch.bfloat16)
    out, lse = _run(sa.sparse_mla_decode, cfg, inp, idx)
    ref_out, ref_lse = _oracle(cfg, inp, idx)
    assert_attention_close(out, ref_out, "rising scores")
    assert_lse_close(lse, ref_lse, "lse")


@pytest.mark.parametrize("fn_name", ["decode", "prefill"])
def test_sparse_mla_leading_empty_tiles(fn_name):
    """Whole 32-key tiles of -1 before and between valid positions (the running
    maximum is still -inf when the first valid key arrives)."""
    fn = sa.sparse_mla_decode if fn_name == "decode" else sa.sparse_mla_prefill
    cfg, inp, idx = _case(2, 128, 256, 1000, seed=31, hole_frac=0.0)
    idx[:, :96] = -1
    idx[1, 160:200] = -1
    out, lse = _run(fn, cfg, inp, idx)
    ref_out, ref_lse = _oracle(cfg, inp, idx)
    assert_attention_close(out, ref_out, "leading empty tiles")
    assert_lse_close(lse, ref_lse, "lse")
    assert sa.check_device_error() == 0


def test_sparse_mla_split_merge_repeatable():
    """Split keys (three rows: sixteen key splits each): the merged output is
    the same on every call, whatever the workspace held before, and one
    workspace serves calls back to back."""
    cfg, inp, idx = _case(3, 128, 2048, 5000, seed=77)
    need = sa.sparse_mla_workspace_size(cfg.rows, cfg.H, cfg.topk, cfg.d_c)

    def call(ws):
        lse = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=DEV)
        out = sa.sparse_mla_decode(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale,
                                   cfg.pages_per_seq, page_table=inp["page_table"], lse=lse, workspace=ws)
        torch.cuda.synchronize()
        return out, lse

    out0, lse0 = call(torch.zeros(need, dtype=torch.uint8, device=DEV))
    for fill in (255, 0x5A):
        out, lse = call(torch.full((need,), fill, dtype=torch.uint8, device=DEV))
        assert torch.equal(out, out0) and torch.equal(lse, lse0)
    ws = torch.full((need,), 255, dtype=torch.uint8, device=DEV)
    for _ in range(3):
        out, lse = call(ws)
        assert torch.equal(out, out0) and torch.equal(lse, lse0)
    ref_out, ref_lse = _oracle(cfg, inp, idx)
    assert_attention_close(out0.cpu().numpy(), ref_out, "split merge")
    assert_lse_close(lse0.cpu().numpy(), ref_lse, "lse")
    assert sa.check_device_error() == 0


def test_sparse_mla_bad_position_is_reported():
    """A selected position past the sequence's page table, then a page-table
    entry outside the pool: the kernel reads pool row 0 for those slots
    (never an address outside the pool), records code 0x700 in the device
    error word, and the rows without a bad slot keep their exact result."""
    cfg, inp, idx = _case(2, 128, 64, 500, seed=9)
    ref_out, _ = _oracle(cfg, inp, idx)
    bad = idx.clone()
    bad[0, 3] = cfg.pages_per_seq * 64 + 5
    out, _ = _run(sa.sparse_mla_decode, cfg, inp, bad)
    assert sa.check_device_error() == 0x700
    assert np.isfinite(out).all()
    assert_attention_close(out[1:], ref_out[1:], "row beside the bad slot")
    pool_pages = inp["c_cache"].shape[0] // 64
    good = idx.clone()
    good[1, 0] = 0  # a slot on page 0 of row 1
    saved = inp["page_table"].clone()
    inp["page_table"][1, 0] = pool_pages + 3
    try:
        out, _ = _run(sa.sparse_mla_decode, cfg, inp, good)
        assert sa.check_device_error() == 0x700
        assert np.isfinite(out).all()
    finally:
        inp["page_table"].copy_(saved)
    out, _ = _run(sa.sparse_mla_decode, cfg, inp, idx)
    assert sa.check_device_error() == 0
    assert_attention_close(out, ref_out, "after the reports")


@pytest.mark.parametrize("fn_name,rows,H,k,L", [
    ("decode", 3, 128, 2048, 5000),   # keys split over several pairs: the combine writes the output
    ("decode", 80, 128, 256, 700),    # one pair per row: the attention kernel writes it
    ("decode", 5, 77, 33, 40),
    ("prefill", 6, 128, 1000, 3000),
])
def test_sparse_mla_bf16_output(fn_name, rows, H, k, L):
    """The bf16-output calls: every element is the fp32 call's output rounded
    to the nearest bf16 (bit for bit), lse as the fp32 call's, and the result
    within the attention tolerance of the oracle."""
    cfg, inp, idx = _case(rows, H, k, L, seed=300 + rows, empty_rows=(1,))
    fn = sa.sparse_mla_decode if fn_name == "decode" else sa.sparse_mla_prefill
    lse32 = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=DEV)
    lse16 = torch.empty_like(lse32)
    o32 = fn(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale, cfg.pages_per_seq,
             page_table=inp["page_table"], lse=lse32)
    o16 = torch.empty(cfg.rows, cfg.H, cfg.d_c, dtype=torch.bfloat16, device=DEV)
    fn(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale, cfg.pages_per_seq,
       page_table=inp["page_table"], out=o16, lse=lse16)
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(lse16, lse32)
    out, lse = _oracle(cfg, inp, idx)
    assert_attention_close(o16.float().cpu().numpy(), out)
    assert sa.check_device_error() == 0

"""GPU parity: dense MLA decode (the short-sequence mode, every visible
position attended) against the fp64 oracle run on all positions of each row,
and against the sparse kernel given the full selection."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_07_b200 as sa
import workloads as W
from _gpu import assert_attention_close, assert_lse_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(lens, H, seed, paged=True):
    rows = len(lens)
    cfg = W.small_dsa(W.RAGGED, n_seqs=rows, rows=rows, lens=tuple(lens), H_I=16, topk=max(lens), H=H, paged=paged)
    inp = W.dsa_inputs(cfg, DEV, seed=seed)
    return cfg, inp


def _oracle_all(cfg, inp, lens):
    """The oracle's sparse MLA with every visible position selected."""
    table = None if inp["page_table"] is None else inp["page_table"].cpu().numpy()
    L = max(lens)
    sel = np.full((len(lens), L), -1, dtype=np.int64)
    flat = []
    for r, n in enumerate(lens):
        pr = oracle.pool_rows(table, cfg.pages_per_seq, r, np.arange(n))
        sel[r, :n] = np.arange(len(flat), len(flat) + n)
        flat.extend(pr.tolist())
    fr = torch.tensor(flat, dtype=torch.long, device=DEV)
    c = inp["c_cache"][fr].double().cpu().numpy()
    kr = inp["kr_cache"][fr].double().cpu().numpy()
    return oracle.sparse_mla(inp["q_lat"].double().cpu().numpy(), inp["q_rope"].double().cpu().numpy(), c, kr,
                             sel, cfg.scale)


@pytest.mark.parametrize("lens,H", [((100, 2048, 3000), 128), ((4097, 64), 77), ((1, 5000), 16)])
def test_dense_mla_vs_oracle(lens, H):
    cfg, inp = _case(lens, H, seed=sum(lens) + H)
    nv = torch.tensor(lens, dtype=torch.int32, device=DEV)
    lse = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=DEV)
    out = sa.dense_mla_decode(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], nv, max(lens), cfg.scale,
                              cfg.pages_per_seq, page_table=inp["page_table"], lse=lse)
    torch.cuda.synchronize()
    ref_out, ref_lse = _oracle_all(cfg, inp, lens)
    assert_attention_close(out.cpu().numpy(), ref_out, f"dense lens={lens} H={H}")
    assert_lse_close(lse.cpu().numpy(), ref_lse, "dense lse")
    assert sa.check_device_error() == 0


def test_dense_equals_sparse_with_full_selection():
    """Dense mode and the sparse kernel given every position compute the same
    thing through the same kernel: identical outputs."""
    lens = (3000, 1500)
    cfg, inp = _case(lens, 128, seed=5)
    L = max(lens)
    nv = torch.tensor(lens, dtype=torch.int32, device=DEV)
    idx = torch.full((len(lens), L), -1, dtype=torch.int32, device=DEV)
    for r, n in enumerate(lens):
        idx[r, :n] = torch.arange(n, dtype=torch.int32, device=DEV)
    dense = sa.dense_mla_decode(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], nv, L, cfg.scale,
                                cfg.pages_per_seq, page_table=inp["page_table"])
    sparse = sa.sparse_mla_decode(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale,
                                  cfg.pages_per_seq, page_table=inp["page_table"])
    torch.cuda.synchronize()
    assert torch.equal(dense, sparse)
    assert sa.check_device_error() == 0


def test_dense_mla_empty_rows():
    lens = (0, 700)
    cfg, inp = _case((1, 700), 128, seed=9)
    nv = torch.tensor(lens, dtype=torch.int32, device=DEV)
    lse = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=DEV)
    out = sa.dense_mla_decode(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], nv, 700, cfg.scale,
                              cfg.pages_per_seq, page_table=inp["page_table"], lse=lse)
    torch.cuda.synchronize()
    assert (out[0] == 0).all() and torch.isneginf(lse[0]).all()
    assert torch.isfinite(out[1]).all()

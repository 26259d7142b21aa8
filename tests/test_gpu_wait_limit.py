"""The bounded-wait failure path on the GPU, made to happen without a fault.

Every wait of the sparse-MLA kernel on another party (a ring slot another
warp fills, the partner CTA's partial scores) has a time limit.  With the
limit set to 200 ns the kernel's waits run out at once: the kernel must
record a sparse-MLA site code in the device error word, drain its own copies
and tensor-core work, free its tensor memory and return (the synchronise
returns), and sa_check_device_error must report SA_ETIMEOUT with that code.
With the default limit restored, the same call must then be correct against
the oracle: the context stays usable."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_07_b200 as sa
import workloads as W
from _gpu import assert_attention_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call(inp, cfg, idx, out):
    return sa.sparse_mla_decode(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], idx, cfg.scale,
                                cfg.pages_per_seq, page_table=inp["page_table"], seq_of_row=inp["seq_of_row"],
                                out=out)


def test_wait_limit_runs_out_and_the_next_call_is_correct():
    cfg = W.small_dsa(W.RAGGED, n_seqs=2, rows=2, lens=(3000, 1500), topk=512)
    inp = W.dsa_inputs(cfg, DEV, seed=41)
    scores = sa.index_scores(inp["q_idx"], inp["w"], inp["k_idx_cache"], inp["n_visible"], cfg.pages_per_seq,
                             page_table=inp["page_table"], seq_of_row=inp["seq_of_row"])
    idx = sa.topk_select(scores, inp["n_visible"], cfg.topk)
    torch.cuda.synchronize()
    assert sa.check_device_error() == 0

    out = torch.empty(cfg.rows, cfg.H, cfg.d_c, dtype=torch.float32, device=DEV)
    sa.set_wait_limit_ns(200)
    try:
        _call(inp, cfg, idx, out)
        torch.cuda.synchronize()  # returns: the kernel gave up instead of waiting
        code = sa.check_device_error()
    finally:
        sa.set_wait_limit_ns(0)
    assert code != 0, "a 200 ns limit must run out"
    assert code & 0xF00 == 0x200, f"expected a sparse-MLA wait site code, got 0x{code:x}"
    assert sa.check_device_error() == 0  # reading the word cleared it

    _call(inp, cfg, idx, out)
    torch.cuda.synchronize()
    assert sa.check_device_error() == 0
    ref = oracle.dsa_step(inp, list(range(cfg.rows)), with_scores=False)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert_attention_close(out.cpu().numpy(), ref["out"], "sparse MLA after the timeout")

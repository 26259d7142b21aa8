"""GPU parity: the per-head projections around sparse MLA (query absorption
with U_K, up-projection with U_V) against the fp64 oracle (oracle.absorb,
oracle.up_project), the pages' worked absorption example on the GPU, and the
whole chain q^C -> q_lat -> sparse MLA -> U_V against oracle.mla_chain."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_07_b200 as sa
from _gpu import assert_attention_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(shape, g, scale=1.0):
    return (torch.randn(shape, generator=g, device=DEV) * scale).to(torch.bfloat16)


def _f64(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("rows,H", [(1, 16), (32, 128), (70, 3)])
def test_absorb_query_vs_oracle(rows, H):
    g = torch.Generator(device=DEV)
    g.manual_seed(rows * 7 + H)
    d_C, d_c = 128, 512
    q_c = _bf16((rows, H, d_C), g)
    U_K = _bf16((H, d_C, d_c), g, 1.0 / np.sqrt(d_C))
    got = _f64(sa.mla_absorb_query(q_c, U_K))
    qn, Un = _f64(q_c), _f64(U_K)
    ref = np.stack([np.stack([oracle.absorb(Un[h], qn[r, h]) for h in range(H)]) for r in range(rows)])
    # fp32 accumulation of bf16 products, output rounded to bf16
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4)
    assert sa.check_device_error() == 0


@pytest.mark.parametrize("rows,H", [(1, 16), (32, 128), (70, 3)])
def test_up_project_vs_oracle(rows, H):
    g = torch.Generator(device=DEV)
    g.manual_seed(rows * 11 + H)
    d_c, d_v = 512, 128
    o_lat = torch.randn(rows, H, d_c, generator=g, device=DEV) * 0.1
    U_V = _bf16((H, d_v, d_c), g, 1.0 / np.sqrt(d_c))
    got = _f64(sa.mla_up_project(o_lat, U_V))
    # the kernel's tensor-core operand is the latent output rounded to bf16
    o_b = _f64(o_lat.to(torch.bfloat16))
    ref = oracle.up_project(_f64(U_V), o_b)
    assert np.abs(got - ref).max() <= 1e-5 + 1e-5 * np.abs(ref).max()
    # and against the unrounded latent output: within the bf16 input rounding
    ref32 = oracle.up_project(_f64(U_V), _f64(o_lat))
    assert np.abs(got - ref32).max() <= 2e-3
    # a bf16 latent output (the _bf16 attention calls) gives the same product bit for bit
    got_b = sa.mla_up_project(o_lat.to(torch.bfloat16), U_V)
    assert np.array_equal(_f64(got_b), got)
    assert sa.check_device_error() == 0


def test_absorbed_example_on_the_gpu():
    """[MLA-S] worked example (latent c=[2,-1], U_K 3x2, q=[1,2,-1] -> U_K^T q =
    [0,3]), embedded in the kernel's smallest supported sizes with zeros."""
    with open(os.path.join(GOLDEN, "absorbed_score.json")) as f:
        gd = json.load(f)
    U = np.array(gd["U_K"])  # [d_C=3][d_c=2]
    q = np.array(gd["query_q"])
    U_K = torch.zeros(1, 64, 128, dtype=torch.bfloat16, device=DEV)
    U_K[0, :3, :2] = torch.tensor(U, dtype=torch.bfloat16)
    q_c = torch.zeros(1, 1, 64, dtype=torch.bfloat16, device=DEV)
    q_c[0, 0, :3] = torch.tensor(q, dtype=torch.bfloat16)
    got = sa.mla_absorb_query(q_c, U_K)[0, 0, :2].float().cpu().numpy()
    assert got.tolist() == gd["absorbed_query"]
    c = np.array(gd["latent_c"])
    assert float(got @ c) == gd["score"]


def test_absorb_mla_up_chain():
    """q^C -> absorbed query -> sparse MLA -> U_V on the GPU against the
    oracle's absorbed chain (itself pinned to the explicit-keys form
    k^C_j = U_K c_j, v_j = U_V c_j)."""
    g = torch.Generator(device=DEV)
    g.manual_seed(21)
    rows, H, d_C, d_c, d_R, d_v, n = 2, 16, 128, 512, 64, 128, 300
    q_c = _bf16((rows, H, d_C), g)
    U_K = _bf16((H, d_C, d_c), g, 1.0 / np.sqrt(d_C))
    U_V = _bf16((H, d_v, d_c), g, 1.0 / np.sqrt(d_c))
    q_rope = _bf16((rows, H, d_R), g)
    pool = (n + 63) // 64 * 64  # one sequence of 64-token pages, shared by both rows
    c = _bf16((pool, d_c), g)
    kr = _bf16((pool, d_R), g)
    idx = torch.arange(n, dtype=torch.int32, device=DEV).repeat(rows, 1)
    idx[1, ::3] = -1
    seq = torch.zeros(rows, dtype=torch.int32, device=DEV)
    scale = 1.0 / np.sqrt(d_C + d_R)
    q_lat = sa.mla_absorb_query(q_c, U_K)
    o_lat = sa.sparse_mla_decode(q_lat, q_rope, c, kr, idx, scale, pages_per_seq=pool // 64, seq_of_row=seq)
    out = _f64(sa.mla_up_project(o_lat, U_V))
    sel = idx.cpu().numpy().astype(np.int64)  # one sequence: pool row = position
    ref = oracle.mla_chain(_f64(q_c), _f64(U_K), _f64(U_V), _f64(q_rope), _f64(c), _f64(kr), sel, scale)
    # q_lat is rounded to bf16 before the scores and o_lat before U_V
    assert_attention_close(out, ref, "absorb -> sparse MLA -> U_V")
    assert sa.check_device_error() == 0

"""Pins for the fp64 oracle: the pages' worked examples, closed forms,
invariants and library routines.  None of these compares the oracle with
itself; each is chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.

CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- MLA scores

def test_absorbed_query_example(golden_dir):
    """MLA-S "先看一条压缩后的表示": score -3 computed directly and via U_K^T q."""
    g = _golden(golden_dir, "absorbed_score.json")
    c, U, q = np.array(g["latent_c"]), np.array(g["U_K"]), np.array(g["query_q"])
    assert (U @ c).tolist() == g["key_k"]
    assert float(q @ (U @ c)) == g["score"]
    qa = oracle.absorb(U, q)
    assert qa.tolist() == g["absorbed_query"]
    # the oracle's score path consumes the absorbed query; with one selected
    # row and scale 1 its log-sum-exp is exactly that row's score
    out, lse = oracle.sparse_mla(qa[None, None], np.zeros((1, 1, 1)), c[None], np.zeros((1, 1)),
                                 np.array([[0]]), 1.0)
    assert lse[0, 0] == g["score"]
    assert out[0, 0].tolist() == c.tolist()      # one row: weight 1, output = that latent


def test_absorbed_identity_random():
    """q^T U_K c_j = (U_K^T q)^T c_j for every row: the oracle on the absorbed
    query equals dense attention on the expanded keys k_j = U_K c_j (values c_j)."""
    rng = np.random.default_rng(7)
    d_k, d_c, n = 24, 16, 9
    U = rng.standard_normal((d_k, d_c))
    q = rng.standard_normal(d_k)
    C = rng.standard_normal((n, d_c))
    keys = C @ U.T
    scale = 0.3
    ref, _ = oracle.dense_attention(q, keys, C, scale)
    out, _ = oracle.sparse_mla(oracle.absorb(U, q)[None, None], np.zeros((1, 1, 1)), C,
                               np.zeros((n, 1)), np.arange(n)[None], scale)
    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-12)


def test_up_project_by_hand():
    """[MLA-S] up-projection o = U_V o_lat on a 3x2 U_V worked by hand:
    rows (1, 0), (0, 2), (1, 1) applied to (2, -1) give (2, -2, 1); a second
    head with its own U_V = identity keeps its latent."""
    U = np.array([[[1.0, 0.0], [0.0, 2.0], [1.0, 1.0]], [[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]]])
    o = np.array([[[2.0, -1.0], [5.0, 7.0]]])
    got = oracle.up_project(U, o)
    assert got.shape == (1, 2, 3)
    assert got[0, 0].tolist() == [2.0, -2.0, 1.0]
    assert got[0, 1].tolist() == [5.0, 7.0, 0.0]


def test_mla_chain_equals_explicit_keys_and_values():
    """[MLA-S] "“吸收矩阵”是交换线性计算的顺序": the absorbed chain (U_K^T q^C
    as the query of the latent rows, latent aggregate, then U_V) equals
    attention computed without absorption, with explicit content keys
    k^C_j = U_K c_j, the RoPE keys, and values v_j = U_V c_j
    (sum_j a_j U_V c_j = U_V sum_j a_j c_j).  Random inputs, empty slots,
    several heads with their own U_K and U_V."""
    rng = np.random.default_rng(17)
    rows, H, d_C, d_c, d_R, d_v, n, k = 2, 3, 6, 10, 4, 5, 23, 9
    q_c = rng.standard_normal((rows, H, d_C))
    U_K = rng.standard_normal((H, d_C, d_c))
    U_V = rng.standard_normal((H, d_v, d_c))
    q_r = rng.standard_normal((rows, H, d_R))
    c = rng.standard_normal((n, d_c))
    kr = rng.standard_normal((n, d_R))
    sel = rng.choice(n, size=(rows, k), replace=True)
    sel[1, ::4] = -1
    scale = 1.0 / math.sqrt(d_C + d_R)
    got = oracle.mla_chain(q_c, U_K, U_V, q_r, c, kr, sel, scale)
    for r in range(rows):
        js = [j for j in sel[r] if j >= 0]
        for h in range(H):
            z = np.array([(q_c[r, h] @ (U_K[h] @ c[j]) + q_r[r, h] @ kr[j]) * scale for j in js])
            a = np.exp(z - z.max())
            a /= a.sum()
            want = sum(a_j * (U_V[h] @ c[j]) for a_j, j in zip(a, js))
            np.testing.assert_allclose(got[r, h], want, rtol=0, atol=1e-12)


def test_content_plus_position_example(golden_dir):
    """MLA-S "分开以后": content 1,1 + RoPE 0,2, /sqrt(4) -> 0.5,1.5 -> 0.269,0.731."""
    g = _golden(golden_dir, "content_position.json")
    # latent rows are unit vectors, so the output is the weight vector itself
    c = np.eye(2)
    q_lat = np.array([[[1.0, 1.0]]])                 # content scores 1 and 1
    q_rope = np.array([[[1.0]]])
    kr = np.array([[0.0], [2.0]])                    # RoPE scores 0 and 2
    out, lse = oracle.sparse_mla(q_lat, q_rope, c, kr, np.array([[0, 1]]), 1.0 / math.sqrt(g["total_dim"]))
    w = out[0, 0]
    assert np.round(w, g["printed_decimals"]).tolist() == g["weights_printed"]
    # closed form: softmax of (0.5, 1.5) is (1/(1+e), e/(1+e))
    np.testing.assert_allclose(w, [1 / (1 + math.e), math.e / (1 + math.e)], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], math.log(math.exp(0.5) + math.exp(1.5)), atol=1e-15)


def test_missed_position_example(golden_dir):
    """MLA-S "稀疏注意力": 8 zero scores, value 8 at one position: dense 1, sparse 0."""
    g = _golden(golden_dir, "missed_position.json")
    n = g["n_positions"]
    c = np.zeros((n, 1)); c[g["evidence_position"], 0] = g["evidence_value"]
    q_lat = np.zeros((1, 1, 1)); q_rope = np.zeros((1, 1, 1)); kr = np.zeros((n, 1))
    dense, _ = oracle.sparse_mla(q_lat, q_rope, c, kr, np.arange(n)[None], 1.0)
    others = [j for j in range(n) if j != g["evidence_position"]]
    sparse, _ = oracle.sparse_mla(q_lat, q_rope, c, kr, np.array([others]), 1.0)
    assert dense[0, 0, 0] == pytest.approx(g["dense_output"], abs=1e-15)
    assert sparse[0, 0, 0] == g["sparse_output_without_it"]


def test_selected_positions_example(golden_dir):
    """MLA-S "一次错选会丢掉什么？": Top-2 of [3,2,1,0] is [0,1]; the dense output
    10e^4/(e^4+3) > 9 while the selection's output is 0."""
    g = _golden(golden_dir, "selected_positions.json")
    chosen = oracle.topk(np.array(g["index_scores"]), len(g["index_scores"]), g["count"])[0]
    assert chosen.tolist() == g["chosen"]
    n = len(g["values"])
    c = np.array(g["values"])[:, None]               # value = latent row
    kr = np.array(g["attention_scores"])[:, None]    # score carried by the RoPE branch
    q_lat = np.zeros((1, 1, 1)); q_rope = np.ones((1, 1, 1))
    dense, _ = oracle.sparse_mla(q_lat, q_rope, c, kr, np.arange(n)[None], 1.0)
    sparse, _ = oracle.sparse_mla(q_lat, q_rope, c, kr, chosen[None].astype(np.int64), 1.0)
    e4 = math.exp(4.0)
    assert dense[0, 0, 0] == pytest.approx(10 * e4 / (e4 + 3), abs=1e-12)
    assert dense[0, 0, 0] > g["dense_output_greater_than"]
    assert sparse[0, 0, 0] == g["sparse_output"]


def test_causal_mask_example(golden_dir):
    """MLA-S causal check: masking before the softmax gives 3 for any future
    score; the plausible mistake (masking after the softmax) gives 2 and then
    below 0.001, so this pin tells the two apart."""
    g = _golden(golden_dir, "causal_mask.json")
    vals, vis = np.array(g["values"]), np.array(g["visible"])

    def mask_after(scores):            # the mistake the page warns about, written here on purpose
        a = np.exp(np.array(scores) - max(scores))
        return float((a * vals * vis).sum() / a.sum())

    for case in g["cases"]:
        assert oracle.masked_attention(case["scores"], vals, vis) == case["mask_before"]
        # the sparse-MLA oracle over the visible set S = {0, 1} agrees
        c = vals[:2, None]; kr = np.array(case["scores"])[:2, None]
        out, _ = oracle.sparse_mla(np.zeros((1, 1, 1)), np.ones((1, 1, 1)), c, kr, np.array([[0, 1]]), 1.0)
        assert out[0, 0, 0] == case["mask_before"]
        if "mask_after" in case:
            assert mask_after(case["scores"]) == case["mask_after"]
        else:
            assert mask_after(case["scores"]) < case["mask_after_below"]


def test_mask_form_equals_renormalisation():
    """Notes §3 vs §2/§6: softmax(S + M) over all positions equals the dense
    weights renormalised by Z on the chosen set, and the sparse-MLA oracle."""
    rng = np.random.default_rng(11)
    n, d = 40, 12
    C = rng.standard_normal((n, d))
    qc = rng.standard_normal(d)
    scale = 0.37
    S = np.sort(rng.choice(n, size=13, replace=False))
    _, alpha = oracle.dense_attention(qc, C, C, scale)
    Z = oracle.dense_mass(alpha, S)
    renorm = (alpha[S, None] / Z * C[S]).sum(0)
    vis = np.zeros(n, dtype=bool); vis[S] = True
    mask_form = np.array([oracle.masked_attention(C @ qc * scale, C[:, j], vis) for j in range(d)])
    out, _ = oracle.sparse_mla(qc[None, None], np.zeros((1, 1, 1)), C, np.zeros((n, 1)), S[None], scale)
    np.testing.assert_allclose(mask_form, renorm, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[0, 0], renorm, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_topk_error_bound(seed):
    """Notes §6: ||o_dense - o_sparse|| <= 2 V_max (1 - Z) with V_max bounding every value."""
    rng = np.random.default_rng(seed)
    n, d = 64, 8
    C = rng.standard_normal((n, d)) * rng.uniform(0.5, 3.0)
    qc = rng.standard_normal(d)
    S = np.sort(rng.choice(n, size=rng.integers(1, n), replace=False))
    dense, alpha = oracle.dense_attention(qc, C, C, 1.0)
    out, _ = oracle.sparse_mla(qc[None, None], np.zeros((1, 1, 1)), C, np.zeros((n, 1)), S[None], 1.0)
    vmax = np.linalg.norm(C, axis=1).max()
    Z = oracle.dense_mass(alpha, S)
    assert np.linalg.norm(dense - out[0, 0]) <= oracle.error_bound(vmax, Z) + 1e-12


def test_k_equals_L_is_dense_attention():
    """Notes §1: selecting every position gives dense attention (torch softmax, fp64)."""
    rng = np.random.default_rng(5)
    n, H, d_c, d_R = 50, 3, 16, 4
    q_lat, q_rope = rng.standard_normal((1, H, d_c)), rng.standard_normal((1, H, d_R))
    C, KR = rng.standard_normal((n, d_c)), rng.standard_normal((n, d_R))
    scale = 1 / math.sqrt(20)
    out, lse = oracle.sparse_mla(q_lat, q_rope, C, KR, np.arange(n)[None], scale)
    t = lambda a: torch.from_numpy(a)
    s = (t(q_lat[0]) @ t(C).T + t(q_rope[0]) @ t(KR).T) * scale
    ref = torch.softmax(s, dim=-1) @ t(C)
    np.testing.assert_allclose(out[0], ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_sparse_mla_heads_independent_and_empty_slots():
    """MLA-S: heads share the rows but not the distribution; -1 slots are skipped."""
    rng = np.random.default_rng(9)
    n, H, d_c, d_R = 20, 4, 8, 2
    q_lat, q_rope = rng.standard_normal((1, H, d_c)), rng.standard_normal((1, H, d_R))
    C, KR = rng.standard_normal((n, d_c)), rng.standard_normal((n, d_R))
    sel = np.array([[3, 7, -1, 11, -1]])
    out, lse = oracle.sparse_mla(q_lat, q_rope, C, KR, sel, 0.5)
    for h in range(H):
        ref, _ = oracle.dense_attention(np.concatenate([q_lat[0, h], q_rope[0, h]]),
                                        np.concatenate([C, KR], 1)[[3, 7, 11]], C[[3, 7, 11]], 0.5)
        np.testing.assert_allclose(out[0, h], ref, atol=1e-12)
    empty_out, empty_lse = oracle.sparse_mla(q_lat, q_rope, C, KR, np.full((1, 3), -1), 0.5)
    assert (empty_out == 0).all() and np.isneginf(empty_lse).all()


# ------------------------------------------------------------------ indexer

def test_index_score_hand_example():
    """Notes §9 by hand: heads (1,2) and (-1,1), weights 0.5 and 2, key (3,-1):
    dots 1 and -4, ReLU 1 and 0, score 0.5.  Key (-1,2): dots 3 and 3 -> 1.5 + 6."""
    q = np.array([[[1.0, 2.0], [-1.0, 1.0]]])
    w = np.array([[0.5, 2.0]])
    keys = np.array([[3.0, -1.0], [-1.0, 2.0]])
    s = oracle.index_scores(q, w, keys, [0], [2])
    assert s[0].tolist() == [0.5, 7.5]


def test_index_scores_vs_einsum_and_causal_bound():
    """Random integer inputs against numpy einsum + maximum (a library routine);
    positions past the visible length are not scored."""
    rng = np.random.default_rng(3)
    rows, H_I, d_I, n = 5, 6, 16, 300
    q = rng.integers(-8, 9, size=(rows, H_I, d_I)).astype(float)
    w = 2.0 ** rng.integers(-4, 2, size=(rows, H_I))
    keys = rng.integers(-8, 9, size=(2 * n, d_I)).astype(float)
    key0 = np.array([0, n, 0, n, n])
    n_vis = np.array([n, n - 7, 1, 0, 123])
    s = oracle.index_scores(q, w, keys, key0, n_vis, out_ld=n)
    for r in range(rows):
        K = keys[key0[r]: key0[r] + n_vis[r]]
        ref = (np.maximum(np.einsum("hd,sd->sh", q[r], K), 0) * w[r]).sum(1)
        assert np.array_equal(s[r, :n_vis[r]], ref)        # integers x 2^-4: exact
        assert np.isnan(s[r, n_vis[r]:]).all()


# --------------------------------------------------------------------- top-k

def test_topk_selected_positions_example(golden_dir):
    g = _golden(golden_dir, "selected_positions.json")
    assert oracle.topk(g["index_scores"], 4, 2)[0].tolist() == g["chosen"]


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce_with_ties(seed):
    """Brute force via numpy lexsort on (-score, position), ascending output."""
    rng = np.random.default_rng(seed)
    rows, n, k = 7, 97, 13
    scores = rng.integers(-3, 4, size=(rows, n)).astype(float)       # many ties
    n_valid = rng.integers(0, n + 1, size=rows)
    got = oracle.topk(scores, n_valid, k)
    for r in range(rows):
        m = n_valid[r]
        order = np.lexsort((np.arange(m), -scores[r, :m]))
        want = np.sort(order[: min(k, m)])
        assert got[r, : len(want)].tolist() == want.tolist()
        assert (got[r, len(want):] == -1).all()


def test_topk_degenerate_cases():
    eq = oracle.topk(np.zeros((1, 50)), 50, 8)[0]
    assert eq.tolist() == list(range(8))                 # all equal: lowest positions
    few = oracle.topk(np.arange(5.0)[None], 5, 8)[0]
    assert few.tolist() == [0, 1, 2, 3, 4, -1, -1, -1]   # k > n: all, then -1
    none = oracle.topk(np.zeros((1, 4)), 0, 3)[0]
    assert none.tolist() == [-1, -1, -1]
    neg = oracle.topk(np.array([[-1.0, -0.0, 0.0, -5.0]]), 4, 2)[0]
    assert neg.tolist() == [1, 2]                        # -0 == +0: tie to lower


# -------------------------------------------------------------- block-sparse

def test_block_toy_example(golden_dir):
    """Ch11 §12.5: n=16, B=4; choosing blocks {0 (sink), 1} reads tokens 0-7.
    The oracle is steered so block 1 is the top-1 block; with one sink block
    and no window its output is dense attention over tokens 0-7."""
    g = _golden(golden_dir, "block_toy.json")
    rng = np.random.default_rng(1)
    n, B, d = g["n"], g["B"], 8
    K = rng.standard_normal((n, d)) * 0.1
    V = rng.standard_normal((n, d))
    q = np.ones(d)
    K[4:8] += 1.0                                        # block 1 has the largest mean key
    out, sel, bs = oracle.block_sparse(q, K, V, B, 1, 1, 0, d ** -0.5)
    assert sel.tolist() == [1]
    toks = [t for b in g["selected_blocks"] for t in range(g["block_tokens"][b][0], g["block_tokens"][b][1] + 1)]
    assert toks == g["tokens_read"]
    ref, _ = oracle.dense_attention(q, K[toks], V[toks], d ** -0.5)
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_block_scores_mean_pool_vs_numpy():
    """Ch11 §12.6: block score = (q . mean(K_block)) * d^-1/2; numpy mean/argsort."""
    rng = np.random.default_rng(2)
    L, D, B = 1000, 16, 64                               # 15 complete blocks + a 40-token tail
    K, V, q = rng.standard_normal((L, D)), rng.standard_normal((L, D)), rng.standard_normal(D)
    pooled = oracle.block_mean_pool(K, B)
    np.testing.assert_allclose(pooled, K[: (L // B) * B].reshape(L // B, B, D).mean(1), atol=1e-14)
    out, sel, bs = oracle.block_sparse(q, K, V, B, 4, 1, 100, D ** -0.5)
    np.testing.assert_allclose(bs, pooled @ q * D ** -0.5, atol=1e-13)
    assert len(bs) == L // B                             # the partial tail block is no candidate
    want = np.sort(np.lexsort((np.arange(len(bs)), -bs))[:4])
    assert sel.tolist() == want.tolist()
    toks = sorted(set(t for b in want for t in range(b * B, b * B + B)) | set(range(B)) | set(range(L - 100, L)))
    ref, _ = oracle.dense_attention(q, K[toks], V[toks], D ** -0.5)
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_block_window_only_is_sliding_window():
    """Notes §4: S = {j : i - w < j <= i}; no blocks, no sink -> last w tokens."""
    rng = np.random.default_rng(4)
    L, D, w = 300, 8, 37
    K, V, q = rng.standard_normal((L, D)), rng.standard_normal((L, D)), rng.standard_normal(D)
    out, sel, _ = oracle.block_sparse(q, K, V, 64, 0, 0, w, 0.25)
    ref, _ = oracle.dense_attention(q, K[L - w:], V[L - w:], 0.25)
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_block_all_blocks_is_dense():
    rng = np.random.default_rng(6)
    L, D = 256, 8
    K, V, q = rng.standard_normal((L, D)), rng.standard_normal((L, D)), rng.standard_normal(D)
    out, sel, _ = oracle.block_sparse(q, K, V, 64, 8, 1, 16, 0.3)
    assert sel.tolist() == [0, 1, 2, 3, -1, -1, -1, -1]
    ref, _ = oracle.dense_attention(q, K, V, 0.3)
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_block_sink_tokens_always_in():
    """Ch11 §12.4 / LLMRes MoBA: the sink block is read even when it scores lowest."""
    rng = np.random.default_rng(8)
    L, D, B = 512, 8, 64
    K, V = rng.standard_normal((L, D)) * 0.01, rng.standard_normal((L, D))
    q = np.ones(D)
    K[:B] -= 5.0                                         # block 0 scores lowest
    out, sel, _ = oracle.block_sparse(q, K, V, B, 1, 1, 0, 1.0)
    assert 0 not in sel.tolist()
    toks = list(range(B)) + list(range(sel[0] * B, sel[0] * B + B))
    ref, _ = oracle.dense_attention(q, K[toks], V[toks], 1.0)
    np.testing.assert_allclose(out, ref, atol=1e-12)


# ------------------------------------------------------------ NSA branches

def _sdpa(q, K, V, scale):
    """torch's attention routine in fp64, one query per row of q."""
    t = lambda a: torch.as_tensor(np.asarray(a, dtype=np.float64))
    o = torch.nn.functional.scaled_dot_product_attention(t(q)[:, None, :], t(K)[None], t(V)[None], scale=scale)
    return o[:, 0, :].numpy()


def test_nsa_shared_choice_example(golden_dir):
    """MLA-S "选块和合并输出，实际算一遍": alone the heads read blocks 0 and 2,
    summed over the group they share block 1."""
    g = _golden(golden_dir, "nsa_shared_choice.json")
    P = g["head_probabilities"]
    assert [oracle.shared_block_choice([h], 1)[0] for h in P] == g["each_head_alone"]
    assert oracle.shared_block_choice(P, g["count"]) == g["shared_choice"]
    assert oracle.shared_block_choice(P, 3) == [1, 0, 2]
    assert oracle.shared_block_choice([[0.5, 0.5]], 1) == [0]   # ties to the lower block


def test_nsa_gate_example(golden_dir):
    """MLA-S same section: independent gates, the mix exceeds every branch."""
    g = _golden(golden_dir, "nsa_gates.json")
    o = [np.array([x]) for x in g["branch_outputs"]]
    got = oracle.nsa_combine(*o, g["gates"])
    assert abs(got[0] - g["output"]) < 1e-12 and got[0] > max(g["branch_outputs"])


def test_nsa_select_scores_aggregation():
    """NSA §3.3 aggregation by hand.  Aligned blocks (l = d = l') leave the
    scores as they are; l = 4, d = 2, l' = 4 on powers of two (so every term
    shows in the sum) gives p0+2p1+p2, p2+2p3+p4, p4."""
    p = np.array([1.0, 2.0, 4.0, 8.0, 16.0])
    np.testing.assert_array_equal(oracle.nsa_select_scores(p, 4, 4, 4), p)
    np.testing.assert_array_equal(oracle.nsa_select_scores(p, 4, 2, 4), [9.0, 36.0, 16.0])
    # l = 2, d = 1, l' = 2: p[2j] + p[2j+1] + p[2j+1] + p[2j+2]
    np.testing.assert_array_equal(oracle.nsa_select_scores(p[:4], 2, 1, 2), [1 + 2 + 2 + 4, 4 + 8 + 8])
    with pytest.raises(ValueError):
        oracle.nsa_select_scores(p, 3, 2, 4)


def _nsa_case(seed, G=4, L=300, D=16):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))


def test_nsa_window_branch_is_sliding_window():
    q, K, V = _nsa_case(11)
    gates = np.tile([0.0, 0.0, 1.0], (4, 1))
    out, _, _ = oracle.nsa_decode_group(q, K, V, 32, 2, 45, gates, 0.25)
    np.testing.assert_allclose(out, _sdpa(q, K[-45:], V[-45:], 0.25), atol=1e-12)
    out, _, _ = oracle.nsa_decode_group(q, K, V, 32, 2, 10**6, gates, 0.25)   # window past the start
    np.testing.assert_allclose(out, _sdpa(q, K, V, 0.25), atol=1e-12)


def test_nsa_selection_of_every_block_is_dense():
    q, K, V = _nsa_case(12, L=256)
    out, chosen, _ = oracle.nsa_decode_group(q, K, V, 32, 8, 0, np.tile([0.0, 1.0, 0.0], (4, 1)), 0.3)
    assert chosen.tolist() == list(range(8))
    np.testing.assert_allclose(out, _sdpa(q, K, V, 0.3), atol=1e-12)


def test_nsa_compression_equals_dense_on_blockwise_constant_history():
    """Keys and values constant inside each block: every token of a block has
    its block's score, so attending to the B copies is attending to the block
    summary once (the factor B cancels) -- which holds only if the summary is
    the block mean.  Block 1 compression is plain dense attention."""
    rng = np.random.default_rng(13)
    G, B, nb, D = 3, 16, 7, 8
    Kb, Vb, q = rng.standard_normal((nb, D)), rng.standard_normal((nb, D)), rng.standard_normal((G, D))
    K, V = np.repeat(Kb, B, axis=0), np.repeat(Vb, B, axis=0)
    gates = np.tile([1.0, 0.0, 0.0], (G, 1))
    out, _, p_cmp = oracle.nsa_decode_group(q, K, V, B, 1, 0, gates, 0.4)
    np.testing.assert_allclose(out, _sdpa(q, K, V, 0.4), atol=1e-12)
    np.testing.assert_allclose(p_cmp.sum(axis=1), 1.0, atol=1e-14)
    q, K, V = _nsa_case(14, G=2, L=50)
    out, _, _ = oracle.nsa_decode_group(q, K, V, 1, 1, 0, np.tile([1.0, 0.0, 0.0], (2, 1)), 0.5)
    np.testing.assert_allclose(out, _sdpa(q, K, V, 0.5), atol=1e-12)


def test_nsa_selection_follows_the_group_not_one_head():
    """Two heads, one KV head: head 0 alone prefers block 0, head 1 block 2, the
    group sum block 1 (the shape of the pages' example).  The selected branch
    reads exactly block 1 for both heads."""
    D, B = 4, 8
    K = np.zeros((3 * B, D))
    K[0:B, 0] = 3.0                    # block 0: head 0's favourite
    K[B:2 * B, 0] = 2.8                # block 1: good for both
    K[B:2 * B, 1] = 2.8
    K[2 * B:, 1] = 3.0                 # block 2: head 1's favourite
    V = np.random.default_rng(15).standard_normal((3 * B, D))
    q = np.array([[1.0, 0.0, 0, 0], [0.0, 1.0, 0, 0]])
    gates = np.tile([0.0, 1.0, 0.0], (2, 1))
    for h in range(2):
        _, alone, _ = oracle.nsa_decode_group(q[h:h + 1], K, V, B, 1, 0, gates[:1], 1.0)
        assert alone.tolist() == [[0], [2]][h]
    out, chosen, _ = oracle.nsa_decode_group(q, K, V, B, 1, 0, gates, 1.0)
    assert chosen.tolist() == [1]
    np.testing.assert_allclose(out, _sdpa(q, K[B:2 * B], V[B:2 * B], 1.0), atol=1e-12)


def test_nsa_incomplete_block_stays_out_of_compression_and_selection():
    """MLA-S causality check: a block that is not complete is never summarised.
    Changing the keys and values of the tail past the last complete block
    moves neither the compression scores nor the choice nor (without the
    window) the output; the window branch does see it."""
    q, K, V = _nsa_case(16, L=300)
    gates = np.tile([0.6, 0.8, 0.0], (4, 1))
    a = oracle.nsa_decode_group(q, K, V, 64, 2, 0, gates, 0.25)
    K2, V2 = K.copy(), V.copy()
    K2[256:] = 50.0 * np.random.default_rng(17).standard_normal((44, 16))
    V2[256:] += 999.0
    b = oracle.nsa_decode_group(q, K2, V2, 64, 2, 0, gates, 0.25)
    assert a[2].shape == (4, 4) and a[1].tolist() == b[1].tolist()
    np.testing.assert_array_equal(a[2], b[2])
    np.testing.assert_array_equal(a[0], b[0])
    c = oracle.nsa_decode_group(q, K2, V2, 64, 2, 16, np.tile([0.0, 0.0, 1.0], (4, 1)), 0.25)
    assert np.all(c[0] > 500.0)


def test_nsa_gates_mix_linearly_and_short_history_has_only_the_window():
    q, K, V = _nsa_case(18, L=200)
    parts = [oracle.nsa_decode_group(q, K, V, 32, 2, 40, np.tile(e, (4, 1)), 0.25)[0] for e in np.eye(3)]
    g = np.random.default_rng(19).uniform(0, 1, (4, 3))
    out, _, _ = oracle.nsa_decode_group(q, K, V, 32, 2, 40, g, 0.25)
    np.testing.assert_allclose(out, sum(g[:, i:i + 1] * parts[i] for i in range(3)), atol=1e-12)
    out, chosen, p_cmp = oracle.nsa_decode_group(q, K[:20], V[:20], 32, 2, 8, g, 0.25)
    assert chosen.size == 0 and p_cmp.shape == (4, 0)
    np.testing.assert_allclose(out, g[:, 2:3] * _sdpa(q, K[12:20], V[12:20], 0.25), atol=1e-12)


def test_bf16_round_matches_torch_and_breaks_ties_to_even():
    """oracle.bf16_round against torch's float32 -> bfloat16 conversion (one
    round-to-nearest-even step; every float32 is exact in float64), and on
    hand-made ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 and goes to
    the even significand 1; 1 + 3*2^-8 goes to 1 + 2^-6; a subnormal tie
    3*2^-134 goes to 2^-132."""
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.randn(20000, generator=g) * 10.0 ** torch.randint(-30, 30, (20000,), generator=g),
                   torch.randn(2000, generator=g) * 2.0 ** -130])
    want = x.to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.bf16_round(x.to(torch.float64).numpy()), want)
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 3 * 2.0 ** -134, 0.0, -0.0])
    np.testing.assert_array_equal(oracle.bf16_round(ties),
                                  [1.0, 1 + 2.0 ** -6, -1.0, 2.0 ** -132, 0.0, 0.0])
    # just off the tie: the nearer neighbour
    assert oracle.bf16_round(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1 + 2.0 ** -7


def test_nsa_compress_stored_cache():
    """The stored cache is the exact block mean rounded to the nearest bf16
    ([Ch11] §12.6 mean compression, kept in the token cache's bf16): exact on
    blocks of small integers (their means are multiples of 1/64, exact in
    fp32, so torch's conversion rounds them once); on N(0,1) bf16 data each
    entry is the bf16 value nearest to the exact rational mean (computed with
    fractions), ties to even."""
    from fractions import Fraction
    g = torch.Generator().manual_seed(21)
    Xi = torch.randint(-8, 9, (4 * 64 + 17, 32), generator=g).to(torch.float64)
    want = Xi[:256].reshape(4, 64, 32).mean(dim=1).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.nsa_compress(Xi.numpy(), 64), want)
    X = torch.randn(64 * 6, 16, generator=g).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.nsa_compress(X, 64)
    assert got.shape == (6, 16)
    for n in range(6):
        for d in range(16):
            exact = sum(Fraction(v) for v in X[n * 64:(n + 1) * 64, d]) / 64
            v = Fraction(got[n, d])
            # the bf16 step in the exact mean's binade (no subnormals here)
            step = Fraction(2) ** (math.floor(math.log2(abs(float(exact)))) - 7)
            assert (v / step).denominator == 1  # v is on that grid (or the binade edge)
            err = abs(exact - v)
            assert err <= step / 2
            if err == step / 2:  # a tie: the even significand
                assert (v / step).numerator % 2 == 0
    assert oracle.nsa_compress(X[:63], 64).shape == (0, 16)


# ------------------------------------------------------------ CSA compression

def _csa_streams(seed, n, c, m):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, c)), rng.standard_normal((n, c)), rng.standard_normal((n, c)),
            rng.standard_normal((n, c)), rng.standard_normal((m, c)), rng.standard_normal((m, c)))


def test_csa_uniform_weights_give_the_mean_of_both_groups():
    """[LLMRes] CSA: equal weights -> entry i is the mean of the 2m rows (group
    i of stream a, group i-1 of stream b); entry 0 has stream a only."""
    m, c = 4, 6
    Ca, Cb, _, _, _, _ = _csa_streams(1, 4 * m + 3, c, m)
    Z, B = np.zeros_like(Ca), np.zeros((m, c))
    out = oracle.csa_compress(Ca, Cb, Z, Z, B, B, m)
    assert out.shape == (4, c)                               # the ragged tail forms no entry
    np.testing.assert_allclose(out[0], Ca[:m].mean(axis=0), atol=1e-14)
    for i in range(1, 4):
        want = np.concatenate([Ca[m * i: m * (i + 1)], Cb[m * (i - 1): m * i]]).mean(axis=0)
        np.testing.assert_allclose(out[i], want, atol=1e-14)


def test_csa_weights_follow_the_logits_and_the_biases():
    """Weight logits log(1..2m) (through Z or through the position biases)
    give weights proportional to 1..2m: a closed form per channel."""
    m, c = 4, 3
    Ca, Cb, _, _, _, _ = _csa_streams(2, 3 * m, c, m)
    lw = np.log(np.arange(1, 2 * m + 1, dtype=np.float64))
    wts = np.arange(1, 2 * m + 1) / np.arange(1, 2 * m + 1).sum()
    Za = np.tile(lw[:m, None], (3, c))
    Zb = np.tile(lw[m:, None], (3, c))
    zero = np.zeros((m, c))
    via_z = oracle.csa_compress(Ca, Cb, Za, Zb, zero, zero, m)
    via_b = oracle.csa_compress(Ca, Cb, np.zeros_like(Ca), np.zeros_like(Cb), np.tile(lw[:m, None], (1, c)),
                                np.tile(lw[m:, None], (1, c)), m)
    for i in (1, 2):
        want = wts[:m] @ Ca[m * i: m * (i + 1)] + wts[m:] @ Cb[m * (i - 1): m * i]
        np.testing.assert_allclose(via_z[i], want, atol=1e-13)
        np.testing.assert_allclose(via_b[i], want, atol=1e-13)
    w0 = np.arange(1, m + 1) / np.arange(1, m + 1).sum()     # entry 0: the softmax over stream a alone
    np.testing.assert_allclose(via_z[0], w0 @ Ca[:m], atol=1e-13)


def test_csa_softmax_is_per_channel_along_the_sequence():
    """Channel 0 puts all weight on row 0 of stream a, channel 1 on row 1 of
    stream b: a softmax over channels, or over both axes, fails this."""
    m, c = 4, 2
    Ca, Cb, _, _, _, _ = _csa_streams(3, 2 * m, c, m)
    Za, Zb = np.zeros_like(Ca), np.zeros_like(Cb)
    Za[m + 0, 0] = 60.0
    Zb[1, 1] = 60.0
    zero = np.zeros((m, c))
    out = oracle.csa_compress(Ca, Cb, Za, Zb, zero, zero, m)
    assert abs(out[1, 0] - Ca[m, 0]) < 1e-20 + 1e-12 * abs(Ca[m, 0])
    assert abs(out[1, 1] - Cb[1, 1]) < 1e-20 + 1e-12 * abs(Cb[1, 1])


def test_csa_entries_see_only_their_own_groups():
    """Entry i reads stream a's group i and stream b's group i-1 only: moving
    any later row (or stream b's group i) leaves entries 0..i unchanged."""
    m, c = 4, 5
    Ca, Cb, Za, Zb, Ba, Bb = _csa_streams(4, 6 * m, c, m)
    ref = oracle.csa_compress(Ca, Cb, Za, Zb, Ba, Bb, m)
    Ca2, Cb2, Za2, Zb2 = Ca.copy(), Cb.copy(), Za.copy(), Zb.copy()
    Ca2[3 * m:] += 7.0
    Za2[3 * m:] -= 3.0
    Cb2[2 * m:] += 5.0
    Zb2[2 * m:] += 2.0
    got = oracle.csa_compress(Ca2, Cb2, Za2, Zb2, Ba, Bb, m)
    np.testing.assert_array_equal(got[:3], ref[:3])
    assert np.abs(got[3:] - ref[3:]).min() > 0


def test_csa_attention_reduces_to_plain_attention():
    """Keys = values = the entries: only compressed entries (no window), or
    only the window, is attention over those rows; both is one softmax over
    their union."""
    rng = np.random.default_rng(5)
    H, c, nc, L = 3, 8, 20, 50
    q, Cc, Cr = rng.standard_normal((H, c)), rng.standard_normal((nc, c)), rng.standard_normal((L, c))
    chosen = np.array([1, 4, 7, 19, -1])
    got = oracle.csa_attend(q, Cc, Cr, chosen, 0, 0.3)
    E = Cc[[1, 4, 7, 19]]
    np.testing.assert_allclose(got, _sdpa(q, E, E, 0.3), atol=1e-12)
    got = oracle.csa_attend(q, Cc, Cr, np.array([-1, -1]), 6, 0.3)
    np.testing.assert_allclose(got, _sdpa(q, Cr[-6:], Cr[-6:], 0.3), atol=1e-12)
    got = oracle.csa_attend(q, Cc, Cr, chosen, 6, 0.3)
    E = np.concatenate([Cc[[1, 4, 7, 19]], Cr[-6:]])
    np.testing.assert_allclose(got, _sdpa(q, E, E, 0.3), atol=1e-12)


def test_csa_workload_indexer_keys_compress_to_their_integers():
    """The CSA workload's indexer-key streams repeat one integer vector over
    the 2m rows each entry merges, so compression (weights summing to one)
    returns exactly that vector and its e4m3 copy is exact."""
    import workloads
    cfg = workloads.CSAConfig(name="t", seed=0, n_seqs=2, L=203, H=4, topk=8, window=8)
    inp = workloads.csa_inputs(cfg, seed=3)
    res = oracle.csa_step(inp, [0, 1])
    for r in range(2):
        want = inp["CIa"][r, :: cfg.m].double().numpy()[: cfg.n_c]
        np.testing.assert_array_equal(res["ki_comp"][r], want)
        assert np.abs(want).max() <= 8 and (want == np.round(want)).all()
    assert res["idx"].shape == (2, 8) and (np.diff(res["idx"], axis=1) > 0).all()


# ------------------------------------------------------------ whole step

def test_dsa_step_placement_invariance():
    """Notes §11: moving KV between storage places (here: a different page
    permutation) leaves the whole step's output unchanged."""
    import workloads
    cfg = workloads.small_dsa(workloads.RAGGED, n_seqs=3, rows=3, lens=(200, 64, 130), H_I=4, d_I=16,
                              topk=40, H=4, d_c=16, d_R=4)
    a = workloads.dsa_inputs(cfg, seed=5)
    b = dict(a)
    table, _ = workloads.page_layout(cfg, 99)
    # move every page's rows to its new place in all three caches
    old = a["page_table"].numpy()
    perm_rows = np.zeros(a["c_cache"].shape[0], dtype=np.int64)
    for s in range(cfg.n_seqs):
        for p in range(cfg.pages_per_seq):
            if old[s, p] >= 0:
                perm_rows[table[s, p] * 64: table[s, p] * 64 + 64] = np.arange(old[s, p] * 64, old[s, p] * 64 + 64)
    idx = torch.from_numpy(perm_rows)
    for key in ("k_idx_cache", "c_cache", "kr_cache"):
        b[key] = a[key][idx]
    b["page_table"] = torch.from_numpy(table)
    ra, rb = oracle.dsa_step(a, range(3)), oracle.dsa_step(b, range(3))
    assert np.array_equal(ra["idx"], rb["idx"])
    np.testing.assert_array_equal(ra["out"], rb["out"])
    np.testing.assert_array_equal(np.nan_to_num(ra["scores"]), np.nan_to_num(rb["scores"]))

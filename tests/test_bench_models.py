"""The algorithmic byte and flop models behind bench.py's roofline figures,
checked against the same quantities written out by hand for each workload
(no GPU: these are host arithmetic only)."""
import bench
import workloads as W


def test_long_decode_step_bytes():
    """32 queries x 32768 e4m3 keys of 128 bytes, then 2048 selected rows of
    512 + 64 bf16 per query: 209,715,200 bytes per step."""
    keys, rows = bench.decode_bytes(W.LONG)
    assert keys == 32 * 32768 * 128 == 134_217_728
    assert rows == 32 * 2048 * (512 + 64) * 2 == 75_497_472
    assert keys + rows == 209_715_200


def test_prefill_flops():
    """Query i of the 4096-query chunk sees 61441 + i keys: the indexer does
    2 * 64 heads * 128 dims flops per visible key, the attention
    2 * 128 heads * (512 + 64 + 512) per selected row (score and aggregate)."""
    idx, mla = bench.prefill_flops(W.PREFILL)
    visible = 4096 * 61441 + 4095 * 4096 // 2
    assert idx == 2 * 64 * 128 * visible == 4_260_641_112_064
    assert mla == 4096 * 2048 * 2 * 128 * 1088 == 2_336_462_209_024


def test_block_sparse_bytes():
    """fp32 pooled keys of 2048 blocks for 8 x 32 (sequence, head) pairs, plus
    K and V (128 bf16 each) of every attended token, plus a bf16 query and an
    fp32 output per pair."""
    nbytes, u = bench.block_bytes(W.BLOCK, 256 * 1300)
    assert u == 256 * 1300
    assert nbytes == 8 * 32 * 2048 * 128 * 4 + 256 * 1300 * 512 + 256 * (256 + 512)


def test_block_union_tokens_by_hand():
    """L = 1000, block 64, sink 1 block, window 100 (tokens 900..999): chosen
    blocks 0 (the sink itself), 3 (192..255) and 14 (896..959, overlapping the
    window by 60 tokens) add 64 + 4 tokens to the 164 of sink and window; a
    second head with no chosen block has only sink and window."""
    cfg = W.BlockConfig(name="t", seed=0, B=1, L=1000, H=2, top_blocks=3, sink_blocks=1, window=100)
    import numpy as np
    sel = np.array([[[0, 3, 14], [-1, -1, -1]]])
    assert bench.block_union_tokens(cfg, sel) == (164 + 64 + 4) + 164


def test_nsa_decode_bytes():
    """Per (sequence, KV head): compressed K and V of 2048 blocks, K and V of
    16 selected 64-token blocks and of the 512-token window (128 bf16 each),
    and for each of the group's 8 heads its bf16 query, three fp32 gates and
    fp32 output: 1,841,248 bytes, 32 of them per step."""
    per_group = (2 * 2048 * 128 * 2 + 16 * 64 * 2 * 128 * 2 + 512 * 2 * 128 * 2
                 + 8 * (128 * 2 + 3 * 4 + 128 * 4))
    assert per_group == 1_841_248
    assert bench.nsa_bytes(W.NSA) == 8 * 4 * per_group == 58_919_936


def test_csa_decode_bytes():
    """32 queries over 32768 compressed e4m3 keys (131072 raw tokens, 4:1),
    then 2048 selected entries plus a 128-token raw window, each a 512-wide
    bf16 row plus the 64 dims read as its RoPE key."""
    keys, rows = bench.csa_bytes(W.CSA)
    assert keys == 32 * (131072 // 4) * 128 == 134_217_728
    assert rows == 32 * (2048 + 128) * (512 + 64) * 2 == 80_216_064


def test_step_working_set_and_e2e_flush_rule():
    """Distinct bytes a step reads, which decides whether the end-to-end loop
    flushes L2 between steps (working set under the 126 MB L2: flush)."""
    import bench
    long_b = bench.step_working_set(W.LONG, None)
    assert long_b == 32 * (32768 * 128 + 2048 * 1152) == 209715200
    assert long_b > bench.L2_BYTES  # streams through L2: no flush
    ragged_b = bench.step_working_set(W.RAGGED, None)
    assert ragged_b == sum(bench.decode_bytes(W.RAGGED)) and ragged_b > bench.L2_BYTES
    prefill_b = bench.step_working_set(W.PREFILL, None)
    assert prefill_b == 65536 * (128 + 1152) < bench.L2_BYTES  # the history once, however many rows read it
    assert bench.step_working_set(W.NSA, None) == bench.nsa_bytes(W.NSA) < bench.L2_BYTES


def test_e2e_input_packing():
    """The end-to-end loop's packed input buffer: every piece starts on a
    16-byte boundary, pieces do not overlap, and each tensor's bytes come back
    unchanged from its slice (fp32, e4m3 and bf16 pieces of odd sizes)."""
    import torch
    import bench
    g = torch.Generator().manual_seed(5)
    ts = [torch.randn(3, 5, generator=g),
          torch.randint(-8, 9, (7,), generator=g).to(torch.float32).to(torch.float8_e4m3fn),
          torch.randn(2, 3, generator=g).to(torch.bfloat16),
          torch.randn(33, generator=g)]
    offs, total = bench.pack_layout(ts)
    assert all(o % 16 == 0 for o, _ in offs)
    ends = [o + nb for o, nb in offs]
    assert all(ends[i] <= offs[i + 1][0] for i in range(len(ts) - 1)) and ends[-1] <= total
    buf = bench.pack_host(ts, offs, total)
    for t, (o, nb) in zip(ts, offs):
        back = torch.empty_like(t)
        back.view(-1).view(torch.uint8).copy_(buf[o:o + nb])
        assert torch.equal(back.view(-1).view(torch.uint8), t.view(-1).view(torch.uint8))

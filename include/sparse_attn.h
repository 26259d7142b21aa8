/*
 * sparse_attn.h — C ABI of the B200 (sm_100a) sparse-attention library
 * (libsparse_attn.so).
 *
 * The library computes DeepSeek-Sparse-Attention-style decode and prefill in
 * three stream-ordered calls, plus a block-sparse (MoBA/NSA-style) decode:
 *
 *   sa_index_scores      lightning indexer  I_{t,s} = sum_j w_{t,j} ReLU(q^I_{t,j} . k^I_s)
 *   sa_topk_select       exact Top-K of I_{t,:} (ties to the lower position)
 *   sa_index_scores_hist / sa_topk_select_hist
 *                        the same two steps, the indexer also counting each row's
 *                        first-digit histogram for the Top-K
 *   sa_index_candidates / sa_topk_from_candidates
 *                        the same two steps for decode, the indexer keeping only
 *                        the keys that can still be in the Top-K
 *   sa_sparse_mla_decode / sa_sparse_mla_prefill (_bf16: bf16 output)
 *                        softmax over the selected set of the absorbed content score
 *                        plus the RoPE score, scaled; output sum_j a_j c_j in latent space
 *   sa_block_mean_pool   mean-pooled block keys (run when blocks complete)
 *   sa_block_sparse_attn top blocks by q . mean(K_block), plus sink and window; softmax
 *                        over the union of their tokens
 *   sa_nsa_compress      NSA compressed cache: bf16 block means of K and V
 *   sa_nsa_decode        NSA three branches (compression, group-shared block
 *                        selection, window), each its own softmax, gated sum
 *   sa_csa_compress      CSA: m-token entries merged by a per-channel softmax
 *   sa_csa_window_index  CSA: selected compressed entries plus the raw window,
 *                        as the index list of sa_sparse_mla_decode
 *
 * Sources, cited by page title and section:
 *   [Notes]  "Sparse Attention 数学学习笔记" (echobase-5bl.pages.dev, 2026.09.14)
 *   [MLA-S]  "MLA 与稀疏注意力：少存一点，还是少看一点？" (tianyi-zhang-02.github.io)
 *   [Ch11]   "第 11 章 稀疏注意力" (book.shippingwang.com)
 *   [LLMRes] "LLM注意力优化：稀疏注意力" (wln20.github.io)
 *
 * Conventions shared by every call:
 *  - Every pointer is device memory owned by the caller unless stated.  The
 *    library allocates nothing and keeps no state between calls other than
 *    one device error word per GPU (see sa_check_device_error) and a cache of
 *    driver entry points.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronise the host.
 *  - Arguments are checked on the host before anything is launched: a bad
 *    count, a null required pointer, or a pointer that breaks the alignment a
 *    call states returns SA_EINVAL; shapes the kernels do not handle return
 *    SA_EUNSUPPORTED.  In both cases nothing is launched.  A failed launch
 *    returns SA_ECUDA.
 *  - Contents the caller promises (finite scores, page ids inside the pool,
 *    positions below the sequence length) are preconditions: they are not
 *    checked on the device, except where a call says so.
 *  - Paging: a cache is a pool of 64-token pages, row = page * 64 + (pos % 64).
 *    `page_table` [n_seqs][pages_per_seq] int32 gives the physical page of each
 *    (sequence, pos / 64); NULL means contiguous: page = seq * pages_per_seq +
 *    pos / 64.  Placement never changes a result ([Notes] §11).
 *  - `seq_of_row` [rows] int32 maps a query row to its sequence; NULL means
 *    row r is sequence r (decode: one query per sequence).
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sa_stream_t; /* same type as cudaStream_t */

typedef enum {
    SA_OK = 0,
    SA_EINVAL = 1,        /* bad argument; nothing launched */
    SA_EUNSUPPORTED = 2,  /* valid for the method, not handled by the kernels; nothing launched */
    SA_ECUDA = 3,         /* a CUDA runtime call or launch failed */
    SA_ETIMEOUT = 4       /* reported by sa_check_device_error: a kernel's bounded wait ran out */
} sa_status;

typedef enum {
    SA_F32 = 0,   /* IEEE binary32 */
    SA_E4M3 = 1,  /* fp8 e4m3 (OCP "e4m3fn", no infinities) */
    SA_BF16 = 2   /* bfloat16 */
} sa_dtype;

/* Short name of a status code (static string). */
const char* sa_status_string(sa_status s);

/* Library version, major*10000 + minor*100 + patch. */
int sa_version(void);

/*
 * Waits for `stream`, then reads and clears this GPU's device error word.
 * Kernels that wait on barriers give every wait a time limit; when one runs
 * out the kernel records a nonzero site code here, abandons its work
 * (outputs of that launch are then undefined) and returns.  The sparse-MLA
 * kernels also record code 0x700 when a selected position lies past the
 * page table or maps to a page outside the pool (row 0 of the pool is read
 * instead).  *code_out gets the code (0 = none; the first code recorded
 * wins).  Returns SA_ETIMEOUT if a code was set, SA_ECUDA if the stream
 * reported an error, else SA_OK.  This call and sa_set_wait_limit_ns are
 * the only calls that synchronise.
 */
sa_status sa_check_device_error(int* code_out, sa_stream_t stream);

/*
 * Sets, for the current GPU, the time limit of the kernels' waits on other
 * parties (a ring slot filled by another warp, a partner CTA's signal), in
 * nanoseconds; 0 restores the default of one second.  Waits of a CTA for its
 * own copies and tensor-core work in flight before it exits always keep the
 * one-second limit, so a kernel whose wait ran out still drains its own work
 * and frees its tensor memory before it returns.  A short limit makes a
 * kernel give up (and record its site code) instead of waiting: a way to
 * exercise the failure path.  The setting applies to launches made after
 * this call returns (it writes device memory synchronously).
 */
sa_status sa_set_wait_limit_ns(unsigned long long limit_ns);

/*
 * Lightning indexer ([Notes] §9, index score I_{t,s}; [MLA-S] "DSA：先用便宜的
 * indexer 选位置"):
 *     scores[r][s] = sum_{j<H_I} w[r][j] * max(0, sum_{d<d_I} q[r][j][d] * k(seq(r), s)[d])
 * for 0 <= s < n_visible[r].  No scale, no softmax.  Entries s >= n_visible[r]
 * are left untouched.  One key per token, shared by all indexer heads.
 *
 *   q         [rows][H_I][d_I]   dtype
 *   w         [rows][H_I]        fp32
 *   k_cache   [pool_pages*64][d_I] dtype (pages as above); a page id outside
 *             [0, pool_pages) reads as zeros and never faults
 *   n_visible [rows]             int32, 0 <= n_visible[r] <= pages_per_seq*64
 *   scores    [rows][scores_ld]  fp32, scores_ld >= max n_visible
 * Products and sums are accumulated in fp32; on integer inputs with
 * power-of-two weights (every partial sum below 2^24 units) the result is
 * exact.  dtype SA_E4M3 with d_I = 128 runs on the tensor cores (tcgen05,
 * kind::f8f6f4); other shapes (d_I <= 128, H_I <= 64, fp32 or e4m3) run on
 * the CUDA cores.  Rows sharing a sequence are batched against one key tile
 * when they are consecutive.  Alignment: k_cache and q 16-byte aligned.
 */
sa_status sa_index_scores(const void* q, const float* w, const void* k_cache, int64_t pool_pages,
                          sa_dtype dtype, const int32_t* page_table, int pages_per_seq,
                          const int32_t* seq_of_row, const int32_t* n_visible,
                          int rows, int H_I, int d_I, int64_t scores_ld, float* scores,
                          sa_stream_t stream);

/*
 * sa_index_scores, and with it the first step of the Top-K selection: every
 * score written also counts in hist[r][key >> 20], where key is the score's
 * order-preserving 32-bit pattern (sign, exponent and three mantissa bits
 * select one of 4096 bins; -0.0 counts as +0.0).  hist [rows][4096] int32
 * must hold zeros on entry (sa_topk_select_hist leaves it zeroed again, so
 * one buffer serves every step).  The scores are those of sa_index_scores.
 */
sa_status sa_index_scores_hist(const void* q, const float* w, const void* k_cache, int64_t pool_pages,
                               sa_dtype dtype, const int32_t* page_table, int pages_per_seq,
                               const int32_t* seq_of_row, const int32_t* n_visible, int rows, int H_I, int d_I,
                               int64_t scores_ld, float* scores, int32_t* hist, sa_stream_t stream);

/*
 * Exact Top-K ([Notes] §9, S_t = {s | I_{t,s} in TopK(I_{t,:}, k)}; [MLA-S]
 * "一次错选会丢掉什么？" orders by (-score, position)):
 * idx_out[r] receives the min(k, n_valid[r]) positions with the largest
 * scores[r][0 .. n_valid[r]-1], equal scores going to the lower position,
 * written in ascending position order, then -1 up to k.  -0.0 equals +0.0.
 * Scores must be finite (precondition).
 *   scores  [rows][scores_ld] fp32;  n_valid [rows] int32 (<= scores_ld)
 *   idx_out [rows][k] int32
 * Limits: 1 <= k; scores_ld <= 262144.
 */
sa_status sa_topk_select(const float* scores, int64_t scores_ld, const int32_t* n_valid,
                         int rows, int k, int32_t* idx_out, sa_stream_t stream);

/*
 * Sparse MLA attention over the selected latent rows ([MLA-S] "分开以后，完整分数
 * 怎么算？" and "“吸收矩阵”是交换线性计算的顺序"; [Notes] §2, §8):
 *   z_j = (q_lat[r][h] . c_j + q_rope[r][h] . kr_j) * scale,   j in S_r
 *   out[r][h] = sum_j softmax_{S_r}(z)_j * c_j         (latent aggregate; U_V is outside)
 *   lse[r][h] = log sum_{j in S_r} exp(z_j)            (natural log; -inf if S_r is empty)
 * S_r = the positions idx[r][0..k-1] that are >= 0, resolved to cache rows
 * through seq(r) and the page table.  The latent row c_j is both the content
 * key and the value; one selection is shared by all heads.
 *
 *   q_lat  [rows][H][d_c] bf16 (absorbed U_K^T q^C);  q_rope [rows][H][d_R] bf16 (rotated)
 *   c_cache  rows of d_c bf16 at stride c_ld elements;  kr_cache rows of d_R bf16 at stride kr_ld;
 *            both pools hold pool_pages*64 rows (a page id outside the pool reads row 0)
 *   idx    [rows][k] int32 positions or -1
 *   out    [rows][H][d_c] fp32;  lse [rows][H] fp32 or NULL
 * Supported: d_c = 512, d_R = 64, 1 <= H <= 128; bf16 inputs, fp32 softmax
 * and accumulation on the tensor cores.  Alignment: every base pointer and
 * row stride a multiple of 16 bytes.
 * Both calls need a caller workspace (256-byte aligned, contents need no
 * initialisation and are scratch after the call): the two CTAs that share a
 * row exchange their partial scores through it (an L2-resident area of
 * sa_sparse_mla_prefill_workspace_size bytes, one slot per SM), and _decode,
 * which splits each row's k positions over several CTA pairs when rows are
 * few, also keeps the partial softmax states there
 * (sa_sparse_mla_workspace_size bytes in all).  A smaller or missing
 * workspace returns SA_EINVAL.  _prefill keeps one row per CTA pair and
 * supports k <= 4096; _decode splits larger k.  Concurrent calls (different
 * streams) need separate workspaces.
 */
size_t sa_sparse_mla_workspace_size(int rows, int H, int k, int d_c);
size_t sa_sparse_mla_prefill_workspace_size(int rows, int H, int k, int d_c);

sa_status sa_sparse_mla_decode(const void* q_lat, const void* q_rope,
                               const void* c_cache, int64_t c_ld, const void* kr_cache, int64_t kr_ld,
                               int64_t pool_pages, const int32_t* page_table, int pages_per_seq,
                               const int32_t* seq_of_row,
                               const int32_t* idx, int rows, int H, int k, int d_c, int d_R, float scale,
                               float* out, float* lse, void* workspace, size_t workspace_bytes,
                               sa_stream_t stream);

sa_status sa_sparse_mla_prefill(const void* q_lat, const void* q_rope,
                                const void* c_cache, int64_t c_ld, const void* kr_cache, int64_t kr_ld,
                                int64_t pool_pages, const int32_t* page_table, int pages_per_seq,
                                const int32_t* seq_of_row,
                                const int32_t* idx, int rows, int H, int k, int d_c, int d_R, float scale,
                                float* out, float* lse, void* workspace, size_t workspace_bytes,
                                sa_stream_t stream);

/*
 * sa_sparse_mla_decode / sa_sparse_mla_prefill with the output stored as bf16:
 * out [rows][H][d_c] bf16, each element the fp32 result of those calls
 * rounded to the nearest bf16 (ties to even) — bit for bit the fp32 call's
 * output so rounded.  Softmax and accumulation stay fp32; lse is fp32 as
 * there.  Half the output bytes (the up-projection reads o_lat as bf16).
 */
sa_status sa_sparse_mla_decode_bf16(const void* q_lat, const void* q_rope,
                                    const void* c_cache, int64_t c_ld, const void* kr_cache, int64_t kr_ld,
                                    int64_t pool_pages, const int32_t* page_table, int pages_per_seq,
                                    const int32_t* seq_of_row,
                                    const int32_t* idx, int rows, int H, int k, int d_c, int d_R, float scale,
                                    void* out, float* lse, void* workspace, size_t workspace_bytes,
                                    sa_stream_t stream);

sa_status sa_sparse_mla_prefill_bf16(const void* q_lat, const void* q_rope,
                                     const void* c_cache, int64_t c_ld, const void* kr_cache, int64_t kr_ld,
                                     int64_t pool_pages, const int32_t* page_table, int pages_per_seq,
                                     const int32_t* seq_of_row,
                                     const int32_t* idx, int rows, int H, int k, int d_c, int d_R, float scale,
                                     void* out, float* lse, void* workspace, size_t workspace_bytes,
                                     sa_stream_t stream);

/*
 * Dense MLA decode: the same attention as sa_sparse_mla_decode over every
 * visible position instead of a selection (row r attends to positions
 * 0 .. n_visible[r]-1 of its sequence).  It is the short-sequence mode of the
 * dual-mode system of [LLMRes] "DeepSeek Sparse Attention (DSA)": below a few
 * thousand tokens the indexer and Top-K cost more than attending to every
 * position, so the caller runs this call without either of them.
 *   n_visible [rows] int32, each <= L_max and inside the page table;
 *   workspace: sa_dense_mla_workspace_size(rows, H, L_max, d_c) bytes.
 * Other arguments, layouts, limits and errors as sa_sparse_mla_decode.
 */
size_t sa_dense_mla_workspace_size(int rows, int H, int L_max, int d_c);

sa_status sa_dense_mla_decode(const void* q_lat, const void* q_rope,
                              const void* c_cache, int64_t c_ld, const void* kr_cache, int64_t kr_ld,
                              int64_t pool_pages, const int32_t* page_table, int pages_per_seq,
                              const int32_t* seq_of_row, const int32_t* n_visible, int rows, int H, int L_max,
                              int d_c, int d_R, float scale, float* out, float* lse, void* workspace,
                              size_t workspace_bytes, sa_stream_t stream);

/*
 * The per-head projections around sparse MLA ([MLA-S] "“吸收矩阵”是交换线性计算的
 * 顺序": q^C . (U_K c_j) = (U_K^T q^C) . c_j, so the query is absorbed once and
 * the output stays in latent space until one up-projection):
 *   q_lat[r][h][j] = sum_i U_K[h][i][j] * q_c[r][h][i]    (the absorbed query)
 *   out[r][h][v]   = sum_j U_V[h][v][j] * o_lat[r][h][j]  (value-space output)
 *   q_c [rows][H][d_C] bf16, U_K [H][d_C][d_c] bf16 (k^C = U_K c), q_lat [rows][H][d_c] bf16 out;
 *   o_lat [rows][H][d_c] fp32 (the sparse-MLA output), U_V [H][d_v][d_c] bf16, out [rows][H][d_v] fp32.
 * bf16 operands (o_lat is rounded to bf16), fp32 accumulation on the tensor
 * cores.  Supported: absorption d_C a multiple of 64 up to 512 and d_c a
 * multiple of 128 up to 512; up-projection d_c a multiple of 64 up to 512 and
 * d_v a multiple of 128.  Alignment: q_c, U_K, o_lat, U_V 16 bytes.
 */
sa_status sa_mla_absorb_query(const void* q_c, const void* U_K, int rows, int H, int d_C, int d_c, void* q_lat,
                              sa_stream_t stream);

sa_status sa_mla_up_project(const float* o_lat, const void* U_V, int rows, int H, int d_c, int d_v, float* out,
                            sa_stream_t stream);

/*
 * sa_mla_up_project with o_lat [rows][H][d_c] bf16 (the output of the _bf16
 * sparse-MLA calls): the same product, bit for bit the fp32 call's result on
 * the fp32 o_lat that rounds to it (that call rounds o_lat to bf16 first).
 */
sa_status sa_mla_up_project_bf16(const void* o_lat, const void* U_V, int rows, int H, int d_c, int d_v, float* out,
                                 sa_stream_t stream);

/*
 * Sparse MLA decode for callers that cannot allocate device memory.  The
 * pages have no counterpart of this call: it is a deployment convenience.
 *
 * Some callers have no allocator to hand the library a workspace: code that
 * runs where cudaMalloc is not allowed or not wanted (inside a host callback
 * or a custom memory manager that owns every byte of the GPU, plugins of a
 * framework that only passes tensors in and out).  This call computes exactly
 * what sa_sparse_mla_decode computes, with the same arguments minus the
 * workspace, and keeps its scratch (the partial-score exchange area and the
 * split-key partial states) in a static device array of
 * SA_STATIC_SCRATCH_BYTES that the library owns.  It calls no cudaMalloc,
 * cudaFree or allocating library routine.
 *
 *  - Every GPU that loads the library holds that array until the process exits.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture begins.
 *  - Shapes whose partial states need more than SA_STATIC_SCRATCH_BYTES
 *    (sa_sparse_mla_workspace_size(rows, H, k, d_c) > SA_STATIC_SCRATCH_BYTES)
 *    return SA_EUNSUPPORTED and launch nothing (no allocation and no launch
 *    happens before this check; the size depends on the device's SM count,
 *    which sets the key splits); use sa_sparse_mla_decode with a caller
 *    workspace for those.  The array holds the exchange area of every SM
 *    slot and the split-key states of up to 80 (row, split) pairs of 128
 *    heads, i.e. every call with k <= 4096 on a GPU of up to 160 SMs (the
 *    library's limit; the B200 has 148).
 *  - All calls share the one array.  Calls that may overlap on the GPU (on
 *    different streams, or on different host threads without ordering)
 *    race on it and give undefined outputs; order them on one stream.  Every
 *    byte a call reads from the array was written earlier in the same call,
 *    so nothing left by a previous call leaks into a result.
 */
#define SA_STATIC_SCRATCH_BYTES (((size_t)40 << 20) + ((size_t)256 << 10))

sa_status sa_sparse_mla_decode_static(const void* q_lat, const void* q_rope,
                                      const void* c_cache, int64_t c_ld, const void* kr_cache, int64_t kr_ld,
                                      int64_t pool_pages, const int32_t* page_table, int pages_per_seq,
                                      const int32_t* seq_of_row,
                                      const int32_t* idx, int rows, int H, int k, int d_c, int d_R, float scale,
                                      float* out, float* lse, sa_stream_t stream);

/*
 * Mean-pooled block keys ([Ch11] §12.6, k_rep = k_blocks.mean(1)):
 *   pooled[b][h][n][d] = (1/block) * sum_{i<block} K[b][n*block+i][h][d]
 * for every complete block n < L / block.
 *   K  bf16, element (b,t,h,d) at b*stride_b + t*stride_t + h*stride_h + d (elements)
 *   pooled [B][H][pooled_ld][D] fp32, pooled_ld >= L / block
 * Supported: D = 128.
 */
sa_status sa_block_mean_pool(const void* K, int64_t stride_b, int64_t stride_t, int64_t stride_h,
                             int B, int L, int H, int D, int block, float* pooled, int64_t pooled_ld,
                             sa_stream_t stream);

/*
 * Block-sparse decode for the query at position L-1 of each (sequence, head)
 * ([Ch11] §12.5-12.6; [LLMRes] MoBA; [Notes] §4 window; [MLA-S] causality of
 * pooling):
 *   score_n = scale * q[b][h] . pooled[b][h][n]  over complete blocks n < L/block
 *   chosen  = the top_blocks blocks by (-score_n, n)
 *   U       = tokens of chosen blocks  u  [0, sink_blocks*block)  u  [L-window, L)
 *   out[b][h] = sum_{t in U} softmax_U(scale * q . K_t) V_t
 *   q [B][H][D] bf16; K, V as in sa_block_mean_pool; out [B][H][D] fp32;
 *   sel_blocks [B][H][top_blocks] int32 (ascending, -1 padded) or NULL.
 * Supported: D = 128, block = 64, 1 <= top_blocks <= 64, L/block <= 4096.
 * K and V need 8-byte alignment and strides that are multiples of 4
 * elements; with 16-byte alignment and strides that are multiples of 8
 * elements the chosen K/V blocks are loaded as tensor-map tiles (faster),
 * otherwise with per-thread loads (same results).  Waits record codes
 * 0x801-0x804 in the device error word when they run out.
 */
sa_status sa_block_sparse_attn(const void* q, const float* pooled, int64_t pooled_ld,
                               const void* K, const void* V, int64_t stride_b, int64_t stride_t,
                               int64_t stride_h, int B, int H, int D, int L, int block,
                               int top_blocks, int sink_blocks, int window, float scale,
                               float* out, int32_t* sel_blocks, sa_stream_t stream);

/*
 * NSA compressed cache ([Ch11] §12.6 mean compression; [MLA-S] NSA: only
 * complete blocks are summarised):
 *   Kc[b][h][n][d] = bf16( (sum_{i<block} K[b][n*block+i][h][d]) / block )
 * with the sum taken in fp64 (exact for bf16 blocks of moderate dynamic
 * range) and the mean rounded once to the nearest bf16, ties to even;
 * Vc likewise from V; for every complete block n < L / block.  Run when a
 * block completes (the decode reads the cache).
 *   K, V bf16, element (b,t,h,d) at b*stride_b + t*stride_t + h*stride_h + d
 *   Kc, Vc [B][H_kv][c_ld][D] bf16, c_ld >= L / block
 * Supported: D = 128.
 */
sa_status sa_nsa_compress(const void* K, const void* V, int64_t stride_b, int64_t stride_t, int64_t stride_h,
                          int B, int L, int H_kv, int D, int block, void* Kc, void* Vc, int64_t c_ld,
                          sa_stream_t stream);

/*
 * NSA three-branch decode for the query at position L-1 of every head
 * ([MLA-S] NSA sections "三条路径，各留住什么？" and "选块和合并输出，实际算一遍";
 * [LLMRes] NSA steps 1-3).  Query head h uses KV head h / G, G = H / H_kv.
 * For each (sequence b, KV head g) and its G query heads, three branches,
 * each with its own softmax over scale * q . k:
 *   compression: the n_b = L / block complete blocks, keys Kc, values Vc;
 *   selection:   the min(top_blocks, n_b) blocks with the largest sum over the
 *                group's heads of the compression probabilities (ties to the
 *                lower block), all their tokens;
 *   window:      positions [max(0, L - window), L);
 *   out[b][h] = gates[b][h][0] o_cmp + gates[b][h][1] o_sel + gates[b][h][2] o_win
 * A branch with no position contributes zero.  The gates are used as given
 * (values of a sigmoid; not normalised).
 *   q [B][H][D] bf16; K, V as in sa_nsa_compress (16-byte aligned rows);
 *   Kc, Vc from sa_nsa_compress (may be NULL when L < block); gates [B][H][3]
 *   fp32; out [B][H][D] fp32; sel_blocks [B][H_kv][top_blocks] int32
 *   (ascending, -1 padded) or NULL.
 * Supported: D = 128, H / H_kv <= 16, block a multiple of 32 up to 256,
 * top_blocks <= 64, window <= 4096, L / block <= 4096, and shapes whose
 * per-CTA shared memory fits (SA_EUNSUPPORTED otherwise).
 */
sa_status sa_nsa_decode(const void* q, const void* K, const void* V, int64_t stride_b, int64_t stride_t,
                        int64_t stride_h, const void* Kc, const void* Vc, int64_t c_ld, const float* gates,
                        int B, int H, int H_kv, int D, int L, int block, int top_blocks, int window, float scale,
                        float* out, int32_t* sel_blocks, sa_stream_t stream);

/*
 * CSA compressed entries ([LLMRes] "DeepSeek CSA & HCA", CSA): for every
 * sequence s and entry g in [g0, g1) (g1 <= L / m: complete groups only),
 *   out[s][g][ch] = sum_{r<m} w_a[r][ch] Ca[s][m g + r][ch]
 *                 + sum_{r<m} w_b[r][ch] Cb[s][m (g-1) + r][ch]
 * where, per channel ch, (w_a, w_b) = softmax over the 2m values
 * (Za[s][m g + r][ch] + Ba[r][ch], Zb[s][m (g-1) + r][ch] + Bb[r][ch]);
 * for g = 0 the stream-b terms are absent (weight 0).  Sums and softmax in
 * fp32, the result rounded to nearest bf16, or to e4m3 with saturation.
 *   Ca, Cb, Za, Zb bf16, element (s, t, ch) at s*seq_stride + t*row_stride + ch
 *   Ba, Bb [m][c] fp32
 *   out: element (s, g, ch) at s*out_seq_stride + g*out_row_stride + ch, in
 *   elements of out_dtype (SA_BF16 or SA_E4M3)
 * Run for the groups that complete (decode: one group every m tokens).
 * Supported: c a multiple of 4 up to 8192, m <= 256.
 */
sa_status sa_csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb, int64_t seq_stride,
                          int64_t row_stride, const float* Ba, const float* Bb, int n_seqs, int L, int m, int c,
                          int g0, int g1, void* out, sa_dtype out_dtype, int64_t out_seq_stride,
                          int64_t out_row_stride, sa_stream_t stream);

/*
 * CSA core-attention slot list ([LLMRes] CSA: the selected compressed entries
 * plus the raw entries of a recent window, attended together):
 *   idx_out[r][j]     = topk_idx[r][j]                          j < k
 *   idx_out[r][k + j] = j < min(window, raw_len[r]) ? win_base + j : -1   j < window
 * idx_out [rows][k + window] int32, the index list of sa_sparse_mla_decode
 * over a latent pool whose positions win_base .. win_base + window - 1 hold
 * the raw entries of each sequence's last tokens (oldest first).
 */
sa_status sa_csa_window_index(const int32_t* topk_idx, int rows, int k, const int32_t* raw_len, int window,
                              int win_base, int32_t* idx_out, sa_stream_t stream);

/*
 * sa_topk_select with the row histograms sa_index_scores_hist counted: the
 * selection starts from them instead of histogramming the scores again, and
 * clears them (zeros on return).  Same output as sa_topk_select.  A row whose
 * counts do not add up to its visible length (a buffer already cleared, say)
 * is selected from its scores alone, as sa_topk_select does.
 */
sa_status sa_topk_select_hist(const float* scores, int64_t scores_ld, const int32_t* n_valid, int rows, int k,
                              int32_t* hist, int32_t* idx_out, sa_stream_t stream);

/*
 * The indexer and the Top-K of one decode step without the dense score rows
 * ([Notes] §9: only the k largest I_{t,s} of each row are used; [MLA-S]
 * "一次错选会丢掉什么？" orders them by (-score, position)).
 * sa_index_candidates computes the scores of sa_index_scores_hist (one query
 * row per sequence; dtype SA_E4M3, d_I = 128, H_I in {16, 32, 64, 128}) and
 * counts them in hist as that call does, but keeps only candidates: while a
 * row streams, the counts so far give a digit d with at least k keys at or
 * above it, and a key whose digit (order key >> 20) is below the latest such d
 * is dropped (it cannot be among the k largest; the counts only grow, so a
 * bound read early is lower, never wrong).  Every key of the final Top-K is
 * kept; how many others are kept depends on timing, not on the result.
 *   cand     [rows][cand_ld] uint64: entries 0 .. cand_cnt[r]-1 of row r are
 *            (order key << 32) | (0xFFFFFFFF - position), in no fixed order
 *   cand_cnt [rows] int32, zeros on entry; hist [rows][4096] int32, zeros on
 *            entry, 16-byte aligned
 *   cand_ld >= pages_per_seq * 64 (<= 262144); n_visible[r] <= pages_per_seq * 64
 * sa_topk_from_candidates then writes idx_out [rows][k] exactly as
 * sa_topk_select does for the same scores (ascending positions, -1 padding),
 * with n_valid = the same n_visible, and leaves hist and cand_cnt zeroed, so
 * one set of buffers serves every step.  A row whose counts do not add up to
 * min(n_valid[r], cand_ld) records code 0x301 in the device error word (its
 * output is then undefined).  Shapes outside the tensor-core indexer return
 * SA_EUNSUPPORTED.  The order key is the score's bit pattern with the sign
 * bit set for non-negative scores and every bit flipped for negative ones
 * (-0.0 as +0.0), so that keys order as the scores do.
 */
sa_status sa_index_candidates(const void* q, const float* w, const void* k_cache, int64_t pool_pages, sa_dtype dtype,
                              const int32_t* page_table, int pages_per_seq, const int32_t* n_visible, int rows,
                              int H_I, int d_I, int k, int64_t cand_ld, uint64_t* cand, int32_t* cand_cnt,
                              int32_t* hist, sa_stream_t stream);

sa_status sa_topk_from_candidates(const uint64_t* cand, int64_t cand_ld, int32_t* cand_cnt, const int32_t* n_valid,
                                  int rows, int k, int32_t* hist, int32_t* idx_out, sa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */

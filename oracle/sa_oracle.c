/*
 * fp64 CPU oracle for the sparse-attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
 * CPU-baseline leg call this code.  The CUDA library never links, loads or
 * calls it, and the two share no source, header, table or helper.
 *
 * Every function below is the plain definition written out in double
 * precision, one query at a time, with its loops in the order the formulas
 * are written.  OpenMP only spreads independent queries over host cores; it
 * never reorders the arithmetic of one query.
 *
 * Sources (cited by page title and section):
 *   [Notes]  "Sparse Attention 数学学习笔记" (echobase-5bl.pages.dev, 2026.09.14)
 *   [MLA-S]  "MLA 与稀疏注意力：少存一点，还是少看一点？" (tianyi-zhang-02.github.io)
 *   [Ch11]   "第 11 章 稀疏注意力" (book.shippingwang.com)
 *   [LLMRes] "LLM注意力优化：稀疏注意力" (wln20.github.io)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Lightning indexer.
 * [Notes] §9, index score:  I_{t,s} = sum_{j=1..H^I} w_{t,j} * ReLU(q_{t,j} . k_s)
 * [MLA-S] "DSA：先用便宜的 indexer 选位置": the same score, candidates s <= t.
 * One key per history token, shared by all indexer heads; no scale, no softmax.
 *
 * q      [rows][H_I][d_I]   indexer queries of each query row
 * w      [rows][H_I]        per-head weights of each query row
 * keys   [n_keys][d_I]      indexer keys, each sequence in logical order
 * key0   [rows]             index in `keys` of position 0 of the row's sequence
 * n_vis  [rows]             number of visible positions (s = 0 .. n_vis-1)
 * out    [rows][out_ld]     I[r][s] for s < n_vis[r]; the rest untouched
 */
void sa_oracle_index_scores(int rows, int H_I, int d_I,
                            const double* q, const double* w,
                            const double* keys, const int64_t* key0,
                            const int64_t* n_vis, double* out, int64_t out_ld)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        const double* qr = q + (int64_t)r * H_I * d_I;
        const double* wr = w + (int64_t)r * H_I;
        for (int64_t s = 0; s < n_vis[r]; ++s) {
            const double* ks = keys + (key0[r] + s) * d_I;
            double I = 0.0;
            for (int j = 0; j < H_I; ++j) {
                double dot = 0.0;
                for (int d = 0; d < d_I; ++d) dot += qr[j * d_I + d] * ks[d];
                double relu = dot > 0.0 ? dot : 0.0;
                I += wr[j] * relu;
            }
            out[(int64_t)r * out_ld + s] = I;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Exact Top-K of the index scores.
 * [Notes] §9:  S_t = { s | I_{t,s} in TopK(I_{t,:}, k) }.
 * [MLA-S] "一次错选会丢掉什么？": positions ordered by (-score, position) and the
 * first `count` kept, so equal scores go to the lower position.
 * Returned set: min(k, n) positions written in ascending order, then -1 up to k.
 */
typedef struct { double v; int64_t i; } sa_oracle_pair;

static int sa_oracle_cmp_desc(const void* a, const void* b)
{
    const sa_oracle_pair* x = (const sa_oracle_pair*)a;
    const sa_oracle_pair* y = (const sa_oracle_pair*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->i > y->i) - (x->i < y->i);
}

static int sa_oracle_cmp_i32(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

void sa_oracle_topk(int rows, const double* scores, int64_t ld, const int64_t* n_valid,
                    int k, int32_t* out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        int64_t n = n_valid[r];
        int32_t* o = out + (int64_t)r * k;
        sa_oracle_pair* p = (sa_oracle_pair*)malloc((size_t)(n > 0 ? n : 1) * sizeof(sa_oracle_pair));
        for (int64_t s = 0; s < n; ++s) { p[s].v = scores[(int64_t)r * ld + s]; p[s].i = s; }
        qsort(p, (size_t)n, sizeof(sa_oracle_pair), sa_oracle_cmp_desc);
        int64_t m = n < k ? n : k;
        for (int64_t j = 0; j < m; ++j) o[j] = (int32_t)p[j].i;
        qsort(o, (size_t)m, sizeof(int32_t), sa_oracle_cmp_i32);
        for (int64_t j = m; j < k; ++j) o[j] = -1;
        free(p);
    }
}

/* ------------------------------------------------------------------------ */
/* Sparse MLA over the selected latent rows.
 * [MLA-S] "分开以后，完整分数怎么算？":
 *     score_{t,j} = ((U_K^T q^C_t)^T c_j + (q^R_t)^T k^R_j) / sqrt(d_C + d_R)
 *   one softmax over the visible (here: selected) positions;
 * [MLA-S] "“吸收矩阵”是交换线性计算的顺序": sum_j a_j U_V c_j = U_V (sum_j a_j c_j), so the
 *   output is the latent aggregate sum_j a_j c_j (U_V is applied outside);
 * [Notes] §2 / §8: a^sparse normalised over S_t only;
 * [MLA-S] masked_scalar_attention: the softmax is shifted by the maximum.
 *
 * q_lat  [rows][H][d_c]   absorbed content queries U_K^T q^C (one per head)
 * q_rope [rows][H][d_R]   rotated RoPE queries
 * c      [n][d_c], kr [n][d_R]   latent and RoPE-key rows shared by all heads
 * sel    [rows][k]        row of c/kr for each selected position, -1 = empty slot
 * out    [rows][H][d_c]   sum_j a_j c_j ; lse [rows][H] = log sum_j exp(score_j)
 * An empty selection gives out = 0 and lse = -inf.
 */
void sa_oracle_sparse_mla(int rows, int H, int d_c, int d_R,
                          const double* q_lat, const double* q_rope,
                          const double* c, const double* kr,
                          const int64_t* sel, int k, double scale,
                          double* out, double* lse)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        double* z = (double*)malloc((size_t)(k > 0 ? k : 1) * sizeof(double));
        const int64_t* sr = sel + (int64_t)r * k;
        for (int h = 0; h < H; ++h) {
            const double* qc = q_lat + ((int64_t)r * H + h) * d_c;
            const double* qr = q_rope + ((int64_t)r * H + h) * d_R;
            double* o = out + ((int64_t)r * H + h) * d_c;
            for (int d = 0; d < d_c; ++d) o[d] = 0.0;
            double m = -INFINITY;
            for (int j = 0; j < k; ++j) {
                if (sr[j] < 0) continue;
                const double* cj = c + sr[j] * d_c;
                const double* kj = kr + sr[j] * d_R;
                double content = 0.0, position = 0.0;
                for (int d = 0; d < d_c; ++d) content += qc[d] * cj[d];
                for (int e = 0; e < d_R; ++e) position += qr[e] * kj[e];
                z[j] = (content + position) * scale;
                if (z[j] > m) m = z[j];
            }
            if (m == -INFINITY) { lse[(int64_t)r * H + h] = -INFINITY; continue; }
            double l = 0.0;
            for (int j = 0; j < k; ++j) if (sr[j] >= 0) l += exp(z[j] - m);
            for (int j = 0; j < k; ++j) {
                if (sr[j] < 0) continue;
                double a = exp(z[j] - m) / l;
                const double* cj = c + sr[j] * d_c;
                for (int d = 0; d < d_c; ++d) o[d] += a * cj[d];
            }
            lse[(int64_t)r * H + h] = m + log(l);
        }
        free(z);
    }
}

/* ------------------------------------------------------------------------ */
/* Block-sparse (MoBA / NSA-style) decode for one (sequence, head).
 * [Ch11] §12.5: the sequence is cut into blocks of `block` consecutive tokens;
 *   a selected block is read whole.
 * [Ch11] §12.6: block representative = mean of the block's keys,
 *   block score = (q . k_rep) * d_h^{-1/2}, the top blocks by score are chosen.
 * [LLMRes] MoBA: affinity s_i = q . mean_pool(K_block_i), top-k blocks; sink and
 *   sliding window are blocks that are always chosen.
 * [MLA-S] "一个不用训练就能检查的错误": only blocks whose every token is visible are
 *   pooled, so the candidates are the complete blocks 0 .. floor(L/block)-1.
 * [Notes] §4 / [Ch11] §11.2: window = the last `window` positions [L-window, L-1].
 * [Notes] §2-3: softmax over the union of the chosen tokens only.
 *
 * Ties between block scores go to the lower block index.
 * q [D], K/V [L][D]; out [D]; sel [top_blocks] chosen blocks ascending, -1 padded;
 * block_scores [floor(L/block)] if not NULL.
 */
void sa_oracle_block_mean_pool(int L, int D, int block, const double* K, double* pooled)
{
    int nb = L / block;
    for (int n = 0; n < nb; ++n)
        for (int d = 0; d < D; ++d) {
            double s = 0.0;
            for (int i = 0; i < block; ++i) s += K[((int64_t)n * block + i) * D + d];
            pooled[(int64_t)n * D + d] = s / block;
        }
}

/* Attention over the token union of given chosen blocks, the sink blocks and
 * the window (the second half of the block-sparse decode above). */
void sa_oracle_block_attend(int L, int D, int block, const int32_t* chosen_blocks, int n_chosen,
                            int sink_blocks, int window, double scale,
                            const double* q, const double* K, const double* V, double* out)
{
    int nb = L / block;
    char* chosen = (char*)calloc((size_t)(nb + 1), 1);
    for (int j = 0; j < n_chosen; ++j)
        if (chosen_blocks[j] >= 0 && chosen_blocks[j] < nb) chosen[chosen_blocks[j]] = 1;
    double* z = (double*)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    char* in_u = (char*)calloc((size_t)(L > 0 ? L : 1), 1);
    double mx = -INFINITY;
    for (int t = 0; t < L; ++t) {
        int b = t / block;
        int keep = (b < nb && chosen[b]) || (t < sink_blocks * block) || (t >= L - window);
        if (!keep) continue;
        in_u[t] = 1;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * K[(int64_t)t * D + d];
        z[t] = dot * scale;
        if (z[t] > mx) mx = z[t];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    double l = 0.0;
    for (int t = 0; t < L; ++t) if (in_u[t]) l += exp(z[t] - mx);
    for (int t = 0; t < L; ++t) {
        if (!in_u[t]) continue;
        double a = exp(z[t] - mx) / l;
        for (int d = 0; d < D; ++d) out[d] += a * V[(int64_t)t * D + d];
    }
    free(chosen); free(z); free(in_u);
}

void sa_oracle_block_sparse(int L, int D, int block, int top_blocks, int sink_blocks, int window,
                            double scale, const double* q, const double* K, const double* V,
                            double* out, int32_t* sel, double* block_scores)
{
    int nb = L / block;
    double* pooled = (double*)malloc((size_t)(nb > 0 ? nb : 1) * D * sizeof(double));
    sa_oracle_block_mean_pool(L, D, block, K, pooled);
    sa_oracle_pair* p = (sa_oracle_pair*)malloc((size_t)(nb > 0 ? nb : 1) * sizeof(sa_oracle_pair));
    for (int n = 0; n < nb; ++n) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * pooled[(int64_t)n * D + d];
        p[n].v = dot * scale;
        p[n].i = n;
        if (block_scores) block_scores[n] = p[n].v;
    }
    qsort(p, (size_t)nb, sizeof(sa_oracle_pair), sa_oracle_cmp_desc);
    int m = nb < top_blocks ? nb : top_blocks;
    for (int j = 0; j < m; ++j) sel[j] = (int32_t)p[j].i;
    qsort(sel, (size_t)m, sizeof(int32_t), sa_oracle_cmp_i32);
    for (int j = m; j < top_blocks; ++j) sel[j] = -1;
    sa_oracle_block_attend(L, D, block, sel, m, sink_blocks, window, scale, q, K, V, out);
    free(pooled); free(p);
}

/* Number of host threads OpenMP will use (reported beside the CPU timings). */
int sa_oracle_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Set the number of host threads the loops above may use (n >= 1); used to
 * time the oracle on one core beside all cores. */
void sa_oracle_set_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n < 1 ? 1 : n);
#else
    (void)n;
#endif
}

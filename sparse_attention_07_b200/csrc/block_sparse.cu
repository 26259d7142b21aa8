// block_sparse.cu — MoBA / NSA-style block-sparse decode.
//
// "第 11 章 稀疏注意力" §12.5-12.6: the history is cut into blocks of `block`
// consecutive tokens; each block is represented by the mean of its keys,
// scored as (q . k_rep) * d^-1/2, and the top blocks are read whole (contiguous
// K/V runs).  "LLM注意力优化：稀疏注意力" (MoBA): sink and sliding window are
// blocks that are always chosen.  "MLA 与稀疏注意力" (causality check): only
// complete blocks are pooled.  "Sparse Attention 数学学习笔记" §2-4: softmax over the
// chosen tokens only; the window is [L-w, L-1].
//
// block_mean_pool: one warp per (b, h, block) sums 64 keys in fp32.
// block_sparse:    one CTA per (b, h): (1) scores of every complete block from
//                  the pooled keys (float4 loads, warp reductions), (2) top
//                  blocks by (-score, block) with block-wide arg-max rounds,
//                  (3) token union = chosen blocks clipped below the window, plus
//                  the sink block and the window, (4) 16 warps stream their share
//                  of the union's K/V rows with an online base-2 softmax, (5) the
//                  warp states are merged in shared memory.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBlocks = 4096;
constexpr int kMaxTop = 64;

__device__ __forceinline__ float4 ld_bf16x4(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ K, int64_t sb, int64_t st,
                                                   int64_t sh, int B, int H, int nb, int block,
                                                   float* __restrict__ pooled, int64_t pooled_ld) {
    const int64_t unit = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (unit >= static_cast<int64_t>(B) * H * nb) return;
    const int n = static_cast<int>(unit % nb);
    const int h = static_cast<int>((unit / nb) % H);
    const int b = static_cast<int>(unit / (static_cast<int64_t>(nb) * H));
    const __nv_bfloat16* base = K + b * sb + h * sh + static_cast<int64_t>(n) * block * st + lane * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int i = 0; i < block; ++i) {
        const float4 v = ld_bf16x4(base + i * st);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
    }
    const float inv = 1.f / static_cast<float>(block);
    float* dst = pooled + ((static_cast<int64_t>(b) * H + h) * pooled_ld + n) * kD + lane * 4;
    *reinterpret_cast<float4*>(dst) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

struct BlkArgs {
    const __nv_bfloat16* q;
    const float* pooled;
    int64_t pooled_ld;
    const __nv_bfloat16* K;
    const __nv_bfloat16* V;
    int64_t sb, st, sh;
    int H, L, block, top, sink_blocks, window;
    float scale;
    float* out;
    int32_t* sel;
};

__global__ void __launch_bounds__(kThreads) block_sparse_kernel(const BlkArgs a) {
    __shared__ float s_score[kMaxBlocks];
    __shared__ __align__(16) float s_q[kD];
    __shared__ float s_bv[kWarps];
    __shared__ int s_bi[kWarps];
    __shared__ int s_chosen[kMaxTop + 1];
    __shared__ uint32_t s_taken[kMaxBlocks / 32];
    __shared__ int s_run_lo[kMaxTop + 2], s_run_hi[kMaxTop + 2], s_run_pre[kMaxTop + 3];
    __shared__ int s_nruns;
    __shared__ float s_wm[kWarps], s_wl[kWarps];
    __shared__ __align__(16) float s_wo[kWarps][kD];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int L = a.L, blk = a.block;
    const int nb = L / blk;  // complete blocks only
    const float c2 = a.scale * 1.4426950408889634f;

    if (tid < kD) s_q[tid] = __bfloat162float(a.q[(static_cast<int64_t>(b) * a.H + h) * kD + tid]);
    __syncthreads();

    // (1) block scores from the pooled keys
    {
        const float4 qv = *reinterpret_cast<const float4*>(&s_q[lane * 4]);
        const float* pb = a.pooled + (static_cast<int64_t>(b) * a.H + h) * a.pooled_ld * kD + lane * 4;
        for (int n0 = warp * 4; n0 < nb; n0 += kWarps * 4) {
            float d[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + j;
                float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
                if (n < nb) p = *reinterpret_cast<const float4*>(pb + static_cast<int64_t>(n) * kD);
                d[j] = qv.x * p.x + qv.y * p.y + qv.z * p.z + qv.w * p.w;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) d[j] = warp_sum(d[j]);
            const float mine = lane == 0 ? d[0] : (lane == 1 ? d[1] : (lane == 2 ? d[2] : d[3]));
            if (lane < 4 && n0 + lane < nb) s_score[n0 + lane] = mine * a.scale;
        }
    }
    __syncthreads();

    // (2) top blocks by (-score, block): repeated block-wide arg-max over the
    //     blocks not taken yet (a bit mask marks the taken ones)
    const int ntop = min(a.top, nb);
    for (int i = tid; i < kMaxBlocks / 32; i += kThreads) s_taken[i] = 0u;
    __syncthreads();
    for (int round = 0; round < ntop; ++round) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int n = tid; n < nb; n += kThreads) {
            if ((s_taken[n >> 5] >> (n & 31)) & 1u) continue;
            const float v = s_score[n];
            if (bi == 0x7fffffff || v > bv || (v == bv && n < bi)) {
                bv = v;
                bi = n;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
                bv = ov;
                bi = oi;
            }
        }
        if (lane == 0) {
            s_bv[warp] = bv;
            s_bi[warp] = bi;
        }
        __syncthreads();
        if (tid == 0) {
            float v = s_bv[0];
            int i = s_bi[0];
            for (int w = 1; w < kWarps; ++w) {
                const int wi = s_bi[w];
                if (wi != 0x7fffffff && (i == 0x7fffffff || s_bv[w] > v || (s_bv[w] == v && wi < i))) {
                    v = s_bv[w];
                    i = wi;
                }
            }
            s_chosen[round] = i;
            s_taken[i >> 5] |= 1u << (i & 31);
        }
        __syncthreads();
    }

    // (3) token runs: chosen and sink blocks clipped below the window, then the window
    if (tid == 0) {
        // sort chosen ascending (ntop <= 64)
        for (int i = 1; i < ntop; ++i) {
            const int v = s_chosen[i];
            int j = i - 1;
            while (j >= 0 && s_chosen[j] > v) {
                s_chosen[j + 1] = s_chosen[j];
                --j;
            }
            s_chosen[j + 1] = v;
        }
        if (a.sel) {
            int32_t* so = a.sel + (static_cast<int64_t>(b) * a.H + h) * a.top;
            for (int i = 0; i < a.top; ++i) so[i] = i < ntop ? s_chosen[i] : -1;
        }
        const int win_lo = max(0, L - a.window);
        const int sink_hi = min(win_lo, a.sink_blocks * blk);
        int nr = 0;
        int cur_lo = 0, cur_hi = 0;  // merge sink range [0, sink_hi) with chosen blocks
        if (sink_hi > 0) {
            cur_lo = 0;
            cur_hi = sink_hi;
        }
        for (int i = 0; i < ntop; ++i) {
            const int lo = s_chosen[i] * blk;
            const int hi = min(lo + blk, win_lo);
            if (hi <= lo) continue;
            if (cur_hi > cur_lo && lo <= cur_hi) {
                cur_hi = max(cur_hi, hi);
            } else {
                if (cur_hi > cur_lo) {
                    s_run_lo[nr] = cur_lo;
                    s_run_hi[nr] = cur_hi;
                    ++nr;
                }
                cur_lo = lo;
                cur_hi = hi;
            }
        }
        if (cur_hi > cur_lo) {
            s_run_lo[nr] = cur_lo;
            s_run_hi[nr] = cur_hi;
            ++nr;
        }
        if (win_lo < L) {
            s_run_lo[nr] = win_lo;
            s_run_hi[nr] = L;
            ++nr;
        }
        s_run_pre[0] = 0;
        for (int i = 0; i < nr; ++i) s_run_pre[i + 1] = s_run_pre[i] + (s_run_hi[i] - s_run_lo[i]);
        s_nruns = nr;
    }
    __syncthreads();

    // (4) online softmax over this warp's slice of the union
    const int nruns = s_nruns;
    const int U = s_run_pre[nruns];
    const int u0 = static_cast<int>(static_cast<int64_t>(warp) * U / kWarps);
    const int u1 = static_cast<int>(static_cast<int64_t>(warp + 1) * U / kWarps);
    const float4 qv = *reinterpret_cast<const float4*>(&s_q[lane * 4]);
    const __nv_bfloat16* Kb = a.K + b * a.sb + h * a.sh + lane * 4;
    const __nv_bfloat16* Vb = a.V + b * a.sb + h * a.sh + lane * 4;
    float m = -INFINITY, l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    int run = 0;
    while (run < nruns && s_run_pre[run + 1] <= u0) ++run;
    for (int u = u0; u < u1; u += 4) {
        int tok[4];
        bool ok[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int uu = u + j;
            ok[j] = uu < u1;
            int rr = run;
            while (ok[j] && rr < nruns && s_run_pre[rr + 1] <= uu) ++rr;
            tok[j] = ok[j] ? s_run_lo[rr] + (uu - s_run_pre[rr]) : 0;
        }
        float4 kv[4], vv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            kv[j] = ld_bf16x4(Kb + static_cast<int64_t>(tok[j]) * a.st);
            vv[j] = ld_bf16x4(Vb + static_cast<int64_t>(tok[j]) * a.st);
        }
        float s[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) s[j] = qv.x * kv[j].x + qv.y * kv[j].y + qv.z * kv[j].z + qv.w * kv[j].w;
#pragma unroll
        for (int j = 0; j < 4; ++j) s[j] = warp_sum(s[j]);
        float mx = m;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s[j] = ok[j] ? s[j] * c2 : -INFINITY;
            mx = fmaxf(mx, s[j]);
        }
        const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - mx);
        l *= alpha;
        o.x *= alpha;
        o.y *= alpha;
        o.z *= alpha;
        o.w *= alpha;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float p = ok[j] ? exp2f(s[j] - mx) : 0.f;
            l += p;
            o.x += p * vv[j].x;
            o.y += p * vv[j].y;
            o.z += p * vv[j].z;
            o.w += p * vv[j].w;
        }
        m = mx;
        while (run < nruns && s_run_pre[run + 1] <= u + 4) ++run;
    }
    if (lane == 0) {
        s_wm[warp] = m;
        s_wl[warp] = l;
    }
    *reinterpret_cast<float4*>(&s_wo[warp][lane * 4]) = o;
    __syncthreads();

    // (5) merge the warp states
    if (tid < kD) {
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_wm[w]);
        float Lsum = 0.f, acc = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            if (s_wm[w] == -INFINITY) continue;
            const float wg = exp2f(s_wm[w] - M);
            Lsum += s_wl[w] * wg;
            acc += s_wo[w][tid] * wg;
        }
        a.out[(static_cast<int64_t>(b) * a.H + h) * kD + tid] = Lsum > 0.f ? acc / Lsum : 0.f;
    }
}

// ------------------------------------------------------------ cluster path
// One cluster of kC CTAs per (sequence, head) (kC = 1 when the batch alone
// fills the GPU, else 4).  CTA r scores its share of the complete blocks, streaming the pooled keys with bulk copies through a
// shared-memory ring; each CTA keeps its top blocks (warp arg-max rounds over
// 64-bit keys: score key, then the lower block), the cluster exchanges them
// through distributed shared memory and every CTA merges the same global set.
// The union is cut into 64-token segments (sink, chosen blocks clipped below
// the window, window); CTA r loads its share of the segments as whole K and V
// tiles (a TMA box of 64 tokens x 128 dims each, through a ring), runs an
// online softmax per warp, and CTA 0 merges the cluster's states.
constexpr int kT2 = 256;                      // threads per CTA
constexpr int kW2 = kT2 / 32;
constexpr int kPoolChunk = 32;                // pooled blocks per bulk copy (16 KB)
constexpr int kPoolStages = 4;
constexpr int kSegTok = 64;                   // tokens per segment (one TMA box)
constexpr int kTileBytes = kSegTok * kD * 2;  // 16 KB of K (or V)
constexpr int kKvStages = 3;
constexpr int kRingBytes = kKvStages * 2 * kTileBytes;  // 96 KB; the pooled ring uses 64 KB of it
constexpr int kPoolRing = kPoolStages * kPoolChunk * kD * 4;  // 64 KB
constexpr int kCSmem = kRingBytes + 1024;
// the block scores (at most kMaxBlocks, one CTA) sit above the pooled ring,
// inside the K/V ring (whose first tiles are issued once the selection is done)
static_assert(kPoolRing + kMaxBlocks * 4 <= kRingBytes, "pooled ring and scores fit the K/V ring");
static_assert(kMaxTop <= 64 && kPoolChunk % kW2 == 0 && kSegTok % kW2 == 0, "shapes");
constexpr int kSelBits = 11;                  // block choice: histogram of the keys' top bits
constexpr int kSelBins = 1 << kSelBits;
constexpr int kSelCap = 256;                  // keys the choosing warp holds (8 per lane)
static_assert(kSelBins * 4 + kSelCap * 8 <= kPoolRing && kSelBins % kT2 == 0, "selection scratch in the pooled ring");
constexpr int kBlkW = kPoolChunk / kW2;       // pooled blocks per warp and chunk
constexpr int kTokW = kSegTok / kW2;          // tokens per warp and segment

struct BlkMaps {
    CUtensorMap K, V;  // 4-d: (d, token, head, sequence), box 128 x 64 x 1 x 1
};

struct BlkArgs2 {
    const __nv_bfloat16* q;
    const float* pooled;
    int64_t pooled_ld;
    int H, L, block, top, sink_blocks, window;
    float scale;
    float* out;
    int32_t* sel;
    int* err;
};

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int o) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), o);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), o);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Selection key of block n: larger for a higher score, then for a lower index
// (0 marks no block: every real key is larger).
__device__ __forceinline__ uint64_t block_key2(float score, int n) {
    return (static_cast<uint64_t>(score_order_key(score)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(n));
}
__device__ __forceinline__ int key_block2(uint64_t key) {
    return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}

// The warp's `ntop` largest of the keys its lanes hold (kPer per lane, taken
// keys are zeroed), written to out[0..ntop) in descending order.
template <int kPer>
__device__ __forceinline__ void warp_top(uint64_t (&v)[kPer], int ntop, uint64_t* out, int lane) {
    for (int t = 0; t < ntop; ++t) {
        uint64_t best = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) best = v[j] > best ? v[j] : best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t x = shfl_xor_u64(best, o);
            best = x > best ? x : best;
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (best != 0 && v[j] == best) v[j] = 0;  // keys are distinct: one lane holds it
        if (lane == 0) out[t] = best;
    }
}

template <int kC>
__global__ void __cluster_dims__(kC, 1, 1) __launch_bounds__(kT2, 2)
    block_sparse_cluster_kernel(const __grid_constant__ BlkMaps maps, const BlkArgs2 a) {
    constexpr int kMaxPer = kMaxBlocks / kC;  // pooled blocks scored by one CTA
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* s_score = reinterpret_cast<float*>(ring + kPoolRing);  // [kMaxPer]
    __shared__ uint64_t bar_pool[kPoolStages], bar_kv[kKvStages];
    __shared__ __align__(16) float s_q[kD];
    __shared__ uint64_t s_wtop[kW2][kMaxTop];     // each warp's best blocks
    __shared__ uint64_t s_ctop[kC][kMaxTop];      // each CTA's best blocks (pushed by every CTA)
    __shared__ int s_chosen[kMaxTop];             // the global choice, ascending
    __shared__ int s_cseg[kMaxTop];               // chosen blocks that add tokens, ascending
    __shared__ int s_ncseg;
    __shared__ float s_wm[kW2], s_wl[kW2];
    __shared__ __align__(16) float s_wo[kW2][kD];
    __shared__ float s_state[kC][kD + 2];         // each CTA's (o, m, l), pushed to CTA 0
    __shared__ int s_abort;
    __shared__ int s_wsel[kW2], s_bstar, s_nge, s_nc;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank();
    const int bh = blockIdx.x / kC;
    const int b = bh / a.H, h = bh % a.H;
    const int L = a.L, blk = a.block;
    const int nb = L / blk;
    const int ntop = min(a.top, nb);
    const float c2 = a.scale * 1.4426950408889634f;
    WaitCtx wc{a.err, &s_abort};
    int pool_issued = 0, kv_issued = 0;  // copies issued (thread 0 issues them all)

    // this CTA's blocks and their bulk-copy chunks
    const int per = (nb + kC - 1) / kC;
    const int blo = min(nb, static_cast<int>(rank) * per), bhi = min(nb, blo + per);
    const int nch = (bhi - blo + kPoolChunk - 1) / kPoolChunk;
    const float* pbase = a.pooled + (static_cast<int64_t>(b) * a.H + h) * a.pooled_ld * kD;
    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < kPoolStages; ++i) mbar_init(&bar_pool[i], 1);
        for (int i = 0; i < kKvStages; ++i) mbar_init(&bar_kv[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&maps.K);
        tma_prefetch_desc(&maps.V);
        for (int c = 0; c < kPoolStages && c < nch; ++c) {
            const int n0 = blo + c * kPoolChunk, nn = min(kPoolChunk, bhi - n0);
            mbar_arrive_expect_tx(&bar_pool[c], static_cast<uint32_t>(nn * kD * 4));
            bulk_copy_g2s(ring + c * (kPoolChunk * kD * 4), pbase + static_cast<int64_t>(n0) * kD,
                          static_cast<uint32_t>(nn * kD * 4), &bar_pool[c]);
            ++pool_issued;
        }
    }
    if (tid < kD) s_q[tid] = __bfloat162float(a.q[(static_cast<int64_t>(b) * a.H + h) * kD + tid]);
    cluster_arrive_relaxed();  // this CTA has started; waited for before the first push
    __syncthreads();

    // (1) scores of this CTA's blocks: warp w takes kBlkW consecutive blocks of a chunk
    const float4 qv = *reinterpret_cast<const float4*>(&s_q[lane * 4]);
    for (int c = 0; c < nch; ++c) {
        const int st = c % kPoolStages;
        const bool got = mbar_wait(&bar_pool[st], static_cast<uint32_t>((c / kPoolStages) & 1), wc, kErrBlockWait | 1);
        const int n0 = c * kPoolChunk, nn = min(kPoolChunk, bhi - blo - n0);
        const float* sp = reinterpret_cast<const float*>(ring + st * (kPoolChunk * kD * 4));
        float d[kBlkW];
#pragma unroll
        for (int j = 0; j < kBlkW; ++j) {
            const int n = warp * kBlkW + j;
            float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
            if (got && n < nn) p = *reinterpret_cast<const float4*>(sp + n * kD + lane * 4);
            d[j] = qv.x * p.x + qv.y * p.y + qv.z * p.z + qv.w * p.w;
        }
#pragma unroll
        for (int j = 0; j < kBlkW; ++j) d[j] = warp_sum(d[j]);
#pragma unroll
        for (int j = 0; j < kBlkW; ++j)
            if (lane == j && warp * kBlkW + j < nn) s_score[n0 + warp * kBlkW + j] = d[j] * a.scale;
        __syncthreads();  // the stage is read: refill it
        if (tid == 0 && c + kPoolStages < nch && !s_abort) {
            const int c2i = c + kPoolStages, m0 = blo + c2i * kPoolChunk, mm = min(kPoolChunk, bhi - m0);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar_pool[st], static_cast<uint32_t>(mm * kD * 4));
            bulk_copy_g2s(ring + st * (kPoolChunk * kD * 4), pbase + static_cast<int64_t>(m0) * kD,
                          static_cast<uint32_t>(mm * kD * 4), &bar_pool[st]);
            ++pool_issued;
        }
    }

    // The window and sink segments come first in the union's order and do not
    // depend on the choice: with one CTA per pair (which takes the segments
    // from the first one on) the first tile pair is loaded now, into the half of
    // the ring that the choice below leaves alone.
    const int win_lo = max(0, L - a.window);
    const int sink_hi = min(win_lo, a.sink_blocks * blk);
    const int n_sink = (sink_hi + kSegTok - 1) / kSegTok;
    const int n_win = (L - win_lo + kSegTok - 1) / kSegTok;
    const bool early = kC == 1 && n_win + n_sink > 0;
    if (early && tid == 0) {
        const int lo = n_win > 0 ? win_lo : 0;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bar_kv[1], 2u * kTileBytes);
        tma_load_4d(ring + 1 * 2 * kTileBytes, &maps.K, &bar_kv[1], 0, lo, h, b);
        tma_load_4d(ring + 1 * 2 * kTileBytes + kTileBytes, &maps.V, &bar_kv[1], 0, lo, h, b);
        ++kv_issued;
    }

    // (2) this CTA's best ntop blocks.  A histogram of the scores' keys
    //     (top 11 bits) in the consumed pooled ring finds the bin of the
    //     ntop-th largest; the keys at or above it (few, unless many scores
    //     tie) are listed and one warp picks the best of them.  Lists too long
    //     for the warp fall back to arg-max rounds in every warp over all keys.
    const int nmine = bhi - blo;
    const int want = min(ntop, nmine);
    uint32_t* hsel = reinterpret_cast<uint32_t*>(ring);                 // [kSelBins]
    uint64_t* cand = reinterpret_cast<uint64_t*>(ring + kSelBins * 4);  // [kSelCap]
    for (int i = tid; i < kSelBins; i += kT2) hsel[i] = 0u;
    if (tid == 0) {
        s_bstar = kSelBins;  // no key qualifies unless a bin is found below
        s_nge = 0;
        s_nc = 0;
    }
    __syncthreads();
    for (int i = tid; i < nmine; i += kT2) atomicAdd(&hsel[score_order_key(s_score[i]) >> (32 - kSelBits)], 1u);
    __syncthreads();
    {
        constexpr int kBinsPer = kSelBins / kT2;       // thread t: bins from the top, highest first
        const int top_bin = kSelBins - 1 - kBinsPer * tid;
        int c[kBinsPer], tot = 0;
#pragma unroll
        for (int j = 0; j < kBinsPer; ++j) {
            c[j] = static_cast<int>(hsel[top_bin - j]);
            tot += c[j];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) s_wsel[warp] = incl;
        __syncthreads();
        int above = incl - tot;
        for (int w = 0; w < warp; ++w) above += s_wsel[w];
        if (want > 0 && above < want && want <= above + tot) {
            int acc = above;
#pragma unroll
            for (int j = 0; j < kBinsPer; ++j) {
                acc += c[j];
                if (acc >= want) {
                    s_bstar = top_bin - j;
                    s_nge = acc;
                    break;
                }
            }
        }
    }
    __syncthreads();
    const bool fast = s_nge <= kSelCap;
    if (fast) {
        const uint32_t bstar = static_cast<uint32_t>(s_bstar);
        for (int i = tid; i < nmine; i += kT2) {
            const uint32_t kk = score_order_key(s_score[i]);
            if ((kk >> (32 - kSelBits)) >= bstar) cand[atomicAdd(&s_nc, 1)] = block_key2(s_score[i], blo + i);
        }
    } else {
        constexpr int kPerLane = kMaxPer / kT2;  // scores per lane (4 or 16)
        uint64_t v[kPerLane];
#pragma unroll
        for (int j = 0; j < kPerLane; ++j) {
            const int i = (warp * kPerLane + j) * 32 + lane;  // warp w: its 32 * kPerLane scores
            v[j] = i < nmine ? block_key2(s_score[i], blo + i) : 0ull;
        }
        warp_top<kPerLane>(v, ntop, s_wtop[warp], lane);
    }
    __syncthreads();
    if (warp == 0) {
        uint64_t* mine = &s_wtop[0][0];  // reused: warp 0 only from here, after the barrier
        if (fast) {
            constexpr int kCP = kSelCap / 32;
            const int nc = s_nc;
            uint64_t v[kCP];
#pragma unroll
            for (int j = 0; j < kCP; ++j) {
                const int i = j * 32 + lane;
                v[j] = i < nc ? cand[i] : 0ull;
            }
            warp_top<kCP>(v, ntop, mine, lane);
        } else {
            constexpr int kM = kW2 * kMaxTop / 32;  // 16 per lane
            uint64_t v[kM];
#pragma unroll
            for (int j = 0; j < kM; ++j) {
                const int i = j * 32 + lane, w = i / kMaxTop, t = i % kMaxTop;
                v[j] = t < ntop ? s_wtop[w][t] : 0ull;
            }
            warp_top<kM>(v, ntop, mine, lane);
        }
        __syncwarp();
        cluster_wait();  // every CTA of the cluster has started
        for (int i = lane; i < kC * ntop; i += 32) {
            const int dst = i / ntop, t = i % ntop;
            const uint64_t x = mine[t];
            const uint32_t at = mapa_u32(smem_u32(&s_ctop[rank][t]), static_cast<uint32_t>(dst));
            asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(at), "r"(static_cast<uint32_t>(x)),
                         "r"(static_cast<uint32_t>(x >> 32))
                         : "memory");
        }
    } else {
        cluster_wait();
    }
    cluster_sync_all();  // every CTA's list is in place
    if (warp == 0) {
        constexpr int kM = (kC * kMaxTop + 31) / 32;  // 2 or 8 per lane
        uint64_t v[kM];
#pragma unroll
        for (int j = 0; j < kM; ++j) {
            const int i = j * 32 + lane, r = i / kMaxTop, t = i % kMaxTop;
            v[j] = (r < kC && t < ntop) ? s_ctop[r][t] : 0ull;
        }
        uint64_t* glob = &s_wtop[1][0];
        warp_top<kM>(v, ntop, glob, lane);
        __syncwarp();
        // ascending block order: each lane ranks its blocks among the chosen
        for (int t = lane; t < ntop; t += 32) {
            const int mine = key_block2(glob[t]);
            int at = 0;
            for (int u = 0; u < ntop; ++u) at += key_block2(glob[u]) < mine ? 1 : 0;
            s_chosen[at] = mine;
        }
        __syncwarp();
        if (lane == 0) {
            const int win_lo = max(0, L - a.window);
            const int sink_hi = min(win_lo, a.sink_blocks * blk);
            int nc = 0;
            for (int t = 0; t < ntop; ++t) {
                const int lo = s_chosen[t] * blk;
                if (lo >= sink_hi && lo < win_lo) s_cseg[nc++] = s_chosen[t];
            }
            s_ncseg = nc;
            if (rank == 0 && a.sel) {
                int32_t* so = a.sel + (static_cast<int64_t>(b) * a.H + h) * a.top;
                for (int i = 0; i < a.top; ++i) so[i] = i < ntop ? s_chosen[i] : -1;
            }
        }
    }
    __syncthreads();

    // (3) the union as 64-token segments (window, sink, chosen blocks); this
    //     CTA's share of them.  Segment i of the share uses ring stage
    //     (i + 1) % kKvStages (stage 1 is the one free during the choice).
    const int n_ch = s_ncseg;
    const int nseg = n_sink + n_ch + n_win;
    const int g0 = static_cast<int>(static_cast<int64_t>(rank) * nseg / kC);
    const int g1 = static_cast<int>(static_cast<int64_t>(rank + 1) * nseg / kC);
    auto seg_of = [&](int g, int& lo, int& hi) {
        if (g < n_win) {
            lo = win_lo + g * kSegTok;
            hi = min(lo + kSegTok, L);
        } else if (g < n_win + n_sink) {
            lo = (g - n_win) * kSegTok;
            hi = min(lo + kSegTok, sink_hi);
        } else {
            lo = s_cseg[g - n_win - n_sink] * blk;
            hi = min(lo + blk, win_lo);
        }
    };
    const int nmy = g1 - g0;
    if (tid == 0) {  // the choice is done (barrier above): the first K/V tiles
        fence_proxy_async_smem();
        for (int i = early ? 1 : 0; i < kKvStages && i < nmy; ++i) {
            const int st = (i + 1) % kKvStages;
            int lo, hi;
            seg_of(g0 + i, lo, hi);
            mbar_arrive_expect_tx(&bar_kv[st], 2u * kTileBytes);
            tma_load_4d(ring + st * 2 * kTileBytes, &maps.K, &bar_kv[st], 0, lo, h, b);
            tma_load_4d(ring + st * 2 * kTileBytes + kTileBytes, &maps.V, &bar_kv[st], 0, lo, h, b);
            ++kv_issued;
        }
    }

    // (4) online softmax: warp w takes tokens kTokW*w .. kTokW*w + kTokW-1 of each segment
    float m = -INFINITY, l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < nmy; ++i) {
        const int st = (i + 1) % kKvStages;
        int lo, hi;
        seg_of(g0 + i, lo, hi);
        const bool got = mbar_wait(&bar_kv[st], static_cast<uint32_t>((i / kKvStages) & 1), wc, kErrBlockWait | 2);
        const uint8_t* kt = ring + st * 2 * kTileBytes;
        const uint8_t* vt = kt + kTileBytes;
        float sc[kTokW];
#pragma unroll
        for (int j = 0; j < kTokW; ++j) {
            const int t = warp * kTokW + j;
            float4 kv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (got) kv = ld_bf16x4(reinterpret_cast<const __nv_bfloat16*>(kt + t * (kD * 2)) + lane * 4);
            sc[j] = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
        }
#pragma unroll
        for (int j = 0; j < kTokW; ++j) sc[j] = warp_sum(sc[j]);
        float mx = m;
#pragma unroll
        for (int j = 0; j < kTokW; ++j) {
            sc[j] = (got && lo + warp * kTokW + j < hi) ? sc[j] * c2 : -INFINITY;
            mx = fmaxf(mx, sc[j]);
        }
        if (mx != -INFINITY) {
            const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - mx);
            l *= alpha;
            o.x *= alpha;
            o.y *= alpha;
            o.z *= alpha;
            o.w *= alpha;
#pragma unroll
            for (int j = 0; j < kTokW; ++j) {
                if (sc[j] == -INFINITY) continue;
                const float p = exp2f(sc[j] - mx);
                const float4 vv = ld_bf16x4(
                    reinterpret_cast<const __nv_bfloat16*>(vt + (warp * kTokW + j) * (kD * 2)) + lane * 4);
                l += p;
                o.x += p * vv.x;
                o.y += p * vv.y;
                o.z += p * vv.z;
                o.w += p * vv.w;
            }
            m = mx;
        }
        __syncthreads();  // the stage is read: refill it
        if (tid == 0 && i + kKvStages < nmy && !s_abort) {
            int nlo, nhi;
            seg_of(g0 + i + kKvStages, nlo, nhi);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar_kv[st], 2u * kTileBytes);
            tma_load_4d(ring + st * 2 * kTileBytes, &maps.K, &bar_kv[st], 0, nlo, h, b);
            tma_load_4d(ring + st * 2 * kTileBytes + kTileBytes, &maps.V, &bar_kv[st], 0, nlo, h, b);
            ++kv_issued;
        }
    }
    if (s_abort && tid == 0) {
        // a wait gave up: every copy issued must land before the CTA leaves
        int dummy = 0;
        WaitCtx dw(a.err, reinterpret_cast<volatile int*>(&dummy), kWaitLimitNs);
        for (int c = max(0, pool_issued - kPoolStages); c < pool_issued; ++c)
            mbar_wait(&bar_pool[c % kPoolStages], static_cast<uint32_t>((c / kPoolStages) & 1), dw, kErrBlockWait | 3);
        for (int i = max(0, kv_issued - kKvStages); i < kv_issued; ++i)
            mbar_wait(&bar_kv[(i + 1) % kKvStages], static_cast<uint32_t>((i / kKvStages) & 1), dw, kErrBlockWait | 4);
    }

    // (5) the warps' states, then the CTAs' states (in CTA 0)
    if (lane == 0) {
        s_wm[warp] = m;
        s_wl[warp] = l;
    }
    *reinterpret_cast<float4*>(&s_wo[warp][lane * 4]) = o;
    __syncthreads();
    if (tid < kD) {
        float M = -INFINITY;
        for (int w = 0; w < kW2; ++w) M = fmaxf(M, s_wm[w]);
        float Ls = 0.f, acc = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < kW2; ++w) {
                if (s_wm[w] == -INFINITY) continue;
                const float wg = exp2f(s_wm[w] - M);
                Ls += s_wl[w] * wg;
                acc += s_wo[w][tid] * wg;
            }
        }
        const uint32_t at = mapa_u32(smem_u32(&s_state[rank][0]), 0u);
        st_cluster_u32(at + 4u * tid, __float_as_uint(acc));
        if (tid == 0) {
            st_cluster_u32(at + 4u * kD, __float_as_uint(M));
            st_cluster_u32(at + 4u * (kD + 1), __float_as_uint(Ls));
        }
    }
    cluster_sync_all();  // the states are in CTA 0; no CTA touches another's memory after this
    if (rank == 0 && tid < kD) {
        float M = -INFINITY;
        for (int r = 0; r < kC; ++r) M = fmaxf(M, s_state[r][kD]);
        float Ls = 0.f, acc = 0.f;
        if (M != -INFINITY) {
            for (int r = 0; r < kC; ++r) {
                if (s_state[r][kD] == -INFINITY) continue;
                const float wg = exp2f(s_state[r][kD] - M);
                Ls += s_state[r][kD + 1] * wg;
                acc += s_state[r][tid] * wg;
            }
        }
        a.out[(static_cast<int64_t>(b) * a.H + h) * kD + tid] = Ls > 0.f ? acc / Ls : 0.f;
    }
}

}  // namespace

sa_status block_mean_pool_launch(const void* K, int64_t sb, int64_t st_, int64_t sh, int B, int L, int H, int D,
                                 int block, float* pooled, int64_t pooled_ld, cudaStream_t st) {
    (void)D;
    const int nb = L / block;
    const int64_t units = static_cast<int64_t>(B) * H * nb;
    if (units == 0) return SA_OK;
    const int64_t grid = (units + 7) / 8;
    pool_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(K), sb, st_, sh, B, H,
                                                             nb, block, pooled, pooled_ld);
    return launch_status(cudaGetLastError());
}

sa_status block_sparse_launch(const void* q, const float* pooled, int64_t pooled_ld, const void* K, const void* V,
                              int64_t sb, int64_t st_, int64_t sh, int B, int H, int D, int L, int block,
                              int top_blocks, int sink_blocks, int window, float scale, float* out,
                              int32_t* sel_blocks, int* err, cudaStream_t st) {
    (void)D;
    // cluster path: K/V tiles by TMA (16-byte aligned base and strides)
    const bool tma_ok = (reinterpret_cast<uintptr_t>(K) & 15) == 0 && (reinterpret_cast<uintptr_t>(V) & 15) == 0 &&
                        sb % 8 == 0 && st_ % 8 == 0 && sh % 8 == 0 && L >= 1;
    if (tma_ok) {
        BlkMaps m;
        const uint64_t dims[4] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(L), static_cast<uint64_t>(H),
                                  static_cast<uint64_t>(B)};
        const uint64_t strides[3] = {static_cast<uint64_t>(st_) * 2, static_cast<uint64_t>(sh) * 2,
                                     static_cast<uint64_t>(sb) * 2};
        const uint32_t box[4] = {static_cast<uint32_t>(kD), static_cast<uint32_t>(kSegTok), 1, 1};
        if (!encode_tiled(&m.K, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, K, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_tiled(&m.V, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, V, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return SA_ECUDA;
        BlkArgs2 a2;
        a2.q = static_cast<const __nv_bfloat16*>(q);
        a2.pooled = pooled;
        a2.pooled_ld = pooled_ld;
        a2.H = H;
        a2.L = L;
        a2.block = block;
        a2.top = top_blocks;
        a2.sink_blocks = sink_blocks;
        a2.window = window;
        a2.scale = scale;
        a2.out = out;
        a2.sel = sel_blocks;
        a2.err = err;
        // one CTA per (sequence, head) once the pairs alone fill the GPU,
        // else clusters of four share each pair's blocks and tokens
        const int64_t pairs = static_cast<int64_t>(B) * H;
        // two CTAs per SM: all of the unified memory as shared memory
        cudaError_t e;
        if (pairs >= sm_count()) {
            e = cudaFuncSetAttribute(block_sparse_cluster_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kCSmem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(block_sparse_cluster_kernel<1>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         100);
            if (e == cudaSuccess) block_sparse_cluster_kernel<1><<<static_cast<unsigned>(pairs), kT2, kCSmem, st>>>(m, a2);
        } else {
            e = cudaFuncSetAttribute(block_sparse_cluster_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kCSmem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(block_sparse_cluster_kernel<4>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         100);
            if (e == cudaSuccess)
                block_sparse_cluster_kernel<4><<<static_cast<unsigned>(pairs) * 4, kT2, kCSmem, st>>>(m, a2);
        }
        if (e != cudaSuccess) return launch_status(e);
        return launch_status(cudaGetLastError());
    }
    BlkArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.pooled = pooled;
    a.pooled_ld = pooled_ld;
    a.K = static_cast<const __nv_bfloat16*>(K);
    a.V = static_cast<const __nv_bfloat16*>(V);
    a.sb = sb;
    a.st = st_;
    a.sh = sh;
    a.H = H;
    a.L = L;
    a.block = block;
    a.top = top_blocks;
    a.sink_blocks = sink_blocks;
    a.window = window;
    a.scale = scale;
    a.out = out;
    a.sel = sel_blocks;
    block_sparse_kernel<<<B * H, kThreads, 0, st>>>(a);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

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
                              int32_t* sel_blocks, cudaStream_t st) {
    (void)D;
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

// topk_select.cu — exact per-row Top-K of the index scores.
//
// S_t = { s | I_{t,s} in TopK(I_{t,:}, k) } ("Sparse Attention 数学学习笔记" §9), with
// positions ranked by (-score, position) so equal scores go to the lower
// position ("MLA 与稀疏注意力", selected_positions), written in ascending order.
//
// One cluster of 8 CTAs per row.  Each CTA copies 1/8 of the row into shared
// memory as order-preserving 32-bit keys (one read of the scores), then the
// cluster runs a most-significant-digit-first radix select with 8-bit digits:
// every CTA builds a histogram of the digit over the keys still in the
// candidate class, the 8 histograms are summed through distributed shared
// memory, and the class shrinks to the digit holding the k-th largest key.
// The search stops as soon as the whole remaining class is taken.  Finally an
// ordered compaction (warp ballots + prefix counts across warps and CTAs)
// writes every key above the class plus the first `remaining` keys of the
// class in position order — ascending output without a sort.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

// fp32 -> uint32 whose unsigned order is the float order; -0 and +0 map alike.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_valid, int k,
                int32_t* __restrict__ out) {
    extern __shared__ uint32_t s_keys[];
    __shared__ int s_hist[2][256];
    __shared__ int s_suf[257];
    __shared__ int s_wsum[8];
    __shared__ int s_warp_gt[kWarps], s_warp_eq[kWarps];
    __shared__ int s_counts[2];
    __shared__ int s_sel[3];  // digit, count above the digit, count of the digit

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x / kCluster;
    const uint32_t rank = cluster_rank();
    int n = n_valid[row];
    n = n < 0 ? 0 : (n > ld ? static_cast<int>(ld) : n);
    int32_t* orow = out + static_cast<int64_t>(row) * k;

    if (n <= k) {  // every position is selected; the rest is padding
        for (int s = static_cast<int>(rank) * kThreads + tid; s < k; s += kCluster * kThreads) orow[s] = s < n ? s : -1;
        return;
    }

    const int chunk = (((n + kCluster - 1) / kCluster) + 3) & ~3;
    const int lo = static_cast<int>(rank) * chunk;
    const int cnt = max(0, min(n, lo + chunk) - lo);
    const float* src = scores + static_cast<int64_t>(row) * ld + lo;
    {
        const int n4 = cnt >> 2;
        for (int i = tid; i < n4; i += kThreads) {
            const float4 v = reinterpret_cast<const float4*>(src)[i];
            s_keys[4 * i + 0] = order_key(v.x);
            s_keys[4 * i + 1] = order_key(v.y);
            s_keys[4 * i + 2] = order_key(v.z);
            s_keys[4 * i + 3] = order_key(v.w);
        }
        for (int i = 4 * n4 + tid; i < cnt; i += kThreads) s_keys[i] = order_key(src[i]);
    }

    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    const int cnt_round = ((cnt + kThreads - 1) / kThreads) * kThreads;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        int* hist = s_hist[pass & 1];
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int base = 0; base < cnt_round; base += kThreads) {
            const int i = base + tid;
            bool active = false;
            uint32_t digit = 0;
            if (i < cnt) {
                const uint32_t key = s_keys[i];
                active = (key & mask) == prefix;
                digit = (key >> shift) & 255u;
            }
            const unsigned am = __ballot_sync(0xffffffffu, active);
            if (active) {
                const unsigned peers = __match_any_sync(am, digit);
                if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
            }
        }
        __syncthreads();
        cluster_sync_all();
        // cluster-wide histogram and its suffix sums (bins 255 .. 0)
        if (tid < 256) {
            const uint32_t my = smem_u32(&hist[tid]);
            int tot = 0;
#pragma unroll
            for (uint32_t r = 0; r < kCluster; ++r) tot += static_cast<int>(ld_cluster_u32(mapa_u32(my, r)));
            int incl = tot;  // suffix within the warp's 32 bins
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += t;
            }
            s_suf[tid] = incl;
            if (lane == 0) s_wsum[warp] = incl;
        }
        __syncthreads();
        if (tid < 256) {
            int add = 0;
            for (int w = warp + 1; w < 8; ++w) add += s_wsum[w];
            s_suf[tid] += add;
            if (tid == 0) s_suf[256] = 0;
        }
        __syncthreads();
        if (tid < 256) {
            const int here = s_suf[tid], above = s_suf[tid + 1];
            if (here >= remaining && above < remaining) {
                s_sel[0] = tid;
                s_sel[1] = above;
                s_sel[2] = here - above;
            }
        }
        __syncthreads();
        remaining -= s_sel[1];
        prefix |= static_cast<uint32_t>(s_sel[0]) << shift;
        mask |= 255u << shift;
        if (s_sel[2] == remaining) break;  // the whole class is taken
    }

    // ---- ordered compaction
    const int seg = (cnt + kWarps - 1) / kWarps;
    const int ws = min(cnt, warp * seg), we = min(cnt, ws + seg);
    int gt_w = 0, eq_w = 0;
    for (int base = ws; base < we; base += 32) {
        const int i = base + lane;
        bool gt = false, eq = false;
        if (i < we) {
            const uint32_t m = s_keys[i] & mask;
            gt = m > prefix;
            eq = m == prefix;
        }
        gt_w += __popc(__ballot_sync(0xffffffffu, gt));
        eq_w += __popc(__ballot_sync(0xffffffffu, eq));
    }
    if (lane == 0) {
        s_warp_gt[warp] = gt_w;
        s_warp_eq[warp] = eq_w;
    }
    __syncthreads();
    if (tid == 0) {
        int g = 0, e = 0;
        for (int w = 0; w < kWarps; ++w) {
            g += s_warp_gt[w];
            e += s_warp_eq[w];
        }
        s_counts[0] = g;
        s_counts[1] = e;
    }
    cluster_sync_all();
    // offsets of this CTA: ranks below take their "above" keys and their share of the class
    int off = 0, eq_before = 0;
    for (uint32_t r = 0; r < rank; ++r) {
        const int g = static_cast<int>(ld_cluster_u32(mapa_u32(smem_u32(&s_counts[0]), r)));
        const int e = static_cast<int>(ld_cluster_u32(mapa_u32(smem_u32(&s_counts[1]), r)));
        const int take = max(0, min(e, remaining - eq_before));
        off += g + take;
        eq_before += e;
    }
    const int take_c = max(0, min(s_counts[1], remaining - eq_before));
    // offsets of this warp inside the CTA
    int sel_before = 0, eqb = 0;
    for (int w = 0; w < warp; ++w) {
        sel_before += s_warp_gt[w] + max(0, min(s_warp_eq[w], take_c - eqb));
        eqb += s_warp_eq[w];
    }
    int eq_run = 0, sel_run = 0;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = ws; base < we; base += 32) {
        const int i = base + lane;
        bool gt = false, eq = false;
        if (i < we) {
            const uint32_t m = s_keys[i] & mask;
            gt = m > prefix;
            eq = m == prefix;
        }
        const unsigned eb = __ballot_sync(0xffffffffu, eq);
        const bool sel = gt || (eq && (eqb + eq_run + __popc(eb & lt)) < take_c);
        const unsigned sb = __ballot_sync(0xffffffffu, sel);
        const int pos = off + sel_before + sel_run + __popc(sb & lt);
        if (sel && pos < k) orow[pos] = lo + i;
        eq_run += __popc(eb);
        sel_run += __popc(sb);
    }
    cluster_sync_all();  // no CTA leaves while another may still read its counts
}

}  // namespace

sa_status topk_select_launch(const float* scores, int64_t ld, const int32_t* n_valid, int rows, int k,
                             int32_t* idx_out, cudaStream_t st) {
    const int chunk = static_cast<int>((((ld + kCluster - 1) / kCluster) + 3) & ~int64_t(3));
    const size_t smem = static_cast<size_t>(chunk) * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return launch_status(e);
    topk_kernel<<<rows * kCluster, kThreads, smem, st>>>(scores, ld, n_valid, k, idx_out);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

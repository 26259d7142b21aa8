// topk_select.cu — exact per-row Top-K of the index scores.
//
// S_t = { s | I_{t,s} in TopK(I_{t,:}, k) } ("Sparse Attention 数学学习笔记" §9), with
// positions ranked by (-score, position) so equal scores go to the lower
// position ("MLA 与稀疏注意力", selected_positions), written in ascending order.
//
// One cluster of 8 CTAs per row.  Each CTA copies 1/8 of the row into shared
// memory as order-preserving 32-bit keys (the only read of the scores) and
// selects with a most-significant-digit-first radix search:
//  1. First digit = key bits 31..20 (sign, exponent, three mantissa bits).
//     When the indexer has counted it (a 4096-bin histogram per row), every
//     CTA reads the counts while its scores are in flight, finds the boundary
//     bin (the bin of the k-th largest key) on its own, and lists the keys of
//     its slice that carry the boundary digit (the candidates) as it loads.
//     Otherwise every CTA builds the histogram while it loads, the cluster
//     reduces it scatter-wise (CTA r sums bins 512r..512r+511 over the eight
//     CTAs and scans them, the eight block totals are exchanged, and the owner
//     of the boundary bin broadcasts the digit, the count above it and the
//     count inside it), and the candidates are listed after.
//  2. The remaining 20 bits (19..12, 11..4, 3..0) are resolved by radix
//     passes over the candidates only; every pass sums its 256-bin histograms
//     through distributed shared memory.  The search stops as soon as the whole
//     remaining class is taken.
//  3. Ordered compaction: each CTA pushes its two counts (keys above the final
//     class, keys in it) into every CTA of the cluster; after one cluster
//     barrier each CTA has its output offset and writes every key above the
//     class plus its share of the first `remaining` keys of the class in
//     position order (warp ballots and prefix counts): ascending output with
//     no sort, and no shared-memory access between CTAs after that barrier.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins0 = 4096;                 // first digit: key bits 31..20
constexpr int kOwn = kBins0 / kCluster;      // first-digit bins reduced by each CTA
constexpr int kBins1 = 256;                  // refinement digits: key bits 19..12, 11..4, 3..0
constexpr int kCandCap = 4096;               // candidate slots per CTA
constexpr int kVec = 4;                      // float4 loads in flight per thread
static_assert(kOwn == kThreads, "one owned bin per thread");
static_assert(kWarps <= 32 && kCluster <= 32, "one warp sums the warp counts and pushes them");

__device__ __forceinline__ uint32_t order_key(float f) { return score_order_key(f); }

// Histogram increment by a whole warp: lanes with equal digits add once.
__device__ __forceinline__ void hist_add(int* hist, bool active, uint32_t digit, int lane) {
    const unsigned am = __ballot_sync(0xffffffffu, active);
    if (active) {
        const unsigned peers = __match_any_sync(am, digit);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
    }
}

// Warp-aggregated append of position i to the candidate list when c holds.
__device__ __forceinline__ void cand_add(int* ncand, uint16_t* cand, bool c, int i, int lane) {
    const unsigned b = __ballot_sync(0xffffffffu, c);
    int wbase = 0;
    if (lane == 0 && b) wbase = atomicAdd(ncand, __popc(b));
    wbase = __shfl_sync(0xffffffffu, wbase, 0);
    const int slot = wbase + __popc(b & ((1u << lane) - 1u));
    if (c && slot < kCandCap) cand[slot] = static_cast<uint16_t>(i);
}

// Lane i receives the sum of lanes i..31.
__device__ __forceinline__ int warp_suffix(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_down_sync(0xffffffffu, v, o);
        if (lane + o < 32) v += t;
    }
    return v;
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 2)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_valid, int k, int chunk,
                int32_t* __restrict__ hist, int32_t* __restrict__ out) {
    extern __shared__ __align__(16) uint32_t s_keys[];  // [chunk] keys of this CTA's slice
    __shared__ int s_hist0[kBins0];
    __shared__ int s_hist[2][kBins1];
    __shared__ int s_suf[kBins1 + 1];
    __shared__ int s_wsum[kWarps];
    __shared__ int s_btot[kCluster];  // first-digit block totals, written by every CTA
    __shared__ int s_sel0[3];         // boundary digit, count above, count inside
    __shared__ int s_sel[3];
    __shared__ int s_ncand;
    __shared__ uint16_t s_cand[kCandCap];  // local positions of the candidates
    __shared__ int s_warp_gt[kWarps], s_warp_eq[kWarps];
    __shared__ int s_counts[kCluster][2];  // (above the class, in the class) of every CTA, pushed by each

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x / kCluster;
    const uint32_t rank = cluster_rank();
    int n = n_valid[row];
    n = n < 0 ? 0 : (n > ld ? static_cast<int>(ld) : n);
    int32_t* orow = out + static_cast<int64_t>(row) * k;

    int32_t* hrow = hist ? hist + static_cast<int64_t>(row) * kHistBins : nullptr;
    if (n <= k) {  // every position is selected; the rest is padding
        for (int s = static_cast<int>(rank) * kThreads + tid; s < k; s += kCluster * kThreads) orow[s] = s < n ? s : -1;
        if (hrow) hrow[static_cast<int>(rank) * kOwn + tid] = 0;  // leave the row's histogram cleared
        return;
    }

    const int lo = static_cast<int>(rank) * chunk;
    const int cnt = max(0, min(n, lo + chunk) - lo);
    const float* src = scores + static_cast<int64_t>(row) * ld + lo;
    const int n4 = cnt >> 2;
    if (tid == 0) s_ncand = 0;

    // the first batch of score loads is in flight while the histogram is read
    float4 v[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
        const int i = u * kThreads + tid;
        if (i < n4) v[u] = reinterpret_cast<const float4*>(src)[i];
    }

    // ---- 1. the boundary digit
    // The row's first-digit histogram may come with the scores (the indexer
    // counted them).  It is used only if its total is the row's length: every
    // CTA of the cluster reads the same counts, so all take the same branch and
    // the same cluster barriers; otherwise the counts are built here.
    bool from_global = false;
    if (hrow) {
        constexpr int kPer = kBins0 / kThreads;  // bins per thread, highest first
        const int b_hi = kBins0 - 1 - tid * kPer;
        int hv[kPer];
        int mine = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            hv[j] = hrow[b_hi - j];
            mine += hv[j];
        }
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) s_wsum[warp] = incl;
        if (tid == 0) {  // defined values should no bin qualify
            s_sel0[0] = 0;
            s_sel0[1] = 0;
            s_sel0[2] = 0;
        }
        __syncthreads();
        int above = incl - mine;  // keys in bins above this thread's bins
        int total = 0;
        for (int w = 0; w < kWarps; ++w) {
            if (w < warp) above += s_wsum[w];
            total += s_wsum[w];
        }
        from_global = total == n;
        if (from_global && above < k && k <= above + mine) {
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                if (k <= above + hv[j]) {
                    s_sel0[0] = b_hi - j;
                    s_sel0[1] = above;
                    s_sel0[2] = hv[j];
                    break;
                }
                above += hv[j];
            }
        }
    }
    if (!from_global)
        for (int i = tid; i < kBins0; i += kThreads) s_hist0[i] = 0;
    __syncthreads();
    // with the boundary digit known, the candidates are listed as the keys are made
    const bool list_now = from_global && s_sel0[2] != k - s_sel0[1];
    const uint32_t d_known = static_cast<uint32_t>(s_sel0[0]);

    // ---- 2. keys of the slice (and the first-digit counts, or the candidates)
    for (int base = 0; base < n4; base += kVec * kThreads) {
        if (base > 0) {
#pragma unroll
            for (int u = 0; u < kVec; ++u) {
                const int i = base + u * kThreads + tid;
                if (i < n4) v[u] = reinterpret_cast<const float4*>(src)[i];
            }
        }
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int i = base + u * kThreads + tid;
            const bool ok = i < n4;
            uint4 kk = make_uint4(0u, 0u, 0u, 0u);
            if (ok) {
                kk = make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z), order_key(v[u].w));
                reinterpret_cast<uint4*>(s_keys)[i] = kk;
            }
            if (!from_global) {
                hist_add(s_hist0, ok, kk.x >> 20, lane);
                hist_add(s_hist0, ok, kk.y >> 20, lane);
                hist_add(s_hist0, ok, kk.z >> 20, lane);
                hist_add(s_hist0, ok, kk.w >> 20, lane);
            } else if (list_now) {
                cand_add(&s_ncand, s_cand, ok && (kk.x >> 20) == d_known, 4 * i, lane);
                cand_add(&s_ncand, s_cand, ok && (kk.y >> 20) == d_known, 4 * i + 1, lane);
                cand_add(&s_ncand, s_cand, ok && (kk.z >> 20) == d_known, 4 * i + 2, lane);
                cand_add(&s_ncand, s_cand, ok && (kk.w >> 20) == d_known, 4 * i + 3, lane);
            }
        }
    }
    if (warp == 0) {  // up to three keys after the last full vector
        const int i = 4 * n4 + lane;
        const bool ok = i < cnt;
        uint32_t key = 0u;
        if (ok) {
            key = order_key(src[i]);
            s_keys[i] = key;
        }
        if (!from_global) hist_add(s_hist0, ok, key >> 20, lane);
        else if (list_now) cand_add(&s_ncand, s_cand, ok && (key >> 20) == d_known, i, lane);
    }
    __syncthreads();

    if (!from_global) {
        cluster_sync_all();
        // CTA `rank` reduces bins rank*512 .. rank*512+511 over the cluster
        const int g = static_cast<int>(rank) * kOwn + tid;
        int tot = 0;
        {
            const uint32_t a = smem_u32(&s_hist0[g]);
            uint32_t hv[kCluster];
#pragma unroll
            for (int r = 0; r < kCluster; ++r) hv[r] = ld_cluster_u32(mapa_u32(a, static_cast<uint32_t>(r)));
#pragma unroll
            for (int r = 0; r < kCluster; ++r) tot += static_cast<int>(hv[r]);
        }
        int incl = warp_suffix(tot, lane);
        if (lane == 0) s_wsum[warp] = incl;
        if (tid == 0) {  // defined values should no bin qualify
            s_sel0[0] = 0;
            s_sel0[1] = 0;
            s_sel0[2] = 0;
        }
        __syncthreads();
        for (int w = warp + 1; w < kWarps; ++w) incl += s_wsum[w];  // keys in bins g.. of this CTA's range
        if (tid < kCluster) {
            int t = 0;
            for (int w = 0; w < kWarps; ++w) t += s_wsum[w];
            st_cluster_u32(mapa_u32(smem_u32(&s_btot[rank]), static_cast<uint32_t>(tid)), static_cast<uint32_t>(t));
        }
        cluster_sync_all();
        for (int r = static_cast<int>(rank) + 1; r < kCluster; ++r) incl += s_btot[r];
        {
            const int above = incl - tot;  // keys in bins above g, cluster-wide
            if (tot > 0 && incl >= k && above < k) {
                for (int r = 0; r < kCluster; ++r) {
                    const uint32_t a = mapa_u32(smem_u32(&s_sel0[0]), static_cast<uint32_t>(r));
                    st_cluster_u32(a, static_cast<uint32_t>(g));
                    st_cluster_u32(a + 4, static_cast<uint32_t>(above));
                    st_cluster_u32(a + 8, static_cast<uint32_t>(tot));
                }
            }
        }
        cluster_sync_all();
    }

    uint32_t prefix = static_cast<uint32_t>(s_sel0[0]) << 20, mask = 0xFFF00000u;
    int remaining = k - s_sel0[1];
    if (s_sel0[2] != remaining) {
        // ---- 3. the candidates (keys carrying the boundary digit), then the refinement passes
        const int cnt_round = ((cnt + kThreads - 1) / kThreads) * kThreads;
        if (!list_now) {
            const uint32_t d0 = static_cast<uint32_t>(s_sel0[0]);
            for (int base = 0; base < cnt_round; base += kThreads) {
                const int i = base + tid;
                cand_add(&s_ncand, s_cand, i < cnt && (s_keys[i] >> 20) == d0, i, lane);
            }
            __syncthreads();
        }
        // a CTA whose candidates overflow the list scans all of its keys instead
        const bool listed = s_ncand <= kCandCap;
        const int nscan = listed ? s_ncand : cnt;
        const int nscan_round = ((nscan + kThreads - 1) / kThreads) * kThreads;
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 12 : (pass == 1 ? 4 : 0);
            const uint32_t dmask = pass == 2 ? 15u : 255u;
            int* h = s_hist[pass & 1];
            if (tid < kBins1) h[tid] = 0;
            __syncthreads();
            for (int base = 0; base < nscan_round; base += kThreads) {
                const int i = base + tid;
                bool active = false;
                uint32_t digit = 0;
                if (i < nscan) {
                    const uint32_t key = s_keys[listed ? static_cast<int>(s_cand[i]) : i];
                    active = (key & mask) == prefix;
                    digit = (key >> shift) & dmask;
                }
                hist_add(h, active, digit, lane);
            }
            cluster_sync_all();
            // cluster-wide histogram and its suffix sums (bins 255 .. 0)
            if (tid < kBins1) {
                const uint32_t my = smem_u32(&h[tid]);
                uint32_t hv[kCluster];
#pragma unroll
                for (int r = 0; r < kCluster; ++r) hv[r] = ld_cluster_u32(mapa_u32(my, static_cast<uint32_t>(r)));
                int t = 0;
#pragma unroll
                for (int r = 0; r < kCluster; ++r) t += static_cast<int>(hv[r]);
                const int in = warp_suffix(t, lane);
                s_suf[tid] = in;
                if (lane == 0) s_wsum[warp] = in;
            }
            __syncthreads();
            if (tid < kBins1) {
                int add = 0;
                for (int w = warp + 1; w < kBins1 / 32; ++w) add += s_wsum[w];
                s_suf[tid] += add;
                if (tid == 0) {
                    s_suf[kBins1] = 0;
                    s_sel[0] = 0;  // defined values should no bin qualify
                    s_sel[1] = 0;
                    s_sel[2] = -1;
                }
            }
            __syncthreads();
            if (tid < kBins1) {
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
            mask |= dmask << shift;
            if (s_sel[2] == remaining) break;  // the whole class is taken
        }
    }

    // ---- 4. ordered compaction
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
    if (warp == 0) {  // this CTA's two counts into every CTA of the cluster
        int g = lane < kWarps ? s_warp_gt[lane] : 0, e = lane < kWarps ? s_warp_eq[lane] : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane < kCluster) {
            const uint32_t a = mapa_u32(smem_u32(&s_counts[rank][0]), static_cast<uint32_t>(lane));
            st_cluster_u32(a, static_cast<uint32_t>(g));
            st_cluster_u32(a + 4, static_cast<uint32_t>(e));
        }
    }
    // Every CTA's counts are in place, and every read of another CTA's shared
    // memory (histograms of the passes) is done: after this barrier no CTA
    // touches another's shared memory, so each may leave when it has written.
    cluster_sync_all();
    if (hrow) hrow[static_cast<int>(rank) * kOwn + tid] = 0;  // every CTA has read it: clear for the next step
    // offsets of this CTA: ranks below take their "above" keys and their share of the class
    int off = 0, eq_before = 0;
    for (int r = 0; r < static_cast<int>(rank); ++r) {
        const int take = max(0, min(s_counts[r][1], remaining - eq_before));
        off += s_counts[r][0] + take;
        eq_before += s_counts[r][1];
    }
    const int take_c = max(0, min(s_counts[rank][1], remaining - eq_before));
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
}

}  // namespace

sa_status topk_select_launch(const float* scores, int64_t ld, const int32_t* n_valid, int rows, int k,
                             int32_t* hist, int32_t* idx_out, cudaStream_t st) {
    const int chunk = static_cast<int>((((ld + kCluster - 1) / kCluster) + 3) & ~int64_t(3));
    const size_t smem = static_cast<size_t>(chunk) * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return launch_status(e);
    topk_kernel<<<rows * kCluster, kThreads, smem, st>>>(scores, ld, n_valid, k, chunk, hist, idx_out);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

// topk_select.cu — exact per-row Top-K of the index scores.
//
// S_t = { s | I_{t,s} in TopK(I_{t,:}, k) } ("Sparse Attention 数学学习笔记" §9), with
// positions ranked by (-score, position) so equal scores go to the lower
// position ("MLA 与稀疏注意力", selected_positions), written in ascending order.
//
// One cluster of 4 CTAs per row; CTA r streams its quarter of the row (the
// scores stay in L2 and are read again where needed, so a CTA holds only the
// candidates in shared memory and two CTAs fit on an SM: 64 rows of up to
// 128K keys run in one wave).  Scores become order-preserving 32-bit keys and
// the selection is a most-significant-digit-first radix search:
//  1. First digit = key bits 31..20 (sign, exponent, three mantissa bits).
//     When the indexer has counted it (a 4096-bin histogram per row), every
//     CTA reads the counts while its first scores are in flight and finds the
//     boundary bin (the bin of the k-th largest key) on its own.  Otherwise
//     every CTA counts its slice, the cluster reduces the histogram
//     scatter-wise through distributed shared memory (CTA r sums bins
//     1024r..1024r+1023 of the four CTAs) and the owner of the boundary bin
//     broadcasts the digit, the count above it and the count inside it.
//  2. One pass over the slice lists, in shared memory, the positions of the
//     keys above the boundary digit (all of them are selected) and the keys
//     that carry it (the candidates) with their positions.
//  3. The remaining 20 bits (19..12, 11..4, 3..0) are resolved by radix
//     passes over the candidates only (a CTA with more candidates than its
//     list holds scans its slice again instead); every pass sums its 256-bin
//     histograms through distributed shared memory.  The search stops as
//     soon as the whole remaining class is taken.
//  4. Ordered compaction from two bitmaps of the slice's positions: one bit
//     per selected position (the listed keys above the boundary digit and the
//     candidates above the final class) and one per member of the final class.
//     A block scan of the class bits ranks the class members by position; each
//     CTA pushes its two counts into every CTA of the cluster; after one
//     cluster barrier each CTA knows its output offset and its share of the
//     first `remaining` class members, sets their bits, and a second block scan
//     places every selected position: ascending output with no sort and no
//     second pass over the scores.  When a list overflowed (or the first digit
//     settled the row) the counts and positions come from passes over the
//     slice instead: each warp counts its contiguous segment, then writes it.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kCluster = 4;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins0 = 4096;                 // first digit: key bits 31..20
constexpr int kOwn = kBins0 / kCluster;      // first-digit bins reduced by each CTA
constexpr int kOwnPer = kOwn / kThreads;     // ... per thread
constexpr int kBins1 = 256;                  // refinement digits: key bits 19..12, 11..4, 3..0
constexpr int kCandCap = 4096;               // candidate slots per CTA
constexpr int kSureCap = 4096;               // slots for the positions above the boundary digit
constexpr int kBmWords = 2048;               // bitmap words: slices of up to 65536 positions
constexpr int kBmPer = kBmWords / kThreads;  // bitmap words owned by each thread
constexpr int kVec = 4;                      // float4 loads in flight per thread
// dynamic shared memory: candidate keys, candidate positions, positions above
// the boundary digit (16-bit: a slice holds at most 65536 positions), bitmaps
constexpr int kOffCPos = kCandCap * 4;
constexpr int kOffSure = kOffCPos + kCandCap * 2;
constexpr int kOffBm = kOffSure + kSureCap * 2;
constexpr int kDynSmem = kOffBm + 2 * kBmWords * 4;
static_assert(kOwnPer * kThreads == kOwn && kOwnPer == 2, "two owned bins per thread");
static_assert(kBmPer * kThreads == kBmWords && kBmWords * 32 == 65536, "bitmaps cover a 65536-position slice");
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

// Lists key `key` at slice position `pos`: above the boundary digit d0 its
// position joins the selected list, on it (key, position) joins the candidate
// list.  Both are rare among a slice's keys, so each hit takes one shared
// atomic of its own; counts past a list's capacity are kept (overflow).
__device__ __forceinline__ void list_key(int* nsure, int* ncand, uint16_t* sure, uint32_t* ckey, uint16_t* cpos,
                                         bool ok, uint32_t key, uint32_t d0, int pos) {
    if (!ok) return;
    const uint32_t d = key >> 20;
    if (d > d0) {
        const int slot = atomicAdd(nsure, 1);
        if (slot < kSureCap) sure[slot] = static_cast<uint16_t>(pos);
    } else if (d == d0) {
        const int slot = atomicAdd(ncand, 1);
        if (slot < kCandCap) {
            ckey[slot] = key;
            cpos[slot] = static_cast<uint16_t>(pos);
        }
    }
}

// Block-wide exclusive prefix of v over the threads (in thread order); also
// returns the block total.  All threads call it; uses `wsum` [kWarps].
__device__ __forceinline__ int block_exclusive(int v, int lane, int warp, int* wsum, int& total) {
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = incl - v;
    total = 0;
    for (int w = 0; w < kWarps; ++w) {
        const int x = wsum[w];
        if (w < warp) before += x;
        total += x;
    }
    return before;
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

// Lane i receives the sum of lanes 0..i-1.
__device__ __forceinline__ int warp_exclusive(int v, int lane) {
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    return incl - v;
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 2)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_valid, int k, int chunk,
                int32_t* __restrict__ hist, int32_t* __restrict__ out) {
    extern __shared__ __align__(16) uint8_t s_dyn[];
    uint32_t* s_ckey = reinterpret_cast<uint32_t*>(s_dyn);             // [kCandCap] candidate keys
    uint16_t* s_cpos = reinterpret_cast<uint16_t*>(s_dyn + kOffCPos);  // [kCandCap] their slice positions
    uint16_t* s_sure = reinterpret_cast<uint16_t*>(s_dyn + kOffSure);  // [kSureCap] positions above the digit
    uint32_t* s_bm_sel = reinterpret_cast<uint32_t*>(s_dyn + kOffBm);  // [kBmWords] selected positions
    uint32_t* s_bm_cls = s_bm_sel + kBmWords;                          // [kBmWords] final-class members
    __shared__ int s_hist0[kBins0];
    __shared__ int s_hist[2][kBins1];
    __shared__ int s_suf[kBins1 + 1];
    __shared__ int s_wsum[kWarps];
    __shared__ int s_btot[kCluster];  // first-digit block totals, written by every CTA
    __shared__ int s_sel0[3];         // boundary digit, count above, count inside
    __shared__ int s_sel[3];
    __shared__ int s_ncand, s_nsure;
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
        if (hrow)  // leave the row's histogram cleared
            for (int j = 0; j < kOwnPer; ++j) hrow[static_cast<int>(rank) * kOwn + j * kThreads + tid] = 0;
        return;
    }
    // this CTA has started; every path waits for the others before its first
    // access to another CTA's shared memory
    cluster_arrive_relaxed();

    const int lo = static_cast<int>(rank) * chunk;
    const int cnt = max(0, min(n, lo + chunk) - lo);
    const float* src = scores + static_cast<int64_t>(row) * ld + lo;
    const int n4 = cnt >> 2;
    if (tid == 0) {
        s_ncand = 0;
        s_nsure = 0;
    }
#pragma unroll
    for (int j = 0; j < kBmPer; ++j) {  // cleared bitmaps (read after several barriers)
        s_bm_sel[tid * kBmPer + j] = 0u;
        s_bm_cls[tid * kBmPer + j] = 0u;
    }

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
    if (!from_global) {
        for (int i = tid; i < kBins0; i += kThreads) s_hist0[i] = 0;
        __syncthreads();
        // the first-digit counts of the slice
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
                const uint4 kk = ok ? make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z),
                                                 order_key(v[u].w))
                                    : make_uint4(0u, 0u, 0u, 0u);
                hist_add(s_hist0, ok, kk.x >> 20, lane);
                hist_add(s_hist0, ok, kk.y >> 20, lane);
                hist_add(s_hist0, ok, kk.z >> 20, lane);
                hist_add(s_hist0, ok, kk.w >> 20, lane);
            }
        }
        if (warp == 0) {  // up to three keys after the last full vector
            const int i = 4 * n4 + lane;
            const bool ok = i < cnt;
            hist_add(s_hist0, ok, ok ? order_key(src[i]) >> 20 : 0u, lane);
        }
        __syncthreads();
        cluster_wait();
        cluster_sync_all();
        // CTA `rank` reduces bins rank*1024 .. rank*1024+1023 over the cluster:
        // thread t owns bins g0 = rank*1024 + 2t and g0 + 1
        const int g0 = static_cast<int>(rank) * kOwn + kOwnPer * tid;
        int t0 = 0, t1 = 0;
        {
            const uint32_t a0 = smem_u32(&s_hist0[g0]);
            uint32_t h0[kCluster], h1[kCluster];
#pragma unroll
            for (int r = 0; r < kCluster; ++r) {
                const uint32_t a = mapa_u32(a0, static_cast<uint32_t>(r));
                h0[r] = ld_cluster_u32(a);
                h1[r] = ld_cluster_u32(a + 4);
            }
#pragma unroll
            for (int r = 0; r < kCluster; ++r) {
                t0 += static_cast<int>(h0[r]);
                t1 += static_cast<int>(h1[r]);
            }
        }
        const int tot = t0 + t1;
        int incl = warp_suffix(tot, lane);
        if (lane == 0) s_wsum[warp] = incl;
        if (tid == 0) {  // defined values should no bin qualify
            s_sel0[0] = 0;
            s_sel0[1] = 0;
            s_sel0[2] = 0;
        }
        __syncthreads();
        for (int w = warp + 1; w < kWarps; ++w) incl += s_wsum[w];  // keys in bins g0.. of this CTA's range
        if (tid < kCluster) {
            int t = 0;
            for (int w = 0; w < kWarps; ++w) t += s_wsum[w];
            st_cluster_u32(mapa_u32(smem_u32(&s_btot[rank]), static_cast<uint32_t>(tid)), static_cast<uint32_t>(t));
        }
        cluster_sync_all();
        for (int r = static_cast<int>(rank) + 1; r < kCluster; ++r) incl += s_btot[r];
        {
            // keys in bins above g0 + 1, cluster-wide; then bin g0 + 1, then bin g0
            const int above1 = incl - tot, above0 = above1 + t1;
            int sel_g = -1, sel_above = 0, sel_in = 0;
            if (t1 > 0 && above1 < k && k <= above1 + t1) {
                sel_g = g0 + 1;
                sel_above = above1;
                sel_in = t1;
            } else if (t0 > 0 && above0 < k && k <= above0 + t0) {
                sel_g = g0;
                sel_above = above0;
                sel_in = t0;
            }
            if (sel_g >= 0) {
                for (int r = 0; r < kCluster; ++r) {
                    const uint32_t a = mapa_u32(smem_u32(&s_sel0[0]), static_cast<uint32_t>(r));
                    st_cluster_u32(a, static_cast<uint32_t>(sel_g));
                    st_cluster_u32(a + 4, static_cast<uint32_t>(sel_above));
                    st_cluster_u32(a + 8, static_cast<uint32_t>(sel_in));
                }
            }
        }
        cluster_sync_all();
    } else {
        __syncthreads();
        cluster_wait();
    }

    uint32_t prefix = static_cast<uint32_t>(s_sel0[0]) << 20, mask = 0xFFF00000u;
    int remaining = k - s_sel0[1];
    bool lists = false;  // the selection can be placed from the two lists
    if (s_sel0[2] != remaining) {
        // ---- 2. the lists: keys above the boundary digit and keys on it
        const uint32_t d0 = static_cast<uint32_t>(s_sel0[0]);
        for (int base = 0; base < n4; base += kVec * kThreads) {
            if (base > 0 || !from_global) {
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
                const uint4 kk = ok ? make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z),
                                                 order_key(v[u].w))
                                    : make_uint4(0u, 0u, 0u, 0u);
                list_key(&s_nsure, &s_ncand, s_sure, s_ckey, s_cpos, ok, kk.x, d0, 4 * i);
                list_key(&s_nsure, &s_ncand, s_sure, s_ckey, s_cpos, ok, kk.y, d0, 4 * i + 1);
                list_key(&s_nsure, &s_ncand, s_sure, s_ckey, s_cpos, ok, kk.z, d0, 4 * i + 2);
                list_key(&s_nsure, &s_ncand, s_sure, s_ckey, s_cpos, ok, kk.w, d0, 4 * i + 3);
            }
        }
        if (warp == 0) {  // up to three keys after the last full vector
            const int i = 4 * n4 + lane;
            const bool ok = i < cnt;
            const uint32_t key = ok ? order_key(src[i]) : 0u;
            list_key(&s_nsure, &s_ncand, s_sure, s_ckey, s_cpos, ok, key, d0, i);
        }
        __syncthreads();
        lists = s_ncand <= kCandCap && s_nsure <= kSureCap;
        // ---- 3. refinement passes; a CTA whose candidates overflow the list
        // scans all of its keys (from L2) instead
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
                    const uint32_t key = listed ? s_ckey[i] : order_key(src[i]);
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

    // ---- 4. ordered compaction.  Each path yields this CTA's two counts
    // (keys above the final class, keys in it); both push them the same way.
    int cta_gt = 0, cta_eq = 0;
    // bitmap path: this thread's words of the two bitmaps and its class rank base
    uint32_t bsel[kBmPer], bcls[kBmPer];
    int cls_before = 0;
    // scan path: this warp's segment of the slice and its counts
    const int seg = (((cnt + kWarps - 1) / kWarps) + 127) & ~127;
    const int ws = min(cnt, warp * seg), we = min(cnt, ws + seg);
    if (lists) {
        const int ns = s_nsure, nc = s_ncand;
        for (int i = tid; i < ns; i += kThreads) {
            const int p = s_sure[i];
            atomicOr(&s_bm_sel[p >> 5], 1u << (p & 31));
        }
        for (int i = tid; i < nc; i += kThreads) {
            const uint32_t m = s_ckey[i] & mask;
            const int p = s_cpos[i];
            if (m > prefix) atomicOr(&s_bm_sel[p >> 5], 1u << (p & 31));
            else if (m == prefix) atomicOr(&s_bm_cls[p >> 5], 1u << (p & 31));
        }
        __syncthreads();
        int nsel = 0, ncls = 0;
#pragma unroll
        for (int j = 0; j < kBmPer; ++j) {
            bsel[j] = s_bm_sel[tid * kBmPer + j];
            bcls[j] = s_bm_cls[tid * kBmPer + j];
            nsel += __popc(bsel[j]);
            ncls += __popc(bcls[j]);
        }
        // both counts are at most 8192 per CTA: one scan of the packed pair
        int tot = 0;
        const int before = block_exclusive((nsel << 16) | ncls, lane, warp, s_wsum, tot);
        cls_before = before & 0xFFFF;
        cta_gt = tot >> 16;
        cta_eq = tot & 0xFFFF;
    } else {
        int gt_w = 0, eq_w = 0;
        for (int base = ws; base < we; base += 128) {
            const int i0 = base + 4 * lane;
            float f[4];
            if (i0 + 3 < we) {
                const float4 q = *reinterpret_cast<const float4*>(src + i0);
                f[0] = q.x;
                f[1] = q.y;
                f[2] = q.z;
                f[3] = q.w;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) f[e] = i0 + e < we ? src[i0 + e] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (i0 + e < we) {
                    const uint32_t m = order_key(f[e]) & mask;
                    gt_w += m > prefix ? 1 : 0;
                    eq_w += m == prefix ? 1 : 0;
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gt_w += __shfl_xor_sync(0xffffffffu, gt_w, o);
            eq_w += __shfl_xor_sync(0xffffffffu, eq_w, o);
        }
        if (lane == 0) {
            s_warp_gt[warp] = gt_w;
            s_warp_eq[warp] = eq_w;
        }
        __syncthreads();
        for (int w = 0; w < kWarps; ++w) {
            cta_gt += s_warp_gt[w];
            cta_eq += s_warp_eq[w];
        }
    }
    if (warp == 0 && lane < kCluster) {  // this CTA's two counts into every CTA of the cluster
        const uint32_t a = mapa_u32(smem_u32(&s_counts[rank][0]), static_cast<uint32_t>(lane));
        st_cluster_u32(a, static_cast<uint32_t>(cta_gt));
        st_cluster_u32(a + 4, static_cast<uint32_t>(cta_eq));
    }
    // Every CTA's counts are in place, and every read of another CTA's shared
    // memory (histograms of the passes) is done: after this barrier no CTA
    // touches another's shared memory, so each may leave when it has written.
    cluster_sync_all();
    if (hrow)  // every CTA has read it: clear for the next step
        for (int j = 0; j < kOwnPer; ++j) hrow[static_cast<int>(rank) * kOwn + j * kThreads + tid] = 0;
    // offsets of this CTA: ranks below take their "above" keys and their share of the class
    int off = 0, eq_before = 0;
    for (int r = 0; r < static_cast<int>(rank); ++r) {
        const int take = max(0, min(s_counts[r][1], remaining - eq_before));
        off += s_counts[r][0] + take;
        eq_before += s_counts[r][1];
    }
    const int take_c = max(0, min(s_counts[rank][1], remaining - eq_before));

    if (lists) {
        // this thread's class members of rank < take_c join the selection
        int r = cls_before, nsel = 0;
#pragma unroll
        for (int j = 0; j < kBmPer; ++j) {
            uint32_t bits = bcls[j];
            while (bits != 0u && r < take_c) {
                const uint32_t low = bits & (0u - bits);
                bsel[j] |= low;
                bits ^= low;
                ++r;
            }
            nsel += __popc(bsel[j]);
        }
        int tot = 0;
        int pos = off + block_exclusive(nsel, lane, warp, s_wsum, tot);
#pragma unroll
        for (int j = 0; j < kBmPer; ++j) {
            uint32_t bits = bsel[j];
            const int p0 = lo + (tid * kBmPer + j) * 32;
            while (bits != 0u) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1u;
                if (pos < k) orow[pos] = p0 + b;
                ++pos;
            }
        }
        return;
    }

    // scan path: offsets of this warp inside the CTA, then its segment in order
    int sel_before = 0, eqb = 0;
    for (int w = 0; w < warp; ++w) {
        sel_before += s_warp_gt[w] + max(0, min(s_warp_eq[w], take_c - eqb));
        eqb += s_warp_eq[w];
    }
    int eq_run = 0, sel_run = 0;
    for (int base = ws; base < we; base += 128) {
        const int i0 = base + 4 * lane;
        float f[4];
        if (i0 + 3 < we) {
            const float4 q = *reinterpret_cast<const float4*>(src + i0);
            f[0] = q.x;
            f[1] = q.y;
            f[2] = q.z;
            f[3] = q.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) f[e] = i0 + e < we ? src[i0 + e] : 0.f;
        }
        bool gt[4], eq[4];
        int neq = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t m = order_key(f[e]) & mask;
            gt[e] = i0 + e < we && m > prefix;
            eq[e] = i0 + e < we && m == prefix;
            neq += eq[e] ? 1 : 0;
        }
        // class rank of each of this lane's keys: keys of the class before it
        int eq_rank = eqb + eq_run + warp_exclusive(neq, lane);
        bool sel[4];
        int nsel = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sel[e] = gt[e] || (eq[e] && eq_rank < take_c);
            eq_rank += eq[e] ? 1 : 0;
            nsel += sel[e] ? 1 : 0;
        }
        int pos = off + sel_before + sel_run + warp_exclusive(nsel, lane);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (sel[e]) {
                if (pos < k) orow[pos] = lo + i0 + e;
                ++pos;
            }
        }
        int tot_eq = neq, tot_sel = nsel;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            tot_eq += __shfl_xor_sync(0xffffffffu, tot_eq, o);
            tot_sel += __shfl_xor_sync(0xffffffffu, tot_sel, o);
        }
        eq_run += tot_eq;
        sel_run += tot_sel;
    }
}

// ------------------------------------------------------------ from candidates
// The selection from the indexer's candidates (keys at or above a proven
// lower bound on each row's k-th largest, as (order key << 32) | ~position)
// and the row's first-digit counts, which cover every key of the row.  One
// CTA per row: the counts give the boundary digit and the number of keys
// above it (all of them are candidates); one pass over the candidates marks
// those keys in a bitmap of the row's positions and lists the keys on the
// boundary digit; 8/8/4-bit passes over that list find the final class; the
// class's lowest positions join the selection, and a block scan of the
// bitmap writes the positions in ascending order.  The counts and the
// candidate count are cleared for the next step.
constexpr int kCMaxN = 262144;          // positions per row (the bitmaps)
constexpr int kCBmWords = kCMaxN / 32;  // 8192
constexpr int kCBmPer = kCBmWords / kThreads;
constexpr int kCListCap = 4096;         // boundary-digit keys held in shared memory
constexpr int kCDynSmem = 2 * kCBmWords * 4 + kCListCap * 8;
static_assert(kCBmPer * kThreads == kCBmWords, "bitmap words per thread");

__global__ void __launch_bounds__(kThreads, 1)
    topk_cand_kernel(const uint64_t* __restrict__ cand, int64_t ld, int32_t* __restrict__ cand_cnt,
                     const int32_t* __restrict__ n_valid, int k, int32_t* __restrict__ hist,
                     int32_t* __restrict__ out, int* err) {
    extern __shared__ __align__(16) uint8_t s_dyn[];
    uint32_t* s_sel = reinterpret_cast<uint32_t*>(s_dyn);         // [kCBmWords] selected positions
    uint32_t* s_cls = s_sel + kCBmWords;                           // [kCBmWords] final-class members
    uint32_t* s_lkey = s_cls + kCBmWords;                          // [kCListCap] boundary keys
    uint32_t* s_lpos = s_lkey + kCListCap;                         // [kCListCap] their positions
    __shared__ int s_h[kBins1];
    __shared__ int s_suf[kBins1 + 1];
    __shared__ int s_wsum[kWarps];
    __shared__ int s_sel0[3], s_pass[3];
    __shared__ int s_nl;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x;
    int n = n_valid[row];
    n = n < 0 ? 0 : (n > ld ? static_cast<int>(ld) : n);
    int32_t* orow = out + static_cast<int64_t>(row) * k;
    int32_t* hrow = hist + static_cast<int64_t>(row) * kHistBins;
    const uint64_t* crow = cand + static_cast<int64_t>(row) * ld;
    const int cnt = min(cand_cnt[row], n);

    if (n <= k) {  // every position is selected; the rest is padding
        for (int s = tid; s < k; s += kThreads) orow[s] = s < n ? s : -1;
    } else {
        // ---- 1. the boundary digit from the row's counts (highest bins first)
        constexpr int kPer = kBins0 / kThreads;
        const int b_hi = kBins0 - 1 - tid * kPer;
        int hv[kPer], mine = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            hv[j] = hrow[b_hi - j];
            mine += hv[j];
        }
        if (tid == 0) {
            s_sel0[0] = 0;
            s_sel0[1] = 0;
            s_sel0[2] = 0;
            s_nl = 0;
        }
#pragma unroll
        for (int j = 0; j < kCBmPer; ++j) {
            s_sel[tid * kCBmPer + j] = 0u;
            s_cls[tid * kCBmPer + j] = 0u;
        }
        int total = 0;
        int above = block_exclusive(mine, lane, warp, s_wsum, total);
        if (tid == 0 && total != n) record_error(err, kErrTopkRow | 1);  // the counts do not cover the row
        if (above < k && k <= above + mine) {
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
        __syncthreads();
        const uint32_t d0 = static_cast<uint32_t>(s_sel0[0]);
        int remaining = k - s_sel0[1];
        // ---- 2. candidates above the boundary digit are selected; those on it are listed
        for (int i = tid; i < cnt; i += kThreads) {
            const uint64_t v = crow[i];
            const uint32_t key = static_cast<uint32_t>(v >> 32), pos = 0xFFFFFFFFu - static_cast<uint32_t>(v);
            if (pos >= static_cast<uint32_t>(n)) continue;
            const uint32_t d = key >> 20;
            if (d > d0) {
                atomicOr(&s_sel[pos >> 5], 1u << (pos & 31));
            } else if (d == d0) {
                const int slot = atomicAdd(&s_nl, 1);
                if (slot < kCListCap) {
                    s_lkey[slot] = key;
                    s_lpos[slot] = pos;
                }
            }
        }
        __syncthreads();
        const bool listed = s_nl <= kCListCap;
        const int nlist = listed ? s_nl : cnt;
        // boundary key j of the list (or candidate j when the list overflowed):
        // returns false when it is not on the boundary digit
        auto bkey = [&](int j, uint32_t& key, uint32_t& pos) -> bool {
            if (listed) {
                key = s_lkey[j];
                pos = s_lpos[j];
                return true;
            }
            const uint64_t v = crow[j];
            key = static_cast<uint32_t>(v >> 32);
            pos = 0xFFFFFFFFu - static_cast<uint32_t>(v);
            return (key >> 20) == d0 && pos < static_cast<uint32_t>(n);
        };
        // ---- 3. refinement passes over the boundary keys (bits 19..12, 11..4, 3..0)
        uint32_t prefix = d0 << 20, mask = 0xFFF00000u;
        if (s_sel0[2] != remaining) {
            for (int pass = 0; pass < 3; ++pass) {
                const int shift = pass == 0 ? 12 : (pass == 1 ? 4 : 0);
                const uint32_t dmask = pass == 2 ? 15u : 255u;
                if (tid < kBins1) s_h[tid] = 0;
                __syncthreads();
                for (int j = tid; j < nlist; j += kThreads) {
                    uint32_t key, pos;
                    if (bkey(j, key, pos) && (key & mask) == prefix) atomicAdd(&s_h[(key >> shift) & dmask], 1);
                }
                __syncthreads();
                if (tid < kBins1) {
                    const int in = warp_suffix(s_h[tid], lane);
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
                        s_pass[0] = 0;
                        s_pass[1] = 0;
                        s_pass[2] = -1;
                    }
                }
                __syncthreads();
                if (tid < kBins1) {
                    const int here = s_suf[tid], up = s_suf[tid + 1];
                    if (here >= remaining && up < remaining) {
                        s_pass[0] = tid;
                        s_pass[1] = up;
                        s_pass[2] = here - up;
                    }
                }
                __syncthreads();
                remaining -= s_pass[1];
                prefix |= static_cast<uint32_t>(s_pass[0]) << shift;
                mask |= dmask << shift;
                const bool whole = s_pass[2] == remaining;
                __syncthreads();  // s_pass is rewritten by the next pass
                if (whole) break;
            }
        }
        // ---- 4. boundary keys above the final class are selected; its members marked
        for (int j = tid; j < nlist; j += kThreads) {
            uint32_t key, pos;
            if (!bkey(j, key, pos)) continue;
            const uint32_t m = key & mask;
            if (m > prefix) atomicOr(&s_sel[pos >> 5], 1u << (pos & 31));
            else if (m == prefix) atomicOr(&s_cls[pos >> 5], 1u << (pos & 31));
        }
        __syncthreads();
        // ---- 5. the class's `remaining` lowest positions join, then ordered writes
        uint32_t bsel[kCBmPer];
        int ncls = 0;
#pragma unroll
        for (int j = 0; j < kCBmPer; ++j) ncls += __popc(s_cls[tid * kCBmPer + j]);
        int tot = 0;
        int r = block_exclusive(ncls, lane, warp, s_wsum, tot);
        int nsel = 0;
#pragma unroll
        for (int j = 0; j < kCBmPer; ++j) {
            uint32_t bits = s_cls[tid * kCBmPer + j];
            uint32_t selw = s_sel[tid * kCBmPer + j];
            while (bits != 0u && r < remaining) {
                const uint32_t low = bits & (0u - bits);
                selw |= low;
                bits ^= low;
                ++r;
            }
            bsel[j] = selw;
            nsel += __popc(selw);
        }
        __syncthreads();  // s_wsum is reused by the next scan
        int pos = block_exclusive(nsel, lane, warp, s_wsum, tot);
#pragma unroll
        for (int j = 0; j < kCBmPer; ++j) {
            uint32_t bits = bsel[j];
            const int p0 = (tid * kCBmPer + j) * 32;
            while (bits != 0u) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1u;
                if (pos < k) orow[pos] = p0 + b;
                ++pos;
            }
        }
    }
    // the row's counts and candidate count, cleared for the next step
    __syncthreads();
    for (int i = tid; i < kHistBins; i += kThreads) hrow[i] = 0;
    if (tid == 0) cand_cnt[row] = 0;
}

}  // namespace

sa_status topk_select_launch(const float* scores, int64_t ld, const int32_t* n_valid, int rows, int k,
                             int32_t* hist, int32_t* idx_out, cudaStream_t st) {
    // each CTA's slice starts on a 16-byte boundary (scores_ld is a multiple of 4)
    const int chunk = static_cast<int>((((ld + kCluster - 1) / kCluster) + 3) & ~int64_t(3));
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
    if (e != cudaSuccess) return launch_status(e);
    topk_kernel<<<rows * kCluster, kThreads, kDynSmem, st>>>(scores, ld, n_valid, k, chunk, hist, idx_out);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

namespace sa {

sa_status topk_cand_launch(const uint64_t* cand, int64_t cand_ld, int32_t* cand_cnt, const int32_t* n_valid,
                           int rows, int k, int32_t* hist, int32_t* idx_out, int* err, cudaStream_t st) {
    if (cand_ld > kCMaxN) return SA_EUNSUPPORTED;
    cudaError_t e = cudaFuncSetAttribute(topk_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCDynSmem);
    if (e != cudaSuccess) return launch_status(e);
    topk_cand_kernel<<<rows, kThreads, kCDynSmem, st>>>(cand, cand_ld, cand_cnt, n_valid, k, hist, idx_out, err);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

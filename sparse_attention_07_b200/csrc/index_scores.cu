// index_scores.cu — lightning-indexer kernels.
//
// Computes I[r][s] = sum_j w[r][j] * ReLU(q[r][j] . k(seq(r), s)) for every
// visible position ("Sparse Attention 数学学习笔记" §9, index score I_{t,s};
// "MLA 与稀疏注意力" DSA section: one key per token shared by all indexer heads,
// per-head queries and weights, no scale, no softmax).
//
// Tensor-core path (fp8 e4m3, d_I = 128): for one sequence the score tile of
// 128 keys x N query-heads is the product K_tile [128 x 128] . Q^T [128 x N]
// (N = R rows x H_I heads), issued as four tcgen05.mma kind::f8f6f4 of
// K = 32 into a TMEM accumulator; the epilogue thread that owns a key (TMEM
// lane) applies ReLU, the weights and the head sum in registers and writes one
// fp32 score per row.  Persistent CTAs walk balanced contiguous ranges of
// (row group, key tile) items; a TMA producer warp streams 16 KB key tiles
// (two 64-token pages) through a ring, an MMA warp issues, and 4 or 8
// epilogue warps drain a ring of 2 or 4 TMEM accumulators.  The producer looks
// up 32 items at a time (one per lane), so its issue loop holds no dependent
// global loads.  A ring stage stays busy from its TMA issue (about 3.4 us to
// land under full load) until its MMAs complete, so the bytes in flight per
// SM set the rate: one-row groups (decode) therefore run two CTAs per SM, each
// with a 5-stage ring, at most 128 registers per thread and 256 TMEM columns
// (4.7 TB/s on the ragged workload against 3.3 TB/s with one 6-stage CTA).
// Grouped rows (prefill) keep one CTA per SM with a 6-stage ring.
//
// CUDA-core path (fp32 or fp8, d_I <= 128, H_I <= 64): one thread per key.
#include <cuda_fp8.h>

#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

// First-digit histogram of the scores a warp writes: lanes with equal digits
// add once (global atomics, one per distinct digit of the warp).
__device__ __forceinline__ void hist_add_global(int32_t* hist, bool active, uint32_t digit, int lane) {
    const unsigned am = __ballot_sync(0xffffffffu, active);
    if (active) {
        const unsigned peers = __match_any_sync(am, digit);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
    }
}

constexpr int kPage = 64;
constexpr int kTileKeys = 128;
constexpr int kStageBytes = kTileKeys * 128;  // 128 keys x 128 fp8
constexpr int kMaxRows = 4096;

__device__ __forceinline__ int clamp_vis(const IdxArgs& a, int r) {
    int n = a.n_visible[r];
    int cap = a.pages_per_seq * kPage;
    if (cap > a.scores_ld) cap = static_cast<int>(a.scores_ld);
    return n < 0 ? 0 : (n > cap ? cap : n);
}

__device__ __forceinline__ int seq_of(const IdxArgs& a, int r) { return a.seq_of_row ? a.seq_of_row[r] : r; }

__device__ __forceinline__ int page_of(const IdxArgs& a, int seq, int p) {
    return a.page_table ? a.page_table[static_cast<int64_t>(seq) * a.pages_per_seq + p]
                        : seq * a.pages_per_seq + p;
}

// In-place block-wide scan over n ints in shared memory (all threads call).
// Sum (exclusive, returns total) or max (inclusive).
template <bool kMax>
__device__ int block_scan(int* a, int n, int* warp_buf) {
    const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
    const int per = (n + nt - 1) / nt;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int acc = kMax ? INT_MIN : 0;
    for (int i = lo; i < hi; ++i) acc = kMax ? max(acc, a[i]) : acc + a[i];
    int incl = acc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl = kMax ? max(incl, v) : incl + v;
    }
    if (lane == 31) warp_buf[wid] = incl;
    __syncthreads();
    if (tid == 0) {
        int run = kMax ? INT_MIN : 0;
        for (int w = 0; w < nw; ++w) {
            int v = warp_buf[w];
            warp_buf[w] = run;
            run = kMax ? max(run, v) : run + v;
        }
        warp_buf[nw] = run;
    }
    __syncthreads();
    int excl_t = incl;  // exclusive prefix of this thread's chunk
    {
        int up = __shfl_up_sync(0xffffffffu, incl, 1);
        int base = warp_buf[wid];
        if (kMax)
            excl_t = lane == 0 ? base : max(base, up);
        else
            excl_t = lane == 0 ? base : base + up;
    }
    int total = warp_buf[nw];
    __syncthreads();
    int run = excl_t;
    for (int i = lo; i < hi; ++i) {
        int v = a[i];
        if (kMax) {
            run = max(run, v);
            a[i] = run;
        } else {
            a[i] = run;
            run += v;
        }
    }
    __syncthreads();
    return total;
}

// Walks the (group, tile) items of one CTA in order.
struct ItemWalk {
    const int* prefix;  // [G+1] tile prefix
    int G, item, end, g, t;
    __device__ bool valid() const { return item < end; }
    __device__ int tiles(int gg) const { return prefix[gg + 1] - prefix[gg]; }
    __device__ void start(int begin, int end_) {
        item = begin;
        end = end_;
        // largest g with prefix[g] <= item (and a nonempty group)
        int lo = 0, hi = G;  // prefix[G] = total > item
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (prefix[mid] <= item) lo = mid; else hi = mid;
        }
        g = lo;
        while (g < G && tiles(g) == 0) ++g;
        t = item - prefix[g];
    }
    __device__ void next() {
        ++item;
        if (++t >= tiles(g)) {
            do { ++g; } while (g < G && tiles(g) == 0);
            t = 0;
        }
    }
};

template <int NH, int R, int NEPI, bool kCand = false>
struct TcCfg {
    static constexpr int N = R * NH;                     // MMA N (rows x heads)
    // accumulator buffers: four where they fit in TMEM (the MMA runs further ahead of the epilogue)
    static constexpr int kAcc = (4 * N <= 512) ? 4 : 2;
    static constexpr int kTmemCols = (kAcc * N <= 32) ? 32 : (kAcc * N <= 64 ? 64 : (kAcc * N <= 128 ? 128 : (kAcc * N <= 256 ? 256 : 512)));
    static constexpr int kQBytes = N * 128;
    // warps: NEPI epilogue, TMA producer, MMA issuer; candidate mode adds the
    // warp that keeps the row's candidate bound up to date
    static constexpr int kThreads = 32 * (NEPI + 2 + (kCand ? 1 : 0));
    // key-tile ring: one-row groups (decode) keep five stages so that two CTAs
    // fit on an SM (shared memory and tensor memory) and stream side by side
    static constexpr int kStages = R == 1 ? 5 : 6;
    // registers per thread: one-row groups with up to 64 heads stay within 128
    // so that two CTAs fit; otherwise whatever one CTA of kThreads can have.
    // The register file is split over the SM's four sub-partitions (16K
    // registers each) and a CTA's warps are spread over them, so the bound is
    // set by the sub-partition holding ceil(warps / 4) warps (10 warps: 168,
    // not 65536 / 320).
    static constexpr int kTwoPerSm = R == 1 && NH <= 64;
    static constexpr int kWarpsPerSubpart = (kThreads / 32 + 3) / 4;
    static constexpr int kRegCap = (16384 / (32 * kWarpsPerSubpart)) & ~7;
    static constexpr int kMaxReg = kTwoPerSm ? 128 : (kRegCap > 255 ? 255 : kRegCap);
    // shared layout (offsets from a 1024-aligned base); the three group tables
    // (prefix, group start, group length) follow, (rows + 1) ints each, rounded
    static constexpr int kOffStages = 0;
    static constexpr int kOffQ = kOffStages + kStages * kStageBytes;
    static constexpr int kOffW = kOffQ + 2 * kQBytes;
    static constexpr int kOffTables = kOffW + NEPI * R * NH * 4;
    static int table_ints(int rows) { return (rows + 1 + 3) & ~3; }
    static size_t smem_bytes(int rows) { return kOffTables + 3 * static_cast<size_t>(table_ints(rows)) * 4 + 1024; }
};

template <int NH, int R, int NEPI, bool kCand>
__global__ void __launch_bounds__((TcCfg<NH, R, NEPI, kCand>::kThreads)) __maxnreg__((TcCfg<NH, R, NEPI, kCand>::kMaxReg))
    idx_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const IdxArgs a) {
    using C = TcCfg<NH, R, NEPI, kCand>;
    static_assert(!kCand || R == 1, "candidates are emitted by one-row groups");
    constexpr int N = C::N;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* s_stage = sm + C::kOffStages;
    uint8_t* s_q = sm + C::kOffQ;
    float* s_w = reinterpret_cast<float*>(sm + C::kOffW);
    const int tab = (a.rows + 1 + 3) & ~3;
    int* s_prefix = reinterpret_cast<int*>(sm + C::kOffTables);
    int* s_gstart = s_prefix + tab;
    int* s_gnk = s_gstart + tab;  // longest visible length in the group

    __shared__ uint64_t bar_full[C::kStages], bar_empty[C::kStages], bar_qfull[2], bar_qempty[2], bar_accfull[C::kAcc],
        bar_accempty[C::kAcc], bar_final;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_warpbuf[40];
    __shared__ int s_G;
    // candidate mode: (row + 1) << 32 | bound digit, published by the bound warp;
    // the epilogue's current row, its tiles done in that row, and "finished"
    __shared__ volatile unsigned long long s_bound;
    __shared__ volatile int s_epi_row, s_epi_tiles, s_epi_done;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WaitCtx wc{a.err, &s_abort};

    if (tid == 0) {
        s_abort = 0;
        s_bound = 0ull;
        s_epi_row = -1;
        s_epi_tiles = 0;
        s_epi_done = 0;
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_qfull[i], 1);
            mbar_init(&bar_qempty[i], 1);
        }
        for (int i = 0; i < C::kAcc; ++i) {
            mbar_init(&bar_accfull[i], 1);
            mbar_init(&bar_accempty[i], NEPI);
        }
        mbar_init(&bar_final, 1);
        fence_mbar_init();
    }
    if (warp == NEPI + 1) {
        tmem_alloc(&s_tmem, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == NEPI && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
    }

    // ---- group table: consecutive rows of one sequence, at most R per group
    const int rows = a.rows;
    int* tmp = reinterpret_cast<int*>(s_stage);  // scratch (stage ring is idle yet)
    int G;
    if (R == 1 || a.seq_of_row == nullptr) {
        G = rows;
        for (int g = tid; g <= rows; g += blockDim.x) s_gstart[g] = g;
        // the group lengths below read entries other warps wrote (g + 1)
        __syncthreads();
    } else {
        int* flag = tmp + kMaxRows;
        for (int r = tid; r < rows; r += blockDim.x)
            tmp[r] = (r == 0 || a.seq_of_row[r] != a.seq_of_row[r - 1]) ? r : 0;
        __syncthreads();
        block_scan<true>(tmp, rows, s_warpbuf);  // run start of each row
        for (int r = tid; r < rows; r += blockDim.x) flag[r] = ((r - tmp[r]) % R == 0) ? 1 : 0;
        __syncthreads();
        for (int r = tid; r < rows; r += blockDim.x) tmp[r] = flag[r];
        __syncthreads();
        G = block_scan<false>(tmp, rows, s_warpbuf);  // group index of group starts
        for (int r = tid; r < rows; r += blockDim.x)
            if (flag[r]) s_gstart[tmp[r]] = r;
        if (tid == 0) s_gstart[G] = rows;
        __syncthreads();
    }
    for (int g = tid; g < G; g += blockDim.x) {
        int nk = 0;
        for (int r = s_gstart[g]; r < s_gstart[g + 1]; ++r) nk = max(nk, clamp_vis(a, r));
        s_gnk[g] = nk;
        s_prefix[g] = (nk + kTileKeys - 1) / kTileKeys;
    }
    __syncthreads();
    const int total = block_scan<false>(s_prefix, G, s_warpbuf);
    if (tid == 0) {
        s_prefix[G] = total;
        s_G = G;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    const int64_t begin = static_cast<int64_t>(blockIdx.x) * total / gridDim.x;
    const int64_t end = static_cast<int64_t>(blockIdx.x + 1) * total / gridDim.x;
    ItemWalk it;
    it.prefix = s_prefix;
    it.G = G;

    if (warp == NEPI) {
        // ------------------------------------------------ TMA producer
        // The warp describes the next 32 items at once (lane i: item + i: its
        // group, key tile and the physical pages of the tile's two 64-key pages),
        // so lane 0's issue loop holds no dependent global loads.
        int stage = 0;
        uint32_t phase = 0;
        int gcount = -1, prev_g = -1;
        int64_t n_issued = 0;
        bool ok = true;
        for (int item = static_cast<int>(begin); ok && item < static_cast<int>(end); item += 32) {
            const int my_item = item + lane;
            int my_g = 0, my_p0 = 0, my_p1 = -1;
            if (my_item < end) {
                int lo = 0, hi = G;  // largest g with prefix[g] <= my_item (a non-empty group)
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (s_prefix[mid] <= my_item) lo = mid; else hi = mid;
                }
                my_g = lo;
                const int t = my_item - s_prefix[lo];
                const int seq = seq_of(a, s_gstart[lo]);
                my_p0 = page_of(a, seq, 2 * t);
                if ((2 * t + 1) * kPage < s_gnk[lo]) my_p1 = page_of(a, seq, 2 * t + 1);
            }
            const int n = min(32, static_cast<int>(end) - item);
            for (int i = 0; i < n; ++i) {
                const int g = __shfl_sync(0xffffffffu, my_g, i);
                const int p0 = __shfl_sync(0xffffffffu, my_p0, i);
                const int p1 = __shfl_sync(0xffffffffu, my_p1, i);
                if (lane == 0) {
                    if (g != prev_g) {
                        ++gcount;
                        prev_g = g;
                        const int qb = gcount & 1;
                        if (gcount >= 2) ok = mbar_wait(&bar_qempty[qb], ((gcount >> 1) - 1) & 1, wc, kErrIdxWait | 1);
                        if (ok) {
                            mbar_arrive_expect_tx(&bar_qfull[qb], C::kQBytes);
                            tma_load_2d(s_q + qb * C::kQBytes, &tm_q, &bar_qfull[qb], 0, s_gstart[g] * NH);
                        }
                    }
                    if (ok) ok = mbar_wait(&bar_empty[stage], phase ^ 1, wc, kErrIdxWait | 2);
                    if (ok) {
                        mbar_arrive_expect_tx(&bar_full[stage], (p1 >= 0 ? 2 : 1) * (kStageBytes / 2));
                        uint8_t* dst = s_stage + stage * kStageBytes;
                        tma_load_2d(dst, &tm_k, &bar_full[stage], 0, p0 * kPage);
                        if (p1 >= 0) tma_load_2d(dst + kStageBytes / 2, &tm_k, &bar_full[stage], 0, p1 * kPage);
                        ++n_issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // drain: every load still in flight lands before the CTA can exit
        if (lane == 0) {
            int dummy = 0;
            WaitCtx dw(a.err, reinterpret_cast<volatile int*>(&dummy), kWaitLimitNs);  // drain: fixed limit
            for (int64_t i = n_issued - C::kStages; i < n_issued; ++i) {
                if (i < 0) continue;
                mbar_wait(&bar_full[i % C::kStages], static_cast<uint32_t>((i / C::kStages) & 1), dw, kErrIdxWait | 7);
            }
        }
        __syncwarp();
    } else if (warp == NEPI + 1) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_f32acc(0, 0, false, false, 128, N);
        int stage = 0;
        uint32_t phase = 0;
        int gcount = -1, prev_g = -1;
        int64_t acc = 0;
        if (begin < end) {
            for (it.start(static_cast<int>(begin), static_cast<int>(end)); it.valid(); it.next()) {
                bool ok = true;
                if (it.g != prev_g) {
                    if (prev_g >= 0 && lane == 0) tc_commit(&bar_qempty[gcount & 1]);
                    ++gcount;
                    prev_g = it.g;
                    if (lane == 0) ok = mbar_wait(&bar_qfull[gcount & 1], (gcount >> 1) & 1, wc, kErrIdxWait | 3);
                }
                const int buf = static_cast<int>(acc % C::kAcc);
                if (ok && lane == 0) ok = mbar_wait(&bar_full[stage], phase, wc, kErrIdxWait | 4);
                if (ok && lane == 0 && acc >= C::kAcc)
                    ok = mbar_wait(&bar_accempty[buf], static_cast<uint32_t>((acc / C::kAcc - 1) & 1), wc, kErrIdxWait | 5);
                if (ok && lane == 0) {
                    tc_fence_after();
                    const uint64_t da = sdesc(smem_u32(s_stage + stage * kStageBytes), 16, 1024, kSw128);
                    const uint64_t db = sdesc(smem_u32(s_q + (gcount & 1) * C::kQBytes), 16, 1024, kSw128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f8_ss(tmem + buf * N, da + 2 * kk, db + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                    tc_commit(&bar_empty[stage]);
                    tc_commit(&bar_accfull[buf]);
                }
                __syncwarp();
                if (s_abort) break;
                ++acc;
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (lane == 0) {  // all issued MMAs complete before TMEM is released
            int dummy = 0;
            WaitCtx dw(a.err, reinterpret_cast<volatile int*>(&dummy), kWaitLimitNs);  // drain: fixed limit
            tc_commit(&bar_final);
            mbar_wait(&bar_final, 0, dw, kErrIdxWait | 8);
        }
        __syncwarp();
    } else if (kCand && warp == NEPI + 2) {
        // ------------------------------------------------ candidate bound
        // Every kBoundTiles tiles of the epilogue's current row, the warp reads
        // the row's first-digit counts (every CTA's keys so far) from the top
        // and publishes the digit d at which they reach k: at least k keys
        // already seen lie at or above d, so no key below d is among the k
        // largest (the counts only grow, so a stale bound is lower, never
        // wrong).  Lane l sums bins 4095-128l down to 3968-128l.
        constexpr int kBoundTiles = 8;
        // The wait limit applies to the epilogue's progress (a row or tile
        // count that stops changing), not to the kernel's whole run.
        int last_row = -1, last_tiles = 0, seen_row = -1, seen_tiles = 0;
        unsigned long long t0 = global_ns();
        while (!s_epi_done) {
            const int row = s_epi_row, tiles = s_epi_tiles;
            if (row != seen_row || tiles != seen_tiles) {
                seen_row = row;
                seen_tiles = tiles;
                t0 = global_ns();
            }
            if (row < 0 || (row == last_row && tiles - last_tiles < kBoundTiles)) {
                if (global_ns() - t0 > wc.limit_ns) {
                    record_error(a.err, kErrIdxWait | 9);
                    break;
                }
                __nanosleep(256);
                continue;
            }
            const int32_t* hr = a.hist + static_cast<int64_t>(row) * kHistBins;
            const int4* src = reinterpret_cast<const int4*>(hr + kHistBins - 128 * (lane + 1));
            int tot = 0;
#pragma unroll 8
            for (int j = 0; j < 32; ++j) {
                const int4 v = __ldcg(src + j);
                tot += v.x + v.y + v.z + v.w;
            }
            int incl = tot;  // keys in this lane's bins and the bins above them
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int above = incl - tot;
            unsigned found = 0u;
            if (above < a.k && a.k <= incl) {
                int run = above;
                for (int j = 31; j >= 0 && !found; --j) {  // highest bins first
                    const int4 v = __ldcg(src + j);
                    const int c4[4] = {v.w, v.z, v.y, v.x};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        run += c4[e];
                        if (!found && run >= a.k) found = static_cast<unsigned>(kHistBins - 128 * (lane + 1) + 4 * j + 3 - e) + 1u;
                    }
                }
            }
            found = __reduce_max_sync(0xffffffffu, found);
            if (lane == 0 && found != 0u)
                s_bound = (static_cast<unsigned long long>(row + 1) << 32) | (found - 1u);
            __syncwarp();
            last_row = row;
            last_tiles = tiles;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0..NEPI-1)
        const int quarter = warp & 3;
        constexpr int kHalves = NEPI / 4;
        constexpr int kRowsPerHalf = (R + kHalves - 1) / kHalves;
        const int half = warp >> 2;
        int64_t acc = 0;
        int prev_g = -1;
        int g_r0 = 0, g_cnt = 0;
        int nvis[kRowsPerHalf];
        float wr[R == 1 ? NH : 1];  // one-row groups: the row's weights
        float* w_own = s_w + warp * R * NH;  // this warp's copy of the group's weights
        if (begin < end) {
            for (it.start(static_cast<int>(begin), static_cast<int>(end)); it.valid(); it.next()) {
                if (it.g != prev_g) {
                    prev_g = it.g;
                    g_r0 = s_gstart[it.g];
                    g_cnt = s_gstart[it.g + 1] - g_r0;
                    if constexpr (R == 1) {
#pragma unroll
                        for (int x = 0; x < NH; ++x) wr[x] = a.w[static_cast<int64_t>(g_r0) * NH + x];
                    }
                    if (kCand && warp == 0 && lane == 0) {
                        s_epi_tiles = 0;
                        s_epi_row = g_r0;
                    }
                    __syncwarp();
                    for (int i = lane; i < R * NH; i += 32) {
                        const int gi = i / NH;
                        w_own[i] = gi < g_cnt ? a.w[static_cast<int64_t>(g_r0 + gi) * NH + (i % NH)] : 0.f;
                    }
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < kRowsPerHalf; ++j) {
                        const int gi = half * kRowsPerHalf + j;
                        nvis[j] = gi < g_cnt ? clamp_vis(a, g_r0 + gi) : 0;
                    }
                }
                const int buf = static_cast<int>(acc % C::kAcc);
                if (!warp_wait(&bar_accfull[buf], static_cast<uint32_t>((acc / C::kAcc) & 1), wc, kErrIdxWait | 6)) break;
                tc_fence_after();
                const int s = it.t * kTileKeys + quarter * 32 + lane;
                if constexpr (R == 1) {
                    // one row per group: its weights sit in registers; four independent
                    // accumulators (on integer inputs every partial sum is exact, so the
                    // order of the additions does not change the result)
                    float acc4[4] = {0.f, 0.f, 0.f, 0.f};
                    const uint32_t col = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * N;
                    if constexpr (NH == 16) {
                        uint32_t v[16];
                        tmem_ld16(col, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int x = 0; x < 16; ++x) acc4[x & 3] = fmaf(wr[x], fmaxf(__uint_as_float(v[x]), 0.f), acc4[x & 3]);
                    } else {
#pragma unroll
                        for (int c = 0; c < NH; c += 64) {
                            uint32_t v0[32], v1[32];
                            tmem_ld32(col + c, v0);
                            if (c + 32 < NH) tmem_ld32(col + c + 32, v1);
                            tmem_ld_wait();
#pragma unroll
                            for (int x = 0; x < 32; ++x)
                                acc4[x & 3] = fmaf(wr[c + x], fmaxf(__uint_as_float(v0[x]), 0.f), acc4[x & 3]);
                            if (c + 32 < NH) {
#pragma unroll
                                for (int x = 0; x < 32; ++x)
                                    acc4[x & 3] = fmaf(wr[c + 32 + x], fmaxf(__uint_as_float(v1[x]), 0.f), acc4[x & 3]);
                            }
                        }
                    }
                    const float sc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
                    const bool live = s < nvis[0] && g_cnt > 0;
                    if constexpr (kCand) {
                        // keys at or above the row's bound, as (key << 32) | ~position
                        const uint32_t key = score_order_key(sc);
                        const unsigned long long bnd = s_bound;
                        const uint32_t thr = static_cast<int>(bnd >> 32) == g_r0 + 1 ? static_cast<uint32_t>(bnd) : 0u;
                        const bool emit = live && (key >> 20) >= thr;
                        const unsigned bm = __ballot_sync(0xffffffffu, emit);
                        if (bm != 0u) {
                            int base = 0;
                            if (lane == 0) base = atomicAdd(a.cand_cnt + g_r0, __popc(bm));
                            base = __shfl_sync(0xffffffffu, base, 0);
                            // a count left over from a step whose Top-K did not run cannot write past the row
                            const int slot = base + __popc(bm & ((1u << lane) - 1u));
                            if (emit && slot < a.cand_ld)
                                a.cand[static_cast<int64_t>(g_r0) * a.cand_ld + slot] =
                                    (static_cast<uint64_t>(key) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(s));
                        }
                    } else {
                        if (live) a.scores[static_cast<int64_t>(g_r0) * a.scores_ld + s] = sc;
                    }
                    if (a.hist) hist_add_global(a.hist + static_cast<int64_t>(g_r0) * kHistBins, live,
                                                score_order_key(sc) >> 20, lane);
                } else {
#pragma unroll
                for (int j = 0; j < kRowsPerHalf; ++j) {
                    const int gi = half * kRowsPerHalf + j;
                    if (gi < R && gi < g_cnt) {
                        float sum = 0.f;
                        const uint32_t col = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * N + gi * NH;
                        if constexpr (NH < 32) {
                            uint32_t v[16];
                            tmem_ld16(col, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int x = 0; x < 16; ++x) sum += w_own[gi * NH + x] * fmaxf(__uint_as_float(v[x]), 0.f);
                        } else {
#pragma unroll
                            for (int c = 0; c < NH; c += 32) {
                                uint32_t v[32];
                                tmem_ld32(col + c, v);
                                tmem_ld_wait();
#pragma unroll
                                for (int x = 0; x < 32; ++x)
                                    sum += w_own[gi * NH + c + x] * fmaxf(__uint_as_float(v[x]), 0.f);
                            }
                        }
                        const bool live = s < nvis[j];
                        if (live) a.scores[static_cast<int64_t>(g_r0 + gi) * a.scores_ld + s] = sum;
                        if (a.hist) hist_add_global(a.hist + static_cast<int64_t>(g_r0 + gi) * kHistBins, live,
                                                    score_order_key(sum) >> 20, lane);
                    }
                }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_accempty[buf]);
                if (kCand && warp == 0 && lane == 0) s_epi_tiles = s_epi_tiles + 1;
                ++acc;
            }
        }
        if (kCand && warp == 0 && lane == 0) s_epi_done = 1;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == NEPI + 1) tmem_dealloc(tmem, C::kTmemCols);
}

// ------------------------------------------------------------ CUDA-core path
template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_fp8_e4m3>(const __nv_fp8_e4m3* p) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    __nv_fp8_e4m3 b[4];
    *reinterpret_cast<uint32_t*>(b) = u;
    return make_float4(float(b[0]), float(b[1]), float(b[2]), float(b[3]));
}

template <typename T, int NH>
__global__ void __launch_bounds__(128) idx_cc_kernel(const T* __restrict__ q, const T* __restrict__ kc, const IdxArgs a) {
    __shared__ float s_q[NH * 128];
    __shared__ float s_w[NH];
    const int r = blockIdx.y;
    const int d_I = a.d_I;
    for (int i = threadIdx.x; i < NH * d_I; i += blockDim.x) {
        const int j = i / d_I, d = i % d_I;
        s_q[j * 128 + d] = j < a.H_I ? float(q[(static_cast<int64_t>(r) * a.H_I + j) * d_I + d]) : 0.f;
    }
    for (int j = threadIdx.x; j < NH; j += blockDim.x) s_w[j] = j < a.H_I ? a.w[static_cast<int64_t>(r) * a.H_I + j] : 0.f;
    __syncthreads();
    const int nv = clamp_vis(a, r);
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= nv) return;
    const int seq = seq_of(a, r);
    const int page = page_of(a, seq, s / kPage);
    if (page < 0 || page >= a.pool_pages) {  // precondition broken: no read outside the pool
        a.scores[static_cast<int64_t>(r) * a.scores_ld + s] = 0.f;
        if (a.hist) atomicAdd(&a.hist[static_cast<int64_t>(r) * kHistBins + (score_order_key(0.f) >> 20)], 1);
        return;
    }
    const int64_t row = static_cast<int64_t>(page) * kPage + (s % kPage);
    const T* kp = kc + row * d_I;
    float dot[NH];
#pragma unroll
    for (int j = 0; j < NH; ++j) dot[j] = 0.f;
    for (int d = 0; d < d_I; d += 4) {
        const float4 kv = load4<T>(kp + d);
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            const float* qq = s_q + j * 128 + d;
            dot[j] += qq[0] * kv.x + qq[1] * kv.y + qq[2] * kv.z + qq[3] * kv.w;
        }
    }
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < NH; ++j) sum += s_w[j] * fmaxf(dot[j], 0.f);
    a.scores[static_cast<int64_t>(r) * a.scores_ld + s] = sum;
    if (a.hist) atomicAdd(&a.hist[static_cast<int64_t>(r) * kHistBins + (score_order_key(sum) >> 20)], 1);
}

template <typename T, int NH>
sa_status launch_cc(const void* q, const void* kc, const IdxArgs& a, cudaStream_t st) {
    const int L = a.pages_per_seq * kPage;
    dim3 grid((L + 127) / 128, a.rows);
    idx_cc_kernel<T, NH><<<grid, 128, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(kc), a);
    return launch_status(cudaGetLastError());
}

template <int NH, int R, int NEPI, bool kCand = false>
sa_status launch_tc(const void* q, const void* kc, const IdxArgs& a, cudaStream_t st) {
    using C = TcCfg<NH, R, NEPI, kCand>;
    CUtensorMap tk, tq;
    // keys: [pool rows][128 bytes]; rows outside the pool read as zero
    const uint64_t kdims[2] = {128, static_cast<uint64_t>(a.pool_pages) * kPage};
    const uint64_t kstr[1] = {128};
    const uint32_t kbox[2] = {128, kPage};
    if (!encode_tiled(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, kc, kdims, kstr, kbox, CU_TENSOR_MAP_SWIZZLE_128B))
        return SA_ECUDA;
    const uint64_t qdims[2] = {128, static_cast<uint64_t>(a.rows) * a.H_I};
    const uint64_t qstr[1] = {128};
    const uint32_t qbox[2] = {128, static_cast<uint32_t>(C::N)};
    if (!encode_tiled(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, qdims, qstr, qbox, CU_TENSOR_MAP_SWIZZLE_128B))
        return SA_ECUDA;
    auto kern = idx_tc_kernel<NH, R, NEPI, kCand>;
    const size_t smem = C::smem_bytes(a.rows);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return launch_status(e);
    // persistent CTAs: two per SM for one-row groups (two accumulator rings
    // fit in tensor memory, two CTAs' shared memory and registers fit the SM),
    // each walking its own item range
    int per_sm = 1;
    if (C::kTwoPerSm && 2 * C::kTmemCols <= 512 && 2 * (smem + 2048) <= 227 * 1024) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);  // all of it as shared
        if (e != cudaSuccess) return launch_status(e);
        per_sm = 2;
    }
    kern<<<sm_count() * per_sm, C::kThreads, smem, st>>>(tk, tq, a);
    return launch_status(cudaGetLastError());
}

}  // namespace

sa_status index_scores_tc(const void* q, const void* kc, const IdxArgs& a, cudaStream_t st) {
    if (a.rows > kMaxRows) return SA_EUNSUPPORTED;
    const bool grouped = a.seq_of_row != nullptr;
    if (a.cand) {  // candidates: one-row groups only
        if (grouped) return SA_EUNSUPPORTED;
        switch (a.H_I) {
            case 16: return launch_tc<16, 1, 4, true>(q, kc, a, st);
            case 32: return launch_tc<32, 1, 4, true>(q, kc, a, st);
            case 64: return launch_tc<64, 1, 4, true>(q, kc, a, st);
            case 128: return launch_tc<128, 1, 4, true>(q, kc, a, st);
            default: return SA_EUNSUPPORTED;
        }
    }
    switch (a.H_I) {
        case 16: return grouped ? launch_tc<16, 16, 8>(q, kc, a, st) : launch_tc<16, 1, 4>(q, kc, a, st);
        case 32: return grouped ? launch_tc<32, 8, 8>(q, kc, a, st) : launch_tc<32, 1, 4>(q, kc, a, st);
        case 64: return grouped ? launch_tc<64, 4, 8>(q, kc, a, st) : launch_tc<64, 1, 4>(q, kc, a, st);
        case 128: return grouped ? launch_tc<128, 2, 8>(q, kc, a, st) : launch_tc<128, 1, 4>(q, kc, a, st);
        default: return SA_EUNSUPPORTED;
    }
}

sa_status index_scores_cc(const void* q, const void* kc, sa_dtype dt, const IdxArgs& a, cudaStream_t st) {
    const int h = a.H_I;
    if (dt == SA_F32) {
        if (h <= 4) return launch_cc<float, 4>(q, kc, a, st);
        if (h <= 16) return launch_cc<float, 16>(q, kc, a, st);
        if (h <= 64) return launch_cc<float, 64>(q, kc, a, st);
    } else if (dt == SA_E4M3) {
        if (h <= 4) return launch_cc<__nv_fp8_e4m3, 4>(q, kc, a, st);
        if (h <= 16) return launch_cc<__nv_fp8_e4m3, 16>(q, kc, a, st);
        if (h <= 64) return launch_cc<__nv_fp8_e4m3, 64>(q, kc, a, st);
    }
    return SA_EUNSUPPORTED;
}

}  // namespace sa

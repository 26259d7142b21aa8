// sparse_mla.cu — sparse MLA attention over the selected latent rows.
//
// For query row r, head h and selected positions S_r ("MLA 与稀疏注意力",
// 分开以后，完整分数怎么算？ and “吸收矩阵”是交换线性计算的顺序):
//   z_j  = (q_lat[h] . c_j + q_rope[h] . kr_j) * scale
//   out  = sum_j softmax_{S_r}(z)_j c_j          (latent aggregate)
// The latent row c_j is key and value at once and one selection serves every
// head ("Sparse Attention 数学学习笔记" §8-9: gather the chosen latent rows only).
//
// Design (one cluster of two CTAs per (row, key split)):
//  * The 576-wide score contraction is split across the pair: CTA 0 owns latent
//    dims 0..255, CTA 1 owns dims 256..511 plus the 64 RoPE dims.  Two
//    producer warps gather only the CTA's slice of every selected row with
//    16-byte cp.async (one warp instruction per 512-byte row slice, written in
//    the 128-byte swizzled layout the tensor cores read) into a 3-stage ring of
//    64-key tiles; padded slots are zero-filled without a read.  Rows of the
//    tile kPrefetch tiles ahead are prefetched into L2, so the ring only has to
//    cover L2 latency.
//  * The CTA's slice of the 128-head query sits in tensor memory and is the A
//    operand of the score MMAs (M=128 heads, N=64 keys, the smallest N at which
//    an MMA is not dominated by its fixed issue cost).
//  * Four exchange warps copy each tile's partial scores from TMEM to shared
//    memory and ship them to the partner in one bulk copy that completes
//    transaction bytes on the partner's barrier (distributed shared memory is
//    the narrowest link of this kernel, so the copy runs off the softmax path);
//    the partner's softmax frees the receive buffer with a remote arrive.
//  * Eight softmax warps: thread = (head = TMEM lane, half of the tile's keys).
//    A pair of warps shares a head range; the two halves swap their tile maxima
//    in shared memory, so both apply the same reference.  Online base-2
//    softmax; O is rescaled only when a tile's maximum exceeds the reference by
//    more than 2^8.  P goes back to TMEM as bf16; both CTAs hold identical
//    scores and probabilities.
//  * O[128 x 256] (+)= P . V on the tensor cores with P from TMEM and V = the
//    gathered latent slice read MN-major: the tile gathered for the scores is
//    reused, so every selected row is read from memory once, and each CTA
//    aggregates its own 256 latent dims.
//  * Rows with few queries split their keys over several clusters; partial
//    (O, m, l) states go to a workspace and a combine kernel merges them.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kPage = 64;
constexpr int kNK = 64;           // keys per tile
constexpr int kHalf = kNK / 2;    // keys per softmax thread
constexpr int kStages = 3;
constexpr int kPrefetch = 4;      // tiles prefetched into L2 ahead of the copy
constexpr int kBlkK = kNK * 128;  // one 64-dim slice of a tile (bytes)
constexpr int kMaxBlk = 5;        // 64-dim slices per CTA (CTA 1: 4 latent + 1 RoPE)
constexpr int kStageBytes = kMaxBlk * kBlkK;
constexpr int kXBytes = 128 * kNK * 4;  // one tile of partial scores (128 heads x 64 keys fp32)
constexpr int kOffStage = 0;
constexpr int kOffX = kOffStage + kStages * kStageBytes;  // partner's halves, 2 buffers
constexpr int kOffL = kOffX + 2 * kXBytes;                // this CTA's half, staged for the copy
constexpr int kSmem = kOffL + kXBytes + 1024;
constexpr int kSmxWarps = 8;
constexpr int kXchgWarp0 = kSmxWarps;
constexpr int kProdWarp0 = kXchgWarp0 + 4;
constexpr int kProdWarps = 2;
constexpr int kMmaWarp = kProdWarp0 + kProdWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // O: 256 fp32 columns
constexpr uint32_t kColS = 256;  // S: 64 fp32 columns
constexpr uint32_t kColP = 320;  // P: 64 bf16 = 32 columns
constexpr uint32_t kColQ = 352;  // query slice: up to 320 bf16 = 160 columns
constexpr float kRescaleLog2 = 8.0f;

static_assert(kSmem <= 232448, "shared memory budget");
static_assert(kColQ + 160 <= kTmemCols, "tensor memory budget");
static_assert(kStageBytes % 1024 == 0 && kXBytes % 1024 == 0, "swizzle atoms stay 1024-byte aligned");

struct MlaKernelArgs {
    MlaArgs a;
    int nsplit;
    float* ws_o;   // [rows][nsplit][H][512] partial outputs (nsplit > 1)
    float* ws_ml;  // [rows][nsplit][H][4] partial (m, l of bf16 P, l of fp32 P, unused)
};

__device__ __forceinline__ int64_t pool_row(const MlaArgs& a, int seq, int p) {
    if (p / kPage >= a.pages_per_seq) return 0;  // position past the table: precondition broken
    const int pg = a.page_table ? a.page_table[static_cast<int64_t>(seq) * a.pages_per_seq + p / kPage]
                                : seq * a.pages_per_seq + p / kPage;
    if (pg < 0 || pg >= a.pool_pages) return 0;  // precondition broken: read a row inside the pool
    return static_cast<int64_t>(pg) * kPage + (p % kPage);
}

__device__ __forceinline__ int idx_at(const MlaArgs& a, int r, int slot) {
    return slot < a.k ? a.idx[static_cast<int64_t>(r) * a.k + slot] : -1;
}

template <int N>
__device__ __forceinline__ float tree_max(float (&v)[N]) {
#pragma unroll
    for (int w = N / 2; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) v[i] = fmaxf(v[i], v[i + w]);
    return v[0];
}

template <int N>
__device__ __forceinline__ float tree_sum(float (&v)[N]) {
#pragma unroll
    for (int w = N / 2; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) v[i] += v[i + w];
    return v[0];
}

// Read 64 fp32 columns of this thread's TMEM lane (two 32-column loads, one wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&v)[64]) {
    uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
    uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
    tmem_ld32(taddr, v0);
    tmem_ld32(taddr + 32, v1);
    tmem_ld_wait();
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1) mla_kernel(const MlaKernelArgs ka) {
    const MlaArgs& a = ka.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sStage = sm + kOffStage;
    uint8_t* sX = sm + kOffX;
    uint8_t* sL = sm + kOffL;

    __shared__ uint64_t bar_full[kStages], bar_empty[kStages], bar_sfull, bar_sfree, bar_xfull[2], bar_xfree[2],
        bar_pfull, bar_pvdone, bar_final;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ volatile int s_xfail;     // written only by exchange threads (see the exchange loop)
    __shared__ volatile int s_pfail[4];  // written only by softmax pair q (see the softmax loop)
    __shared__ float s_pmax[2][2][128];  // [tile parity][key half][head] tile maxima
    __shared__ float s_psum[2][2][128];  // (l, lx) of the two key halves, for the output

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank(), partner = rank ^ 1u;
    const int nblk = 4 + static_cast<int>(rank);  // 64-dim slices this CTA contracts
    const int cl = blockIdx.x >> 1;
    const int r = cl / ka.nsplit, split = cl % ka.nsplit;
    const int T = (a.k + kNK - 1) / kNK;
    const int t0 = static_cast<int>(static_cast<int64_t>(split) * T / ka.nsplit);
    const int t1 = static_cast<int>(static_cast<int64_t>(split + 1) * T / ka.nsplit);
    const int nt = t1 - t0;
    const int seq = a.seq_of_row ? a.seq_of_row[r] : r;
    WaitCtx wc{a.err, &s_abort};

    if (tid == 0) {
        s_abort = 0;
        s_xfail = 0;
        for (int q = 0; q < 4; ++q) s_pfail[q] = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bar_full[i], 32 * kProdWarps);
            mbar_init(&bar_empty[i], 1);
        }
        mbar_init(&bar_sfull, 1);
        mbar_init(&bar_sfree, kSmxWarps + 4);  // softmax and exchange warps both read S
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_xfull[i], 1);
            mbar_init(&bar_xfree[i], kSmxWarps);  // the partner's softmax warps
        }
        mbar_init(&bar_pfull, kSmxWarps);
        mbar_init(&bar_pvdone, 1);
        mbar_init(&bar_final, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync_all();  // partner's barriers exist before any remote write
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp < 4) {
        // The query slice of head `tid` into its TMEM lane: column c holds
        // elements 2c, 2c+1 (rows beyond H are zero and never written out).
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const bool live = tid < a.H;
        const uint4* ql = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q_lat) +
                                                         (static_cast<int64_t>(r) * a.H + (live ? tid : 0)) * 512 +
                                                         rank * 256);
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 u = live ? ql[c / 4 + j] : make_uint4(0u, 0u, 0u, 0u);
                v[4 * j] = u.x;
                v[4 * j + 1] = u.y;
                v[4 * j + 2] = u.z;
                v[4 * j + 3] = u.w;
            }
            tmem_st32(tmem + lane_base + kColQ + c, v);
        }
        if (rank == 1) {
            const uint4* qr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q_rope) +
                                                             (static_cast<int64_t>(r) * a.H + (live ? tid : 0)) * 64);
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 u = live ? qr[j] : make_uint4(0u, 0u, 0u, 0u);
                v[4 * j] = u.x;
                v[4 * j + 1] = u.y;
                v[4 * j + 2] = u.z;
                v[4 * j + 3] = u.w;
            }
            tmem_st32(tmem + lane_base + kColQ + 128, v);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp >= kProdWarp0 && warp < kMmaWarp) {
        // ------------------------------------------------ producers: gathered row slices
        // Warp p copies keys p, p+2, ... of each tile: lane = 16-byte chunk of the
        // 512-byte latent slice (slice b = lane / 8, chunk lane % 8); CTA 1 adds the
        // 128-byte RoPE keys, 4 keys per instruction.  Lane i holds the pool row of
        // the warp's i-th key (or -1 for a padded slot), for the kPrefetch tiles in
        // flight between the L2 prefetch and the copy.
        const int pw = warp - kProdWarp0;
        const __nv_bfloat16* cbase = static_cast<const __nv_bfloat16*>(a.c_cache) + rank * 256 + lane * 8;
        const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(a.kr_cache) + (lane & 7) * 8;
        constexpr int kPer = kNK / kProdWarps;  // 32 keys per warp per tile
        auto row_of = [&](int t) -> int {
            const int p = idx_at(a, r, (t0 + t) * kNK + pw + kProdWarps * lane);
            return p >= 0 ? static_cast<int>(pool_row(a, seq, p)) : -1;
        };
        auto prefetch_rows = [&](int row) {
            if (row < 0) return;
            const char* c = reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(a.c_cache) +
                                                          static_cast<int64_t>(row) * a.c_ld + rank * 256);
#pragma unroll
            for (int o = 0; o < 512; o += 128) prefetch_l2(c + o);
            if (rank == 1)
                prefetch_l2(static_cast<const __nv_bfloat16*>(a.kr_cache) + static_cast<int64_t>(row) * a.kr_ld);
        };
        int ring[kPrefetch];  // rows of tiles t .. t + kPrefetch - 1
#pragma unroll
        for (int d = 0; d < kPrefetch; ++d) {
            ring[d] = d < nt ? row_of(d) : -1;
            prefetch_rows(ring[d]);
        }
        int stage = 0;
        uint32_t phase = 0;
        for (int t = 0; t < nt; ++t) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&bar_empty[stage], phase ^ 1, wc, kErrMlaWait | 1);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            const int myrow = ring[0];
            const uint32_t sbase = smem_u32(sStage + stage * kStageBytes);
            const int b = lane >> 3, c = lane & 7;
#pragma unroll 8
            for (int i = 0; i < kPer; ++i) {
                const int j = pw + kProdWarps * i;
                const int row = __shfl_sync(0xffffffffu, myrow, i);
                const uint32_t dst = sbase + b * kBlkK + j * 128 + ((c ^ (j & 7)) << 4);
                cp_async16(dst, cbase + static_cast<int64_t>(row < 0 ? 0 : row) * a.c_ld, row < 0 ? 0u : 16u);
            }
            if (rank == 1) {
#pragma unroll
                for (int i0 = 0; i0 < kPer; i0 += 4) {
                    const int i = i0 + (lane >> 3);
                    const int j = pw + kProdWarps * i;
                    const int row = __shfl_sync(0xffffffffu, myrow, i);
                    const uint32_t dst = sbase + 4 * kBlkK + j * 128 + ((c ^ (j & 7)) << 4);
                    cp_async16(dst, kbase + static_cast<int64_t>(row < 0 ? 0 : row) * a.kr_ld, row < 0 ? 0u : 16u);
                }
            }
            cp_async_arrive_noinc(&bar_full[stage]);
#pragma unroll
            for (int d = 0; d + 1 < kPrefetch; ++d) ring[d] = ring[d + 1];
            ring[kPrefetch - 1] = t + kPrefetch < nt ? row_of(t + kPrefetch) : -1;
            prefetch_rows(ring[kPrefetch - 1]);
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1;
            }
        }
        cp_async_wait_all();  // every copy lands before the CTA can exit
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t id_qk = idesc_f32acc(1, 1, false, false, 128, kNK);
        constexpr uint32_t id_pv = idesc_f32acc(1, 1, false, true, 128, 256);
        bool ok = true;
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0; i <= nt && ok; ++i) {
                if (i < nt) {
                    ok = mbar_wait(&bar_full[stage], phase, wc, kErrMlaWait | 4);
                    if (ok && i >= 1) ok = mbar_wait(&bar_sfree, static_cast<uint32_t>((i - 1) & 1), wc, kErrMlaWait | 5);
                    if (!ok) break;
                    fence_proxy_async_smem();  // cp.async writes -> tensor-core reads
                    tc_fence_after();
                    uint8_t* stg = sStage + stage * kStageBytes;
                    for (int b = 0; b < nblk; ++b) {
                        const uint64_t kd = sdesc(smem_u32(stg + b * kBlkK), 16, 1024, kSw128);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_ts(tmem + kColS, tmem + kColQ + 32 * b + 8 * kk, kd + 2 * kk, id_qk,
                                        (b | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&bar_sfull);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                const int u = i - 1;
                if (u >= 0) {
                    ok = mbar_wait(&bar_pfull, static_cast<uint32_t>(u & 1), wc, kErrMlaWait | 3);
                    if (!ok) break;
                    tc_fence_after();
                    const int st = u % kStages;
                    const uint64_t vd = sdesc(smem_u32(sStage + st * kStageBytes), kBlkK, 1024, kSw128);
#pragma unroll
                    for (int kk = 0; kk < kNK / 16; ++kk)
                        mma_bf16_ts(tmem + kColO, tmem + kColP + 8 * kk, vd + 128 * kk, id_pv, (u > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_empty[st]);
                    tc_commit(&bar_pvdone);
                }
            }
        }
        if (lane == 0) {
            int dummy = 0;
            WaitCtx dw{a.err, reinterpret_cast<volatile int*>(&dummy)};
            tc_commit(&bar_final);
            mbar_wait(&bar_final, 0, dw, kErrMlaWait | 11);
        }
        __syncwarp();
    } else if (warp >= kXchgWarp0) {
        // ------------------------------------------------ exchange: this CTA's partial scores -> partner
        // Named barrier 2 spans the 128 exchange threads.  A failed (timed-out)
        // wait is recorded in s_xfail, which only exchange threads write, before
        // the barrier, and every exchange thread reads it after the barrier: the
        // four warps always leave the loop together, never one of them stuck in
        // bar.sync.
        const int h = tid - 32 * kXchgWarp0;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t x_remote = mapa_u32(smem_u32(sX), partner);
        const uint32_t xfull_remote = mapa_u32(smem_u32(&bar_xfull[0]), partner);
        for (int t = 0; t < nt; ++t) {
            const int xb = t & 1;
            uint32_t v[64];
            const bool got = warp_wait(&bar_sfull, static_cast<uint32_t>(t & 1), wc, kErrMlaWait | 14);
            if (got) {
                tc_fence_after();
                tmem_ld64(tmem + lane_base + kColS, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_sfree);
            } else if (lane == 0) {
                s_xfail = 1;
            }
            // the partner's softmax has read its buffer xb (tile t - 2); the previous copy has read L
            if (h == 0) {
                if (t >= 2 && !mbar_wait<true>(&bar_xfree[xb], static_cast<uint32_t>(((t >> 1) - 1) & 1), wc,
                                               kErrMlaWait | 15))
                    s_xfail = 1;
                bulk_wait_read_all();
            }
            named_sync(2, 128);
            if (s_xfail) break;
            uint8_t* lrow = sL + h * 256;
#pragma unroll
            for (int c = 0; c < 16; ++c)
                *reinterpret_cast<uint4*>(lrow + ((c ^ (h & 7)) << 4)) =
                    make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            fence_proxy_async_smem();
            named_sync(2, 128);
            if (h == 0) bulk_copy_to_cluster(x_remote + xb * kXBytes, sL, kXBytes, xfull_remote + 8 * xb);
        }
        if (h == 0) bulk_wait_all();
    } else {
        // ------------------------------------------------ softmax + output
        // Thread = (head h = TMEM lane, key half kh).  Warps q and q + 4 form
        // pair q and meet at named barrier 3 + q (64 threads) once per tile.  A
        // failed wait is recorded in s_pfail[q], written only by pair q before
        // that barrier and read by both warps after it, so the pair always
        // leaves the loop together.
        const int q = warp & 3, kh = warp >> 2;
        const int h = 32 * q + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const float c2 = a.scale * 1.4426950408889634f;  // scores in base-2 units
        float m = -INFINITY, l = 0.f, lx = 0.f;  // l: sum of bf16 P (normalises O); lx: fp32 sum (lse)
        const uint32_t xfree_remote = mapa_u32(smem_u32(&bar_xfree[0]), partner);
        bool ok = true;
        // validity of this half's 32 slots of the next tile (slot = 32 kh + lane)
        int i_next = nt > 0 ? idx_at(a, r, t0 * kNK + kHalf * kh + lane) : -1;
        for (int t = 0; t < nt; ++t) {
            const int xb = t & 1;
            const unsigned vmask = __ballot_sync(0xffffffffu, i_next >= 0);
            if (t + 1 < nt) i_next = idx_at(a, r, (t0 + t + 1) * kNK + kHalf * kh + lane);
            if (tid == 0) mbar_arrive_expect_tx(&bar_xfull[xb], kXBytes);  // the partner's half of tile t
            float s[kHalf];
            bool got = warp_wait(&bar_sfull, static_cast<uint32_t>(t & 1), wc, kErrMlaWait | 6);
            if (got) {
                tc_fence_after();
                uint32_t v[kHalf];
                tmem_ld32(tmem + lane_base + kColS + kHalf * kh, v);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_sfree);
                got = warp_wait<true>(&bar_xfull[xb], static_cast<uint32_t>((t >> 1) & 1), wc, kErrMlaWait | 7);
                if (got) {
                    const uint8_t* xl = sX + xb * kXBytes + h * 256;
#pragma unroll
                    for (int c = 0; c < kHalf / 4; ++c) {
                        const int cc = 8 * kh + c;  // 16-byte chunk of the row (4 keys)
                        const float4 x = *reinterpret_cast<const float4*>(xl + ((cc ^ (h & 7)) << 4));
                        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 4 * c + e;
                            s[j] = ((vmask >> j) & 1u) ? (__uint_as_float(v[j]) + xs[e]) * c2 : -INFINITY;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(xfree_remote + 8 * xb);  // the partner may refill it
                }
            }
            float mx;
            {
                float tmp[kHalf];
#pragma unroll
                for (int j = 0; j < kHalf; ++j) tmp[j] = got ? s[j] : -INFINITY;
                mx = tree_max(tmp);
            }
            s_pmax[t & 1][kh][h] = mx;  // by parity: the partner may still read tile t - 1
            if (!got && lane == 0) s_pfail[q] = 1;
            named_sync(3 + q, 64);
            if (s_pfail[q]) {
                ok = false;
                break;
            }
            mx = fmaxf(mx, s_pmax[t & 1][kh ^ 1][h]);
            if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
                const float m_new = fmaxf(m, mx);
                const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
                if (t > 0) {  // O holds tiles < t: wait for the last product, then scale this half of it
                    if (warp_wait(&bar_pvdone, static_cast<uint32_t>((t - 1) & 1), wc, kErrMlaWait | 8)) {
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 128 * kh; c < 128 * kh + 128; c += 32) {
                            uint32_t o[32];
                            tmem_ld32(tmem + lane_base + kColO + c, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                            tmem_st32(tmem + lane_base + kColO + c, o);
                        }
                        tmem_st_wait();
                    }
                }
                l *= alpha;
                lx *= alpha;
                m = m_new;
            }
            // masked slots are -inf and give exactly 0; a fully masked prefix keeps m at -inf
            const float mref = (m == -INFINITY) ? 0.f : m;
            uint32_t pk[kHalf / 2];
            float lb[kHalf / 2], lf[kHalf / 2];
#pragma unroll
            for (int j = 0; j < kHalf / 2; ++j) {
                const float p0 = fast_exp2(s[2 * j] - mref);
                const float p1 = fast_exp2(s[2 * j + 1] - mref);
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                lb[j] = __low2float(b2) + __high2float(b2);
                lf[j] = p0 + p1;
                pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            l += tree_sum(lb);
            lx += tree_sum(lf);
            // the product of tile t - 1 has read P before it is overwritten
            if (t >= 1) warp_wait(&bar_pvdone, static_cast<uint32_t>((t - 1) & 1), wc, kErrMlaWait | 12);
            tc_fence_after();
            tmem_st16(tmem + lane_base + kColP + (kHalf / 2) * kh, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_pfull);
        }
        // ---- output: this thread's half (128 latent dims) of the CTA's 256 dims of head h
        s_psum[kh][0][h] = l;
        s_psum[kh][1][h] = lx;
        named_sync(3 + q, 64);
        const float lt = s_psum[0][0][h] + s_psum[1][0][h];
        const float lxt = s_psum[0][1][h] + s_psum[1][1][h];
        if (ok && nt > 0)
            ok = warp_wait(&bar_pvdone, static_cast<uint32_t>((nt - 1) & 1), wc, kErrMlaWait | 13);
        if (ok && !s_abort) {
            tc_fence_after();
            const bool partial = ka.nsplit > 1;
            const float inv = (lt > 0.f && !partial) ? 1.f / lt : 1.f;
            float* dst;
            if (partial)
                dst = ka.ws_o + ((static_cast<int64_t>(r) * ka.nsplit + split) * a.H + h) * 512 + rank * 256;
            else
                dst = a.out + (static_cast<int64_t>(r) * a.H + h) * a.d_c + rank * 256;
#pragma unroll 1
            for (int c = 128 * kh; c < 128 * kh + 128; c += 32) {
                uint32_t o[32];
                if (nt > 0) {
                    tmem_ld32(tmem + lane_base + kColO + c, o);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = 0u;
                }
                if (h < a.H) {
                    const bool empty = !(lt > 0.f);
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float4 f;
                        f.x = empty ? 0.f : __uint_as_float(o[j + 0]) * inv;
                        f.y = empty ? 0.f : __uint_as_float(o[j + 1]) * inv;
                        f.z = empty ? 0.f : __uint_as_float(o[j + 2]) * inv;
                        f.w = empty ? 0.f : __uint_as_float(o[j + 3]) * inv;
                        *reinterpret_cast<float4*>(dst + c + j) = f;
                    }
                }
            }
            if (h < a.H && rank == 0 && kh == 0) {
                if (partial) {
                    float* ml = ka.ws_ml + ((static_cast<int64_t>(r) * ka.nsplit + split) * a.H + h) * 4;
                    ml[0] = m;
                    ml[1] = lt;
                    ml[2] = lxt;
                } else if (a.lse) {
                    a.lse[static_cast<int64_t>(r) * a.H + h] = lt > 0.f ? (m + log2f(lxt)) * 0.6931471805599453f : -INFINITY;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the partner no longer writes into this CTA's shared memory
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// Merge the split partial states of every (row, head).
__global__ void __launch_bounds__(128) mla_combine_kernel(const MlaKernelArgs ka) {
    const MlaArgs& a = ka.a;
    const int r = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int ns = ka.nsplit;
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) {
        const float* ml = ka.ws_ml + ((static_cast<int64_t>(r) * ns + s) * a.H + h) * 4;
        if (ml[1] > 0.f) M = fmaxf(M, ml[0]);
    }
    float L = 0.f, LX = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int d = threadIdx.x * 4;
    for (int s = 0; s < ns; ++s) {
        const int64_t base = (static_cast<int64_t>(r) * ns + s) * a.H + h;
        const float* ml = ka.ws_ml + base * 4;
        if (!(ml[1] > 0.f)) continue;
        const float wgt = exp2f(ml[0] - M);
        L += ml[1] * wgt;
        LX += ml[2] * wgt;
        const float4 o = *reinterpret_cast<const float4*>(ka.ws_o + base * 512 + d);
        acc.x += o.x * wgt;
        acc.y += o.y * wgt;
        acc.z += o.z * wgt;
        acc.w += o.w * wgt;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    float* dst = a.out + (static_cast<int64_t>(r) * a.H + h) * a.d_c + d;
    *reinterpret_cast<float4*>(dst) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (threadIdx.x == 0 && a.lse)
        a.lse[static_cast<int64_t>(r) * a.H + h] = L > 0.f ? (M + log2f(LX)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace

int mla_decode_splits(int rows, int k) {
    const int T = (k + kNK - 1) / kNK;
    int ns = sm_count() / (2 * rows);
    if (ns < 1) ns = 1;
    if (ns > T) ns = T;
    if (ns > 16) ns = 16;
    return ns;
}

size_t mla_workspace_bytes(int rows, int H, int k, int d_c, int nsplit) {
    (void)k;
    if (nsplit <= 1) return 0;
    const size_t o = static_cast<size_t>(rows) * nsplit * H * d_c * 4;
    const size_t ml = static_cast<size_t>(rows) * nsplit * H * 4 * 4;
    return ((o + 255) & ~size_t(255)) + ((ml + 255) & ~size_t(255));
}

sa_status sparse_mla_launch(const MlaArgs& a, int nsplit, void* ws, size_t ws_bytes, cudaStream_t st) {
    MlaKernelArgs ka;
    ka.a = a;
    ka.nsplit = nsplit;
    ka.ws_o = nullptr;
    ka.ws_ml = nullptr;
    if (nsplit > 1) {
        const size_t need = mla_workspace_bytes(a.rows, a.H, a.k, a.d_c, nsplit);
        if (ws == nullptr || ws_bytes < need) return SA_EINVAL;
        const size_t o = static_cast<size_t>(a.rows) * nsplit * a.H * a.d_c * 4;
        ka.ws_o = static_cast<float*>(ws);
        ka.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ((o + 255) & ~size_t(255)));
    }
    cudaError_t e = cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return launch_status(e);
    mla_kernel<<<2 * a.rows * nsplit, kThreads, kSmem, st>>>(ka);
    e = cudaGetLastError();
    if (e != cudaSuccess) return launch_status(e);
    if (nsplit > 1) {
        mla_combine_kernel<<<a.rows * a.H, 128, 0, st>>>(ka);
        e = cudaGetLastError();
    }
    return launch_status(e);
}

}  // namespace sa

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
//    dims 0..255, CTA 1 owns dims 256..511 plus the 64 RoPE dims, and each CTA
//    aggregates its own 256 latent dims of the output, so every selected row is
//    read from memory once.
//  * Prologue: the pool rows of all of the CTA's selected slots go into a table
//    in shared memory (-1 for padded slots); the gather loop then does no
//    dependent global loads.
//  * Six producer warps gather the CTA's slice of every selected row with
//    16-byte cp.async (one warp instruction per 512-byte row slice, written in
//    the 128-byte swizzled layout the tensor cores read) into a 5-stage ring of
//    64-key tiles; padded slots are zero-filled without a read.
//  * The CTA's slice of the 128-head query sits in tensor memory and is the A
//    operand of the score MMAs (M=128 heads, N=64 keys).
//  * Four exchange warps copy each tile's partial scores from tensor memory
//    (which frees the score accumulator for the next tile at once) to this
//    CTA's slot of an L2-resident scratch buffer and signal both softmaxes: this
//    CTA's through a local barrier, the partner's through a remote arrive.
//    Distributed shared memory carries only those barrier arrivals.
//  * Four softmax warps, thread = head = TMEM lane: the thread adds the two
//    partial scores of its head for the tile's 64 keys, runs an online base-2
//    softmax (O is rescaled only when a tile's maximum exceeds the reference by
//    more than 2^8) and writes P as bf16 to tensor memory.  Both CTAs compute
//    the same P.
//  * O[128 x 256] (+)= P . V on the tensor cores with P from TMEM and V = the
//    gathered latent slice read MN-major.  The MMA warp issues whichever of the
//    next score MMA and the next aggregation is ready, so the scores of later
//    tiles run ahead of the softmax.
//  * The output leaves through shared memory, one bulk copy per head.
//  * Rows with few queries split their keys over several clusters; partial
//    (O, m, l) states go to a workspace and a combine kernel merges them.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kPage = 64;
constexpr int kNK = 64;           // keys per tile
constexpr int kStages = 5;
constexpr int kBlkK = kNK * 128;  // one 64-dim slice of a tile (bytes)
constexpr int kMaxBlk = 5;        // 64-dim slices per CTA (CTA 1: 4 latent + 1 RoPE)
constexpr int kStageBytes = kMaxBlk * kBlkK;
constexpr int kOffStage = 0;
constexpr int kOffRows = kOffStage + kStages * kStageBytes;  // [kMaxTilesPerCta * kNK] pool rows
constexpr int kSmem = kOffRows + kMaxTilesPerCta * kNK * 4 + 1024;
constexpr int kORowBytes = 256 * 4 + 16;  // one head's output row staged in shared memory (padded)
constexpr int kSmxWarps = 4;
constexpr int kXchgWarp0 = kSmxWarps;
constexpr int kProdWarp0 = kXchgWarp0 + 4;
constexpr int kProdWarps = 6;
constexpr int kMmaWarp = kProdWarp0 + kProdWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // O: 256 fp32 columns
constexpr uint32_t kColS = 256;  // S: 64 fp32 columns
constexpr uint32_t kColP = 320;  // P: 64 bf16 = 32 columns
constexpr uint32_t kColQ = 352;  // query slice: up to 320 bf16 = 160 columns
constexpr float kRescaleLog2 = 8.0f;
constexpr int kXFloats = kMlaXBytes / 4;  // floats per exchange buffer

static_assert(kSmem <= 232448 - 2048, "shared memory budget");
static_assert(kColQ + 160 <= kTmemCols, "tensor memory budget");
static_assert(kStageBytes % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
static_assert(128 * kORowBytes <= kStages * kStageBytes, "the output rows fit in the stage ring");
static_assert(kMlaXBytes == 128 * kNK * 4, "one exchange buffer holds a tile of fp32 partial scores");

struct MlaKernelArgs {
    MlaArgs a;
    int nsplit;
    float* xs;     // exchange scratch: [kMlaScratchSlots][kMlaXBuf][16 chunks][128 heads][4] fp32
    float* ws_o;   // [rows][nsplit][H][512] partial outputs (nsplit > 1)
    float* ws_ml;  // [rows][nsplit][H][4] partial (m, l of bf16 P, l of fp32 P, unused)
};

// Pool row of position p of sequence `seq`, or -2 when p lies past the page
// table or its page is outside the pool (the caller's preconditions are
// broken: the caller records that and reads row 0 of the pool instead).
__device__ __forceinline__ int64_t pool_row(const MlaArgs& a, int seq, int p) {
    if (p / kPage >= a.pages_per_seq) return -2;
    const int pg = a.page_table ? a.page_table[static_cast<int64_t>(seq) * a.pages_per_seq + p / kPage]
                                : seq * a.pages_per_seq + p / kPage;
    if (pg < 0 || pg >= a.pool_pages) return -2;
    return static_cast<int64_t>(pg) * kPage + (p % kPage);
}

// Position held by slot `slot` of row r: the selection, or in dense mode (no
// selection) every visible position in order.
__device__ __forceinline__ int idx_at(const MlaArgs& a, int r, int slot) {
    if (slot >= a.k) return -1;
    if (a.idx) return a.idx[static_cast<int64_t>(r) * a.k + slot];
    return slot < a.n_visible[r] ? slot : -1;
}

// Four fp32 values rounded to bf16 (nearest, ties to even), packed in order.
__device__ __forceinline__ uint2 bf16x4_bits(float4 f) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(f.x, f.y), hi = __floats2bfloat162_rn(f.z, f.w);
    return make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
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

__device__ __forceinline__ uint32_t sm_id() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1) mla_kernel(const MlaKernelArgs ka) {
    // The split combine that follows may take the idle SMs now and wait there
    // for this grid (measured: attention 1.6 us shorter; the same overlap from
    // the indexer to the Top-K made the back-to-back step 6 us longer).
    pdl_trigger();
    const MlaArgs& a = ka.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sStage = sm + kOffStage;
    int* sRows = reinterpret_cast<int*>(sm + kOffRows);

    __shared__ uint64_t bar_full[kStages], bar_empty[kStages], bar_sfull, bar_sfree, bar_lfull[kMlaXBuf],
        bar_lfree[kMlaXBuf], bar_xfull[kMlaXBuf], bar_xfree[kMlaXBuf], bar_pfull, bar_pvdone, bar_final;
    __shared__ uint32_t s_tmem;
    __shared__ uint32_t s_slot;  // this CTA's scratch slot (its SM id); the partner reads it remotely
    __shared__ int s_abort;
    __shared__ volatile int s_xfail;  // written only by exchange threads (see the exchange loop)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank(), partner = rank ^ 1u;
    const int nblk = 4 + static_cast<int>(rank);  // 64-dim slices this CTA contracts
    const int cl = blockIdx.x >> 1;
    const int r = cl / ka.nsplit, split = cl % ka.nsplit;
    const int T = (a.k + kNK - 1) / kNK;
    const int t0 = static_cast<int>(static_cast<int64_t>(split) * T / ka.nsplit);
    const int t1 = static_cast<int>(static_cast<int64_t>(split + 1) * T / ka.nsplit);
    const int nt = t1 - t0;  // at most kMaxTilesPerCta (the host picks the splits)
    WaitCtx wc{a.err, &s_abort};

    if (tid == 0) {
        const uint32_t slot = sm_id();
        s_slot = slot;
        s_abort = 0;
        s_xfail = 0;
        if (slot >= static_cast<uint32_t>(kMlaScratchSlots) || nt > kMaxTilesPerCta) {
            record_error(a.err, kErrMlaWait | 20);  // no scratch slot for this SM: do nothing
            s_abort = 1;
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bar_full[i], 32 * kProdWarps);
            mbar_init(&bar_empty[i], 1);
        }
        mbar_init(&bar_sfull, 1);
        mbar_init(&bar_sfree, 4);  // the exchange warps read S
        for (int i = 0; i < kMlaXBuf; ++i) {
            mbar_init(&bar_lfull[i], 1);          // exchange thread 0
            mbar_init(&bar_lfree[i], kSmxWarps);  // this CTA's softmax warps
            mbar_init(&bar_xfull[i], 1);          // the partner's exchange thread 0
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
    __syncthreads();  // the TMEM address is published
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int seq = a.seq_of_row ? a.seq_of_row[r] : r;

    if (warp < 4) {
        // The query slice of head `tid` into its TMEM lane: column c holds
        // elements 2c, 2c+1 (rows beyond H are zero and never written out).
        // Sixteen 16-byte loads in flight per round.
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const bool live = tid < a.H;
        const uint4* ql = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q_lat) +
                                                         (static_cast<int64_t>(r) * a.H + (live ? tid : 0)) * 512 +
                                                         rank * 256);
#pragma unroll 1
        for (int c = 0; c < 128; c += 64) {
            uint32_t v[64];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint4 u = live ? ql[c / 4 + j] : make_uint4(0u, 0u, 0u, 0u);
                v[4 * j] = u.x;
                v[4 * j + 1] = u.y;
                v[4 * j + 2] = u.z;
                v[4 * j + 3] = u.w;
            }
            tmem_st32(tmem + lane_base + kColQ + c, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_st32(tmem + lane_base + kColQ + c + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
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
    } else if (nt <= kMaxTilesPerCta) {
        // pool rows of every slot of this CTA's tiles (-1: padded slot), four
        // selection reads in flight per thread
        const int n = nt * kNK, nthr = kThreads - 128;
        bool broken = false;
        for (int i0 = tid - 128; i0 < n; i0 += 4 * nthr) {
            int pos[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * nthr;
                pos[u] = i < n ? idx_at(a, r, t0 * kNK + i) : -1;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * nthr;
                if (i < n) {
                    int row = pos[u] >= 0 ? static_cast<int>(pool_row(a, seq, pos[u])) : -1;
                    if (row == -2) {
                        broken = true;
                        row = 0;
                    }
                    sRows[i] = row;
                }
            }
        }
        if (broken) record_error(a.err, kErrMlaIndex);
    }
    tc_fence_before();
    cluster_sync_all();  // query, row table and slot are in place, and the partner has started
    tc_fence_after();
    const uint32_t my_slot = s_slot;
    const uint32_t peer_slot = ld_cluster_u32(mapa_u32(smem_u32(&s_slot), partner));
    // both CTAs skip the work alike when either has no scratch slot (recorded above)
    const bool run = my_slot < static_cast<uint32_t>(kMlaScratchSlots) &&
                     peer_slot < static_cast<uint32_t>(kMlaScratchSlots) && nt <= kMaxTilesPerCta;

    if (!run) {
        // nothing to do: fall through to the teardown
    } else if (warp >= kProdWarp0 && warp < kMmaWarp) {
        // ------------------------------------------------ producers: gathered row slices
        // Warp p copies keys p, p + 6, ... of each tile: lane = 16-byte chunk of the
        // 512-byte latent slice (slice b = lane / 8, chunk lane % 8).  CTA 1 adds the
        // 128-byte RoPE keys, 4 keys per instruction.
        const int pw = warp - kProdWarp0;
        const __nv_bfloat16* cbase = static_cast<const __nv_bfloat16*>(a.c_cache) + rank * 256 + lane * 8;
        const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(a.kr_cache) + (lane & 7) * 8;
        const int b = lane >> 3, c = lane & 7;
        int stage = 0;
        uint32_t phase = 0;
        for (int t = 0; t < nt; ++t) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&bar_empty[stage], phase ^ 1, wc, kErrMlaWait | 1);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            const int* trow = sRows + t * kNK;
            const uint32_t sbase = smem_u32(sStage + stage * kStageBytes);
#pragma unroll 4
            for (int j = pw; j < kNK; j += kProdWarps) {
                const int row = trow[j];
                const uint32_t dst = sbase + b * kBlkK + j * 128 + ((c ^ (j & 7)) << 4);
                cp_async16(dst, cbase + static_cast<int64_t>(row < 0 ? 0 : row) * a.c_ld, row < 0 ? 0u : 16u);
            }
            if (rank == 1) {
                for (int j0 = 4 * pw; j0 < kNK; j0 += 4 * kProdWarps) {
                    const int j = j0 + (lane >> 3);
                    const int row = trow[j];
                    const uint32_t dst = sbase + 4 * kBlkK + j * 128 + ((c ^ (j & 7)) << 4);
                    cp_async16(dst, kbase + static_cast<int64_t>(row < 0 ? 0 : row) * a.kr_ld, row < 0 ? 0u : 16u);
                }
            }
            cp_async_arrive_noinc(&bar_full[stage]);
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1;
            }
        }
        cp_async_wait_all();  // every copy lands before the CTA can exit
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        // Polls (without blocking) for the next score tile (its rows landed and the
        // exchange warps have read the previous scores) and for the next
        // aggregation (its P is written), and issues whichever is ready.
        constexpr uint32_t id_qk = idesc_f32acc(1, 1, false, false, 128, kNK);
        constexpr uint32_t id_pv = idesc_f32acc(1, 1, false, true, 128, 256);
        if (lane == 0) {
            int iq = 0, ip = 0;  // next score tile, next aggregation tile
            int qstage = 0;
            uint32_t qphase = 0;
            unsigned long long t_last = global_ns();
            while (ip < nt) {
                bool did = false;
                if (iq < nt && mbar_test_wait(&bar_full[qstage], qphase) &&
                    (iq == 0 || mbar_test_wait(&bar_sfree, static_cast<uint32_t>((iq - 1) & 1)))) {
                    fence_proxy_async_smem();  // cp.async writes -> tensor-core reads
                    tc_fence_after();
                    uint8_t* stg = sStage + qstage * kStageBytes;
                    for (int bb = 0; bb < nblk; ++bb) {
                        const uint64_t kd = sdesc(smem_u32(stg + bb * kBlkK), 16, 1024, kSw128);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_ts(tmem + kColS, tmem + kColQ + 32 * bb + 8 * kk, kd + 2 * kk, id_qk,
                                        (bb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&bar_sfull);
                    ++iq;
                    if (++qstage == kStages) {
                        qstage = 0;
                        qphase ^= 1;
                    }
                    did = true;
                }
                if (ip < iq && mbar_test_wait(&bar_pfull, static_cast<uint32_t>(ip & 1))) {
                    tc_fence_after();
                    const int st = ip % kStages;
                    const uint64_t vd = sdesc(smem_u32(sStage + st * kStageBytes), kBlkK, 1024, kSw128);
#pragma unroll
                    for (int kk = 0; kk < kNK / 16; ++kk)
                        mma_bf16_ts(tmem + kColO, tmem + kColP + 8 * kk, vd + 128 * kk, id_pv,
                                    (ip > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_empty[st]);
                    tc_commit(&bar_pvdone);
                    ++ip;
                    did = true;
                }
                if (did) {
                    t_last = global_ns();
                } else {
                    if (*wc.abort) break;
                    if (global_ns() - t_last > wc.limit_ns) {
                        record_error(a.err, kErrMlaWait | 4);
                        s_abort = 1;
                        break;
                    }
                }
            }
            int dummy = 0;
            WaitCtx dw(a.err, reinterpret_cast<volatile int*>(&dummy), kWaitLimitNs);  // drain: fixed limit
            tc_commit(&bar_final);
            mbar_wait(&bar_final, 0, dw, kErrMlaWait | 11);
        }
        __syncwarp();
    } else if (warp >= kXchgWarp0) {
        // ------------------------------------------------ exchange: partial scores -> L2 scratch
        // Thread h moves head h's 64 partial scores of tile t into buffer t % kMlaXBuf
        // of this CTA's scratch slot (layout [16-byte chunk][head], so each warp
        // store covers 512 contiguous bytes).  Named barrier 2 spans the 128
        // exchange threads.  A failed (timed-out) wait is recorded in s_xfail,
        // which only exchange threads write, before the barrier, and every
        // exchange thread reads it after the barrier: the four warps always leave
        // the loop together, never one of them stuck in bar.sync.
        const int h = tid - 32 * kXchgWarp0;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        float* myx = ka.xs + static_cast<size_t>(my_slot) * kMlaXBuf * kXFloats;
        const uint32_t xfull_remote = mapa_u32(smem_u32(&bar_xfull[0]), partner);
        for (int t = 0; t < nt; ++t) {
            const int xb = t % kMlaXBuf;
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
            // buffer xb last held tile t - kMlaXBuf: both softmaxes must have read it
            if (h == 0 && t >= kMlaXBuf) {
                const uint32_t par = static_cast<uint32_t>((t / kMlaXBuf - 1) & 1);
                if (!mbar_wait(&bar_lfree[xb], par, wc, kErrMlaWait | 16)) s_xfail = 1;
                if (!mbar_wait<true>(&bar_xfree[xb], par, wc, kErrMlaWait | 15)) s_xfail = 1;
            }
            named_sync(2, 128);
            if (s_xfail) break;
            float4* dst = reinterpret_cast<float4*>(myx + xb * kXFloats);
#pragma unroll
            for (int c = 0; c < 16; ++c) st_cg_v4(dst + c * 128 + h, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            named_sync(2, 128);
            if (h == 0) {
                // release arrivals (this CTA's softmax at CTA scope, the partner's at
                // cluster scope): the stores of all 128 exchange threads precede them
                // through the named barrier, and each softmax acquires its arrival
                mbar_arrive(&bar_lfull[xb]);
                mbar_arrive_cluster(xfull_remote + 8 * xb);
            }
        }
    } else {
        // ------------------------------------------------ softmax + output (thread = head h)
        const int h = tid;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float c2 = a.scale * 1.4426950408889634f;  // scores in base-2 units
        float m = -INFINITY, l = 0.f, lx = 0.f;  // l: sum of bf16 P (normalises O); lx: fp32 sum (lse)
        const float4* myx = reinterpret_cast<const float4*>(ka.xs + static_cast<size_t>(my_slot) * kMlaXBuf * kXFloats);
        const float4* px = reinterpret_cast<const float4*>(ka.xs + static_cast<size_t>(peer_slot) * kMlaXBuf * kXFloats);
        const uint32_t xfree_remote = mapa_u32(smem_u32(&bar_xfree[0]), partner);
        bool ok = true;
        for (int t = 0; t < nt; ++t) {
            const int xb = t % kMlaXBuf;
            const uint32_t par = static_cast<uint32_t>((t / kMlaXBuf) & 1);
            // which of the tile's 64 slots hold a key
            const unsigned vm0 = __ballot_sync(0xffffffffu, sRows[t * kNK + lane] >= 0);
            const unsigned vm1 = __ballot_sync(0xffffffffu, sRows[t * kNK + 32 + lane] >= 0);
            ok = warp_wait(&bar_lfull[xb], par, wc, kErrMlaWait | 6);
            if (ok) ok = warp_wait<true>(&bar_xfull[xb], par, wc, kErrMlaWait | 7);
            if (!ok) break;
            float s[kNK];
            {
                const float4* ow = myx + xb * (kXFloats / 4) + h;
                const float4* pw4 = px + xb * (kXFloats / 4) + h;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float4 u = ld_cg_v4(ow + c * 128);
                    const float4 w = ld_cg_v4(pw4 + c * 128);
                    s[4 * c + 0] = (u.x + w.x) * c2;
                    s[4 * c + 1] = (u.y + w.y) * c2;
                    s[4 * c + 2] = (u.z + w.z) * c2;
                    s[4 * c + 3] = (u.w + w.w) * c2;
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar_lfree[xb]);
                mbar_arrive_cluster_relaxed(xfree_remote + 8 * xb);  // the partner may refill its buffer
            }
#pragma unroll
            for (int j = 0; j < kNK; ++j) {
                const unsigned bit = j < 32 ? (vm0 >> j) & 1u : (vm1 >> (j - 32)) & 1u;
                if (!bit) s[j] = -INFINITY;
            }
            float mx;
            {
                float tmp[kNK];
#pragma unroll
                for (int j = 0; j < kNK; ++j) tmp[j] = s[j];
                mx = tree_max(tmp);
            }
            if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
                const float m_new = fmaxf(m, mx);
                const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
                if (t > 0) {  // O holds tiles < t: wait for the last product, then scale this head's row
                    if (!warp_wait(&bar_pvdone, static_cast<uint32_t>((t - 1) & 1), wc, kErrMlaWait | 8)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 256; c += 32) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_base + kColO + c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        tmem_st32(tmem + lane_base + kColO + c, o);
                    }
                    tmem_st_wait();
                }
                l *= alpha;
                lx *= alpha;
                m = m_new;
            }
            // masked slots are -inf and give exactly 0; a fully masked prefix keeps m at -inf
            const float mref = (m == -INFINITY) ? 0.f : m;
            uint32_t pk[kNK / 2];
            float lb[kNK / 2], lf[kNK / 2];
#pragma unroll
            for (int j = 0; j < kNK / 2; ++j) {
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
            if (t >= 1 && !warp_wait(&bar_pvdone, static_cast<uint32_t>((t - 1) & 1), wc, kErrMlaWait | 12)) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_st32(tmem + lane_base + kColP, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_pfull);
        }
        // ---- output: head h's 256 latent dims of this CTA, staged in the idle stage
        // ring (padded rows: no bank conflicts) and sent with one bulk copy per head
        if (ok && nt > 0)
            ok = warp_wait(&bar_pvdone, static_cast<uint32_t>((nt - 1) & 1), wc, kErrMlaWait | 13);
        if (ok && !*wc.abort) {
            tc_fence_after();
            const bool partial = ka.nsplit > 1;
            const bool bf = !partial && a.out_bf16 != nullptr;  // final output rounded to bf16
            const bool empty = !(l > 0.f);
            const float inv = (!empty && !partial) ? 1.f / l : 1.f;
            float* srow = reinterpret_cast<float*>(sStage + h * kORowBytes);
#pragma unroll 1
            for (int c = 0; c < 256; c += 32) {
                uint32_t o[32];
                if (nt > 0) {
                    tmem_ld32(tmem + lane_base + kColO + c, o);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = 0u;
                }
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 f;
                    f.x = empty ? 0.f : __uint_as_float(o[j + 0]) * inv;
                    f.y = empty ? 0.f : __uint_as_float(o[j + 1]) * inv;
                    f.z = empty ? 0.f : __uint_as_float(o[j + 2]) * inv;
                    f.w = empty ? 0.f : __uint_as_float(o[j + 3]) * inv;
                    if (bf)
                        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(srow) + 2 * (c + j)) = bf16x4_bits(f);
                    else
                        *reinterpret_cast<float4*>(srow + c + j) = f;
                }
            }
            fence_proxy_async_smem();  // generic-proxy writes -> bulk-copy reads
            if (h < a.H && bf) {
                uint8_t* dst = static_cast<uint8_t*>(a.out_bf16) +
                               ((static_cast<int64_t>(r) * a.H + h) * a.d_c + rank * 256) * 2;
                bulk_copy_s2g(dst, srow, 256 * 2);
                if (rank == 0 && a.lse)
                    a.lse[static_cast<int64_t>(r) * a.H + h] =
                        l > 0.f ? (m + log2f(lx)) * 0.6931471805599453f : -INFINITY;
                bulk_wait_all();
            } else if (h < a.H) {
                float* dst = partial ? ka.ws_o + ((static_cast<int64_t>(r) * ka.nsplit + split) * a.H + h) * 512 + rank * 256
                                     : a.out + (static_cast<int64_t>(r) * a.H + h) * a.d_c + rank * 256;
                bulk_copy_s2g(dst, srow, 256 * 4);
                if (rank == 0) {
                    if (partial) {
                        float* ml = ka.ws_ml + ((static_cast<int64_t>(r) * ka.nsplit + split) * a.H + h) * 4;
                        ml[0] = m;
                        ml[1] = l;
                        ml[2] = lx;
                    } else if (a.lse) {
                        a.lse[static_cast<int64_t>(r) * a.H + h] =
                            l > 0.f ? (m + log2f(lx)) * 0.6931471805599453f : -INFINITY;
                    }
                }
                bulk_wait_all();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the partner no longer arrives on this CTA's barriers
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// Merge the split partial states of every (row, head).  Thread = (row, head,
// four 16-byte pieces d, d + 128, d + 256, d + 384 of the 512 latent dims):
// 32 threads per head, eight heads per CTA, three CTAs per SM; the loads of
// two splits (their states and outputs) are in flight together.
constexpr int kCombThreads = 256;
constexpr int kCombHeads = kCombThreads / 32;
constexpr int kCombChunk = 2;  // splits whose loads are issued together

__global__ void __launch_bounds__(kCombThreads, 3) mla_combine_kernel(const MlaKernelArgs ka) {
    pdl_wait();  // the partial states of the kernel before are complete
    const MlaArgs& a = ka.a;
    const int64_t rh = static_cast<int64_t>(blockIdx.x) * kCombHeads + (threadIdx.x >> 5);
    if (rh >= static_cast<int64_t>(a.rows) * a.H) return;
    const int r = static_cast<int>(rh / a.H), h = static_cast<int>(rh % a.H);
    const int ns = ka.nsplit;
    const int d = (threadIdx.x & 31) * 4;
    const int64_t base0 = static_cast<int64_t>(r) * ns * a.H + h;  // (row, split 0, head)
    float M = -INFINITY;
    for (int s0 = 0; s0 < ns; s0 += kCombChunk) {
        float mv[kCombChunk], lv[kCombChunk];
#pragma unroll
        for (int j = 0; j < kCombChunk; ++j) {
            mv[j] = -INFINITY;
            lv[j] = 0.f;
            if (s0 + j < ns) {
                const float* ml = ka.ws_ml + (base0 + static_cast<int64_t>(s0 + j) * a.H) * 4;
                mv[j] = ml[0];
                lv[j] = ml[1];
            }
        }
#pragma unroll
        for (int j = 0; j < kCombChunk; ++j)
            if (lv[j] > 0.f) M = fmaxf(M, mv[j]);
    }
    float L = 0.f, LX = 0.f;
    float4 acc[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) acc[p] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < ns; s0 += kCombChunk) {
        float mv[kCombChunk], lv[kCombChunk], xv[kCombChunk];
        float4 o[kCombChunk][4];
#pragma unroll
        for (int j = 0; j < kCombChunk; ++j) {
            mv[j] = 0.f;
            lv[j] = 0.f;
            xv[j] = 0.f;
#pragma unroll
            for (int p = 0; p < 4; ++p) o[j][p] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s0 + j < ns) {
                const int64_t row = base0 + static_cast<int64_t>(s0 + j) * a.H;
                const float* ml = ka.ws_ml + row * 4;
                mv[j] = ml[0];
                lv[j] = ml[1];
                xv[j] = ml[2];
                const float4* src = reinterpret_cast<const float4*>(ka.ws_o + row * 512 + d);
#pragma unroll
                for (int p = 0; p < 4; ++p) o[j][p] = src[32 * p];
            }
        }
#pragma unroll
        for (int j = 0; j < kCombChunk; ++j) {  // in split order
            if (!(lv[j] > 0.f)) continue;
            const float wgt = exp2f(mv[j] - M);
            L += lv[j] * wgt;
            LX += xv[j] * wgt;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                acc[p].x += o[j][p].x * wgt;
                acc[p].y += o[j][p].y * wgt;
                acc[p].z += o[j][p].z * wgt;
                acc[p].w += o[j][p].w * wgt;
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int64_t o0 = (static_cast<int64_t>(r) * a.H + h) * a.d_c + d;
    if (a.out_bf16) {
        uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.out_bf16) + o0 * 2);
#pragma unroll
        for (int p = 0; p < 4; ++p)
            dst[32 * p] = bf16x4_bits(make_float4(acc[p].x * inv, acc[p].y * inv, acc[p].z * inv, acc[p].w * inv));
    } else {
        float* dst = a.out + o0;
#pragma unroll
        for (int p = 0; p < 4; ++p)
            *reinterpret_cast<float4*>(dst + 128 * p) =
                make_float4(acc[p].x * inv, acc[p].y * inv, acc[p].z * inv, acc[p].w * inv);
    }
    if ((threadIdx.x & 31) == 0 && a.lse)
        a.lse[static_cast<int64_t>(r) * a.H + h] = L > 0.f ? (M + log2f(LX)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace

int mla_decode_splits(int rows, int k) {
    const int T = (k + kNK - 1) / kNK;
    int ns = sm_count() / (2 * rows);
    if (ns > T) ns = T;
    if (ns > 16) ns = 16;
    const int need = (T + kMaxTilesPerCta - 1) / kMaxTilesPerCta;  // tiles per CTA fit the row table
    if (ns < need) ns = need;
    if (ns < 1) ns = 1;
    return ns;
}

size_t mla_exchange_bytes() { return static_cast<size_t>(kMlaScratchSlots) * kMlaXBuf * kMlaXBytes; }

size_t mla_workspace_bytes(int rows, int H, int k, int d_c, int nsplit) {
    (void)k;
    size_t total = mla_exchange_bytes();
    if (nsplit > 1) {
        const size_t o = static_cast<size_t>(rows) * nsplit * H * d_c * 4;
        const size_t ml = static_cast<size_t>(rows) * nsplit * H * 4 * 4;
        total += ((o + 255) & ~size_t(255)) + ((ml + 255) & ~size_t(255));
    }
    return total;
}

sa_status sparse_mla_launch(const MlaArgs& a, int nsplit, void* ws, size_t ws_bytes, cudaStream_t st) {
    MlaKernelArgs ka;
    ka.a = a;
    ka.nsplit = nsplit;
    ka.ws_o = nullptr;
    ka.ws_ml = nullptr;
    const int T = (a.k + kNK - 1) / kNK;
    if ((T + nsplit - 1) / nsplit > kMaxTilesPerCta) return SA_EUNSUPPORTED;
    if (sm_count() > kMlaScratchSlots) return SA_EUNSUPPORTED;
    const size_t need = mla_workspace_bytes(a.rows, a.H, a.k, a.d_c, nsplit);
    if (ws == nullptr || ws_bytes < need) return SA_EINVAL;
    uint8_t* w = static_cast<uint8_t*>(ws);
    ka.xs = reinterpret_cast<float*>(w);
    w += mla_exchange_bytes();
    if (nsplit > 1) {
        const size_t o = static_cast<size_t>(a.rows) * nsplit * a.H * a.d_c * 4;
        ka.ws_o = reinterpret_cast<float*>(w);
        ka.ws_ml = reinterpret_cast<float*>(w + ((o + 255) & ~size_t(255)));
    }
    cudaError_t e = cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return launch_status(e);
    mla_kernel<<<2 * a.rows * nsplit, kThreads, kSmem, st>>>(ka);
    e = cudaGetLastError();
    if (e != cudaSuccess) return launch_status(e);
    if (nsplit > 1) {
        const int64_t heads = static_cast<int64_t>(a.rows) * a.H;
        e = launch_pdl(mla_combine_kernel, dim3(static_cast<unsigned>((heads + kCombHeads - 1) / kCombHeads)),
                       dim3(kCombThreads), 0, st, ka);
    }
    return launch_status(e);
}

}  // namespace sa

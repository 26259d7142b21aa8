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
//    dims 0..255, CTA 1 owns dims 256..511 plus the 64 RoPE dims.  Each CTA
//    keeps its slice of the 128-head query in shared memory (A operand,
//    K-major, 128B swizzle) and gathers only its slice of every selected row
//    with TMA tile::gather4 (4 rows x 128 B per instruction) into a 4-stage ring.
//  * Per 32-key tile, tcgen05.mma (M=128 heads, N=32 keys, K=16) forms the
//    CTA's partial scores in TMEM; the softmax warps (thread = head) read them,
//    swap them with the partner through distributed shared memory and add, so
//    both CTAs hold identical full scores and identical probabilities.
//  * Each CTA then aggregates its own 256 latent dims: O[128 x 256] (+)= P . V
//    with P (bf16, interleaved K-major) from shared memory and V = the gathered
//    latent slice read MN-major — the tile gathered for the scores is reused,
//    so every selected row is read from memory exactly once.
//  * Online softmax in base 2 with a lazy reference: O in TMEM is rescaled
//    only when a tile's maximum exceeds the reference by more than 2^8.
//  * Rows with few queries split their keys over several clusters; partial
//    (O, m, l) states go to a workspace and a combine kernel merges them.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kPage = 64;
constexpr int kNK = 32;          // keys per tile
constexpr int kStages = 4;
constexpr int kBlkQ = 128 * 128;  // one 64-dim slice of the 128-head query (bytes)
constexpr int kBlkK = kNK * 128;  // one 64-dim slice of a 32-key tile (bytes)
constexpr int kMaxBlk = 5;
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kMaxBlk * kBlkQ;
constexpr int kOffX = kOffStage + kStages * kMaxBlk * kBlkK;
constexpr int kXBytes = 128 * kNK * 4;
constexpr int kOffP = kOffX + 2 * kXBytes;
constexpr int kPBytes = 128 * kNK * 2;
constexpr int kSmem = kOffP + 2 * kPBytes + 1024;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.0f;

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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_kernel(const __grid_constant__ CUtensorMap tm_qlat, const __grid_constant__ CUtensorMap tm_qrope,
               const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_kr,
               const MlaKernelArgs ka) {
    const MlaArgs& a = ka.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = sm + kOffQ;
    uint8_t* sStage = sm + kOffStage;
    uint8_t* sX = sm + kOffX;
    uint8_t* sP = sm + kOffP;

    __shared__ uint64_t bar_q, bar_full[kStages], bar_empty[kStages], bar_sfull[2], bar_sfree[2], bar_xfull[2],
        bar_pfull[2], bar_pvdone[2], bar_final;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

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
        mbar_init(&bar_q, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_sfull[i], 1);
            mbar_init(&bar_sfree[i], 4);
            mbar_init(&bar_xfull[i], 128);
            mbar_init(&bar_pfull[i], 4);
            mbar_init(&bar_pvdone[i], 1);
        }
        mbar_init(&bar_final, 1);
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync_all();  // partner's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 4) {
        // ------------------------------------------------ producer: query slice + gathered rows
        if (lane == 0) {
            tma_prefetch_desc(&tm_c);
            mbar_arrive_expect_tx(&bar_q, nblk * kBlkQ);
            for (int b = 0; b < 4; ++b)
                tma_load_3d(sQ + b * kBlkQ, &tm_qlat, &bar_q, static_cast<int>(rank) * 256 + b * 64, 0, r);
            if (rank == 1) tma_load_3d(sQ + 4 * kBlkQ, &tm_qrope, &bar_q, 0, 0, r);
        }
        int stage = 0;
        uint32_t phase = 0;
        int64_t n_issued = 0;
        for (int t = 0; t < nt; ++t) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&bar_empty[stage], phase ^ 1, wc, kErrMlaWait | 1);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            const int slot = (t0 + t) * kNK + lane;
            const int p = slot < a.k ? a.idx[static_cast<int64_t>(r) * a.k + slot] : -1;
            const int row = p >= 0 ? static_cast<int>(pool_row(a, seq, p)) : 0;
            if (lane == 0) mbar_arrive_expect_tx(&bar_full[stage], nblk * kBlkK);
            __syncwarp();
            const int g = lane & 7, b = lane >> 3;
            const int y0 = __shfl_sync(0xffffffffu, row, 4 * g + 0), y1 = __shfl_sync(0xffffffffu, row, 4 * g + 1);
            const int y2 = __shfl_sync(0xffffffffu, row, 4 * g + 2), y3 = __shfl_sync(0xffffffffu, row, 4 * g + 3);
            uint8_t* dst = sStage + stage * (kMaxBlk * kBlkK);
            tma_gather4(dst + b * kBlkK + g * 512, &tm_c, &bar_full[stage], static_cast<int>(rank) * 256 + b * 64, y0,
                        y1, y2, y3);
            if (rank == 1 && b == 0) tma_gather4(dst + 4 * kBlkK + g * 512, &tm_kr, &bar_full[stage], 0, y0, y1, y2, y3);
            ++n_issued;
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1;
            }
        }
        if (lane == 0) {  // drain loads in flight
            int dummy = 0;
            WaitCtx dw{a.err, reinterpret_cast<volatile int*>(&dummy)};
            mbar_wait(&bar_q, 0, dw, kErrMlaWait | 9);
            for (int64_t i = n_issued - kStages; i < n_issued; ++i)
                if (i >= 0) mbar_wait(&bar_full[i % kStages], static_cast<uint32_t>((i / kStages) & 1), dw, kErrMlaWait | 10);
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t id_qk = idesc_f32acc(1, 1, false, false, 128, kNK);
        constexpr uint32_t id_pv = idesc_f32acc(1, 1, false, true, 128, 256);
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&bar_q, 0, wc, kErrMlaWait | 2);
        auto issue_pv = [&](int u) -> bool {
            const int pb = u & 1;
            if (!mbar_wait(&bar_pfull[pb], static_cast<uint32_t>((u >> 1) & 1), wc, kErrMlaWait | 3)) return false;
            tc_fence_after();
            const int st = u % kStages;
            const uint64_t pd = sdesc(smem_u32(sP + pb * kPBytes), 128, 512, kSwNone);
            const uint64_t vd = sdesc(smem_u32(sStage + st * (kMaxBlk * kBlkK)), 4096, 1024, kSw128);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
                mma_bf16_ss(tmem + kColO, pd + 16 * kk, vd + 128 * kk, id_pv, (u > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&bar_empty[st]);
            tc_commit(&bar_pvdone[pb]);
            return true;
        };
        if (lane == 0 && ok) {
            int stage = 0;
            uint32_t phase = 0;
            for (int t = 0; t < nt && ok; ++t) {
                ok = mbar_wait(&bar_full[stage], phase, wc, kErrMlaWait | 4);
                const int sb = t & 1;
                if (ok && t >= 2) ok = mbar_wait(&bar_sfree[sb], static_cast<uint32_t>(((t >> 1) - 1) & 1), wc, kErrMlaWait | 5);
                if (!ok) break;
                tc_fence_after();
                uint8_t* stg = sStage + stage * (kMaxBlk * kBlkK);
                for (int b = 0; b < nblk; ++b) {
                    const uint64_t qd = sdesc(smem_u32(sQ + b * kBlkQ), 16, 1024, kSw128);
                    const uint64_t kd = sdesc(smem_u32(stg + b * kBlkK), 16, 1024, kSw128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tmem + sb * kNK, qd + 2 * kk, kd + 2 * kk, id_qk, (b | kk) != 0 ? 1u : 0u);
                }
                tc_commit(&bar_sfull[sb]);
                if (t >= 1) ok = issue_pv(t - 1);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (ok && nt > 0) issue_pv(nt - 1);
        }
        if (lane == 0) {
            int dummy = 0;
            WaitCtx dw{a.err, reinterpret_cast<volatile int*>(&dummy)};
            tc_commit(&bar_final);
            mbar_wait(&bar_final, 0, dw, kErrMlaWait | 11);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax + exchange + output (thread = head)
        const int h = tid;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float c2 = a.scale * 1.4426950408889634f;  // scores in base-2 units
        float m = -INFINITY, l = 0.f, lx = 0.f;  // l: sum of bf16 P (normalises O); lx: fp32 sum (lse)
        const uint32_t x_remote = mapa_u32(smem_u32(sX), partner);
        const uint32_t xfull_remote0 = mapa_u32(smem_u32(&bar_xfull[0]), partner);
        const uint32_t xfull_remote1 = mapa_u32(smem_u32(&bar_xfull[1]), partner);
        bool ok = true;
        for (int t = 0; t < nt; ++t) {
            const int sb = t & 1;
            if (!(ok = warp_wait(&bar_sfull[sb], static_cast<uint32_t>((t >> 1) & 1), wc, kErrMlaWait | 6))) break;
            tc_fence_after();
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + sb * kNK, v);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sfree[sb]);
            // swap partial scores with the partner (row h, 8 chunks of 16 B, xor-swizzled)
            const uint32_t xrow = x_remote + sb * kXBytes + h * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_cluster_v4(xrow + ((c ^ (h & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            mbar_arrive_cluster(sb ? xfull_remote1 : xfull_remote0);
            if (!(ok = warp_wait<true>(&bar_xfull[sb], static_cast<uint32_t>((t >> 1) & 1), wc, kErrMlaWait | 7))) break;
            const uint8_t* xl = sX + sb * kXBytes + h * 128;
            float s[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = *reinterpret_cast<const float4*>(xl + ((c ^ (h & 7)) << 4));
                s[4 * c + 0] = __uint_as_float(v[4 * c + 0]) + x.x;
                s[4 * c + 1] = __uint_as_float(v[4 * c + 1]) + x.y;
                s[4 * c + 2] = __uint_as_float(v[4 * c + 2]) + x.z;
                s[4 * c + 3] = __uint_as_float(v[4 * c + 3]) + x.w;
            }
            const int slot = (t0 + t) * kNK + lane;
            const bool vld = slot < a.k && a.idx[static_cast<int64_t>(r) * a.k + slot] >= 0;
            const unsigned vmask = __ballot_sync(0xffffffffu, vld);
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                s[j] = ((vmask >> j) & 1u) ? s[j] * c2 : -INFINITY;
                mx = fmaxf(mx, s[j]);
            }
            const bool need = mx > m + kRescaleLog2;
            if (__any_sync(0xffffffffu, need)) {
                const float m_new = fmaxf(m, mx);
                const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
                if (t > 0) {  // O holds tiles < t: wait for the last product, then scale it
                    if (!(ok = warp_wait(&bar_pvdone[(t - 1) & 1], static_cast<uint32_t>(((t - 1) >> 1) & 1), wc,
                                         kErrMlaWait | 8)))
                        break;
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
                    tc_fence_before();
                }
                l *= alpha;
                lx *= alpha;
                m = m_new;
            }
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                // masked slots contribute exactly 0 (also while m is still -inf)
                const float p0 = ((vmask >> (2 * j)) & 1u) ? exp2f(s[2 * j] - m) : 0.f;
                const float p1 = ((vmask >> (2 * j + 1)) & 1u) ? exp2f(s[2 * j + 1] - m) : 0.f;
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                l += __low2float(b2) + __high2float(b2);
                lx += p0 + p1;
                pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            const int pb = t & 1;
            if (t >= 2 &&
                !(ok = warp_wait(&bar_pvdone[pb], static_cast<uint32_t>(((t >> 1) - 1) & 1), wc, kErrMlaWait | 12)))
                break;
            uint8_t* prow = sP + pb * kPBytes + (h >> 3) * 512 + (h & 7) * 16;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(prow + c * 128) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_pfull[pb]);
        }
        // ---- output: this CTA's 256 latent dims of every head
        if (ok && nt > 0)
            ok = warp_wait(&bar_pvdone[(nt - 1) & 1], static_cast<uint32_t>(((nt - 1) >> 1) & 1), wc, kErrMlaWait | 13);
        if (ok) {
            tc_fence_after();
            const bool partial = ka.nsplit > 1;
            const float inv = (l > 0.f && !partial) ? 1.f / l : 1.f;
            float* dst;
            if (partial)
                dst = ka.ws_o + ((static_cast<int64_t>(r) * ka.nsplit + split) * a.H + h) * 512 + rank * 256;
            else
                dst = a.out + (static_cast<int64_t>(r) * a.H + h) * a.d_c + rank * 256;
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
                if (h < a.H) {
                    const bool empty = !(l > 0.f);
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
            if (h < a.H && rank == 0) {
                if (partial) {
                    float* ml = ka.ws_ml + ((static_cast<int64_t>(r) * ka.nsplit + split) * a.H + h) * 4;
                    ml[0] = m;
                    ml[1] = l;
                    ml[2] = lx;
                } else if (a.lse) {
                    a.lse[static_cast<int64_t>(r) * a.H + h] = l > 0.f ? (m + log2f(lx)) * 0.6931471805599453f : -INFINITY;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the partner no longer writes into this CTA's shared memory
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, kTmemCols);
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
    const uint64_t pool_rows = static_cast<uint64_t>(a.pool_pages) * kPage;
    CUtensorMap tq, tqr, tc, tkr;
    {
        const uint64_t dims[3] = {512, static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.rows)};
        const uint64_t str[2] = {512 * 2, static_cast<uint64_t>(a.H) * 512 * 2};
        const uint32_t box[3] = {64, 128, 1};
        if (!encode_tiled(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.q_lat, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SA_ECUDA;
    }
    {
        const uint64_t dims[3] = {64, static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.rows)};
        const uint64_t str[2] = {64 * 2, static_cast<uint64_t>(a.H) * 64 * 2};
        const uint32_t box[3] = {64, 128, 1};
        if (!encode_tiled(&tqr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.q_rope, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SA_ECUDA;
    }
    {
        const uint64_t dims[2] = {512, pool_rows};
        const uint64_t str[1] = {static_cast<uint64_t>(a.c_ld) * 2};
        const uint32_t box[2] = {64, 1};
        if (!encode_tiled(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.c_cache, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SA_ECUDA;
    }
    {
        const uint64_t dims[2] = {64, pool_rows};
        const uint64_t str[1] = {static_cast<uint64_t>(a.kr_ld) * 2};
        const uint32_t box[2] = {64, 1};
        if (!encode_tiled(&tkr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.kr_cache, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SA_ECUDA;
    }
    cudaError_t e = cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return launch_status(e);
    mla_kernel<<<2 * a.rows * nsplit, kThreads, kSmem, st>>>(tq, tqr, tc, tkr, ka);
    e = cudaGetLastError();
    if (e != cudaSuccess) return launch_status(e);
    if (nsplit > 1) {
        mla_combine_kernel<<<a.rows * a.H, 128, 0, st>>>(ka);
        e = cudaGetLastError();
    }
    return launch_status(e);
}

}  // namespace sa

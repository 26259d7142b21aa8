// head_gemm.cu — the two per-head projections around sparse MLA.
//
// "MLA 与稀疏注意力" (“吸收矩阵”是交换线性计算的顺序): with the content key
// k^C_j = U_K c_j of head h, the content score q^C . k^C_j equals
// (U_K^T q^C) . c_j, so the query is absorbed once per row and head,
//   q_lat[r][h] = U_K[h]^T q_c[r][h]            (d_c outputs, d_C inputs),
// and the attention output stays in latent space until one up-projection
//   out[r][h]   = U_V[h] o_lat[r][h]            (d_v outputs, d_c inputs).
//
// Both are batched GEMMs over heads: for head h and a tile of 128 output
// features m, D[m][n] = sum_k A_h[m][k] X_h[n][k] over the rows n of the call.
// A is the head's weight, streamed by TMA in 64-wide K chunks through a ring
// (K-major for U_V[h] [d_v][d_c]; M-major for U_K[h] [d_C][d_c], whose rows
// are the reduction); X (the activations of up to 64 rows of the head) is
// converted to bf16 and staged whole in shared memory in the prologue.  One
// thread issues tcgen05 MMAs (M=128, N = rows rounded up to 16, K=16) into a
// TMEM accumulator; four warps write the outputs (thread = output feature,
// one column per row: coalesced across the warp).
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kGStages = 4;
constexpr int kGChunkK = 64;                  // K elements per ring stage (one 128-byte swizzle atom)
constexpr int kGStageBytes = 128 * kGChunkK * 2;  // A tile: 128 x 64 bf16
constexpr int kGMaxRows = 64;                 // activation rows per CTA (N <= 64)
constexpr int kGMaxK = 512;
constexpr int kGXChunkBytes = kGMaxRows * 128;  // one 64-wide K chunk of X (64 rows x 128 bytes)
// shared layout: min(kGStages, K chunks) A stages, then the K chunks of X
__host__ __device__ constexpr int g_stages(int nk) { return nk < kGStages ? nk : kGStages; }
__host__ __device__ constexpr int g_smem(int nk) { return g_stages(nk) * kGStageBytes + nk * kGXChunkBytes + 1024; }
constexpr int kGThreads = 192;                // 4 epilogue/staging warps, TMA warp, MMA warp

struct GemmArgs {
    const void* x;      // activations [rows][H][K] (bf16 or fp32)
    int x_fp32;         // 1: x is fp32 (converted to bf16 while staging)
    int rows, H, M, K;
    int a_mn_major;     // 1: A_h stored [K][M] (U_K); 0: [M][K] (U_V)
    void* y;            // [rows][H][M] outputs
    int y_fp32;         // 1: fp32 outputs, 0: bf16
    int* err;
};

__global__ void __launch_bounds__(kGThreads)
    head_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const GemmArgs g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nk = g.K / kGChunkK;
    const int nst = g_stages(nk);
    uint8_t* sX = sm + nst * kGStageBytes;
    __shared__ uint64_t bar_full[kGStages], bar_empty[kGStages], bar_acc;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * 128, h = blockIdx.y, n0 = blockIdx.z * kGMaxRows;
    const int nrows = min(kGMaxRows, g.rows - n0);
    const int npad = (nrows + 15) & ~15;  // MMA N
    WaitCtx wc{g.err, &s_abort};

    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < nst; ++i) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], 1);
        }
        mbar_init(&bar_acc, 1);
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&s_tmem, 64);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) tma_prefetch_desc(&tm_a);
    // X of this head: row n, K chunk c -> 128-byte row n of chunk c, 16-byte
    // pieces swizzled by (n & 7); rows past nrows are zero.  Four pieces per
    // thread are loaded before any is stored (loads in flight together).
    {
        constexpr int kU = 4;
        const int total = nk * kGMaxRows * 8;
        for (int base = tid; base < total; base += kU * kGThreads) {
            uint4 v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = base + u * kGThreads;
                const int c = i / (kGMaxRows * 8), n = (i / 8) % kGMaxRows, p = i % 8;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (i < total && n < nrows) {
                    const int64_t e = ((static_cast<int64_t>(n0 + n) * g.H + h) * g.K) + c * kGChunkK + p * 8;
                    if (g.x_fp32) {
                        const float4* f = reinterpret_cast<const float4*>(static_cast<const float*>(g.x) + e);
                        const float4 a = __ldg(f), b = __ldg(f + 1);
                        v[u] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                                          pack_bf16x2(b.z, b.w));
                    } else {
                        v[u] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(g.x) + e));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = base + u * kGThreads;
                if (i < total) {
                    const int c = i / (kGMaxRows * 8), n = (i / 8) % kGMaxRows, p = i % 8;
                    *reinterpret_cast<uint4*>(sX + c * kGXChunkBytes + n * 128 + ((p ^ (n & 7)) << 4)) = v[u];
                }
            }
        }
    }
    fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 4) {
        // ------------------------------------------------ TMA: A chunks
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int c = 0; c < nk; ++c) {
                if (!mbar_wait(&bar_empty[stage], phase ^ 1, wc, kErrGemmWait | 1)) break;
                uint8_t* dst = sm + stage * kGStageBytes;
                mbar_arrive_expect_tx(&bar_full[stage], kGStageBytes);
                if (g.a_mn_major) {
                    // two 64 (M) x 64 (K) boxes: M = m0..m0+63 and m0+64..m0+127
                    tma_load_3d(dst, &tm_a, &bar_full[stage], m0, c * kGChunkK, h);
                    tma_load_3d(dst + kGStageBytes / 2, &tm_a, &bar_full[stage], m0 + 64, c * kGChunkK, h);
                } else {
                    tma_load_3d(dst, &tm_a, &bar_full[stage], c * kGChunkK, m0, h);  // 128 (M) x 64 (K)
                }
                if (++stage == nst) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_f32acc(1, 1, g.a_mn_major != 0, false, 128, npad);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int c = 0; c < nk && ok; ++c) {
                ok = mbar_wait(&bar_full[stage], phase, wc, kErrGemmWait | 2);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(sm + stage * kGStageBytes);
                const uint64_t ad = g.a_mn_major ? sdesc(a_addr, kGStageBytes / 2, 1024, kSw128)
                                                 : sdesc(a_addr, 16, 1024, kSw128);
                const uint64_t bd = sdesc(smem_u32(sX + c * kGXChunkBytes), 16, 1024, kSw128);
#pragma unroll
                for (int kk = 0; kk < kGChunkK / 16; ++kk) {
                    // K advance: 32 bytes along a K-major row, or 16 rows of 128 bytes M-major
                    const uint64_t a_k = g.a_mn_major ? ad + 128 * kk : ad + 2 * kk;
                    mma_bf16_ss(tmem, a_k, bd + 2 * kk, idesc, (c | kk) != 0 ? 1u : 0u);
                }
                tc_commit(&bar_empty[stage]);
                if (++stage == nst) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            tc_commit(&bar_acc);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue: thread = output feature m0 + tid
        const int m = m0 + tid;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        if (warp_wait(&bar_acc, 0, wc, kErrGemmWait | 3)) {
            tc_fence_after();
            for (int c0 = 0; c0 < npad; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + lane_base + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c0 + j;
                    if (n < nrows && m < g.M) {
                        const int64_t e = (static_cast<int64_t>(n0 + n) * g.H + h) * g.M + m;
                        if (g.y_fp32)
                            static_cast<float*>(g.y)[e] = __uint_as_float(v[j]);
                        else
                            static_cast<__nv_bfloat16*>(g.y)[e] = __float2bfloat16_rn(__uint_as_float(v[j]));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 64);
}

sa_status head_gemm_launch(const void* a, const GemmArgs& g, cudaStream_t st) {
    CUtensorMap tm;
    bool ok;
    if (g.a_mn_major) {
        // A_h stored [K][M]: dims {M, K, H}, box 64 (M) x 64 (K)
        const uint64_t dims[3] = {static_cast<uint64_t>(g.M), static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.H)};
        const uint64_t str[2] = {static_cast<uint64_t>(g.M) * 2, static_cast<uint64_t>(g.M) * g.K * 2};
        const uint32_t box[3] = {64, kGChunkK, 1};
        ok = encode_tiled(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        // A_h stored [M][K]: dims {K, M, H}, box 64 (K) x 128 (M)
        const uint64_t dims[3] = {static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.M), static_cast<uint64_t>(g.H)};
        const uint64_t str[2] = {static_cast<uint64_t>(g.K) * 2, static_cast<uint64_t>(g.M) * g.K * 2};
        const uint32_t box[3] = {kGChunkK, 128, 1};
        ok = encode_tiled(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!ok) return SA_ECUDA;
    const int smem = g_smem(g.K / kGChunkK);
    cudaError_t e = cudaFuncSetAttribute(head_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         g_smem(kGMaxK / kGChunkK));
    if (e != cudaSuccess) return launch_status(e);
    const dim3 grid(g.M / 128, g.H, (g.rows + kGMaxRows - 1) / kGMaxRows);
    head_gemm_kernel<<<grid, kGThreads, smem, st>>>(tm, g);
    return launch_status(cudaGetLastError());
}

}  // namespace

sa_status mla_absorb_query_launch(const void* q_c, const void* U_K, int rows, int H, int d_C, int d_c, void* q_lat,
                                  int* err, cudaStream_t st) {
    GemmArgs g{q_c, 0, rows, H, d_c, d_C, 1, q_lat, 0, err};
    return head_gemm_launch(U_K, g, st);
}

sa_status mla_up_project_launch(const void* o_lat, bool o_lat_fp32, const void* U_V, int rows, int H, int d_c,
                                int d_v, float* out, int* err, cudaStream_t st) {
    GemmArgs g{o_lat, o_lat_fp32 ? 1 : 0, rows, H, d_v, d_c, 0, out, 1, err};
    return head_gemm_launch(U_V, g, st);
}

}  // namespace sa

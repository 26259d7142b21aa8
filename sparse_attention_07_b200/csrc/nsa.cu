// nsa.cu — NSA three-branch decode over a GQA group.
//
// "MLA 与稀疏注意力：少存一点，还是少看一点？" (NSA sections "三条路径，各留住什么？"
// and "选块和合并输出，实际算一遍") and "LLM注意力优化：稀疏注意力" (NSA steps
// 1-3): for one decode query per head, three attention branches over the
// history of the KV head the group shares, each with its own softmax:
//   compression  over the mean of every complete block of keys / values
//                ("第 11 章 稀疏注意力" §12.6 mean compression; only complete
//                blocks are summarised);
//   selection    over all tokens of the top blocks, chosen once for the group
//                by the sum over its heads of the compression probabilities
//                (shared_block_choice; ties to the lower block);
//   window       over the last `window` positions;
// mixed by independent gates: out = g_c o_c + g_s o_s + g_w o_w.
//
// nsa_compress: one warp per (sequence, KV head, block, K|V) sums the block's
// rows in fp32 in token order and stores mean rounded to bf16 (the compressed
// cache, built when a block completes).
//
// nsa_decode: a cluster of kC CTAs per (sequence, KV head).  Every CTA streams
// its share of the data through one ring of 32-row items (cp.async, padded
// rows): window K rows, compressed K rows (its chunk of blocks), window V,
// compressed V, then selected-block K and V.  Contractions run on mma.sync
// m16n8k16 bf16 with the group's heads as N = 8 (scores as S^T = K Q^T,
// outputs as O^T = V^T P^T): with at most 16 query rows per KV head, tcgen05's
// smallest tile (M = 64) would be mostly padding, and the kernel is bound by
// HBM, not by the tensor pipe.  After the compressed keys, the CTAs exchange
// per-head softmax statistics through distributed shared memory, form the
// group's block probabilities for their chunk, and agree on the top blocks by
// merging per-CTA candidate lists (each CTA merges the same lists, so all hold
// the same choice).  Partial (max, sum, output) states of the three branches
// are combined through distributed shared memory at the end.
#include <algorithm>

#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kD = 128;
constexpr int kC = 8;                  // CTAs per (sequence, KV head)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 32;              // rows per ring item
constexpr int kRowB = 2 * kD + 16;     // padded bf16 row: 272 B keeps ldmatrix rows on distinct banks
constexpr int kItemB = kRows * kRowB;  // 8704 B
constexpr int kStages = 8;
constexpr int kRingB = kStages * kItemB;
constexpr int kMaxTop = 64;
constexpr int kMaxG = 16;
constexpr float kLog2e = 1.4426950408889634f;

// --------------------------------------------------------------- compression
__global__ void __launch_bounds__(256) nsa_compress_kernel(const __nv_bfloat16* __restrict__ K,
                                                           const __nv_bfloat16* __restrict__ V, int64_t sb,
                                                           int64_t st, int64_t sh, int Hkv, int nb, int block,
                                                           __nv_bfloat16* __restrict__ Kc,
                                                           __nv_bfloat16* __restrict__ Vc, int64_t c_ld,
                                                           int64_t units) {
    const int64_t unit = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (unit >= units) return;
    const int which = static_cast<int>(unit & 1);  // 0: keys, 1: values
    const int64_t u = unit >> 1;
    const int n = static_cast<int>(u % nb);
    const int h = static_cast<int>((u / nb) % Hkv);
    const int64_t b = u / (static_cast<int64_t>(nb) * Hkv);
    const __nv_bfloat16* src = (which ? V : K) + b * sb + h * sh + static_cast<int64_t>(n) * block * st + lane * 4;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
    for (int i = 0; i < block; ++i) {  // token order, plain fp32 adds
        const uint2 raw = *reinterpret_cast<const uint2*>(src + i * st);
        const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        a0 = __fadd_rn(a0, __low2float(x));
        a1 = __fadd_rn(a1, __high2float(x));
        a2 = __fadd_rn(a2, __low2float(y));
        a3 = __fadd_rn(a3, __high2float(y));
    }
    const float inv = 1.f / static_cast<float>(block);
    uint2 o;
    o.x = pack_bf16x2(__fmul_rn(a0, inv), __fmul_rn(a1, inv));
    o.y = pack_bf16x2(__fmul_rn(a2, inv), __fmul_rn(a3, inv));
    __nv_bfloat16* dst = (which ? Vc : Kc) + ((b * Hkv + h) * c_ld + n) * kD + lane * 4;
    *reinterpret_cast<uint2*>(dst) = o;
}

// --------------------------------------------------------------- decode
struct NsaArgs {
    const __nv_bfloat16* q;  // [B][H][D]
    const __nv_bfloat16* K;
    const __nv_bfloat16* V;
    int64_t sb, st, sh;      // token cache strides (elements)
    const __nv_bfloat16* Kc; // [B][Hkv][c_ld][D]
    const __nv_bfloat16* Vc;
    int64_t c_ld;
    const float* gates;      // [B][H][3]: compression, selection, window
    float* out;              // [B][H][D]
    int32_t* sel;            // [B][Hkv][top] or null
    int H, Hkv, G, L, block, top, window;
    float scale;
    int per;                 // compressed blocks per CTA (multiple of kRows)
    int ftok;                // capacity of the fine-branch score rows (multiple of kRows)
};

// Shared-memory plan (bytes from the dynamic base); every region 16-byte aligned.
struct Smem {
    int q, sc, pc, sf, pf, keyw, cand, glob, total;
    int ld_sc, ld_pc, ld_sf, ld_pf;  // row strides in elements
};

__host__ __device__ inline Smem smem_plan(int gp, int per, int ftok, int top) {
    Smem s;
    s.ld_sc = per + 4;   // fp32 rows: stride = 4 mod 32 words spreads the fragment stores over the banks
    s.ld_pc = per + 8;   // bf16 rows: stride = 4 mod 8 words, conflict-free B-fragment loads
    s.ld_sf = ftok + 4;
    s.ld_pf = ftok + 8;
    int off = kRingB;
    auto take = [&](int bytes) {
        const int at = off;
        off += (bytes + 15) & ~15;
        return at;
    };
    s.q = take(gp * kRowB);
    s.sc = take(gp * s.ld_sc * 4);
    s.pc = take(gp * s.ld_pc * 2);
    s.sf = take(gp * s.ld_sf * 4);
    s.pf = take(gp * s.ld_pf * 2);
    s.keyw = take(per * 8);
    s.cand = take(kWarps * top * 8);
    s.glob = take(kC * top * 8);
    s.total = off;
    return s;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most n (0 <= n < kStages) of this thread's cp.async groups are pending.
__device__ __forceinline__ void cp_async_wait_n(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
        case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    }
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int o) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), o);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), o);
    return (static_cast<unsigned long long>(hi) << 32) | lo;
}

// One warp: the `count` largest nonzero keys of keys[0, n) into out[0, count)
// (zero where fewer exist), largest first.  Keys are unique; taken keys are
// zeroed in place.
__device__ void warp_top(unsigned long long* keys, int n, int count, unsigned long long* out, int lane) {
    for (int round = 0; round < count; ++round) {
        unsigned long long best = 0ull;
        int bj = -1;
        for (int j = lane; j < n; j += 32) {
            const unsigned long long k = keys[j];
            if (k > best) {
                best = k;
                bj = j;
            }
        }
        unsigned long long w = best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long x = shfl_xor_u64(w, o);
            w = x > w ? x : w;
        }
        if (w != 0ull && best == w) keys[bj] = 0ull;
        if (lane == 0) out[round] = w;
        __syncwarp();
    }
}

// Block key: larger is better; probability bits (nonnegative floats order as
// their bit patterns) above the complemented block index (ties to the lower
// block).  Zero is reserved for "no block".
__device__ __forceinline__ unsigned long long block_key(float p, int n) {
    return (static_cast<unsigned long long>(__float_as_uint(p)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(n));
}

__device__ __forceinline__ int key_block(unsigned long long k) {
    return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(k));
}

// Softmax of one branch from its score rows s[h][0, npos) (log2 units, -inf
// for positions that do not exist): per head the max m, P = bf16(2^(s - m))
// into the bf16 rows p, l = sum of P as rounded (the normaliser of the output
// the tensor cores form from P).  With `keep`, the fp32 2^(s - m) replaces the
// scores and its sum goes to Lsel (the compression probabilities that choose
// blocks).  One warp per head; heads G .. GP-1 (padding) get P = 0.
__device__ void branch_softmax(float* s, int ld_s, __nv_bfloat16* p, int ld_p, int npos, int G, int GP, bool keep,
                               float* m_out, float* l_out, float* lsel_out, int warp, int lane) {
    for (int h = warp; h < GP; h += kWarps) {
        float* row = s + h * ld_s;
        __nv_bfloat16* prow = p + h * ld_p;
        if (h >= G) {
            for (int j = lane; j < npos; j += 32) prow[j] = __float2bfloat16_rn(0.f);
            continue;
        }
        float m = -INFINITY;
        for (int j = lane; j < npos; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f, ls = 0.f;
        for (int j = lane; j < npos; j += 32) {
            const float e = m == -INFINITY ? 0.f : fast_exp2(row[j] - m);
            const __nv_bfloat16 eb = __float2bfloat16_rn(e);
            prow[j] = eb;
            l += __bfloat162float(eb);
            ls += e;
            if (keep) row[j] = e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            l += __shfl_xor_sync(0xffffffffu, l, o);
            ls += __shfl_xor_sync(0xffffffffu, ls, o);
        }
        if (lane == 0) {
            m_out[h] = m;
            l_out[h] = l;
            if (lsel_out) lsel_out[h] = ls;
        }
    }
}

struct Plan {
    int b, kvh, r;
    int nwi, nci, nsi, nA, n_items;  // items: window K, compressed K, window V, compressed V, selected K, selected V
    int w_lo, n_lo, n_hi, ipb;
};

// cp.async of ring item i (32 rows of 256 B) into its slot; rows that do not
// exist are zero-filled.  Every thread copies two 16-byte pieces.
__device__ __forceinline__ void issue_item(const NsaArgs& a, const Plan& p, int i, uint32_t ring_s,
                                           const int* chosen) {
    const uint32_t base = ring_s + static_cast<uint32_t>((i % kStages) * kItemB);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int idx = static_cast<int>(threadIdx.x) + k * kThreads;
        const int row = idx >> 4, ch = idx & 15;
        const __nv_bfloat16* src = a.Kc;
        bool ok;
        int j = i;
        if (j < p.nwi || (j >= p.nwi + p.nci && j < 2 * p.nwi + p.nci)) {  // window rows
            const bool isv = j >= p.nwi;
            if (isv) j -= p.nwi + p.nci;
            const int t = p.w_lo + kRows * (p.r + kC * j) + row;
            ok = t < a.L;
            if (ok) src = (isv ? a.V : a.K) + p.b * a.sb + static_cast<int64_t>(t) * a.st + p.kvh * a.sh;
        } else if (j < p.nA) {  // compressed rows
            const bool isv = j >= 2 * p.nwi + p.nci;
            j -= isv ? 2 * p.nwi + p.nci : p.nwi;
            const int n = p.n_lo + kRows * j + row;
            ok = n < p.n_hi;
            if (ok) src = (isv ? a.Vc : a.Kc) + ((static_cast<int64_t>(p.b) * a.Hkv + p.kvh) * a.c_ld + n) * kD;
        } else {  // rows of the selected blocks
            j -= p.nA;
            const bool isv = j >= p.nsi;
            if (isv) j -= p.nsi;
            const int blk = chosen[p.r + kC * (j / p.ipb)];
            const int t = blk * a.block + kRows * (j % p.ipb) + row;
            ok = true;
            src = (isv ? a.V : a.K) + p.b * a.sb + static_cast<int64_t>(t) * a.st + p.kvh * a.sh;
        }
        cp_async16(base + static_cast<uint32_t>(row * kRowB + ch * 16), ok ? src + ch * 8 : a.Kc, ok ? 16u : 0u);
    }
}

// Scores of one item: S^T[32 rows x GP heads] = rows . Q^T on warps
// (m-tile, n-tile) < (2, NT); results (log2 units) into dst[h][pos0 + row],
// -inf where the row does not exist.
template <int NT>
__device__ __forceinline__ void item_scores(uint32_t item_s, const uint32_t (&qb)[8][2], float* dst, int ld,
                                            int pos0, int nvalid_rows, float c2, int warp, int lane) {
    if (warp >= 2 * NT) return;
    const int mt = warp & 1, nt = warp >> 1;
    const int g = lane >> 2, c4 = lane & 3;
    const uint32_t abase =
        item_s + static_cast<uint32_t>((16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8) * kRowB + (lane >> 4) * 16);
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        uint32_t af[4];
        ldsm_x4(abase + kk * 32, af);
        mma_bf16_16816(d, af, qb[kk][0], qb[kk][1]);
    }
    const int r0 = 16 * mt + g, r1 = r0 + 8;
    const int h0 = 8 * nt + 2 * c4;
    dst[h0 * ld + pos0 + r0] = r0 < nvalid_rows ? d[0] * c2 : -INFINITY;
    dst[(h0 + 1) * ld + pos0 + r0] = r0 < nvalid_rows ? d[1] * c2 : -INFINITY;
    dst[h0 * ld + pos0 + r1] = r1 < nvalid_rows ? d[2] * c2 : -INFINITY;
    dst[(h0 + 1) * ld + pos0 + r1] = r1 < nvalid_rows ? d[3] * c2 : -INFINITY;
}

// O^T[16 dims of this warp x GP heads] += rows^T . P^T over one item's 32 rows.
template <int NT>
__device__ __forceinline__ void item_pv(uint32_t item_s, const __nv_bfloat16* P, int ldp, int pos0, float (&acc)[NT][4],
                                        int warp, int lane) {
    const int g = lane >> 2, c4 = lane & 3;
    const uint32_t vbase = item_s + static_cast<uint32_t>(((lane & 7) + ((lane >> 4) & 1) * 8) * kRowB +
                                                          (16 * warp + ((lane >> 3) & 1) * 8) * 2);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t af[4];
        ldsm_x4_trans(vbase + ks * 16 * kRowB, af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const __nv_bfloat16* pr = P + (8 * nt + g) * ldp + pos0 + 16 * ks + 2 * c4;
            mma_bf16_16816(acc[nt], af, *reinterpret_cast<const uint32_t*>(pr),
                           *reinterpret_cast<const uint32_t*>(pr + 8));
        }
    }
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) { return __uint_as_float(ld_cluster_u32(addr)); }

template <int NT>
__global__ void __cluster_dims__(kC, 1, 1) __launch_bounds__(kThreads, 2) nsa_decode_kernel(const NsaArgs a) {
    constexpr int GP = 8 * NT;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ float s_m[3][kMaxG], s_l[3][kMaxG];  // per branch (compression, selection, window) and head
    __shared__ float s_lsel[kMaxG], s_fac[kMaxG];
    __shared__ float s_pub_m[kMaxG], s_pub_L[kMaxG];  // read by the other CTAs of the cluster
    __shared__ unsigned long long s_pub_top[kMaxTop];
    __shared__ int s_chosen[kMaxTop];
    __shared__ int s_nch;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G;
    const Smem sp = smem_plan(GP, a.per, a.ftok, a.top);
    const uint32_t ring_s = smem_u32(smem);
    float* s_sc = reinterpret_cast<float*>(smem + sp.sc);
    __nv_bfloat16* s_pc = reinterpret_cast<__nv_bfloat16*>(smem + sp.pc);
    float* s_sf = reinterpret_cast<float*>(smem + sp.sf);
    __nv_bfloat16* s_pf = reinterpret_cast<__nv_bfloat16*>(smem + sp.pf);
    unsigned long long* keyw = reinterpret_cast<unsigned long long*>(smem + sp.keyw);
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + sp.cand);
    unsigned long long* glob = reinterpret_cast<unsigned long long*>(smem + sp.glob);

    Plan p;
    p.r = static_cast<int>(cluster_rank());
    {
        const int pair = static_cast<int>(blockIdx.x) / kC;
        p.b = pair / a.Hkv;
        p.kvh = pair % a.Hkv;
    }
    const int nb = a.L / a.block;
    p.n_lo = p.r * a.per;
    p.n_hi = min(nb, p.n_lo + a.per);
    const int nvc = max(0, p.n_hi - p.n_lo);
    p.nci = (nvc + kRows - 1) / kRows;
    const int nw = min(a.window, a.L);
    p.w_lo = a.L - nw;
    const int tw = (nw + kRows - 1) / kRows;
    p.nwi = tw > p.r ? (tw - p.r + kC - 1) / kC : 0;
    const int ntop = min(a.top, nb);
    p.ipb = a.block / kRows;
    p.nsi = (ntop > p.r ? (ntop - p.r + kC - 1) / kC : 0) * p.ipb;
    p.nA = 2 * (p.nwi + p.nci);
    p.n_items = p.nA + 2 * p.nsi;
    const float c2 = a.scale * kLog2e;

    // the group's queries, zero rows for padding heads
    const int64_t qrow0 = static_cast<int64_t>(p.b) * a.H + static_cast<int64_t>(p.kvh) * G;
    for (int idx = tid; idx < GP * 16; idx += kThreads) {
        const int h = idx >> 4, ch = idx & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (h < G) v = *reinterpret_cast<const uint4*>(a.q + (qrow0 + h) * kD + ch * 8);
        *reinterpret_cast<uint4*>(smem + sp.q + h * kRowB + ch * 16) = v;
    }
    if (tid < 3 * kMaxG) {
        s_m[tid / kMaxG][tid % kMaxG] = -INFINITY;
        s_l[tid / kMaxG][tid % kMaxG] = 0.f;
    }
    __syncthreads();
    uint32_t qb[8][2];
    {
        const int nt = (warp >> 1) < NT ? (warp >> 1) : 0;
        const uint8_t* qr = smem + sp.q + (8 * nt + (lane >> 2)) * kRowB + (lane & 3) * 4;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qb[kk][0] = *reinterpret_cast<const uint32_t*>(qr + kk * 32);
            qb[kk][1] = *reinterpret_cast<const uint32_t*>(qr + kk * 32 + 16);
        }
    }

    float acc_c[NT][4], acc_s[NT][4], acc_w[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc_c[nt][e] = acc_s[nt][e] = acc_w[nt][e] = 0.f;

    bool ready = false;  // the selected blocks are known
    int issued = 0;
    auto top_up = [&](int limit) {
        while (issued < limit && issued < p.n_items && (issued < p.nA || ready)) {
            issue_item(a, p, issued, ring_s, s_chosen);
            cp_async_commit();
            ++issued;
        }
    };

    // Compression softmax, the cluster's exchange of its statistics, the
    // group's block probabilities and the shared choice of blocks; also the
    // window softmax (its scores are complete by then).
    auto choose = [&]() {
        __syncthreads();
        branch_softmax(s_sf, sp.ld_sf, s_pf, sp.ld_pf, kRows * p.nwi, G, GP, false, s_m[2], s_l[2], nullptr, warp,
                       lane);
        branch_softmax(s_sc, sp.ld_sc, s_pc, sp.ld_pc, kRows * p.nci, G, GP, true, s_m[0], s_l[0], s_lsel, warp,
                       lane);
        __syncthreads();
        if (tid < kMaxG) {
            s_pub_m[tid] = tid < G ? s_m[0][tid] : -INFINITY;
            s_pub_L[tid] = tid < G ? s_lsel[tid] : 0.f;
        }
        cluster_sync_all();
        if (tid < G) {
            float mr[kC], Lr[kC];
            float M = -INFINITY;
#pragma unroll
            for (int rr = 0; rr < kC; ++rr) {
                mr[rr] = ld_cluster_f32(mapa_u32(smem_u32(&s_pub_m[tid]), rr));
                Lr[rr] = ld_cluster_f32(mapa_u32(smem_u32(&s_pub_L[tid]), rr));
                M = fmaxf(M, mr[rr]);
            }
            float Lt = 0.f;
#pragma unroll
            for (int rr = 0; rr < kC; ++rr)
                if (mr[rr] != -INFINITY) Lt += Lr[rr] * exp2f(mr[rr] - M);
            const float mine = s_m[0][tid];
            s_fac[tid] = (mine != -INFINITY && Lt > 0.f) ? exp2f(mine - M) / Lt : 0.f;
        }
        __syncthreads();
        // the group's probability of each block of this chunk, as a key
        for (int n = tid; n < kRows * p.nci; n += kThreads) {
            unsigned long long k = 0ull;
            if (n < nvc) {
                float pg = 0.f;
                for (int h = 0; h < G; ++h) pg += s_sc[h * sp.ld_sc + n] * s_fac[h];
                k = block_key(pg, p.n_lo + n);
            }
            keyw[n] = k;
        }
        __syncthreads();
        if (ntop > 0) {
            const int span = kRows * p.nci;
            const int sl = (span + kWarps - 1) / kWarps;
            const int lo = min(span, warp * sl);
            warp_top(keyw + lo, min(span, lo + sl) - lo, ntop, cand + warp * ntop, lane);
        }
        __syncthreads();
        if (warp == 0 && ntop > 0) warp_top(cand, kWarps * ntop, ntop, s_pub_top, lane);
        cluster_sync_all();
        if (warp == 0) {
            if (ntop > 0) {
                for (int j = lane; j < kC * ntop; j += 32) {
                    const uint32_t ra = mapa_u32(smem_u32(&s_pub_top[j % ntop]), static_cast<uint32_t>(j / ntop));
                    const uint32_t lo = ld_cluster_u32(ra), hi = ld_cluster_u32(ra + 4);
                    glob[j] = (static_cast<unsigned long long>(hi) << 32) | lo;
                }
                __syncwarp();
                warp_top(glob, kC * ntop, ntop, cand, lane);
                __syncwarp();
                if (lane == 0) {
                    int nch = 0;
                    for (int j = 0; j < ntop; ++j) {
                        if (cand[j] == 0ull) continue;
                        const int v = key_block(cand[j]);
                        int t = nch++;
                        while (t > 0 && s_chosen[t - 1] > v) {
                            s_chosen[t] = s_chosen[t - 1];
                            --t;
                        }
                        s_chosen[t] = v;
                    }
                    s_nch = nch;
                }
            } else if (lane == 0) {
                s_nch = 0;
            }
        }
        __syncthreads();
        if (p.r == 0 && a.sel != nullptr && tid < a.top)
            a.sel[(static_cast<int64_t>(p.b) * a.Hkv + p.kvh) * a.top + tid] = tid < s_nch ? s_chosen[tid] : -1;
        ready = true;
    };

    top_up(kStages - 1);
    if (p.nwi + p.nci == 0) {
        choose();
        top_up(kStages - 1);
    }
    for (int i = 0; i < p.n_items; ++i) {
        cp_async_wait_n(issued - i - 1);
        __syncthreads();
        top_up(i + kStages);  // into the slot of item i - 1
        const uint32_t item_s = ring_s + static_cast<uint32_t>((i % kStages) * kItemB);
        if (i < p.nwi) {
            const int t0 = p.w_lo + kRows * (p.r + kC * i);
            item_scores<NT>(item_s, qb, s_sf, sp.ld_sf, kRows * i, a.L - t0, c2, warp, lane);
        } else if (i < p.nwi + p.nci) {
            const int j = i - p.nwi;
            item_scores<NT>(item_s, qb, s_sc, sp.ld_sc, kRows * j, nvc - kRows * j, c2, warp, lane);
        } else if (i < 2 * p.nwi + p.nci) {
            item_pv<NT>(item_s, s_pf, sp.ld_pf, kRows * (i - p.nwi - p.nci), acc_w, warp, lane);
        } else if (i < p.nA) {
            item_pv<NT>(item_s, s_pc, sp.ld_pc, kRows * (i - 2 * p.nwi - p.nci), acc_c, warp, lane);
        } else if (i < p.nA + p.nsi) {
            item_scores<NT>(item_s, qb, s_sf, sp.ld_sf, kRows * (i - p.nA), kRows, c2, warp, lane);
        } else {
            item_pv<NT>(item_s, s_pf, sp.ld_pf, kRows * (i - p.nA - p.nsi), acc_s, warp, lane);
        }
        if (i + 1 == p.nwi + p.nci) {
            choose();
            top_up(i + kStages);
        }
        if (p.nsi > 0 && i + 1 == p.nA + p.nsi) {
            __syncthreads();
            branch_softmax(s_sf, sp.ld_sf, s_pf, sp.ld_pf, kRows * p.nsi, G, GP, false, s_m[1], s_l[1], nullptr, warp,
                           lane);
        }
    }
    __syncthreads();  // every item consumed: the ring holds the partial states now

    float* pm = reinterpret_cast<float*>(smem);  // [3][kMaxG]
    float* pl = pm + 3 * kMaxG;                  // [3][kMaxG]
    float* po = pl + 3 * kMaxG;                  // [3][GP][kD]
    if (tid < 3 * kMaxG) {
        pm[tid] = s_m[tid / kMaxG][tid % kMaxG];
        pl[tid] = s_l[tid / kMaxG][tid % kMaxG];
    }
    {
        const int g = lane >> 2, c4 = lane & 3;
        const int d0 = 16 * warp + g;
#pragma unroll
        for (int br = 0; br < 3; ++br) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float* acc = br == 0 ? acc_c[nt] : (br == 1 ? acc_s[nt] : acc_w[nt]);
                float* o = po + (br * GP + 8 * nt + 2 * c4) * kD;
                o[d0] = acc[0];
                o[kD + d0] = acc[1];
                o[d0 + 8] = acc[2];
                o[kD + d0 + 8] = acc[3];
            }
        }
    }
    cluster_sync_all();
    {
        const int h = p.r + kC * (tid >> 7), d = tid & (kD - 1);
        if (h < G) {
            float res = 0.f;
#pragma unroll
            for (int br = 0; br < 3; ++br) {
                float mr[kC];
                float M = -INFINITY;
#pragma unroll
                for (int rr = 0; rr < kC; ++rr) {
                    mr[rr] = ld_cluster_f32(mapa_u32(smem_u32(pm + br * kMaxG + h), rr));
                    M = fmaxf(M, mr[rr]);
                }
                float num = 0.f, den = 0.f;
#pragma unroll
                for (int rr = 0; rr < kC; ++rr) {
                    if (mr[rr] == -INFINITY) continue;
                    const float w = exp2f(mr[rr] - M);
                    den += w * ld_cluster_f32(mapa_u32(smem_u32(pl + br * kMaxG + h), rr));
                    num += w * ld_cluster_f32(mapa_u32(smem_u32(po + (br * GP + h) * kD + d), rr));
                }
                const float o = den > 0.f ? num / den : 0.f;
                res += a.gates[(qrow0 + h) * 3 + br] * o;
            }
            a.out[(qrow0 + h) * kD + d] = res;
        }
    }
    cluster_sync_all();  // the other CTAs have read this CTA's partial states
}

}  // namespace

sa_status nsa_compress_launch(const void* K, const void* V, int64_t sb, int64_t st_, int64_t sh, int B, int L,
                              int Hkv, int block, void* Kc, void* Vc, int64_t c_ld, cudaStream_t st) {
    const int nb = L / block;
    const int64_t units = 2 * static_cast<int64_t>(B) * Hkv * nb;
    if (units == 0) return SA_OK;
    const int64_t grid = (units + 7) / 8;
    nsa_compress_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), sb, st_, sh, Hkv, nb, block,
        static_cast<__nv_bfloat16*>(Kc), static_cast<__nv_bfloat16*>(Vc), c_ld, units);
    return launch_status(cudaGetLastError());
}

int nsa_decode_smem(int G, int L, int block, int top, int window, int* per_out, int* ftok_out) {
    const int nb = L / block;
    const int per = std::max(kRows, (nb + kC * kRows - 1) / (kC * kRows) * kRows);
    const int nw = std::min(window, L);
    const int tw = (nw + kRows - 1) / kRows;
    const int ntop = std::min(top, nb);
    const int fitems = std::max((tw + kC - 1) / kC, (ntop + kC - 1) / kC * (block / kRows));
    const int ftok = std::max(1, fitems) * kRows;
    if (per_out) *per_out = per;
    if (ftok_out) *ftok_out = ftok;
    return smem_plan(G <= 8 ? 8 : 16, per, ftok, top).total;
}

sa_status nsa_decode_launch(const void* q, const void* K, const void* V, int64_t sb, int64_t st_, int64_t sh,
                            const void* Kc, const void* Vc, int64_t c_ld, const float* gates, int B, int H, int Hkv,
                            int L, int block, int top, int window, float scale, float* out, int32_t* sel,
                            cudaStream_t st) {
    NsaArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.K = static_cast<const __nv_bfloat16*>(K);
    a.V = static_cast<const __nv_bfloat16*>(V);
    a.sb = sb;
    a.st = st_;
    a.sh = sh;
    a.Kc = static_cast<const __nv_bfloat16*>(Kc);
    a.Vc = static_cast<const __nv_bfloat16*>(Vc);
    a.c_ld = c_ld;
    a.gates = gates;
    a.out = out;
    a.sel = sel;
    a.H = H;
    a.Hkv = Hkv;
    a.G = H / Hkv;
    a.L = L;
    a.block = block;
    a.top = top;
    a.window = window;
    a.scale = scale;
    const int smem = nsa_decode_smem(a.G, L, block, top, window, &a.per, &a.ftok);
    if (smem > kNsaMaxSmem) return SA_EUNSUPPORTED;
    const unsigned grid = static_cast<unsigned>(B) * Hkv * kC;
    cudaError_t e;
    if (a.G <= 8) {
        e = cudaFuncSetAttribute(nsa_decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess) nsa_decode_kernel<1><<<grid, kThreads, smem, st>>>(a);
    } else {
        e = cudaFuncSetAttribute(nsa_decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess) nsa_decode_kernel<2><<<grid, kThreads, smem, st>>>(a);
    }
    if (e != cudaSuccess) return launch_status(e);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

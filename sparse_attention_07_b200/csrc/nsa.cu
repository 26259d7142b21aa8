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
// rows in fp64 and stores the mean rounded once to bf16 (the compressed cache,
// built when a block completes).
//
// nsa_decode: a cluster of kC CTAs per (sequence, KV head).  Every CTA streams
// its share of the data through one ring of 32-row items (one TMA box each,
// both 64-dim halves of the rows, 128-byte swizzle, one mbarrier per slot): compressed K rows (its
// chunk of blocks), window K rows, window V, compressed V, then selected-block
// K and V.  Contractions run on mma.sync
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
constexpr int kRowB = 2 * kD + 16;     // padded bf16 row of the query tile: 272 B, conflict-free fragment loads
constexpr int kHalfB = kRows * 128;    // one TMA box: 32 rows x 64 dims, 128-byte swizzle
constexpr int kItemB = 2 * kHalfB;     // an item: dims 0-63, then dims 64-127
constexpr int kStages = 8;
constexpr int kRingB = kStages * kItemB;
constexpr int kMaxTop = 64;
constexpr int kMaxG = 16;
constexpr float kLog2e = 1.4426950408889634f;

// --------------------------------------------------------------- compression
// Bits of the bf16 value nearest to x (ties to the even significand), for
// finite x whose rounding stays within the bf16 range: bf16 keeps 8
// significant bits with the fp32 exponent range, so the step in the binade
// [2^e, 2^(e+1)) is 2^(e-7), and 2^-133 among the subnormals.  Scaling by
// that step is exact, rint() rounds half to even, and the rounded value is
// exact in fp32, whose upper 16 bits are then the bf16 encoding.
__device__ __forceinline__ uint32_t bf16_bits_rn(double x) {
    if (x == 0.0) return __double_as_longlong(x) < 0 ? 0x8000u : 0u;
    int ex;
    (void)frexp(x, &ex);  // |x| = f * 2^ex, 0.5 <= f < 1
    const int step = max(ex - 1, -126) - 7;
    const double r = ldexp(rint(ldexp(x, -step)), step);
    return __float_as_uint(static_cast<float>(r)) >> 16;
}

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
    // fp64 sums in token order: a bf16 value has 8 significant bits, so the
    // sum of a block whose magnitudes span less than 2^45 is exact, and the
    // stored value is the exact mean rounded once to bf16
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
#pragma unroll 8
    for (int i = 0; i < block; ++i) {
        const uint2 raw = *reinterpret_cast<const uint2*>(src + i * st);
        const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        a0 += static_cast<double>(__low2float(x));
        a1 += static_cast<double>(__high2float(x));
        a2 += static_cast<double>(__low2float(y));
        a3 += static_cast<double>(__high2float(y));
    }
    const double nblk = static_cast<double>(block);
    uint2 o;
    o.x = bf16_bits_rn(a0 / nblk) | (bf16_bits_rn(a1 / nblk) << 16);
    o.y = bf16_bits_rn(a2 / nblk) | (bf16_bits_rn(a3 / nblk) << 16);
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
    int* err;
    int H, Hkv, G, L, block, top, window;
    float scale;
    int per;                 // compressed blocks per CTA (multiple of kRows)
    int ftok;                // capacity of the fine-branch score rows (multiple of kRows)
};

// Shared-memory plan (bytes from the dynamic base); every region 16-byte aligned.
struct Smem {
    int q, sc, pc, sf, pf, part, keyw, cand, glob, recv, recv_ml, total;
    int ld_sc, ld_pc, ld_sf, ld_pf;  // row strides in elements
    int hpc;                         // heads each CTA finishes
};

__host__ __device__ inline Smem smem_plan(int G, int per, int ftok, int top) {
    const int gp = G <= 8 ? 8 : 16;
    Smem s;
    s.ld_sc = per + 4;   // fp32 rows: stride = 4 mod 32 words spreads the fragment stores over the banks
    s.ld_pc = per + 8;   // bf16 rows: stride = 4 mod 8 words, conflict-free B-fragment loads
    s.ld_sf = ftok + 4;
    s.ld_pf = ftok + 8;
    s.hpc = (G + kC - 1) / kC;
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
    s.part = take(3 * 2 * (gp / 8) * 32 * 16);   // split-k partial score fragments
    s.keyw = take(per * 8);
    s.cand = take(kWarps * top * 8);
    s.glob = take(kC * top * 8);
    s.recv = take(kC * 3 * s.hpc * kD * 4);      // partial outputs pushed by the cluster, [rank][branch][head][d]
    s.recv_ml = take(kC * 3 * s.hpc * 2 * 4);    // their (max, sum)
    s.total = off + 1024;                        // the ring starts on a 1024-byte boundary (swizzle atoms)
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

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                            int w, int v) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
        "%6, %7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(v)
        : "memory");
}

// Byte offset of the 16-byte chunk c (0..7) of row r in a 128-byte-swizzled box.
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_cluster_u64(uint32_t addr, unsigned long long v) {
    asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(static_cast<uint32_t>(v)),
                 "r"(static_cast<uint32_t>(v >> 32))
                 : "memory");
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int o) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), o);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), o);
    return (static_cast<unsigned long long>(hi) << 32) | lo;
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) { return a > b ? a : b; }
__device__ __forceinline__ unsigned long long umin64(unsigned long long a, unsigned long long b) { return a > b ? b : a; }

// Bitonic sort, descending, of the warp's 32 (TWO: 64) keys: element e sits in
// lane e % 32, slot e / 32.  Afterwards element 0 is the largest.
template <bool TWO>
__device__ __forceinline__ void warp_sort_desc(unsigned long long& v0, unsigned long long& v1, int lane) {
#pragma unroll
    for (int k = 2; k <= (TWO ? 64 : 32); k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {  // k = 64: the partner is the other slot of this lane; one descending run
                const unsigned long long hi = umax64(v0, v1), lo = umin64(v0, v1);
                v0 = hi;
                v1 = lo;
                continue;
            }
            const bool is_lo = (lane & j) == 0;
            {
                const unsigned long long p = shfl_xor_u64(v0, j);
                const bool desc = (lane & k) == 0;  // k <= 32 here or k = 64 (lane & 64 = 0)
                v0 = (is_lo == desc) ? umax64(v0, p) : umin64(v0, p);
            }
            if (TWO) {
                const unsigned long long p = shfl_xor_u64(v1, j);
                const bool desc = ((lane + 32) & k) == 0;
                v1 = (is_lo == desc) ? umax64(v1, p) : umin64(v1, p);
            }
        }
    }
}

// Rank of key x (its position in descending order) among 8 descending lists
// of n keys each (lists[l * n + i]), x being element `pos` of list `self`:
// pos plus, for every other list, the number of its keys larger than x
// (binary lifting with p2 > n, the 8 searches independent of one another).
__device__ int rank_in_lists(const unsigned long long* lists, int n, int p2, int self, int pos,
                             unsigned long long x) {
    int c[8];
#pragma unroll
    for (int l = 0; l < 8; ++l) c[l] = 0;
#pragma unroll 1
    for (int step = p2 >> 1; step > 0; step >>= 1) {
#pragma unroll
        for (int l = 0; l < 8; ++l)
            if (c[l] + step <= n && lists[l * n + c[l] + step - 1] > x) c[l] += step;
    }
    int rank = pos;
#pragma unroll
    for (int l = 0; l < 8; ++l) rank += l == self ? 0 : c[l];
    return rank;
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
// scores and its sum goes to lsel (the compression probabilities that choose
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
    int nwi, nci, nsi, nA, n_items;  // items: compressed K, window K, window V, compressed V, selected K, selected V
    int w_lo, n_lo, n_hi, ipb;
};

struct Maps {
    // Dims (64 dims, row, dim half, KV head, sequence): one box of 64 x 32 x 2 x 1 x 1
    // lands as [half][row][64 dims], 128-byte swizzled.
    CUtensorMap K, V;    // token cache: rows = positions
    CUtensorMap Kc, Vc;  // compressed cache: rows = complete blocks
};

// The tensor map and first row (y) of ring item i: compressed K rows, window K,
// window V, compressed V, then the rows of the selected blocks, K and V.
__device__ __forceinline__ const CUtensorMap* locate_item(const Maps& m, const Plan& p, int i, const int* chosen,
                                                         int block, int& y, int& z) {
    int j = i;
    const CUtensorMap* map;
    if (j >= p.nci && j < p.nci + 2 * p.nwi) {  // window rows
        j -= p.nci;
        const bool isv = j >= p.nwi;
        if (isv) j -= p.nwi;
        map = isv ? &m.V : &m.K;
        y = p.w_lo + kRows * (p.r + kC * j);
        z = p.kvh;
    } else if (j < p.nA) {  // compressed rows
        const bool isv = j >= p.nci;
        if (isv) j -= p.nci + 2 * p.nwi;
        map = isv ? &m.Vc : &m.Kc;
        y = p.n_lo + kRows * j;
        z = p.kvh;
    } else {  // rows of the selected blocks
        j -= p.nA;
        const bool isv = j >= p.nsi;
        if (isv) j -= p.nsi;
        map = isv ? &m.V : &m.K;
        y = chosen[p.r + kC * (j / p.ipb)] * block + kRows * (j % p.ipb);
        z = p.kvh;
    }
    return map;
}

// One thread: the TMA box of ring item i (both halves, dims 0-63 and 64-127)
// into its slot, completing on the slot's mbarrier.  Rows past the end of the
// history (or of the complete blocks) are zero-filled by the copy.
__device__ __forceinline__ void issue_item(const Maps& m, const Plan& p, int i, uint8_t* ring, uint64_t* full,
                                           const int* chosen, int block) {
    const int slot = i % kStages;
    uint8_t* dst = ring + slot * kItemB;
    mbar_arrive_expect_tx(&full[slot], kItemB);
    int y, z;
    const CUtensorMap* map = locate_item(m, p, i, chosen, block, y, z);
    tma_load_5d(dst, map, &full[slot], 0, y, 0, z, p.b);  // y = first row, z = KV head
}

// Scores of one item: S^T[32 rows x GP heads] = rows . Q^T, split over the
// 8 warps as (m-tile = warp & 1) x (quarter of the 128 dims = warp >> 1).
// The first quarter's warp adds the three other partial fragments in order
// (deterministic), then writes the scores (log2 units) to dst[h][pos0 + row],
// -inf where the row does not exist.
template <int NT>
__device__ __forceinline__ void item_scores(uint32_t item_s, const uint32_t (&qb)[2][NT][2], float4* part, float* dst,
                                            int ld, int pos0, int nvalid_rows, float c2, int warp, int lane) {
    const int mt = warp & 1, kq = warp >> 1;
    const int R = 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
    const uint32_t hbase = item_s + static_cast<uint32_t>((kq >> 1) * kHalfB);
    const int c0 = (kq & 1) * 4 + (lane >> 4);
    float d[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.f;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        uint32_t af[4];
        ldsm_x4(hbase + swz(R, c0 + 2 * s), af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(d[nt], af, qb[s][nt][0], qb[s][nt][1]);
    }
    if (kq != 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            part[(((kq - 1) * 2 + mt) * NT + nt) * 32 + lane] = make_float4(d[nt][0], d[nt][1], d[nt][2], d[nt][3]);
        named_arrive(1 + mt, 128);
        return;
    }
    named_sync(1 + mt, 128);
    const int g = lane >> 2, c4 = lane & 3;
    const int r0 = 16 * mt + g, r1 = r0 + 8;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int q = 1; q < 4; ++q) {
            const float4 v = part[(((q - 1) * 2 + mt) * NT + nt) * 32 + lane];
            d[nt][0] += v.x;
            d[nt][1] += v.y;
            d[nt][2] += v.z;
            d[nt][3] += v.w;
        }
        const int h0 = 8 * nt + 2 * c4;
        dst[h0 * ld + pos0 + r0] = r0 < nvalid_rows ? d[nt][0] * c2 : -INFINITY;
        dst[(h0 + 1) * ld + pos0 + r0] = r0 < nvalid_rows ? d[nt][1] * c2 : -INFINITY;
        dst[h0 * ld + pos0 + r1] = r1 < nvalid_rows ? d[nt][2] * c2 : -INFINITY;
        dst[(h0 + 1) * ld + pos0 + r1] = r1 < nvalid_rows ? d[nt][3] * c2 : -INFINITY;
    }
}

// O^T[16 dims of this warp x GP heads] += rows^T . P^T over one item's 32 rows.
template <int NT>
__device__ __forceinline__ void item_pv(uint32_t item_s, const __nv_bfloat16* P, int ldp, int pos0, float (&acc)[NT][4],
                                        int warp, int lane) {
    const int g = lane >> 2, c4 = lane & 3;
    const uint32_t hbase = item_s + static_cast<uint32_t>((warp >> 2) * kHalfB);
    const int c = 2 * (warp & 3) + ((lane >> 3) & 1);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t af[4];
        ldsm_x4_trans(hbase + swz(16 * ks + (lane & 7) + ((lane >> 4) & 1) * 8, c), af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const __nv_bfloat16* pr = P + (8 * nt + g) * ldp + pos0 + 16 * ks + 2 * c4;
            mma_bf16_16816(acc[nt], af, *reinterpret_cast<const uint32_t*>(pr),
                           *reinterpret_cast<const uint32_t*>(pr + 8));
        }
    }
}

template <int NT>
__global__ void __cluster_dims__(kC, 1, 1) __launch_bounds__(kThreads, 2)
    nsa_decode_kernel(const __grid_constant__ Maps maps, const NsaArgs a) {
    constexpr int GP = 8 * NT;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t s_full[kStages];
    __shared__ float s_m[3][kMaxG], s_l[3][kMaxG];  // per branch (compression, selection, window) and head
    __shared__ float s_lsel[kMaxG], s_fac[kMaxG];
    __shared__ float s_allm[kC][kMaxG], s_allL[kC][kMaxG];  // compression statistics pushed by the cluster
    __shared__ unsigned long long s_ctop[kMaxTop], s_gtop[kMaxTop];
    __shared__ int s_chosen[kMaxTop];
    __shared__ float s_gate[kMaxG][3];
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G;
    const Smem sp = smem_plan(G, a.per, a.ftok, a.top);
    uint8_t* ring = smem;
    const uint32_t ring_s = smem_u32(ring);
    float* s_sc = reinterpret_cast<float*>(smem + sp.sc);
    __nv_bfloat16* s_pc = reinterpret_cast<__nv_bfloat16*>(smem + sp.pc);
    float* s_sf = reinterpret_cast<float*>(smem + sp.sf);
    __nv_bfloat16* s_pf = reinterpret_cast<__nv_bfloat16*>(smem + sp.pf);
    float4* part = reinterpret_cast<float4*>(smem + sp.part);
    unsigned long long* keyw = reinterpret_cast<unsigned long long*>(smem + sp.keyw);
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + sp.cand);
    unsigned long long* glob = reinterpret_cast<unsigned long long*>(smem + sp.glob);
    float* recv = reinterpret_cast<float*>(smem + sp.recv);
    float* recv_ml = reinterpret_cast<float*>(smem + sp.recv_ml);

    cluster_arrive_relaxed();  // this CTA has started; the matching wait precedes the first push into another CTA

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
    if (tid < kMaxTop) s_ctop[tid] = 0ull;
    if (tid < 3 * G) s_gate[tid / 3][tid % 3] = a.gates[qrow0 * 3 + tid];
    if (tid == 0) {
        tma_prefetch_desc(&maps.K);
        tma_prefetch_desc(&maps.V);
        tma_prefetch_desc(&maps.Kc);
        tma_prefetch_desc(&maps.Vc);
        for (int i = 0; i < kStages; ++i) mbar_init(&s_full[i], 1);
        fence_mbar_init();
        s_abort = 0;
    }
    __syncthreads();
    uint32_t qb[2][NT][2];
    {
        const int kq = warp >> 1;
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint8_t* qr = smem + sp.q + (8 * nt + (lane >> 2)) * kRowB + (16 * (2 * kq + s) + 2 * (lane & 3)) * 2;
                qb[s][nt][0] = *reinterpret_cast<const uint32_t*>(qr);
                qb[s][nt][1] = *reinterpret_cast<const uint32_t*>(qr + 16);
            }
    }
    const WaitCtx wc{a.err, &s_abort};

    float acc_c[NT][4], acc_s[NT][4], acc_w[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc_c[nt][e] = acc_s[nt][e] = acc_w[nt][e] = 0.f;

    bool ready = false;  // the selected blocks are known
    int issued = 0;      // the same count in every thread; warp 0 issues
    auto top_up = [&](int limit) {
        while (issued < limit && issued < p.n_items && (issued < p.nA || ready)) {
            if (tid == 0) issue_item(maps, p, issued, ring, s_full, s_chosen, a.block);
            ++issued;
        }
    };

    // The group's choice of blocks, in three steps placed between ring items
    // so that the cluster's exchanges overlap the streaming of window and
    // compressed-value rows:
    //  E1 (after the compressed keys): compression softmax; every CTA's
    //     per-head (max, sum) pushed to every CTA of the cluster; arrive.
    //  E2 (after the window keys): window softmax; wait; the group's block
    //     probabilities of this chunk; its top blocks (warp sorts, then a
    //     merge of the warps' lists) pushed to every CTA; arrive.
    //  E3 (after the window values): wait; merge of the CTAs' lists into the
    //     group's top blocks, ascending -> the selected-block rows may load.
    const int e1 = p.nci, e2 = p.nci + p.nwi, e3 = p.nci + 2 * p.nwi;
    int p2 = 1;
    while (p2 <= ntop) p2 <<= 1;
    auto events = [&](int done) {
        if (done == e1) {
            __syncthreads();
            branch_softmax(s_sc, sp.ld_sc, s_pc, sp.ld_pc, kRows * p.nci, G, GP, true, s_m[0], s_l[0], s_lsel, warp,
                           lane);
            __syncthreads();
            cluster_wait();  // every CTA of the cluster has started
            for (int t = tid; t < kC * G; t += kThreads) {
                const uint32_t dst = static_cast<uint32_t>(t / G), h = static_cast<uint32_t>(t % G);
                st_cluster_u32(mapa_u32(smem_u32(&s_allm[p.r][h]), dst), __float_as_uint(s_m[0][h]));
                st_cluster_u32(mapa_u32(smem_u32(&s_allL[p.r][h]), dst), __float_as_uint(s_lsel[h]));
            }
            cluster_arrive();
        }
        if (done == e2) {
            __syncthreads();
            branch_softmax(s_sf, sp.ld_sf, s_pf, sp.ld_pf, kRows * p.nwi, G, GP, false, s_m[2], s_l[2], nullptr,
                           warp, lane);
            cluster_wait();
            if (tid < G) {
                float M = -INFINITY;
#pragma unroll
                for (int rr = 0; rr < kC; ++rr) M = fmaxf(M, s_allm[rr][tid]);
                float Lt = 0.f;
#pragma unroll
                for (int rr = 0; rr < kC; ++rr)
                    Lt += s_allm[rr][tid] == -INFINITY ? 0.f : s_allL[rr][tid] * fast_exp2(s_allm[rr][tid] - M);
                const float mine = s_m[0][tid];
                s_fac[tid] = (mine != -INFINITY && Lt > 0.f) ? fast_exp2(mine - M) / Lt : 0.f;
            }
            __syncthreads();
            // the group's probability of each block of this chunk, as a key (0: no block)
            for (int n = tid; n < a.per; n += kThreads) {
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
                const int kw = a.per / kWarps;  // 4 .. 64 keys per warp
                const unsigned long long* src = keyw + warp * kw;
                unsigned long long v0 = lane < kw ? src[lane] : 0ull;
                unsigned long long v1 = lane + 32 < kw ? src[lane + 32] : 0ull;
                if (kw > 32) warp_sort_desc<true>(v0, v1, lane);
                else warp_sort_desc<false>(v0, v1, lane);
                if (lane < ntop) cand[warp * ntop + lane] = v0;
                if (lane + 32 < ntop) cand[warp * ntop + lane + 32] = kw > 32 ? v1 : 0ull;
                __syncthreads();
                for (int c = tid; c < kWarps * ntop; c += kThreads) {
                    const unsigned long long x = cand[c];
                    if (x == 0ull) continue;
                    const int rank = rank_in_lists(cand, ntop, p2, c / ntop, c % ntop, x);
                    if (rank < ntop) s_ctop[rank] = x;
                }
                __syncthreads();
                for (int t = tid; t < kC * ntop; t += kThreads) {
                    const uint32_t dst = static_cast<uint32_t>(t / ntop);
                    const int j = t % ntop;
                    st_cluster_u64(mapa_u32(smem_u32(glob + p.r * ntop + j), dst), s_ctop[j]);
                }
            }
            cluster_arrive();
        }
        if (done == e3) {
            cluster_wait();
            if (ntop > 0) {
                for (int c = tid; c < kC * ntop; c += kThreads) {
                    const unsigned long long x = glob[c];
                    if (x == 0ull) continue;
                    const int rank = rank_in_lists(glob, ntop, p2, c / ntop, c % ntop, x);
                    if (rank < ntop) s_gtop[rank] = x;
                }
                __syncthreads();
                if (tid < ntop) {
                    const int blk = key_block(s_gtop[tid]);
                    int at = 0;
                    for (int u = 0; u < ntop; ++u) at += key_block(s_gtop[u]) < blk;
                    s_chosen[at] = blk;
                }
            }
            __syncthreads();
            if (p.r == 0 && a.sel != nullptr && tid < a.top)
                a.sel[(static_cast<int64_t>(p.b) * a.Hkv + p.kvh) * a.top + tid] = tid < ntop ? s_chosen[tid] : -1;
            ready = true;
        }
        if (p.nsi > 0 && done == p.nA + p.nsi) {
            __syncthreads();
            branch_softmax(s_sf, sp.ld_sf, s_pf, sp.ld_pf, kRows * p.nsi, G, GP, false, s_m[1], s_l[1], nullptr, warp,
                           lane);
        }
    };

    top_up(kStages - 1);
    events(0);
    top_up(kStages - 1);
    for (int i = 0; i < p.n_items; ++i) {
        const int slot = i % kStages;
        const bool got = warp_wait(&s_full[slot], static_cast<uint32_t>((i / kStages) & 1), wc, kErrNsaWait | slot);
        const bool ok = __syncthreads_and(got) != 0;  // also: every warp is done with item i - 1
        top_up(i + kStages);                           // into the slot of item i - 1
        const uint32_t item_s = ring_s + static_cast<uint32_t>(slot * kItemB);
        if (ok) {
            if (i < e1) {
                item_scores<NT>(item_s, qb, part, s_sc, sp.ld_sc, kRows * i, nvc - kRows * i, c2, warp, lane);
            } else if (i < e2) {
                const int j = i - e1;
                const int t0 = p.w_lo + kRows * (p.r + kC * j);
                item_scores<NT>(item_s, qb, part, s_sf, sp.ld_sf, kRows * j, a.L - t0, c2, warp, lane);
            } else if (i < e3) {
                item_pv<NT>(item_s, s_pf, sp.ld_pf, kRows * (i - e2), acc_w, warp, lane);
            } else if (i < p.nA) {
                item_pv<NT>(item_s, s_pc, sp.ld_pc, kRows * (i - e3), acc_c, warp, lane);
            } else if (i < p.nA + p.nsi) {
                item_scores<NT>(item_s, qb, part, s_sf, sp.ld_sf, kRows * (i - p.nA), kRows, c2, warp, lane);
            } else {
                item_pv<NT>(item_s, s_pf, sp.ld_pf, kRows * (i - p.nA - p.nsi), acc_s, warp, lane);
            }
        }
        events(i + 1);
        if (i + 1 == e3) top_up(i + kStages);
    }
    __syncthreads();  // every item consumed: the ring is free for the partial outputs

    // partial outputs to this CTA's shared memory, then pushed to the CTA that finishes each head
    float* po = reinterpret_cast<float*>(ring);  // [3][GP][kD]
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
    __syncthreads();
    const int hpc = sp.hpc;
    for (int t = tid; t < 3 * G * 32; t += kThreads) {
        const int br = t / (G * 32), h = (t / 32) % G, c16 = t % 32;
        const float4 v = *reinterpret_cast<const float4*>(po + (br * GP + h) * kD + 4 * c16);
        const uint32_t at = smem_u32(recv + (((p.r * 3 + br) * hpc + h / kC) * kD + 4 * c16));
        st_cluster_v4(mapa_u32(at, static_cast<uint32_t>(h % kC)), __float_as_uint(v.x), __float_as_uint(v.y),
                      __float_as_uint(v.z), __float_as_uint(v.w));
    }
    for (int t = tid; t < 3 * G; t += kThreads) {
        const int br = t / G, h = t % G;
        const uint32_t at = smem_u32(recv_ml + ((p.r * 3 + br) * hpc + h / kC) * 2);
        const uint32_t dst = static_cast<uint32_t>(h % kC);
        st_cluster_u32(mapa_u32(at, dst), __float_as_uint(s_m[br][h]));
        st_cluster_u32(mapa_u32(at + 4, dst), __float_as_uint(s_l[br][h]));
    }
    cluster_sync_all();
    {
        const int sl = tid >> 7, d = tid & (kD - 1);
        const int h = p.r + kC * sl;
        if (sl < hpc && h < G) {
            float res = 0.f;
#pragma unroll
            for (int br = 0; br < 3; ++br) {
                float M = -INFINITY;
#pragma unroll
                for (int rr = 0; rr < kC; ++rr) M = fmaxf(M, recv_ml[((rr * 3 + br) * hpc + sl) * 2]);
                float num = 0.f, den = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int rr = 0; rr < kC; ++rr) {
                        const float mr = recv_ml[((rr * 3 + br) * hpc + sl) * 2];
                        if (mr == -INFINITY) continue;
                        const float w = exp2f(mr - M);
                        den += w * recv_ml[((rr * 3 + br) * hpc + sl) * 2 + 1];
                        num += w * recv[((rr * 3 + br) * hpc + sl) * kD + d];
                    }
                }
                const float o = den > 0.f ? num / den : 0.f;
                res += s_gate[h][br] * o;
            }
            a.out[(qrow0 + h) * kD + d] = res;
        }
    }
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
    return smem_plan(G, per, ftok, top).total;
}

sa_status nsa_decode_launch(const void* q, const void* K, const void* V, int64_t sb, int64_t st_, int64_t sh,
                            const void* Kc, const void* Vc, int64_t c_ld, const float* gates, int B, int H, int Hkv,
                            int L, int block, int top, int window, float scale, float* out, int32_t* sel, int* err,
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
    a.err = err;
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
    Maps m;
    {
        const uint64_t tdims[5] = {64, static_cast<uint64_t>(L), 2, static_cast<uint64_t>(Hkv),
                                   static_cast<uint64_t>(B)};
        const uint64_t tstr[4] = {static_cast<uint64_t>(st_) * 2, 128, static_cast<uint64_t>(sh) * 2,
                                  static_cast<uint64_t>(sb) * 2};
        const uint64_t cdims[5] = {64, static_cast<uint64_t>(std::max(1, L / block)), 2, static_cast<uint64_t>(Hkv),
                                   static_cast<uint64_t>(B)};
        const uint64_t cstr[4] = {static_cast<uint64_t>(kD) * 2, 128, static_cast<uint64_t>(c_ld) * kD * 2,
                                  static_cast<uint64_t>(c_ld) * kD * 2 * Hkv};
        const uint32_t box[5] = {64, kRows, 2, 1, 1};
        const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
        if (!encode_tiled(&m.K, bf, 5, K, tdims, tstr, box, sw) || !encode_tiled(&m.V, bf, 5, V, tdims, tstr, box, sw) ||
            !encode_tiled(&m.Kc, bf, 5, Kc, cdims, cstr, box, sw) ||
            !encode_tiled(&m.Vc, bf, 5, Vc, cdims, cstr, box, sw))
            return SA_ECUDA;
    }
    const unsigned grid = static_cast<unsigned>(B) * Hkv * kC;
    cudaError_t e;
    if (a.G <= 8) {
        e = cudaFuncSetAttribute(nsa_decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess) nsa_decode_kernel<1><<<grid, kThreads, smem, st>>>(m, a);
    } else {
        e = cudaFuncSetAttribute(nsa_decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess) nsa_decode_kernel<2><<<grid, kThreads, smem, st>>>(m, a);
    }
    if (e != cudaSuccess) return launch_status(e);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

// sa_internal.h — host-side declarations shared by the library's translation
// units (launchers and helpers behind the C ABI in include/sparse_attn.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sparse_attn.h"

namespace sa {

// Device address of this GPU's error word (kernels record wait timeouts here).
int* device_error_word();
// Number of SMs of the current device (cached).
int sm_count();
// Tensor-map encoder from the driver, fetched once through the runtime.
bool encode_tiled(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz);
sa_status launch_status(cudaError_t e);

// Launch with programmatic serialization: the kernel may be scheduled while
// the previous kernel of the stream still runs (once that kernel's CTAs have
// all called pdl_trigger() or exited) and must call pdl_wait() before it
// reads anything the previous kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

struct IdxArgs {
    const float* w = nullptr;
    const int32_t* page_table = nullptr;
    int pages_per_seq = 0;
    int64_t pool_pages = 0;
    const int32_t* seq_of_row = nullptr;
    const int32_t* n_visible = nullptr;
    int rows = 0;
    int H_I = 0;
    int d_I = 0;
    float* scores = nullptr;
    int64_t scores_ld = 0;
    int32_t* hist = nullptr;  // [rows][kHistBins] first-digit counts of the scores written, or null
    int* err = nullptr;
    // candidate mode (one-row groups): no scores; every key whose first digit is
    // at or above a proven lower bound on the row's k-th largest is written as
    // (order key << 32) | ~position to cand[row][cand_cnt[row]++]
    uint64_t* cand = nullptr;
    int64_t cand_ld = 0;
    int32_t* cand_cnt = nullptr;
    int k = 0;
};

sa_status index_scores_tc(const void* q, const void* k_cache, const IdxArgs& a, cudaStream_t st);
sa_status index_scores_cc(const void* q, const void* k_cache, sa_dtype dt, const IdxArgs& a, cudaStream_t st);

sa_status topk_select_launch(const float* scores, int64_t ld, const int32_t* n_valid, int rows, int k,
                             int32_t* hist, int32_t* idx_out, cudaStream_t st);
sa_status topk_cand_launch(const uint64_t* cand, int64_t cand_ld, int32_t* cand_cnt, const int32_t* n_valid,
                           int rows, int k, int32_t* hist, int32_t* idx_out, int* err, cudaStream_t st);

struct MlaArgs {
    const void* q_lat;
    const void* q_rope;
    const void* c_cache;
    int64_t c_ld;
    const void* kr_cache;
    int64_t kr_ld;
    const int32_t* page_table;
    int pages_per_seq;
    int64_t pool_pages;
    const int32_t* seq_of_row;
    const int32_t* idx;        // [rows][k] selected positions; null: dense mode
    const int32_t* n_visible;  // dense mode: row r attends to positions 0 .. n_visible[r]-1
    int rows, H, k, d_c, d_R;
    float scale;
    float* out;
    float* lse;
    int* err;
    void* out_bf16 = nullptr;  // [rows][H][d_c] bf16 output in place of `out` when set
};

// Sparse MLA: the two CTAs of a pair exchange partial scores through an
// L2-resident scratch area with one slot per SM (a CTA uses the slot of the SM
// it runs on; one CTA fits on an SM), kMlaXBuf tiles of kMlaXBytes per slot.
constexpr int kMlaXBuf = 4;
constexpr int kMlaXBytes = 128 * 64 * 4;
constexpr int kMlaScratchSlots = 160;
constexpr int kMaxTilesPerCta = 64;  // 64-key tiles per CTA (the row table in shared memory)

size_t mla_exchange_bytes();
size_t mla_workspace_bytes(int rows, int H, int k, int d_c, int nsplit);
int mla_decode_splits(int rows, int k);
sa_status sparse_mla_launch(const MlaArgs& a, int nsplit, void* ws, size_t ws_bytes, cudaStream_t st);

sa_status mla_absorb_query_launch(const void* q_c, const void* U_K, int rows, int H, int d_C, int d_c, void* q_lat,
                                  int* err, cudaStream_t st);
sa_status mla_up_project_launch(const void* o_lat, bool o_lat_fp32, const void* U_V, int rows, int H, int d_c,
                                int d_v, float* out, int* err, cudaStream_t st);

sa_status block_mean_pool_launch(const void* K, int64_t sb, int64_t st_, int64_t sh, int B, int L, int H, int D,
                                 int block, float* pooled, int64_t pooled_ld, cudaStream_t st);
sa_status block_sparse_launch(const void* q, const float* pooled, int64_t pooled_ld, const void* K, const void* V,
                              int64_t sb, int64_t st_, int64_t sh, int B, int H, int D, int L, int block,
                              int top_blocks, int sink_blocks, int window, float scale, float* out,
                              int32_t* sel_blocks, int* err, cudaStream_t st);

// NSA three-branch decode (nsa.cu).
constexpr int kNsaMaxSmem = 227 * 1024 - 4096;  // dynamic part; the kernel also has ~3 KB of static shared memory
sa_status nsa_compress_launch(const void* K, const void* V, int64_t sb, int64_t st_, int64_t sh, int B, int L,
                              int Hkv, int block, void* Kc, void* Vc, int64_t c_ld, cudaStream_t st);
int nsa_decode_smem(int G, int L, int block, int top, int window, int* per_out, int* ftok_out);
sa_status nsa_decode_launch(const void* q, const void* K, const void* V, int64_t sb, int64_t st_, int64_t sh,
                            const void* Kc, const void* Vc, int64_t c_ld, const float* gates, int B, int H, int Hkv,
                            int L, int block, int top, int window, float scale, float* out, int32_t* sel, int* err,
                            cudaStream_t st);

// CSA compression and window slots (csa.cu).
sa_status csa_compress_launch(const void* Ca, const void* Cb, const void* Za, const void* Zb, int64_t seq_stride,
                              int64_t row_stride, const float* Ba, const float* Bb, int n_seqs, int m, int c, int g0,
                              int g1, void* out, int out_e4m3, int64_t out_seq_stride, int64_t out_row_stride,
                              cudaStream_t st);
sa_status csa_window_index_launch(const int32_t* topk_idx, int rows, int k, const int32_t* raw_len, int window,
                                  int win_base, int32_t* idx_out, cudaStream_t st);

}  // namespace sa

// sa_api.cu — the C ABI (include/sparse_attn.h): argument checks, then the
// launches.  Every check happens on the host before anything is launched.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kMaxDevices = 64;
__device__ ErrBlock g_error_block;  // one per GPU that loads the library: error word + wait limit
int* g_error_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return -1;
    return d;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

sa_status launch_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ECUDA; }

int* device_error_word() {
    const int d = current_device();
    if (d < 0 || d >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_error_ptr[d]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_block) != cudaSuccess) return nullptr;
        g_error_ptr[d] = &static_cast<ErrBlock*>(p)->err;
    }
    return g_error_ptr[d];
}

int sm_count() {
    const int d = current_device();
    if (d < 0 || d >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_sm_count[d]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
        g_sm_count[d] = n;
    }
    return g_sm_count[d];
}

bool encode_tiled(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return false;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
    }
    cuuint64_t gd[5];
    cuuint64_t gs[4];
    cuuint32_t bd[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bd[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) gs[i] = strides_bytes[i];
    }
    const CUresult r = g_encode(map, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gd, gs, bd, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace sa

using namespace sa;

extern "C" {

const char* sa_status_string(sa_status s) {
    switch (s) {
        case SA_OK: return "SA_OK";
        case SA_EINVAL: return "SA_EINVAL";
        case SA_EUNSUPPORTED: return "SA_EUNSUPPORTED";
        case SA_ECUDA: return "SA_ECUDA";
        case SA_ETIMEOUT: return "SA_ETIMEOUT";
    }
    return "SA_UNKNOWN";
}

int sa_version(void) { return 100; }

sa_status sa_set_wait_limit_ns(unsigned long long limit_ns) {
    int* w = device_error_word();
    if (!w) return SA_ECUDA;
    void* lim = reinterpret_cast<char*>(w) + offsetof(ErrBlock, wait_limit_ns);
    return cudaMemcpy(lim, &limit_ns, sizeof(limit_ns), cudaMemcpyHostToDevice) == cudaSuccess ? SA_OK : SA_ECUDA;
}

sa_status sa_check_device_error(int* code_out, sa_stream_t stream) {
    if (!code_out) return SA_EINVAL;
    *code_out = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ECUDA;
    int* w = device_error_word();
    if (!w) return SA_ECUDA;
    int v = 0;
    if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SA_ECUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return SA_ECUDA;
    }
    *code_out = v;
    return v ? SA_ETIMEOUT : SA_OK;
}

static sa_status index_scores_impl(const void* q, const float* w, const void* k_cache, int64_t pool_pages,
                                   sa_dtype dtype, const int32_t* page_table, int pages_per_seq,
                                   const int32_t* seq_of_row, const int32_t* n_visible, int rows, int H_I, int d_I,
                                   int64_t scores_ld, float* scores, int32_t* hist, sa_stream_t stream) {
    if (rows < 0 || H_I < 1 || d_I < 1 || pages_per_seq < 1 || pool_pages < 1 || scores_ld < 1) return SA_EINVAL;
    if (rows == 0) return SA_OK;
    if (!q || !w || !k_cache || !n_visible || !scores) return SA_EINVAL;
    if (hist && !aligned(hist, 4)) return SA_EINVAL;
    if (dtype != SA_F32 && dtype != SA_E4M3) return SA_EUNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(w, 4) || !aligned(scores, 4)) return SA_EINVAL;
    if (pool_pages * 64 > (int64_t(1) << 31)) return SA_EUNSUPPORTED;
    IdxArgs a;
    a.w = w;
    a.page_table = page_table;
    a.pages_per_seq = pages_per_seq;
    a.pool_pages = pool_pages;
    a.seq_of_row = seq_of_row;
    a.n_visible = n_visible;
    a.rows = rows;
    a.H_I = H_I;
    a.d_I = d_I;
    a.scores = scores;
    a.scores_ld = scores_ld;
    a.hist = hist;
    a.err = device_error_word();
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool tc_shape = dtype == SA_E4M3 && d_I == 128 && (H_I == 16 || H_I == 32 || H_I == 64 || H_I == 128) &&
                          rows <= 4096;
    if (tc_shape) return index_scores_tc(q, k_cache, a, st);
    if (d_I % 4 != 0 || d_I > 128 || H_I > 64) return SA_EUNSUPPORTED;
    return index_scores_cc(q, k_cache, dtype, a, st);
}

sa_status sa_index_scores(const void* q, const float* w, const void* k_cache, int64_t pool_pages, sa_dtype dtype,
                          const int32_t* page_table, int pages_per_seq, const int32_t* seq_of_row,
                          const int32_t* n_visible, int rows, int H_I, int d_I, int64_t scores_ld, float* scores,
                          sa_stream_t stream) {
    return index_scores_impl(q, w, k_cache, pool_pages, dtype, page_table, pages_per_seq, seq_of_row, n_visible,
                             rows, H_I, d_I, scores_ld, scores, nullptr, stream);
}

sa_status sa_index_scores_hist(const void* q, const float* w, const void* k_cache, int64_t pool_pages,
                               sa_dtype dtype, const int32_t* page_table, int pages_per_seq,
                               const int32_t* seq_of_row, const int32_t* n_visible, int rows, int H_I, int d_I,
                               int64_t scores_ld, float* scores, int32_t* hist, sa_stream_t stream) {
    if (!hist) return SA_EINVAL;
    return index_scores_impl(q, w, k_cache, pool_pages, dtype, page_table, pages_per_seq, seq_of_row, n_visible,
                             rows, H_I, d_I, scores_ld, scores, hist, stream);
}

static sa_status topk_impl(const float* scores, int64_t scores_ld, const int32_t* n_valid, int rows, int k,
                           int32_t* hist, int32_t* idx_out, sa_stream_t stream) {
    if (rows < 0 || k < 1 || scores_ld < 1) return SA_EINVAL;
    if (rows == 0) return SA_OK;
    if (!scores || !n_valid || !idx_out) return SA_EINVAL;
    if (!aligned(scores, 16) || scores_ld % 4 != 0 || !aligned(idx_out, 4) || (hist && !aligned(hist, 4)))
        return SA_EINVAL;
    if (scores_ld > 262144) return SA_EUNSUPPORTED;
    return topk_select_launch(scores, scores_ld, n_valid, rows, k, hist, idx_out,
                              reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_topk_select(const float* scores, int64_t scores_ld, const int32_t* n_valid, int rows, int k,
                         int32_t* idx_out, sa_stream_t stream) {
    return topk_impl(scores, scores_ld, n_valid, rows, k, nullptr, idx_out, stream);
}

sa_status sa_topk_select_hist(const float* scores, int64_t scores_ld, const int32_t* n_valid, int rows, int k,
                              int32_t* hist, int32_t* idx_out, sa_stream_t stream) {
    if (!hist) return SA_EINVAL;
    return topk_impl(scores, scores_ld, n_valid, rows, k, hist, idx_out, stream);
}

sa_status sa_index_candidates(const void* q, const float* w, const void* k_cache, int64_t pool_pages, sa_dtype dtype,
                              const int32_t* page_table, int pages_per_seq, const int32_t* n_visible, int rows,
                              int H_I, int d_I, int k, int64_t cand_ld, uint64_t* cand, int32_t* cand_cnt,
                              int32_t* hist, sa_stream_t stream) {
    if (rows < 0 || H_I < 1 || d_I < 1 || k < 1 || pages_per_seq < 1 || pool_pages < 1) return SA_EINVAL;
    if (cand_ld < static_cast<int64_t>(pages_per_seq) * 64) return SA_EINVAL;
    if (rows == 0) return SA_OK;
    if (!q || !w || !k_cache || !n_visible || !cand || !cand_cnt || !hist) return SA_EINVAL;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(w, 4) || !aligned(cand, 8) || !aligned(cand_cnt, 4) ||
        !aligned(hist, 16))
        return SA_EINVAL;
    if (dtype != SA_E4M3 || d_I != 128 || rows > 4096) return SA_EUNSUPPORTED;
    if (cand_ld > 262144 || pool_pages * 64 > (int64_t(1) << 31)) return SA_EUNSUPPORTED;
    IdxArgs a;
    a.w = w;
    a.page_table = page_table;
    a.pages_per_seq = pages_per_seq;
    a.pool_pages = pool_pages;
    a.n_visible = n_visible;
    a.rows = rows;
    a.H_I = H_I;
    a.d_I = d_I;
    a.scores_ld = cand_ld;
    a.hist = hist;
    a.cand = cand;
    a.cand_ld = cand_ld;
    a.cand_cnt = cand_cnt;
    a.k = k;
    a.err = device_error_word();
    return index_scores_tc(q, k_cache, a, reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_topk_from_candidates(const uint64_t* cand, int64_t cand_ld, int32_t* cand_cnt, const int32_t* n_valid,
                                  int rows, int k, int32_t* hist, int32_t* idx_out, sa_stream_t stream) {
    if (rows < 0 || k < 1 || cand_ld < 1) return SA_EINVAL;
    if (rows == 0) return SA_OK;
    if (!cand || !cand_cnt || !n_valid || !hist || !idx_out) return SA_EINVAL;
    if (!aligned(cand, 8) || !aligned(cand_cnt, 4) || !aligned(hist, 4) || !aligned(idx_out, 4)) return SA_EINVAL;
    if (cand_ld > 262144) return SA_EUNSUPPORTED;
    return topk_cand_launch(cand, cand_ld, cand_cnt, n_valid, rows, k, hist, idx_out, device_error_word(),
                            reinterpret_cast<cudaStream_t>(stream));
}

size_t sa_sparse_mla_workspace_size(int rows, int H, int k, int d_c) {
    if (rows < 1 || H < 1 || k < 1 || d_c < 1) return 0;
    return mla_workspace_bytes(rows, H, k, d_c, mla_decode_splits(rows, k));
}

static sa_status mla_common(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                            const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                            int pages_per_seq, const int32_t* seq_of_row, const int32_t* idx, int rows, int H, int k,
                            int d_c, int d_R, float scale, void* out, bool out_bf16, float* lse, MlaArgs* a) {
    if (rows < 0 || H < 1 || k < 1 || pages_per_seq < 1 || pool_pages < 1 || !std::isfinite(scale)) return SA_EINVAL;
    if (!q_lat || !q_rope || !c_cache || !kr_cache || !out) return SA_EINVAL;
    if (d_c != 512 || d_R != 64 || H > 128) return SA_EUNSUPPORTED;
    if (c_ld < d_c || kr_ld < d_R || c_ld % 8 != 0 || kr_ld % 8 != 0) return SA_EINVAL;
    if (!aligned(q_lat, 16) || !aligned(q_rope, 16) || !aligned(c_cache, 16) || !aligned(kr_cache, 16) ||
        !aligned(out, 16) || (idx && !aligned(idx, 4)) || (lse && !aligned(lse, 4)))
        return SA_EINVAL;
    if (pool_pages * 64 > (int64_t(1) << 31)) return SA_EUNSUPPORTED;
    a->q_lat = q_lat;
    a->q_rope = q_rope;
    a->c_cache = c_cache;
    a->c_ld = c_ld;
    a->kr_cache = kr_cache;
    a->kr_ld = kr_ld;
    a->page_table = page_table;
    a->pages_per_seq = pages_per_seq;
    a->pool_pages = pool_pages;
    a->seq_of_row = seq_of_row;
    a->idx = idx;
    a->n_visible = nullptr;
    a->rows = rows;
    a->H = H;
    a->k = k;
    a->d_c = d_c;
    a->d_R = d_R;
    a->scale = scale;
    a->out = out_bf16 ? nullptr : static_cast<float*>(out);
    a->out_bf16 = out_bf16 ? out : nullptr;
    a->lse = lse;
    a->err = device_error_word();
    return SA_OK;
}

static sa_status mla_decode_impl(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                                 const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                                 int pages_per_seq, const int32_t* seq_of_row, const int32_t* idx, int rows, int H,
                                 int k, int d_c, int d_R, float scale, void* out, bool out_bf16, float* lse,
                                 void* workspace, size_t workspace_bytes, sa_stream_t stream) {
    if (rows == 0) return SA_OK;
    if (!idx) return SA_EINVAL;
    MlaArgs a;
    sa_status s = mla_common(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                             seq_of_row, idx, rows, H, k, d_c, d_R, scale, out, out_bf16, lse, &a);
    if (s != SA_OK) return s;
    const int ns = mla_decode_splits(rows, k);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < mla_workspace_bytes(rows, H, k, d_c, ns))
        return SA_EINVAL;
    return sparse_mla_launch(a, ns, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t sa_sparse_mla_prefill_workspace_size(int rows, int H, int k, int d_c) {
    if (rows < 1 || H < 1 || k < 1 || d_c < 1) return 0;
    return mla_workspace_bytes(rows, H, k, d_c, 1);
}

static sa_status mla_prefill_impl(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                                  const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                                  int pages_per_seq, const int32_t* seq_of_row, const int32_t* idx, int rows, int H,
                                  int k, int d_c, int d_R, float scale, void* out, bool out_bf16, float* lse,
                                  void* workspace, size_t workspace_bytes, sa_stream_t stream) {
    if (rows == 0) return SA_OK;
    if (!idx) return SA_EINVAL;
    MlaArgs a;
    sa_status s = mla_common(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                             seq_of_row, idx, rows, H, k, d_c, d_R, scale, out, out_bf16, lse, &a);
    if (s != SA_OK) return s;
    if (k > 64 * kMaxTilesPerCta) return SA_EUNSUPPORTED;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < mla_workspace_bytes(rows, H, k, d_c, 1))
        return SA_EINVAL;
    return sparse_mla_launch(a, 1, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_sparse_mla_decode(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                               const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                               int pages_per_seq, const int32_t* seq_of_row, const int32_t* idx, int rows, int H,
                               int k, int d_c, int d_R, float scale, float* out, float* lse, void* workspace,
                               size_t workspace_bytes, sa_stream_t stream) {
    return mla_decode_impl(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                           seq_of_row, idx, rows, H, k, d_c, d_R, scale, out, false, lse, workspace,
                           workspace_bytes, stream);
}

sa_status sa_sparse_mla_decode_bf16(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                                    const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                                    int pages_per_seq, const int32_t* seq_of_row, const int32_t* idx, int rows, int H,
                                    int k, int d_c, int d_R, float scale, void* out, float* lse, void* workspace,
                                    size_t workspace_bytes, sa_stream_t stream) {
    return mla_decode_impl(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                           seq_of_row, idx, rows, H, k, d_c, d_R, scale, out, true, lse, workspace,
                           workspace_bytes, stream);
}

sa_status sa_sparse_mla_prefill(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                                const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                                int pages_per_seq, const int32_t* seq_of_row, const int32_t* idx, int rows, int H,
                                int k, int d_c, int d_R, float scale, float* out, float* lse, void* workspace,
                                size_t workspace_bytes, sa_stream_t stream) {
    return mla_prefill_impl(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                            seq_of_row, idx, rows, H, k, d_c, d_R, scale, out, false, lse, workspace,
                            workspace_bytes, stream);
}

sa_status sa_sparse_mla_prefill_bf16(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                                     const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                                     int pages_per_seq, const int32_t* seq_of_row, const int32_t* idx, int rows, int H,
                                     int k, int d_c, int d_R, float scale, void* out, float* lse, void* workspace,
                                     size_t workspace_bytes, sa_stream_t stream) {
    return mla_prefill_impl(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                            seq_of_row, idx, rows, H, k, d_c, d_R, scale, out, true, lse, workspace,
                            workspace_bytes, stream);
}

size_t sa_dense_mla_workspace_size(int rows, int H, int L_max, int d_c) {
    return sa_sparse_mla_workspace_size(rows, H, L_max, d_c);
}

sa_status sa_dense_mla_decode(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                              const void* kr_cache, int64_t kr_ld, int64_t pool_pages, const int32_t* page_table,
                              int pages_per_seq, const int32_t* seq_of_row, const int32_t* n_visible, int rows,
                              int H, int L_max, int d_c, int d_R, float scale, float* out, float* lse,
                              void* workspace, size_t workspace_bytes, sa_stream_t stream) {
    if (rows == 0) return SA_OK;
    if (!n_visible || !aligned(n_visible, 4)) return SA_EINVAL;
    MlaArgs a;
    sa_status s = mla_common(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                             seq_of_row, nullptr, rows, H, L_max, d_c, d_R, scale, out, false, lse, &a);
    if (s != SA_OK) return s;
    a.n_visible = n_visible;
    const int ns = mla_decode_splits(rows, L_max);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < mla_workspace_bytes(rows, H, L_max, d_c, ns))
        return SA_EINVAL;
    return sparse_mla_launch(a, ns, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------ decode without a caller workspace
namespace {

// Split-key partial states of sa_sparse_mla_decode_static live here; every
// GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[SA_STATIC_SCRATCH_BYTES];
// The exchange area of every slot plus the split-key states (outputs, then
// (m, l) words, each rounded to 256 bytes) of kMlaScratchSlots / 2 (row,
// split) pairs of 128 heads: every decode with k <= 4096 on up to
// kMlaScratchSlots SMs (splits are chosen so that rows * splits <= SMs / 2).
static_assert(SA_STATIC_SCRATCH_BYTES >= static_cast<size_t>(kMlaScratchSlots) * kMlaXBuf * kMlaXBytes +
                                             static_cast<size_t>(kMlaScratchSlots / 2) * 128 * 512 * 4 +
                                             ((static_cast<size_t>(kMlaScratchSlots / 2) * 128 * 16 + 255) & ~size_t(255)),
              "the static array covers k <= 4096 on every supported GPU");
void* g_static_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  The array's name in
// host code is only a host-side stand-in, so the address is looked up once per
// device, with that device current, and cached.
void* static_scratch() {
    const int d = current_device();
    if (d < 0 || d >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_static_scratch_ptr[d]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_static_scratch_ptr[d] = p;
    }
    return g_static_scratch_ptr[d];
}

}  // namespace

extern "C" {

sa_status sa_sparse_mla_decode_static(const void* q_lat, const void* q_rope, const void* c_cache, int64_t c_ld,
                                      const void* kr_cache, int64_t kr_ld, int64_t pool_pages,
                                      const int32_t* page_table, int pages_per_seq, const int32_t* seq_of_row,
                                      const int32_t* idx, int rows, int H, int k, int d_c, int d_R, float scale,
                                      float* out, float* lse, sa_stream_t stream) {
    if (rows == 0) return SA_OK;
    if (!idx) return SA_EINVAL;
    MlaArgs a;
    sa_status s = mla_common(q_lat, q_rope, c_cache, c_ld, kr_cache, kr_ld, pool_pages, page_table, pages_per_seq,
                             seq_of_row, idx, rows, H, k, d_c, d_R, scale, out, false, lse, &a);
    if (s != SA_OK) return s;
    const int ns = mla_decode_splits(rows, k);
    const size_t need = mla_workspace_bytes(rows, H, k, d_c, ns);
    if (need > SA_STATIC_SCRATCH_BYTES) return SA_EUNSUPPORTED;  // no allocation or launch before this check
    void* ws = static_scratch();
    if (ws == nullptr) return SA_ECUDA;
    return sparse_mla_launch(a, ns, ws, SA_STATIC_SCRATCH_BYTES, reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_mla_absorb_query(const void* q_c, const void* U_K, int rows, int H, int d_C, int d_c, void* q_lat,
                              sa_stream_t stream) {
    if (rows < 0 || H < 1 || d_C < 1 || d_c < 1) return SA_EINVAL;
    if (rows == 0) return SA_OK;
    if (!q_c || !U_K || !q_lat) return SA_EINVAL;
    if (d_C % 64 != 0 || d_C > 512 || d_c % 128 != 0 || d_c > 512 || H > 65535) return SA_EUNSUPPORTED;
    if (!aligned(q_c, 16) || !aligned(U_K, 16) || !aligned(q_lat, 2)) return SA_EINVAL;
    return mla_absorb_query_launch(q_c, U_K, rows, H, d_C, d_c, q_lat, device_error_word(),
                                   reinterpret_cast<cudaStream_t>(stream));
}

static sa_status up_project_impl(const void* o_lat, bool o_lat_fp32, const void* U_V, int rows, int H, int d_c,
                                 int d_v, float* out, sa_stream_t stream) {
    if (rows < 0 || H < 1 || d_c < 1 || d_v < 1) return SA_EINVAL;
    if (rows == 0) return SA_OK;
    if (!o_lat || !U_V || !out) return SA_EINVAL;
    if (d_c % 64 != 0 || d_c > 512 || d_v % 128 != 0 || H > 65535) return SA_EUNSUPPORTED;
    if (!aligned(o_lat, 16) || !aligned(U_V, 16) || !aligned(out, 4)) return SA_EINVAL;
    return mla_up_project_launch(o_lat, o_lat_fp32, U_V, rows, H, d_c, d_v, out, device_error_word(),
                                 reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_mla_up_project(const float* o_lat, const void* U_V, int rows, int H, int d_c, int d_v, float* out,
                            sa_stream_t stream) {
    return up_project_impl(o_lat, true, U_V, rows, H, d_c, d_v, out, stream);
}

sa_status sa_mla_up_project_bf16(const void* o_lat, const void* U_V, int rows, int H, int d_c, int d_v, float* out,
                                 sa_stream_t stream) {
    return up_project_impl(o_lat, false, U_V, rows, H, d_c, d_v, out, stream);
}

sa_status sa_block_mean_pool(const void* K, int64_t stride_b, int64_t stride_t, int64_t stride_h, int B, int L,
                             int H, int D, int block, float* pooled, int64_t pooled_ld, sa_stream_t stream) {
    if (B < 0 || L < 0 || H < 0 || block < 1) return SA_EINVAL;
    if (D != 128) return SA_EUNSUPPORTED;
    if (B == 0 || H == 0 || L / block == 0) return SA_OK;
    if (!K || !pooled || pooled_ld < L / block) return SA_EINVAL;
    if (!aligned(K, 8) || !aligned(pooled, 16) || stride_b % 4 || stride_t % 4 || stride_h % 4) return SA_EINVAL;
    return block_mean_pool_launch(K, stride_b, stride_t, stride_h, B, L, H, D, block, pooled, pooled_ld,
                                  reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_block_sparse_attn(const void* q, const float* pooled, int64_t pooled_ld, const void* K, const void* V,
                               int64_t stride_b, int64_t stride_t, int64_t stride_h, int B, int H, int D, int L,
                               int block, int top_blocks, int sink_blocks, int window, float scale, float* out,
                               int32_t* sel_blocks, sa_stream_t stream) {
    if (B < 0 || H < 0 || L < 0 || block < 1 || top_blocks < 0 || sink_blocks < 0 || window < 0 ||
        !std::isfinite(scale))
        return SA_EINVAL;
    if (D != 128 || block != 64 || top_blocks > 64 || L / block > 4096) return SA_EUNSUPPORTED;
    if (B == 0 || H == 0) return SA_OK;
    if (!q || !K || !V || !out || (L / block > 0 && !pooled) || pooled_ld < L / block) return SA_EINVAL;
    if (!aligned(q, 2) || !aligned(K, 8) || !aligned(V, 8) || !aligned(out, 4) || (pooled && !aligned(pooled, 16)) ||
        stride_b % 4 || stride_t % 4 || stride_h % 4)
        return SA_EINVAL;
    return block_sparse_launch(q, pooled, pooled_ld, K, V, stride_b, stride_t, stride_h, B, H, D, L, block,
                               top_blocks, sink_blocks, window, scale, out, sel_blocks, device_error_word(),
                               reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_nsa_compress(const void* K, const void* V, int64_t stride_b, int64_t stride_t, int64_t stride_h, int B,
                          int L, int H_kv, int D, int block, void* Kc, void* Vc, int64_t c_ld, sa_stream_t stream) {
    if (B < 0 || L < 0 || H_kv < 0 || block < 1) return SA_EINVAL;
    if (D != 128) return SA_EUNSUPPORTED;
    if (B == 0 || H_kv == 0 || L / block == 0) return SA_OK;
    if (!K || !V || !Kc || !Vc || c_ld < L / block) return SA_EINVAL;
    if (!aligned(K, 8) || !aligned(V, 8) || !aligned(Kc, 8) || !aligned(Vc, 8) || stride_b % 4 || stride_t % 4 ||
        stride_h % 4)
        return SA_EINVAL;
    return nsa_compress_launch(K, V, stride_b, stride_t, stride_h, B, L, H_kv, block, Kc, Vc, c_ld,
                               reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_nsa_decode(const void* q, const void* K, const void* V, int64_t stride_b, int64_t stride_t,
                        int64_t stride_h, const void* Kc, const void* Vc, int64_t c_ld, const float* gates, int B,
                        int H, int H_kv, int D, int L, int block, int top_blocks, int window, float scale,
                        float* out, int32_t* sel_blocks, sa_stream_t stream) {
    if (B < 0 || H < 1 || H_kv < 1 || H % H_kv != 0 || L < 1 || block < 1 || top_blocks < 0 || window < 0 ||
        !std::isfinite(scale))
        return SA_EINVAL;
    if (D != 128 || H / H_kv > 16 || block % 32 != 0 || block > 256 || top_blocks > 64 || window > 4096 ||
        L / block > 4096 || static_cast<int64_t>(B) * H_kv * 8 > 0x7fffffff)
        return SA_EUNSUPPORTED;
    if (nsa_decode_smem(H / H_kv, L, block, top_blocks, window, nullptr, nullptr) > kNsaMaxSmem)
        return SA_EUNSUPPORTED;
    if (B == 0) return SA_OK;
    if (!q || !K || !V || !gates || !out || (L / block > 0 && (!Kc || !Vc)) || c_ld < L / block) return SA_EINVAL;
    if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 4) || !aligned(gates, 4) ||
        (Kc && !aligned(Kc, 16)) || (Vc && !aligned(Vc, 16)) || stride_b % 8 || stride_t % 8 || stride_h % 8)
        return SA_EINVAL;
    return nsa_decode_launch(q, K, V, stride_b, stride_t, stride_h, Kc ? Kc : K, Vc ? Vc : V, c_ld, gates, B, H,
                             H_kv, L, block, top_blocks, window, scale, out, sel_blocks, device_error_word(),
                             reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb, int64_t seq_stride,
                          int64_t row_stride, const float* Ba, const float* Bb, int n_seqs, int L, int m, int c,
                          int g0, int g1, void* out, sa_dtype out_dtype, int64_t out_seq_stride,
                          int64_t out_row_stride, sa_stream_t stream) {
    if (n_seqs < 0 || L < 0 || m < 1 || c < 1 || g0 < 0 || g1 < g0 || g1 > L / m) return SA_EINVAL;
    if (c % 4 != 0 || c > 8192 || m > 256 || (out_dtype != SA_BF16 && out_dtype != SA_E4M3)) return SA_EUNSUPPORTED;
    if (n_seqs == 0 || g1 == g0) return SA_OK;
    if (!Ca || !Cb || !Za || !Zb || !Ba || !Bb || !out) return SA_EINVAL;
    if (row_stride < c || out_row_stride < c) return SA_EINVAL;
    const size_t oa = out_dtype == SA_E4M3 ? 4 : 8;
    if (!aligned(Ca, 8) || !aligned(Cb, 8) || !aligned(Za, 8) || !aligned(Zb, 8) || !aligned(Ba, 16) ||
        !aligned(Bb, 16) || !aligned(out, oa) || seq_stride % 4 || row_stride % 4 || out_seq_stride % 4 ||
        out_row_stride % 4)
        return SA_EINVAL;
    return csa_compress_launch(Ca, Cb, Za, Zb, seq_stride, row_stride, Ba, Bb, n_seqs, m, c, g0, g1, out,
                               out_dtype == SA_E4M3 ? 1 : 0, out_seq_stride, out_row_stride,
                               reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_csa_window_index(const int32_t* topk_idx, int rows, int k, const int32_t* raw_len, int window,
                              int win_base, int32_t* idx_out, sa_stream_t stream) {
    if (rows < 0 || k < 0 || window < 0 || win_base < 0 || k + window < 1) return SA_EINVAL;
    if (rows == 0) return SA_OK;
    if ((k > 0 && !topk_idx) || !raw_len || !idx_out) return SA_EINVAL;
    if ((topk_idx && !aligned(topk_idx, 4)) || !aligned(raw_len, 4) || !aligned(idx_out, 4)) return SA_EINVAL;
    return csa_window_index_launch(topk_idx, rows, k, raw_len, window, win_base, idx_out,
                                   reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

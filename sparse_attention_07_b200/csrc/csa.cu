// csa.cu — CSA (compressed sparse attention): m-token compressed entries and
// the index list that adds the raw window to the selected entries.
//
// "LLM注意力优化：稀疏注意力", section "DeepSeek CSA & HCA": the entries of
// every m tokens are merged into one.  Entry i takes group i of stream a and
// group i-1 of stream b; the 2m weight rows (Z plus the position bias B of the
// row's place in its group) are normalised by a softmax along the sequence,
// separately in every channel, and weight the 2m entry rows, summed (for
// i = 0 stream b has weight zero).  DSA then selects k compressed entries per
// query, and the core attention also reads the raw entries of a recent
// window; keys and values are the entries themselves.
//
// csa_compress: one thread per (sequence, entry, 4 channels), an online
// softmax over the 2m rows (running max, rescaled sum and weighted sum in
// fp32), 8-byte bf16 loads (a warp covers 128 channels of one row: 256
// contiguous bytes per stream row); output rounded to bf16 or e4m3.
// csa_window_index: per query row, the k selected entry positions followed by
// the positions of the window slots.
#include <cuda_fp8.h>

#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

struct CsaArgs {
    const __nv_bfloat16* Ca;
    const __nv_bfloat16* Cb;
    const __nv_bfloat16* Za;
    const __nv_bfloat16* Zb;
    int64_t seq_stride, row_stride;  // elements, shared by the four streams
    const float* Ba;                 // [m][c]
    const float* Bb;
    int m, c, g0, ng;                // entries g0 .. g0 + ng - 1
    void* out;
    int out_e4m3;
    int64_t out_seq_stride, out_row_stride;  // elements of the output type
    int64_t units;
};

__device__ __forceinline__ float4 ld_bf16x4(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}

// One weight logit z with entry value v joins the running softmax-weighted sum
// of one channel: (mx, sum, acc) hold max, sum of e^(z - mx), sum of e^(z - mx) v.
__device__ __forceinline__ void online_add(float z, float v, float& mx, float& sum, float& acc) {
    if (z > mx) {
        const float s = expf(mx - z);  // mx = -inf -> 0
        sum = sum * s + 1.f;
        acc = acc * s + v;
        mx = z;
    } else {
        const float e = expf(z - mx);
        sum += e;
        acc += e * v;
    }
}

__global__ void __launch_bounds__(256) csa_compress_kernel(const CsaArgs a) {
    const int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (u >= a.units) return;
    const int nq = a.c / 4;
    const int q4 = static_cast<int>(u % nq) * 4;
    const int64_t rest = u / nq;
    const int g = a.g0 + static_cast<int>(rest % a.ng);
    const int64_t seq = rest / a.ng;
    float mx[4], sum[4], acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        mx[j] = -INFINITY;
        sum[j] = 0.f;
        acc[j] = 0.f;
    }
    const int64_t base = seq * a.seq_stride + q4;
    for (int r = 0; r < a.m; ++r) {  // group g of stream a
        const int64_t row = base + (static_cast<int64_t>(g) * a.m + r) * a.row_stride;
        const float4 z = ld_bf16x4(a.Za + row), v = ld_bf16x4(a.Ca + row);
        const float4 bias = *reinterpret_cast<const float4*>(a.Ba + r * a.c + q4);
        online_add(z.x + bias.x, v.x, mx[0], sum[0], acc[0]);
        online_add(z.y + bias.y, v.y, mx[1], sum[1], acc[1]);
        online_add(z.z + bias.z, v.z, mx[2], sum[2], acc[2]);
        online_add(z.w + bias.w, v.w, mx[3], sum[3], acc[3]);
    }
    if (g > 0) {
        for (int r = 0; r < a.m; ++r) {  // group g - 1 of stream b
            const int64_t row = base + (static_cast<int64_t>(g - 1) * a.m + r) * a.row_stride;
            const float4 z = ld_bf16x4(a.Zb + row), v = ld_bf16x4(a.Cb + row);
            const float4 bias = *reinterpret_cast<const float4*>(a.Bb + r * a.c + q4);
            online_add(z.x + bias.x, v.x, mx[0], sum[0], acc[0]);
            online_add(z.y + bias.y, v.y, mx[1], sum[1], acc[1]);
            online_add(z.z + bias.z, v.z, mx[2], sum[2], acc[2]);
            online_add(z.w + bias.w, v.w, mx[3], sum[3], acc[3]);
        }
    }
    float o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = acc[j] / sum[j];
    const int64_t at = seq * a.out_seq_stride + static_cast<int64_t>(g) * a.out_row_stride + q4;
    if (a.out_e4m3) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(o[0], o[1]), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(o[2], o[3]), __NV_SATFINITE, __NV_E4M3);
        *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.out) + at) =
            static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    } else {
        uint2 v;
        v.x = pack_bf16x2(o[0], o[1]);
        v.y = pack_bf16x2(o[2], o[3]);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + at) = v;
    }
}

__global__ void __launch_bounds__(256) csa_window_index_kernel(const int32_t* __restrict__ topk_idx, int k,
                                                               const int32_t* __restrict__ raw_len, int window,
                                                               int win_base, int32_t* __restrict__ idx_out) {
    const int r = blockIdx.x;
    const int kk = k + window;
    const int wl = min(window, raw_len[r]);
    for (int j = threadIdx.x; j < kk; j += blockDim.x) {
        int v;
        if (j < k) v = topk_idx[static_cast<int64_t>(r) * k + j];
        else v = (j - k) < wl ? win_base + (j - k) : -1;
        idx_out[static_cast<int64_t>(r) * kk + j] = v;
    }
}

}  // namespace

sa_status csa_compress_launch(const void* Ca, const void* Cb, const void* Za, const void* Zb, int64_t seq_stride,
                              int64_t row_stride, const float* Ba, const float* Bb, int n_seqs, int m, int c, int g0,
                              int g1, void* out, int out_e4m3, int64_t out_seq_stride, int64_t out_row_stride,
                              cudaStream_t st) {
    CsaArgs a;
    a.Ca = static_cast<const __nv_bfloat16*>(Ca);
    a.Cb = static_cast<const __nv_bfloat16*>(Cb);
    a.Za = static_cast<const __nv_bfloat16*>(Za);
    a.Zb = static_cast<const __nv_bfloat16*>(Zb);
    a.seq_stride = seq_stride;
    a.row_stride = row_stride;
    a.Ba = Ba;
    a.Bb = Bb;
    a.m = m;
    a.c = c;
    a.g0 = g0;
    a.ng = g1 - g0;
    a.out = out;
    a.out_e4m3 = out_e4m3;
    a.out_seq_stride = out_seq_stride;
    a.out_row_stride = out_row_stride;
    a.units = static_cast<int64_t>(n_seqs) * a.ng * (c / 4);
    if (a.units == 0) return SA_OK;
    const int64_t grid = (a.units + 255) / 256;
    csa_compress_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(a);
    return launch_status(cudaGetLastError());
}

sa_status csa_window_index_launch(const int32_t* topk_idx, int rows, int k, const int32_t* raw_len, int window,
                                  int win_base, int32_t* idx_out, cudaStream_t st) {
    if (rows == 0) return SA_OK;
    csa_window_index_kernel<<<rows, 256, 0, st>>>(topk_idx, k, raw_len, window, win_base, idx_out);
    return launch_status(cudaGetLastError());
}

}  // namespace sa

// KV cache append: the step before decode.  Each new token's 576 values
// (c_kv 512 then k_pe 64, bf16) go into its slot of the paged cache: copied
// for a bf16 cache; for an FP8 cache quantised with one fp32 scale per token,
// scale = max|x| / 448 (1 for an all-zero row), code = e4m3(x / scale),
// round to nearest even, saturating at 448.  The FP8 cache computing its
// scale as it is written is what the pages hold responsible for its slower
// decode steps ("Kimi K2.6 DFlash on 8x MI300X", comparison of FP8 and BF16
// KV); a per-token scale makes the writer a single pass over the row.
//
// CTA = one (sequence b, new token t), 96 threads: thread j < 72 owns values
// 8j .. 8j+7 (16 bytes of bf16 in, 8 e4m3 bytes or 16 bf16 bytes out); the
// row maximum is a warp reduction plus three shared-memory words.  Token t of
// a sequence whose context (which already counts the T new tokens) is ctx
// lands at position ctx - T + t.
#include <cuda_fp8.h>

#include "mla_common.cuh"

namespace mla {
namespace {

constexpr int kThreads = 96;
constexpr int kUnits = kD / 8;  // 72

struct AppendArgs {
    const __nv_bfloat16 *c_kv_new;  // [B,T,512]
    const __nv_bfloat16 *k_pe_new;  // [B,T,64]
    void *kv;                       // [P,16,576] bf16 or e4m3 bytes
    float *kv_scale;                // [P,16] (FP8)
    const int32_t *page_table;      // [B, stride]
    const int32_t *ctx_lens;        // [B]
    int32_t *err;                   // {code, info} or null
    int B, T, num_pages, max_pages, pt_stride;
    int per_tensor;                 // FP8: kv_scale[0] is the cache's static scale (read, not written)
};

__device__ __forceinline__ void append_error(int32_t *err, int code, int info) {
    if (err) report_error(err, code, info);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads) append_kernel(AppendArgs a) {
    __shared__ float wmax[kThreads / 32];
    const int b = blockIdx.x / a.T, t = blockIdx.x % a.T;
    const int tid = threadIdx.x;
    const int ctx = __ldg(a.ctx_lens + b);
    if (ctx < a.T || ctx > a.max_pages * kPage) {
        if (tid == 0 && t == 0) append_error(a.err, MLA_DEV_BAD_CTX, b);
        return;
    }
    const int pos = ctx - a.T + t;
    const int page = __ldg(a.page_table + (int64_t)b * a.pt_stride + pos / kPage);
    if (page < 0 || page >= a.num_pages) {
        if (tid == 0) append_error(a.err, MLA_DEV_BAD_PAGE, b);
        return;
    }
    const int64_t row = (int64_t)page * kPage + pos % kPage;
    const int64_t tok = (int64_t)b * a.T + t;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tid < kUnits)
        v = tid < kDl / 8 ? __ldg(reinterpret_cast<const uint4 *>(a.c_kv_new + tok * kDl) + tid)
                          : __ldg(reinterpret_cast<const uint4 *>(a.k_pe_new + tok * kDr) + (tid - kDl / 8));
    if constexpr (!kFp8) {
        if (tid < kUnits) reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.kv) + row * kD)[tid] = v;
        return;
    } else {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
        float x[8];
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            x[2 * e] = f.x;
            x[2 * e + 1] = f.y;
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((tid & 31) == 0) wmax[tid >> 5] = amax;
        __syncthreads();
        amax = fmaxf(fmaxf(wmax[0], wmax[1]), wmax[2]);
        float scale = __fdiv_rn(amax, 448.f);
        if (!(scale > 0.f)) scale = 1.f;
        if (a.per_tensor) scale = __ldg(a.kv_scale);
        if (tid < kUnits) {
            uint32_t w[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t word = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float y = fminf(fmaxf(__fdiv_rn(x[4 * q + e], scale), -448.f), 448.f);
                    const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
                    word |= (uint32_t)c << (8 * e);
                }
                w[q] = word;
            }
            reinterpret_cast<uint2 *>(static_cast<uint8_t *>(a.kv) + row * kD)[tid] = make_uint2(w[0], w[1]);
        }
        if (tid == 0 && !a.per_tensor) a.kv_scale[row] = scale;
    }
}

}  // namespace

int launch_append(const void *c_kv_new, const void *k_pe_new, void *kv_pages, float *kv_scale,
                  const int32_t *page_table, const int32_t *ctx_lens, int B, int T, int num_pages, int max_pages,
                  int pt_stride, int fp8, int per_tensor, int32_t *err, cudaStream_t stream) {
    AppendArgs a;
    a.c_kv_new = static_cast<const __nv_bfloat16 *>(c_kv_new);
    a.k_pe_new = static_cast<const __nv_bfloat16 *>(k_pe_new);
    a.kv = kv_pages;
    a.kv_scale = kv_scale;
    a.page_table = page_table;
    a.ctx_lens = ctx_lens;
    a.err = err;
    a.B = B;
    a.T = T;
    a.num_pages = num_pages;
    a.max_pages = max_pages;
    a.pt_stride = pt_stride;
    a.per_tensor = per_tensor;
    const unsigned grid = (unsigned)((int64_t)B * T);
    if (fp8)
        append_kernel<true><<<grid, kThreads, 0, stream>>>(a);
    else
        append_kernel<false><<<grid, kThreads, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

}  // namespace mla

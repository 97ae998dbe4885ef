// Exact merge of partial attention results through their log-sum-exps.
//
// Partial answers computed over disjoint position sets each carry their
// normaliser, so they combine exactly ("Inside Kimi K3 optimisation work",
// section 1, DCP; section 4, history split):
//   L = max_i lse_i,  w_i = exp(lse_i - L),
//   out = sum_i w_i out_i / sum_i w_i,  lse = L + ln sum_i w_i.
//
// One CTA per (output row, quarter of the 512 latent dims), 256 threads:
// thread (grp, c) = (tid / 32, tid % 32) accumulates dims 128q + 4c .. +3
// over the parts i = grp (mod 8), four parts in flight at a time; the eight
// groups are then summed through shared memory.  Rows x 4 CTAs keep every
// SM streaming even when a single sequence has few query rows.
#include "mla_common.cuh"

namespace mla {
namespace {

constexpr int kThreads = 256;
constexpr int kGroups = kThreads / 32;
constexpr int kQuarters = 4;

struct MergeSmem {
    float4 acc[kGroups - 1][32];
    float wsum[kGroups];
    float red[kGroups];
    int nan_flag;
};

// parts i of this row: out at o0 + i*o_stride, lse at l0 + i*l_stride.
__device__ __forceinline__ void merge_row(const float *o0, int64_t o_stride, const float *l0,
                                          int64_t l_stride, int n, void *out, int64_t out_row,
                                          int out_f32, float *lse_out, int quarter, MergeSmem &sm) {
    const int tid = threadIdx.x, c = tid & 31, grp = tid >> 5;
    // 1) max lse, NaN detection
    float L = -INFINITY;
    int has_nan = 0;
    for (int i = tid; i < n; i += kThreads) {
        const float l = __ldg(l0 + i * l_stride);
        if (isnan(l)) has_nan = 1;
        L = fmaxf(L, l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, o));
    has_nan = __any_sync(0xffffffffu, has_nan);
    if (tid == 0) sm.nan_flag = 0;
    __syncthreads();
    if (c == 0) {
        sm.red[grp] = L;
        if (has_nan) sm.nan_flag = 1;
    }
    __syncthreads();
    L = sm.red[0];
#pragma unroll
    for (int w = 1; w < kGroups; ++w) L = fmaxf(L, sm.red[w]);
    const bool nan_row = sm.nan_flag != 0;

    // 2) weighted sums, parts strided over the groups
    const float4 *v0 = reinterpret_cast<const float4 *>(o0) + quarter * 32 + c;
    const int64_t v_stride = o_stride / 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (!nan_row && L != -INFINITY) {
        int i = grp;
        for (; i + 3 * kGroups < n; i += 4 * kGroups) {
            float w[4];
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = i + u * kGroups;
                w[u] = __ldg(l0 + k * l_stride);
                v[u] = __ldg(v0 + k * v_stride);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                // a part that saw nothing weighs nothing, whatever its out holds
                const bool empty = w[u] == -INFINITY;
                const float ww = empty ? 0.f : expf(w[u] - L);
                if (empty) v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                wsum += ww;
                acc.x = fmaf(ww, v[u].x, acc.x);
                acc.y = fmaf(ww, v[u].y, acc.y);
                acc.z = fmaf(ww, v[u].z, acc.z);
                acc.w = fmaf(ww, v[u].w, acc.w);
            }
        }
        for (; i < n; i += kGroups) {
            const float l = __ldg(l0 + i * l_stride);
            if (l == -INFINITY) continue;
            const float ww = expf(l - L);
            const float4 v = __ldg(v0 + i * v_stride);
            wsum += ww;
            acc.x = fmaf(ww, v.x, acc.x);
            acc.y = fmaf(ww, v.y, acc.y);
            acc.z = fmaf(ww, v.z, acc.z);
            acc.w = fmaf(ww, v.w, acc.w);
        }
    }
    if (grp > 0) sm.acc[grp - 1][c] = acc;
    if (c == 0) sm.wsum[grp] = wsum;
    __syncthreads();
    if (grp == 0) {
        float W = sm.wsum[0];
#pragma unroll
        for (int g2 = 1; g2 < kGroups; ++g2) {
            const float4 a = sm.acc[g2 - 1][c];
            acc.x += a.x;
            acc.y += a.y;
            acc.z += a.z;
            acc.w += a.w;
            W += sm.wsum[g2];
        }
        float4 o;
        float lse;
        if (nan_row) {
            o = make_float4(NAN, NAN, NAN, NAN);
            lse = NAN;
        } else if (L == -INFINITY) {
            o = make_float4(0.f, 0.f, 0.f, 0.f);
            lse = -INFINITY;
        } else {
            const float inv = 1.f / W;
            o = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
            lse = L + logf(W);
        }
        const int64_t base = out_row * kDl + 128 * quarter + 4 * c;
        if (out_f32) {
            reinterpret_cast<float4 *>(static_cast<float *>(out) + base)[0] = o;
        } else {
            const __nv_bfloat162 lo2 = __floats2bfloat162_rn(o.x, o.y);
            const __nv_bfloat162 hi2 = __floats2bfloat162_rn(o.z, o.w);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t *>(&lo2);
            pk.y = *reinterpret_cast<const uint32_t *>(&hi2);
            reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + base)[0] = pk;
        }
        if (c == 0 && quarter == 0 && lse_out) lse_out[out_row] = lse;
    }
}

// Rows of sequences that were split into several pieces by mla_decode.
__global__ void __launch_bounds__(kThreads) merge_internal_kernel(Problem p) {
    __shared__ MergeSmem sm;
    const int64_t grow = blockIdx.x / kQuarters;  // b * R + r
    const int quarter = blockIdx.x % kQuarters;
    const int b = (int)(grow / p.R), r = (int)(grow % p.R);
    int n_pieces = 0, piece_base = 0;
    bool bad = false;
    pieces_of(p, b, &n_pieces, &piece_base, &bad);
    if (n_pieces < 2) return;  // finished by the decode kernel
    const float *o0 = p.part_o + ((int64_t)piece_base * p.R + r) * kDl;
    const float *l0 = p.part_lse + (int64_t)piece_base * p.R + r;
    merge_row(o0, (int64_t)p.R * kDl, l0, p.R, n_pieces, p.out, grow, p.out_f32, p.lse, quarter, sm);
}

// mla_merge_partials: parts laid out [n_parts, rows, 512] and [n_parts, rows].
__global__ void __launch_bounds__(kThreads) merge_public_kernel(const float *out_parts,
                                                                const float *lse_parts, int n_parts,
                                                                int64_t rows, void *out, int out_f32,
                                                                float *lse_out) {
    __shared__ MergeSmem sm;
    const int64_t row = blockIdx.x / kQuarters;
    const int quarter = blockIdx.x % kQuarters;
    merge_row(out_parts + row * kDl, rows * kDl, lse_parts + row, rows, n_parts, out, row, out_f32,
              lse_out, quarter, sm);
}

}  // namespace

int launch_merge_internal(const Problem &p, cudaStream_t stream) {
    const int64_t rows = (int64_t)p.B * p.R;
    if (rows <= 0) return MLA_OK;
    merge_internal_kernel<<<(unsigned)(rows * kQuarters), kThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

int launch_merge_public(const float *out_parts, const float *lse_parts, int n_parts, int64_t rows,
                        void *out, int out_f32, float *lse_out, cudaStream_t stream) {
    if (rows == 0) return MLA_OK;
    merge_public_kernel<<<(unsigned)(rows * kQuarters), kThreads, 0, stream>>>(out_parts, lse_parts, n_parts,
                                                                               rows, out, out_f32, lse_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

}  // namespace mla

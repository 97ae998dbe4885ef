// Exact merge of partial attention results through their log-sum-exps.
//
// Partial answers computed over disjoint position sets each carry their
// normaliser, so they combine exactly ("Inside Kimi K3 optimisation work",
// section 1, DCP; section 4, history split):
//   L = max_i lse_i,  w_i = exp(lse_i - L),
//   out = sum_i w_i out_i / sum_i w_i,  lse = L + ln sum_i w_i.
//
// Work unit = (output row, quarter of the 512 latent dims): 32 lanes x 4 dims.
// Each lane combines its parts online, one pass over them:
//   m <- max(m, lse_i);  s, acc rescaled by exp(m_old - m);  then += w_i, w_i out_i
// which is the formula above with L replaced by a running maximum.  Loads are
// issued eight parts at a time before any is used.
//   * few parts: one warp per unit, eight units per CTA;
//   * many parts: one CTA per unit, eight warps each taking every eighth part,
//     their (m, s, acc) then combined through shared memory.
#include "mla_common.cuh"

namespace mla {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kQuarters = 4;
constexpr int kFewParts = 16;
constexpr int kBatch = 8;     // parts in flight per lane, one warp per unit
constexpr int kCtaBatch = 10; // the same, eight warps per unit: 80 parts in one round of loads

struct Online {
    float m = -INFINITY, s = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    bool nan = false;
};

// Four consecutive dims of a part: fp32 (mla_merge_partials) or bf16 (the
// decode's own split-KV partials).
__device__ __forceinline__ float4 load4(const float *q) { return __ldg(reinterpret_cast<const float4 *>(q)); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *q) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(q));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

// parts first, first + step, ... < n of one unit: lse at l0[i*l_stride], the
// lane's four dims at v0 + i*v_stride (elements)
template <int kB, typename T>
__device__ __forceinline__ void combine_parts(Online &st, const float *l0, int64_t l_stride, const T *v0,
                                              int64_t v_stride, int first, int step, int n) {
    for (int base = first; base < n; base += kB * step) {
        float l[kB];
        float4 v[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int i = base + u * step;
            l[u] = -INFINITY;
            if (i < n) {
                l[u] = __ldg(l0 + i * l_stride);
                v[u] = load4(v0 + i * v_stride);
            }
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            if (isnan(l[u])) st.nan = true;
            // a part that saw nothing weighs nothing, whatever its out holds
            if (!(l[u] > -INFINITY)) continue;
            if (l[u] > st.m) {
                const float sc = __expf(st.m - l[u]);  // m = -inf -> 0
                st.s *= sc;
                st.acc.x *= sc;
                st.acc.y *= sc;
                st.acc.z *= sc;
                st.acc.w *= sc;
                st.m = l[u];
            }
            const float w = __expf(l[u] - st.m);
            st.s += w;
            st.acc.x = fmaf(w, v[u].x, st.acc.x);
            st.acc.y = fmaf(w, v[u].y, st.acc.y);
            st.acc.z = fmaf(w, v[u].z, st.acc.z);
            st.acc.w = fmaf(w, v[u].w, st.acc.w);
        }
    }
}

__device__ __forceinline__ void write_unit(const Online &st, void *out, int64_t out_row, int quarter, int lane,
                                           int out_f32, float *lse_out) {
    float4 o;
    float lse;
    if (st.nan) {
        o = make_float4(NAN, NAN, NAN, NAN);
        lse = NAN;
    } else if (!(st.s > 0.f)) {
        o = make_float4(0.f, 0.f, 0.f, 0.f);
        lse = -INFINITY;
    } else {
        const float inv = 1.f / st.s;
        o = make_float4(st.acc.x * inv, st.acc.y * inv, st.acc.z * inv, st.acc.w * inv);
        lse = st.m + logf(st.s);
    }
    const int64_t base = out_row * kDl + 128 * quarter + 4 * lane;
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
    if (lane == 0 && quarter == 0 && lse_out) lse_out[out_row] = lse;
}

struct MergeSmem {
    float4 acc[kWarps][32];
    float m[kWarps], s[kWarps];
    int nan[kWarps];
};

// One unit, all eight warps of the CTA over its parts (many parts).
template <typename T>
__device__ __forceinline__ void merge_unit_cta(const T *o0, int64_t o_stride, const float *l0, int64_t l_stride,
                                               int n, void *out, int64_t out_row, int quarter, int out_f32,
                                               float *lse_out, MergeSmem &sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    Online st;
    combine_parts<kCtaBatch>(st, l0, l_stride, o0 + quarter * 128 + lane * 4, o_stride, warp, kWarps, n);
    sm.acc[warp][lane] = st.acc;
    if (lane == 0) {
        sm.m[warp] = st.m;
        sm.s[warp] = st.s;
        sm.nan[warp] = st.nan;
    }
    __syncthreads();
    if (warp == 0) {
        Online t;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) t.m = fmaxf(t.m, sm.m[w]);
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            t.nan |= sm.nan[w] != 0;
            if (!(sm.s[w] > 0.f)) continue;
            const float sc = __expf(sm.m[w] - t.m);
            const float4 a = sm.acc[w][lane];
            t.s = fmaf(sc, sm.s[w], t.s);
            t.acc.x = fmaf(sc, a.x, t.acc.x);
            t.acc.y = fmaf(sc, a.y, t.acc.y);
            t.acc.z = fmaf(sc, a.z, t.acc.z);
            t.acc.w = fmaf(sc, a.w, t.acc.w);
        }
        write_unit(t, out, out_row, quarter, lane, out_f32, lse_out);
    }
}

// One unit per warp (few parts).
template <typename T>
__device__ __forceinline__ void merge_unit_warp(const T *o0, int64_t o_stride, const float *l0, int64_t l_stride,
                                                int n, void *out, int64_t out_row, int quarter, int out_f32,
                                                float *lse_out) {
    const int lane = threadIdx.x & 31;
    Online st;
    combine_parts<kBatch>(st, l0, l_stride, o0 + quarter * 128 + lane * 4, o_stride, 0, 1, n);
    write_unit(st, out, out_row, quarter, lane, out_f32, lse_out);
}

// Rows of sequences that were split into several pieces by mla_decode.
// kCta: one unit per CTA (many pieces), else one unit per warp.
// three unit-CTAs per SM: a row set of one sequence (96 rows x 4 quarters) is one wave;
// the warp-per-unit form runs four CTAs per SM (64 registers), which keeps twice
// the loads in flight of two (the DCP-8 combine of 322 MB: 63.6 against 79.9 us)
template <bool kCta>
__global__ void __launch_bounds__(kThreads, kCta ? 3 : 4) merge_internal_kernel(Problem p) {
    __shared__ MergeSmem sm;
    __shared__ int row_info[kWarps / kQuarters][2];  // warp per unit: pieces of the CTA's rows
    const int warp = threadIdx.x >> 5;
    const int64_t unit = kCta ? (int64_t)blockIdx.x : (int64_t)blockIdx.x * kWarps + warp;
    const int64_t grow = unit / kQuarters;  // b * R + r
    const bool valid = grow < (int64_t)p.B * p.R;
    const int quarter = (int)(unit % kQuarters);
    const int b = valid ? (int)(grow / p.R) : 0, r = valid ? (int)(grow % p.R) : 0;
    int n_pieces = 0, piece_base = 0;
    bool bad = false;
    if (kCta) {
        if (!valid) return;
        // one warp scans the schedule for the CTA's row
        if (warp == 0) {
            pieces_of(p, b, &n_pieces, &piece_base, &bad);
            if ((threadIdx.x & 31) == 0) {
                row_info[0][0] = n_pieces;
                row_info[0][1] = piece_base;
            }
        }
        __syncthreads();
        n_pieces = row_info[0][0];
        piece_base = row_info[0][1];
    } else {
        // the CTA's warps cover kWarps / kQuarters rows, four warps each: the
        // first warp of each row scans the schedule for the row's sequence
        if (warp % kQuarters == 0) {
            if (valid) pieces_of(p, b, &n_pieces, &piece_base, &bad);
            if ((threadIdx.x & 31) == 0) {
                row_info[warp / kQuarters][0] = n_pieces;
                row_info[warp / kQuarters][1] = piece_base;
            }
        }
        __syncthreads();
        if (!valid) return;
        n_pieces = row_info[warp / kQuarters][0];
        piece_base = row_info[warp / kQuarters][1];
    }
    if (n_pieces < 2) return;  // finished by the decode kernel
    // The kernel may start while the attention kernel is finishing (its
    // schedule needs only ctx_lens); the partials are read after it is done.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the pieces of row r are contiguous: [r][piece][512]
    const __nv_bfloat16 *o0 = p.part_o + ((int64_t)r * p.max_pieces + piece_base) * kDl;
    const float *l0 = p.part_lse + (int64_t)r * p.max_pieces + piece_base;
    if (kCta)
        merge_unit_cta(o0, kDl, l0, 1, n_pieces, p.out, grow, quarter, p.out_f32, p.lse, sm);
    else
        merge_unit_warp(o0, kDl, l0, 1, n_pieces, p.out, grow, quarter, p.out_f32, p.lse);
}

// mla_merge_partials: parts laid out [n_parts, rows, 512] and [n_parts, rows].
template <bool kCta>
__global__ void __launch_bounds__(kThreads, kCta ? 3 : 4) merge_public_kernel(const float *out_parts, const float *lse_parts,
                                                                int n_parts, int64_t rows, void *out, int out_f32,
                                                                float *lse_out) {
    __shared__ MergeSmem sm;
    const int64_t unit = kCta ? (int64_t)blockIdx.x : (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t row = unit / kQuarters;
    if (row >= rows) return;
    const int quarter = (int)(unit % kQuarters);
    if (kCta)
        merge_unit_cta(out_parts + row * kDl, rows * kDl, lse_parts + row, rows, n_parts, out, row, quarter, out_f32,
                       lse_out, sm);
    else
        merge_unit_warp(out_parts + row * kDl, rows * kDl, lse_parts + row, rows, n_parts, out, row, quarter,
                        out_f32, lse_out);
}

}  // namespace

int launch_merge_internal(const Problem &p, cudaStream_t stream) {
    const int64_t rows = (int64_t)p.B * p.R;
    if (rows <= 0) return MLA_OK;
    // Slots much more numerous than sequences mean many pieces per sequence:
    // eight warps per unit.  Otherwise a warp per unit (it handles any number
    // of pieces, only more slowly when there are many).  The choice depends on
    // the schedule alone, not on the row count, so that padding the heads of
    // a call changes none of its results: the two forms combine the parts in
    // different orders.
    const bool many = p.n_slots > 2 * p.B;
    const int64_t units = rows * kQuarters;
    // a programmatic dependent of the attention kernel before it in the stream
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (many) {
        cfg.gridDim = dim3((unsigned)units);
        e = cudaLaunchKernelEx(&cfg, merge_internal_kernel<true>, p);
    } else {
        cfg.gridDim = dim3((unsigned)((units + kWarps - 1) / kWarps));
        e = cudaLaunchKernelEx(&cfg, merge_internal_kernel<false>, p);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

int launch_merge_public(const float *out_parts, const float *lse_parts, int n_parts, int64_t rows,
                        void *out, int out_f32, float *lse_out, cudaStream_t stream) {
    if (rows == 0) return MLA_OK;
    const int64_t units = rows * kQuarters;
    if (n_parts > kFewParts)
        merge_public_kernel<true><<<(unsigned)units, kThreads, 0, stream>>>(out_parts, lse_parts, n_parts, rows, out,
                                                                           out_f32, lse_out);
    else
        merge_public_kernel<false><<<(unsigned)((units + kWarps - 1) / kWarps), kThreads, 0, stream>>>(
            out_parts, lse_parts, n_parts, rows, out, out_f32, lse_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

}  // namespace mla

// Plain CUDA-core decode kernel: fp32 arithmetic, one page at a time.
//
// This is the simple GPU path: it shares the split-KV schedule, the partial
// layout and the merge kernel with the tensor-core kernel, and exists so that
// two independent GPU implementations can be compared at sizes the CPU
// oracle cannot finish.  It is not tuned.
//
// CTA = one (KV range, group of 16 query rows).  256 threads: thread
// (row, j) = (tid / 16, tid % 16) owns one score of the current page; for the
// value sum, thread tid owns latent dims 2*tid and 2*tid+1 of all 16 rows.
#include <cuda_fp8.h>

#include "mla_common.cuh"

namespace mla {
namespace {

constexpr int kRows = 16;
constexpr int kThreads = 256;
constexpr int kLd = kD + 1;  // padded smem row: conflict-free column reads

struct SimtSmem {
    float q[kRows][kLd];
    float kv[kPage][kLd];
    float p[kRows][kPage + 1];
    float alpha[kRows];
    float l[kRows];
    float m[kRows];
    int vis[kRows];
    int row_ok[kRows];
    int page_ok;
};

__device__ __forceinline__ float load_kv(const Problem &p, bool fp8, int64_t row, int d) {
    if (fp8) {
        const uint8_t *kv = static_cast<const uint8_t *>(p.kv);
        __nv_fp8_e4m3 v;
        v.__x = kv[row * kD + d];
        return float(v) * __ldg(p.kv_scale + (p.kv_scale_per_tensor ? 0 : row));
    }
    const __nv_bfloat16 *kv = static_cast<const __nv_bfloat16 *>(p.kv);
    return __bfloat162float(kv[row * kD + d]);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads) simt_decode_kernel(Problem p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem &sm = *reinterpret_cast<SimtSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int slot = blockIdx.x / p.n_groups;
    const int g = blockIdx.x % p.n_groups;
    const int r0 = g * kRows;
    const int lr = tid / kPage;  // score row
    const int j = tid % kPage;   // score position within the page

    for_each_piece(p, slot, [&](const Piece &pc) {
        __syncthreads();  // previous piece fully consumed smem
        // query rows (zero rows past R are padding, never written out)
        for (int i = tid; i < kRows * kD; i += kThreads) {
            int rr = i / kD, d = i % kD;
            int r = r0 + rr;
            float v = 0.f;
            if (r < p.R) {
                int64_t qrow = (int64_t)pc.b * p.R + r;
                v = d < kDl ? __bfloat162float(p.q_lat[qrow * kDl + d])
                            : __bfloat162float(p.q_pe[qrow * kDr + (d - kDl)]);
            }
            sm.q[rr][d] = v;
        }
        if (tid < kRows) {
            int r = r0 + tid;
            int vis = 0, ok = 1;
            if (pc.bad_ctx) {
                ok = 0;
            } else if (r < p.R) {
                vis = visible(p, pc.b, r / p.H, pc.ctx);
                if (vis < 0) {
                    ok = 0;
                    vis = 0;
                    if (r % p.H == 0) report_error(p.err, MLA_DEV_BAD_VIS, pc.b * p.T + r / p.H);
                }
            }
            sm.vis[tid] = vis;
            sm.row_ok[tid] = ok;
        }
        if (tid == 0 && pc.bad_ctx && g == 0) report_error(p.err, MLA_DEV_BAD_CTX, pc.b);
        float m_run = -INFINITY, l_run = 0.f;  // replicated across the 16 threads of a row
        float acc[kRows][2];
#pragma unroll
        for (int rr = 0; rr < kRows; ++rr) acc[rr][0] = acc[rr][1] = 0.f;
        bool piece_ok = true;

        for (int pg = pc.page_lo; pg < pc.page_hi; ++pg) {
            __syncthreads();  // kv/p of the previous page consumed
            int page = __ldg(p.page_table + (int64_t)pc.b * p.pt_stride + pg);
            bool pok = page >= 0 && page < p.num_pages;
            if (!pok) {
                piece_ok = false;
                if (tid == 0) report_error(p.err, MLA_DEV_BAD_PAGE, pc.b);
            } else {
                // Slots past the context hold undefined data (possibly NaN);
                // they get zero weight, and 0 * NaN would still poison the
                // value sum, so they are staged as zeros.
                const int valid = pc.ctx - pg * kPage;
                for (int i = tid; i < kPage * kD; i += kThreads) {
                    int s = i / kD, d = i % kD;
                    sm.kv[s][d] = s < valid ? load_kv(p, kFp8, (int64_t)page * kPage + s, d) : 0.f;
                }
            }
            __syncthreads();
            // score of (row lr, position j), in log2 units
            const int pos = pg * kPage + j;
            float s = -INFINITY;
            if (pok && pos < sm.vis[lr]) {
                float dot = 0.f;
#pragma unroll 8
                for (int d = 0; d < kD; ++d) dot = fmaf(sm.q[lr][d], sm.kv[j][d], dot);
                s = dot * p.sm_scale_log2;
            }
            float tmax = s;
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
            float m_new = fmaxf(m_run, tmax);
            float alpha = 1.f, pr = 0.f;
            if (m_new != -INFINITY) {
                alpha = exp2f(m_run - m_new);          // m_run == -inf -> 0
                pr = s == -INFINITY ? 0.f : exp2f(s - m_new);
            }
            float psum = pr;
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
            l_run = l_run * alpha + psum;
            m_run = m_new;
            sm.p[lr][j] = pr;
            if (j == 0) sm.alpha[lr] = alpha;
            __syncthreads();
            if (pok) {
                const int d0 = 2 * tid;
#pragma unroll
                for (int rr = 0; rr < kRows; ++rr) {
                    float a0 = acc[rr][0] * sm.alpha[rr], a1 = acc[rr][1] * sm.alpha[rr];
#pragma unroll
                    for (int jj = 0; jj < kPage; ++jj) {
                        float w = sm.p[rr][jj];
                        a0 = fmaf(w, sm.kv[jj][d0], a0);
                        a1 = fmaf(w, sm.kv[jj][d0 + 1], a1);
                    }
                    acc[rr][0] = a0;
                    acc[rr][1] = a1;
                }
            }
        }
        if (j == 0) {
            sm.l[lr] = l_run;
            sm.m[lr] = m_run;
        }
        __syncthreads();
        // epilogue: normalised output and log-sum-exp, final or partial
        const int d0 = 2 * tid;
        for (int rr = 0; rr < kRows; ++rr) {
            int r = r0 + rr;
            if (r >= p.R) break;
            float l = sm.l[rr];
            bool ok = piece_ok && sm.row_ok[rr];
            float inv = l > 0.f ? 1.f / l : 0.f;
            float o0 = ok ? acc[rr][0] * inv : NAN;
            float o1 = ok ? acc[rr][1] * inv : NAN;
            float lse = !ok ? NAN : (l > 0.f ? (sm.m[rr] + log2f(l)) * kLn2 : -INFINITY);
            int64_t grow = (int64_t)pc.b * p.R + r;
            if (pc.single) {
                store_out(p.out, grow * kDl + d0, o0, p.out_f32);
                store_out(p.out, grow * kDl + d0 + 1, o1, p.out_f32);
                if (tid == 0 && p.lse) p.lse[grow] = lse;
            } else {
                int64_t prow = (int64_t)r * p.max_pieces + pc.piece;
                p.part_o[prow * kDl + d0] = __float2bfloat16_rn(o0);
                p.part_o[prow * kDl + d0 + 1] = __float2bfloat16_rn(o1);
                if (tid == 0) p.part_lse[prow] = lse;
            }
        }
    });
}

}  // namespace

int launch_simt(const Problem &p, cudaStream_t stream) {
    const size_t smem = sizeof(SimtSmem);
    const dim3 grid(p.n_slots * p.n_groups), block(kThreads);
    // The shared-memory opt-in is per device; setting it again is harmless.
    cudaError_t e;
    if (p.kv_scale) {
        e = cudaFuncSetAttribute(simt_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) simt_decode_kernel<true><<<grid, block, smem, stream>>>(p);
    } else {
        e = cudaFuncSetAttribute(simt_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) simt_decode_kernel<false><<<grid, block, smem, stream>>>(p);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

}  // namespace mla

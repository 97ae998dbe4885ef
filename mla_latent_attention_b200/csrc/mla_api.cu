// C ABI entry points: argument validation, workspace layout, kernel dispatch.
#include <atomic>
#include <cstring>
#include <mutex>

#include "mla_common.cuh"

namespace mla {

static std::atomic<int> g_last_cuda{0};

void note_cuda_error(cudaError_t e) { g_last_cuda.store((int)e); }

namespace {

constexpr int kSimtRows = 16;
constexpr int kTcRows = 48;
constexpr int kMaxT = 8;
constexpr int kMaxRows = 1024;

int device_sm_count(int *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
    int kernel;
    int rows_per_group;
    int n_groups;
    int n_slots;
    int64_t max_pieces;
    size_t lse_off, o_off, bytes;
};

// Checks that need no CUDA call.
int check_dims(const mla_dims *d) {
    if (!d) return MLA_ERR_INVALID_ARG;
    if (d->B < 1 || d->T < 1 || d->T > kMaxT || d->H < 1 || (int64_t)d->T * d->H > kMaxRows)
        return MLA_ERR_INVALID_ARG;
    if ((int64_t)d->B * d->T * d->H > ((int64_t)1 << 29) - 1) return MLA_ERR_INVALID_ARG;  // merge grid
    if (d->num_pages < 1 || d->max_pages_per_seq < 1 || d->page_table_stride < d->max_pages_per_seq)
        return MLA_ERR_INVALID_ARG;
    // the device schedule sums page counts of all sequences in 32-bit integers
    if ((int64_t)d->B * d->max_pages_per_seq > (int64_t)INT32_MAX) return MLA_ERR_INVALID_ARG;
    if (d->kv_dtype != MLA_KV_BF16 && d->kv_dtype != MLA_KV_FP8_E4M3) return MLA_ERR_INVALID_ARG;
    if (d->kv_scale_per_tensor != 0 && d->kv_scale_per_tensor != 1) return MLA_ERR_INVALID_ARG;
    if (d->kv_scale_per_tensor && d->kv_dtype != MLA_KV_FP8_E4M3) return MLA_ERR_INVALID_ARG;
    if (d->out_dtype != MLA_OUT_BF16 && d->out_dtype != MLA_OUT_F32) return MLA_ERR_INVALID_ARG;
    if (d->num_splits < 0 || d->wait_limit_kcycles < 0) return MLA_ERR_INVALID_ARG;
    if (d->kernel != MLA_KERNEL_AUTO && d->kernel != MLA_KERNEL_SIMT && d->kernel != MLA_KERNEL_TCGEN05)
        return MLA_ERR_INVALID_ARG;
    return MLA_OK;
}

int make_plan(const mla_dims *d, Plan *pl) {
    int rc = check_dims(d);
    if (rc) return rc;
    int sms = 0;
    rc = device_sm_count(&sms);
    if (rc) return rc;
    pl->kernel = d->kernel == MLA_KERNEL_AUTO ? MLA_KERNEL_TCGEN05 : d->kernel;
    pl->rows_per_group = pl->kernel == MLA_KERNEL_SIMT ? kSimtRows : kTcRows;
    const int R = d->T * d->H;
    pl->n_groups = (R + pl->rows_per_group - 1) / pl->rows_per_group;
    int64_t slots;
    if (d->num_splits > 0) {
        slots = d->num_splits;
    } else {
        const int ctas_per_sm = pl->kernel == MLA_KERNEL_SIMT ? 2 : 1;
        slots = (int64_t)sms * ctas_per_sm / pl->n_groups;
        // no range shorter than 16 pages (two 128-position tiles) on average:
        // a CTA with less work spends most of its time in its fixed costs, and
        // a history that fits one range needs no merge kernel at all
        const int64_t page_bound = ((int64_t)d->B * d->max_pages_per_seq + 15) / 16;
        if (slots > page_bound) slots = page_bound;
        if (slots < 1) slots = 1;
    }
    if (slots * pl->n_groups > (int64_t)INT32_MAX) return MLA_ERR_INVALID_ARG;
    pl->n_slots = (int)slots;
    // a range cuts at most one sequence at each of its two ends
    pl->max_pieces = pl->n_slots > 1 ? (int64_t)pl->n_slots + d->B : 0;
    pl->lse_off = kWsHeaderBytes;
    pl->o_off = align256(pl->lse_off + (size_t)pl->max_pieces * R * sizeof(float));
    pl->bytes = pl->o_off + (size_t)pl->max_pieces * R * kDl * sizeof(__nv_bfloat16);
    return MLA_OK;
}

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Checks of mla_decode's arguments that need no CUDA call (the workspace aside).
int check_decode_args(const void *q_lat, const void *q_pe, const void *kv_pages, const float *kv_scale,
                      const int32_t *page_table, const int32_t *ctx_lens, float sm_scale, const void *out,
                      const float *lse, const mla_dims *dims) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!q_lat || !q_pe || !kv_pages || !page_table || !ctx_lens || !out) return MLA_ERR_INVALID_ARG;
    if ((dims->kv_dtype == MLA_KV_FP8_E4M3) != (kv_scale != nullptr)) return MLA_ERR_INVALID_ARG;
    if (!aligned(q_lat, 16) || !aligned(q_pe, 16) || !aligned(kv_pages, 16) || !aligned(out, 16) ||
        !aligned(page_table, 4) || !aligned(ctx_lens, 4) || (kv_scale && !aligned(kv_scale, 16)) ||
        (lse && !aligned(lse, 4)))
        return MLA_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || sm_scale == INFINITY || sm_scale == -INFINITY) return MLA_ERR_INVALID_ARG;
    return MLA_OK;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

int64_t mla_decode_workspace_size(const mla_dims *dims) {
    Plan pl;
    int rc = make_plan(dims, &pl);
    return rc ? (int64_t)rc : (int64_t)pl.bytes;
}

int mla_decode(const void *q_lat, const void *q_pe, const void *kv_pages, const float *kv_scale,
               const int32_t *page_table, const int32_t *ctx_lens, float sm_scale, void *out,
               float *lse, const mla_dims *dims, void *workspace, size_t workspace_bytes,
               mla_stream_t stream) {
    int rc = check_decode_args(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, out, lse, dims);
    if (rc) return rc;
    if (!workspace || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
    Plan pl;
    rc = make_plan(dims, &pl);
    if (rc) return rc;
    if (workspace_bytes < pl.bytes) return MLA_ERR_WORKSPACE;

    Problem p;
    std::memset(&p, 0, sizeof p);
    p.q_lat = static_cast<const __nv_bfloat16 *>(q_lat);
    p.q_pe = static_cast<const __nv_bfloat16 *>(q_pe);
    p.kv = kv_pages;
    p.kv_scale = kv_scale;
    p.page_table = page_table;
    p.ctx_lens = ctx_lens;
    p.vis_lens = dims->vis_lens;
    p.out = out;
    p.lse = lse;
    char *ws = static_cast<char *>(workspace);
    p.err = reinterpret_cast<int32_t *>(ws);
    p.part_lse = reinterpret_cast<float *>(ws + pl.lse_off);
    p.part_o = reinterpret_cast<__nv_bfloat16 *>(ws + pl.o_off);
    p.max_pieces = pl.max_pieces;
    p.B = dims->B;
    p.T = dims->T;
    p.H = dims->H;
    p.R = dims->T * dims->H;
    p.num_pages = dims->num_pages;
    p.max_pages = dims->max_pages_per_seq;
    p.pt_stride = dims->page_table_stride;
    p.out_f32 = dims->out_dtype == MLA_OUT_F32;
    p.kv_scale_per_tensor = dims->kv_scale_per_tensor;
    p.n_slots = pl.n_slots;
    p.n_groups = pl.n_groups;
    p.rows_per_group = pl.rows_per_group;
    p.sm_scale_log2 = sm_scale * kLog2e;
    p.wait_limit = (uint64_t)dims->wait_limit_kcycles * 1000u;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = pl.kernel == MLA_KERNEL_SIMT ? launch_simt(p, s) : launch_tc(p, s);
    if (rc) return rc;
    if (dims->stage_event) {
        // inside a stream capture the record becomes an external event node
        // (readable after each replay); outside one it is a plain record
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaError_t e = cudaStreamIsCapturing(s, &cs);
        if (e == cudaSuccess)
            e = cudaEventRecordWithFlags(static_cast<cudaEvent_t>(dims->stage_event), s,
                                         cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                             : cudaEventRecordDefault);
        if (e != cudaSuccess) {
            note_cuda_error(e);
            return MLA_ERR_CUDA;
        }
    }
    if (pl.n_slots > 1) rc = launch_merge_internal(p, s);
    return rc;
}

// ---------------------------------------------------------------------------
// Allocation-free decode.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point
// where they decode: runtimes whose device memory is entirely owned by another
// allocator arena, or plugins that must not grow the process's device
// footprint per call.  For them the library keeps one fixed scratch array in
// device memory (every GPU that loads the library holds it until the process
// exits) and runs the ordinary decode with that array as its workspace.
// ---------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
static constexpr int kMaxDevices = 64;
static void *g_noalloc_ptr[kMaxDevices];
static std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in: the address must come from the runtime, once per
// device, with that device current.  The address is kept for the life of the
// process, so it does not survive a reset of the device (cudaDeviceReset) or
// a re-created primary context.
static int noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr) {
            note_cuda_error(e);
            return MLA_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return MLA_OK;
}

int mla_decode_noalloc(const void *q_lat, const void *q_pe, const void *kv_pages, const float *kv_scale,
                       const int32_t *page_table, const int32_t *ctx_lens, float sm_scale, void *out,
                       float *lse, const mla_dims *dims, mla_stream_t stream) {
    // every check that can fail without a CUDA call comes before anything is enqueued
    int rc = check_decode_args(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, out, lse, dims);
    if (rc) return rc;
    const int64_t need = mla_decode_workspace_size(dims);
    if (need < 0) return (int)need;
    if ((size_t)need > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE;
    void *ws = nullptr;
    rc = noalloc_scratch(&ws);
    if (rc) return rc;
    // the array keeps the previous call's contents: the error word must start clear
    cudaError_t e = cudaMemsetAsync(ws, 0, kWsHeaderBytes, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return mla_decode(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, out, lse, dims, ws,
                      kNoAllocScratchBytes, stream);
}

int mla_merge_partials(const float *out_parts, const float *lse_parts, int32_t n_parts, int64_t rows,
                       void *out, int32_t out_dtype, float *lse_out, mla_stream_t stream) {
    if (!out_parts || !lse_parts || !out) return MLA_ERR_INVALID_ARG;
    if (n_parts < 1 || n_parts > 4096 || rows < 0 || rows > ((int64_t)1 << 29) - 1) return MLA_ERR_INVALID_ARG;
    if (out_dtype != MLA_OUT_BF16 && out_dtype != MLA_OUT_F32) return MLA_ERR_INVALID_ARG;
    if (!aligned(out_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16) ||
        (lse_out && !aligned(lse_out, 4)))
        return MLA_ERR_INVALID_ARG;
    return launch_merge_public(out_parts, lse_parts, n_parts, rows, out, out_dtype == MLA_OUT_F32,
                               lse_out, reinterpret_cast<cudaStream_t>(stream));
}

int mla_append_kv(const void *c_kv_new, const void *k_pe_new, void *kv_pages, float *kv_scale,
                  const int32_t *page_table, const int32_t *ctx_lens, const mla_dims *d, int32_t *device_error,
                  mla_stream_t stream) {
    if (!c_kv_new || !k_pe_new || !kv_pages || !page_table || !ctx_lens || !d) return MLA_ERR_INVALID_ARG;
    if (d->B < 1 || d->T < 1 || d->T > kMaxT || d->num_pages < 1 || d->max_pages_per_seq < 1 ||
        d->page_table_stride < d->max_pages_per_seq)
        return MLA_ERR_INVALID_ARG;
    if ((int64_t)d->B * d->T > (int64_t)INT32_MAX) return MLA_ERR_INVALID_ARG;
    const bool fp8 = d->kv_dtype == MLA_KV_FP8_E4M3;
    if (!fp8 && d->kv_dtype != MLA_KV_BF16) return MLA_ERR_INVALID_ARG;
    if (d->kv_scale_per_tensor != 0 && d->kv_scale_per_tensor != 1) return MLA_ERR_INVALID_ARG;
    if (d->kv_scale_per_tensor && !fp8) return MLA_ERR_INVALID_ARG;
    if (fp8 != (kv_scale != nullptr)) return MLA_ERR_INVALID_ARG;
    if (!aligned(c_kv_new, 16) || !aligned(k_pe_new, 16) || !aligned(kv_pages, 16) || !aligned(page_table, 4) ||
        !aligned(ctx_lens, 4) || (kv_scale && !aligned(kv_scale, 4)) || (device_error && !aligned(device_error, 4)))
        return MLA_ERR_INVALID_ARG;
    return launch_append(c_kv_new, k_pe_new, kv_pages, kv_scale, page_table, ctx_lens, d->B, d->T, d->num_pages,
                         d->max_pages_per_seq, d->page_table_stride, fp8, d->kv_scale_per_tensor, device_error,
                         reinterpret_cast<cudaStream_t>(stream));
}

int mla_read_device_error(const void *workspace, int32_t *code, int32_t *info, mla_stream_t stream) {
    if (!workspace || !code) return MLA_ERR_INVALID_ARG;
    int32_t word[2] = {0, 0};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(word, workspace, sizeof word, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    *code = word[0];
    if (info) *info = word[1];
    return MLA_OK;
}

int mla_reset_device_error(void *workspace, mla_stream_t stream) {
    if (!workspace) return MLA_ERR_INVALID_ARG;
    cudaError_t e = cudaMemsetAsync(workspace, 0, 2 * sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

const char *mla_status_string(int status) {
    switch (status) {
        case MLA_OK: return "ok";
        case MLA_ERR_INVALID_ARG: return "invalid argument";
        case MLA_ERR_UNSUPPORTED: return "unsupported";
        case MLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MLA_ERR_CUDA: return "CUDA error";
        default: return "unknown status";
    }
}

int mla_last_cuda_error(void) { return g_last_cuda.load(); }

}  // extern "C"

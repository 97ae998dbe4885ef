/*
 * mla.h -- C ABI of the B200 (sm_100a) paged MLA latent-attention decode library.
 *
 * The library computes decode-time Multi-head Latent Attention over a paged,
 * compressed KV cache.  Every cached position stores 576 values: a 512-wide
 * latent vector c_kv followed by a 64-wide RoPE key k_pe.  The cache
 * holds one such row per position, shared by all query heads; its size is
 * 576 values (576 FP8 bytes) per position per layer ("Inside Kimi K3
 * optimisation work", section 1 'Cache', DCP paragraph: 24 layers x 142,000
 * positions x 576 FP8 bytes ~ 1.96 GB).  Rows live in 16-token pages
 * ("Kimi K2.6 DFlash on 8x MI300X", hardware stack: BLOCK_SIZE=16).
 *
 * For query row (b, t, h) -- sequence b, query token t of T, head h of H:
 *     n      = visible positions of (b, t)
 *     s_j    = sm_scale * (q_lat[b,t,h,:] . c_kv_j + q_pe[b,t,h,:] . k_pe_j),  j < n
 *     lse    = ln sum_j exp(s_j)
 *     out[:] = sum_j exp(s_j - lse) * c_kv_j
 * Each head attends independently ("Inside Kimi K3 optimisation work",
 * section 4, head padding), so any head count works; heads are packed with
 * query tokens into matrix tiles on chip and never padded in memory.
 *
 * Visibility: the last T cached positions of a sequence are its T query
 * tokens (1 token, or 1 + st speculative drafts, "Inside Kimi K3 optimisation
 * work", section 1, multi-token verification #51705); token t sits at
 * position ctx - T + t and sees positions 0 .. ctx - T + t, i.e.
 * n = ctx_lens[b] - T + t + 1, unless mla_dims.vis_lens gives n explicitly.
 * vis_lens also carries a batch whose sequences have different draft depths:
 * a sequence with k < T tokens puts them in slots 0..k-1 with
 * n = ctx_lens[b] - k + t + 1 and gives the unused slots n = 0.
 *
 * Long histories are split across the GPU's SMs and the partial answers are
 * merged exactly through their log-sum-exp normalisers ("Inside Kimi K3
 * optimisation work", section 4: the history is split into parallel pieces
 * whose results are combined; section 1: each partial answer carries
 * normalisation information so shards are weighted correctly on merge).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  Inputs
 *     are read-only; outputs are fully overwritten.  The library allocates
 *     and frees nothing and does not synchronise, except where stated.
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream of the current device).  The current CUDA device must be the one
 *     that owns the pointers.
 *   - Tensors are dense, row-major, with the shapes given below (innermost
 *     dimension last), except page_table whose row stride is explicit.
 *   - Return value: MLA_OK (0) or a negative mla_status.  A host-detected
 *     error launches nothing.  Data-dependent problems that only the device
 *     can see (a page index out of range, a context length that does not fit
 *     the page table) set a sticky error word in the workspace and turn the
 *     affected rows' out and lse into NaN; no kernel traps.
 */
#ifndef MLA_B200_MLA_H
#define MLA_B200_MLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *mla_stream_t;

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = -1,  /* null pointer, non-positive size, bad enum, misalignment */
    MLA_ERR_UNSUPPORTED = -2,  /* valid request the library cannot run here (e.g. no sm_100 device) */
    MLA_ERR_WORKSPACE = -3,    /* workspace missing, misaligned or smaller than required */
    MLA_ERR_CUDA = -4          /* a CUDA runtime/driver call failed; see mla_last_cuda_error */
} mla_status;

typedef enum { MLA_KV_BF16 = 0, MLA_KV_FP8_E4M3 = 1 } mla_kv_dtype;
typedef enum { MLA_OUT_BF16 = 0, MLA_OUT_F32 = 1 } mla_out_dtype;

typedef enum {
    MLA_KERNEL_AUTO = 0,    /* tcgen05 tensor-core kernel */
    MLA_KERNEL_SIMT = 1,    /* plain CUDA-core kernel (slow; a second GPU path for checking) */
    MLA_KERNEL_TCGEN05 = 2  /* tcgen05 (5th-generation tensor core) kernel */
} mla_kernel;

/* Device-side error codes found in the workspace error word. */
typedef enum {
    MLA_DEV_OK = 0,
    MLA_DEV_BAD_PAGE = 1,   /* page_table entry outside [0, num_pages); info = sequence */
    MLA_DEV_BAD_CTX = 2,    /* ctx_lens[b] < 0, > max_pages_per_seq*16, or < T without vis_lens; info = b */
    MLA_DEV_BAD_VIS = 3,    /* vis_lens[b,t] < 0 or > ctx_lens[b]; info = b*T + t */
    MLA_DEV_TIMEOUT = 4     /* a bounded on-chip wait gave up (the CTA stopped cleanly); info = CTA */
} mla_device_error;

typedef struct mla_dims {
    int32_t B;                  /* sequences, >= 1 (B*T*H <= 2^29 - 1) */
    int32_t T;                  /* query tokens per sequence (1 + drafts), 1..8 */
    int32_t H;                  /* query heads, >= 1 (T*H <= 1024) */
    int32_t num_pages;          /* P: pages in kv_pages */
    int32_t max_pages_per_seq;  /* usable columns of page_table */
    int32_t page_table_stride;  /* int32 elements between rows of page_table (>= max_pages_per_seq) */
    int32_t kv_dtype;           /* mla_kv_dtype */
    int32_t out_dtype;          /* mla_out_dtype of `out` */
    int32_t num_splits;         /* 0 = automatic; else number of KV ranges the pages are cut into */
    int32_t kernel;             /* mla_kernel */
    const int32_t *vis_lens;    /* device [B,T] visible positions per query token, or NULL */
    void *stage_event;          /* optional cudaEvent_t, recorded on `stream` after the
                                   attention kernel and before the merge kernel (inside a stream
                                   capture as an external event node, readable after each
                                   replay); NULL for none */
    int32_t kv_scale_per_tensor;  /* FP8 only: 0 = kv_scale is [P,16], one scale per cached
                                     position; 1 = kv_scale points to ONE fp32 scale for the
                                     whole cache (a static, calibrated scale: "Kimi K2.6 DFlash
                                     on 8x MI300X", next steps) */
    int32_t wait_limit_kcycles;   /* 0 = default: an on-chip wait of the tensor-core kernel
                                     (for a copy, an MMA or another warp) gives up after about
                                     4e9 SM cycles (about 2 s).  > 0: after this many thousand
                                     cycles instead, for a tighter watchdog or to exercise the
                                     stop.  A CTA whose wait gives up records MLA_DEV_TIMEOUT,
                                     lets its copies and MMAs in flight finish, frees its tensor
                                     memory and exits; its rows' results are unspecified.
                                     Must be >= 0. */
} mla_dims;

/*
 * Bytes of device workspace mla_decode needs for `dims` on the current
 * device (partial outputs of split histories plus the error word), or a
 * negative mla_status.  The value depends on B, T, H, num_splits, kernel and
 * the device's SM count only.  Returns at least 256.
 */
MLA_API int64_t mla_decode_workspace_size(const mla_dims *dims);

/*
 * Paged MLA decode attention.
 *
 *   q_lat      [B,T,H,512] bf16     latent-space query (already absorbed)
 *   q_pe       [B,T,H,64]  bf16     RoPE part of the query
 *   kv_pages   [P,16,576]           bf16 (1152 B per position), or FP8 e4m3fn
 *                                   bytes (576 B per position); values 0..511
 *                                   are c_kv (also the attention value),
 *                                   512..575 are k_pe.  16-byte aligned.
 *   kv_scale   [P,16] fp32          FP8 only: dequantised value = e4m3 * scale
 *                                   of its position.  16-byte aligned.  Must be
 *                                   NULL for bf16.  With dims->kv_scale_per_tensor
 *                                   it is one fp32 scale for every position.
 *   page_table [B, stride] int32    page_table[b][i] = physical page of the
 *                                   sequence's positions 16i .. 16i+15.  Only
 *                                   entries i < ceil(ctx_lens[b]/16) are read.
 *   ctx_lens   [B] int32            cached positions of each sequence,
 *                                   including its T query tokens.
 *   sm_scale   softmax scale applied to the 576-wide dot products.
 *   out        [B,T,H,512]          bf16 or fp32 (dims->out_dtype): the
 *                                   attention output, normalised.
 *   lse        [B,T,H] fp32         natural-log log-sum-exp of the scaled
 *                                   scores; -inf for a row that sees nothing
 *                                   (whose out is then 0).  May be NULL.
 *   workspace  device scratch of at least mla_decode_workspace_size(dims)
 *              bytes, 256-byte aligned.  Not shared between calls in flight.
 *              Its first 8 bytes are the sticky device error word, which
 *              mla_decode only ever sets: clear it once before the first call
 *              (mla_reset_device_error, or zero the whole workspace) if it is
 *              going to be read with mla_read_device_error.
 *
 * Rows with no visible position (only possible with vis_lens) produce out = 0
 * and lse = -inf, the identity of the merge below.
 */
MLA_API int mla_decode(const void *q_lat, const void *q_pe, const void *kv_pages, const float *kv_scale,
               const int32_t *page_table, const int32_t *ctx_lens, float sm_scale, void *out,
               float *lse, const mla_dims *dims, void *workspace, size_t workspace_bytes,
               mla_stream_t stream);

/*
 * mla_decode without a caller-provided workspace, for callers that cannot
 * allocate device memory when they decode (for example a runtime whose device
 * memory all belongs to another allocator, or a plugin that must not grow the
 * process's device footprint per call).  The pages describe no such entry
 * point; it is a service of this library, not part of the method.
 *
 * Same arguments and results as mla_decode, minus the workspace.  The scratch
 * is one fixed 32 MiB array in device memory, defined in the library, held by
 * every GPU that loads the library until the process exits.  The call
 * allocates and frees nothing:
 *   - If mla_decode_workspace_size(dims) exceeds 32 MiB it returns
 *     MLA_ERR_WORKSPACE and launches nothing.
 *   - The first call on each device looks up the array's device address (a
 *     host-side runtime query, made with that device current).  Make that
 *     first call before any stream capture on the device.  The address is
 *     kept for the life of the process: after cudaDeviceReset (or any loss of
 *     the device's primary context) this entry point must not be called again.
 *   - Argument errors are reported before anything is enqueued, as for
 *     mla_decode.
 *   - Each call clears the array's error word on `stream`, then runs the
 *     decode there.  The device error word is not reported.
 *   - All calls share the one array, so calls that can overlap on the GPU
 *     (different streams, or several host threads) race and corrupt each
 *     other's results.  Serialise them, e.g. on one stream.
 */
MLA_API int mla_decode_noalloc(const void *q_lat, const void *q_pe, const void *kv_pages,
                               const float *kv_scale, const int32_t *page_table,
                               const int32_t *ctx_lens, float sm_scale, void *out, float *lse,
                               const mla_dims *dims, mla_stream_t stream);

/*
 * Exact merge of partial attention results over disjoint position sets
 * (split-KV pieces, or context-parallel ranks each holding a subset of the
 * positions): "Inside Kimi K3 optimisation work", section 1, DCP -- each
 * partial answer carries normalisation information so that shards are
 * weighted correctly when merged.
 *
 *   out_parts [n_parts, rows, 512] fp32  each part's normalised output
 *   lse_parts [n_parts, rows] fp32       each part's natural-log log-sum-exp
 *   out       [rows, 512]                bf16 or fp32 (out_dtype)
 *   lse_out   [rows] fp32 or NULL
 *
 * L = max_i lse_i; w_i = exp(lse_i - L); out = sum_i w_i out_i / sum_i w_i;
 * lse = L + ln sum_i w_i.  Parts with lse = -inf weigh nothing; a row whose
 * parts are all -inf gets out = 0, lse = -inf; a NaN lse makes the row NaN.
 * 1 <= n_parts <= 4096, 0 <= rows <= 2^29 - 1 (rows == 0 launches nothing).
 */
MLA_API int mla_merge_partials(const float *out_parts, const float *lse_parts, int32_t n_parts,
                       int64_t rows, void *out, int32_t out_dtype, float *lse_out,
                       mla_stream_t stream);

/*
 * Writes the T new tokens of every sequence into the paged cache: the step
 * before mla_decode.  For an FP8 cache each token is quantised as it is
 * written, with one fp32 scale per token ("Kimi K2.6 DFlash on 8x MI300X",
 * comparison of FP8 and BF16 KV: the FP8 cache computes a dynamic scale):
 *
 *   x         = the token's 576 values, c_kv (512) then k_pe (64), widened
 *   scale     = max|x| / 448 in binary32 (1 if that is 0)
 *   code_d    = e4m3fn(clamp(x_d / scale, -448, 448)), round to nearest even
 *
 * A bf16 cache receives the values unchanged (kv_scale must be NULL).
 *
 *   c_kv_new   [B,T,512] bf16   16-byte aligned
 *   k_pe_new   [B,T,64]  bf16   16-byte aligned
 *   kv_pages   [P,16,576]       the cache (dims->kv_dtype), 16-byte aligned
 *   kv_scale   [P,16] fp32      FP8 only; with dims->kv_scale_per_tensor one
 *                               fp32 static scale, read and left unchanged
 *   page_table, ctx_lens        as for mla_decode; ctx_lens[b] already counts
 *                               the T new tokens, so token t of sequence b
 *                               goes to position ctx_lens[b] - T + t
 *   dims                        B, T (1..8), num_pages, max_pages_per_seq,
 *                               page_table_stride, kv_dtype are read
 *   device_error               NULL, or a device {code, info} pair that
 *                               receives MLA_DEV_BAD_CTX (ctx < T or beyond the
 *                               page table) or MLA_DEV_BAD_PAGE like the
 *                               workspace error word; such tokens are skipped
 *
 * Inputs must be finite.  Asynchronous on `stream`; writes only the new
 * tokens' slots (and their scales).
 */
MLA_API int mla_append_kv(const void *c_kv_new, const void *k_pe_new, void *kv_pages, float *kv_scale,
                          const int32_t *page_table, const int32_t *ctx_lens, const mla_dims *dims,
                          int32_t *device_error, mla_stream_t stream);

/*
 * Copies the workspace error word to the host.  SYNCHRONISES `stream`.
 * *code receives an mla_device_error (the first one raised since the last
 * reset), *info its detail (may be NULL).
 */
MLA_API int mla_read_device_error(const void *workspace, int32_t *code, int32_t *info,
                          mla_stream_t stream);

/* Clears the workspace error word (asynchronous, on `stream`). */
MLA_API int mla_reset_device_error(void *workspace, mla_stream_t stream);

/* Static string for an mla_status. */
MLA_API const char *mla_status_string(int status);

/* The cudaError_t of the last failing CUDA call inside the library (0 if none). */
MLA_API int mla_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_MLA_H */

// Device-side pieces shared by the decode kernels and the merge kernel:
// problem description, the split-KV schedule, error reporting.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

constexpr int kPage = 16;     // tokens per page
constexpr int kDl = 512;      // latent width (also the value width)
constexpr int kDr = 64;       // RoPE key width
constexpr int kD = kDl + kDr; // 576 values per cached position
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr size_t kWsHeaderBytes = 256;  // error word block at the start of the workspace

// Everything a decode kernel needs, passed by value.
struct Problem {
    const __nv_bfloat16 *q_lat;   // [B,T,H,512]
    const __nv_bfloat16 *q_pe;    // [B,T,H,64]
    const void *kv;               // [P,16,576] bf16 or e4m3 bytes
    const float *kv_scale;        // [P,16] (FP8)
    const int32_t *page_table;    // [B,stride]
    const int32_t *ctx_lens;      // [B]
    const int32_t *vis_lens;      // [B,T] or null
    void *out;                    // [B,T,H,512]
    float *lse;                   // [B,T,H] or null
    // split-KV partials, row-major over pieces: the pieces of one query row
    // sit next to each other, so the merge reads each row's parts as one
    // contiguous run (no large power-of-two stride that lands every part of a
    // row in the same cache slices)
    // bf16: the partials are half the bytes the attention kernel writes and the
    // merge reads (2^-9 relative error each, far inside the parity tolerance)
    __nv_bfloat16 *part_o;        // [R, max_pieces, 512] normalised partial outputs
    float *part_lse;              // [R, max_pieces]
    int64_t max_pieces;           // piece stride of the partials
    int32_t *err;                 // workspace error word {code, info}
    int B, T, H, R;               // R = T*H query rows per sequence
    int num_pages, max_pages, pt_stride;
    int out_f32;
    int kv_scale_per_tensor;      // FP8: kv_scale[0] scales every cached value
    int n_slots;                  // KV ranges the global page sequence is cut into
    int n_groups;                 // row groups per sequence
    int rows_per_group;
    float sm_scale_log2;          // sm_scale * log2(e)
    uint64_t wait_limit;          // SM cycles before an on-chip wait gives up; 0 = the kernel's default
};

__device__ __forceinline__ void report_error(int32_t *err, int code, int info) {
    if (atomicCAS(err, 0, code) == 0) atomicExch(err + 1, info);
}

// Pages of sequence b; 0 (and *bad) when its context length cannot be valid.
__device__ __forceinline__ int seq_pages(const Problem &p, int b, bool *bad) {
    int c = __ldg(p.ctx_lens + b);
    bool ok = c >= 0 && c <= p.max_pages * kPage && (p.vis_lens != nullptr || c >= p.T);
    *bad = !ok;
    return ok ? (c + kPage - 1) / kPage : 0;
}

// Visible positions of query token t of sequence b (ctx known valid);
// -1 when an explicit count is out of range.
__device__ __forceinline__ int visible(const Problem &p, int b, int t, int ctx) {
    if (p.vis_lens) {
        int v = __ldg(p.vis_lens + b * p.T + t);
        return (v < 0 || v > ctx) ? -1 : v;
    }
    return ctx - p.T + t + 1;
}

// ---------------------------------------------------------------------------
// Split-KV schedule.
//
// Sequences' pages are laid end to end (sequence 0 first) into one global
// page sequence of `total` pages, which is cut into n_slots equal ranges of
// `per` pages.  Every (range, row group) pair is one CTA.  The part of a
// sequence that falls in one range is a "piece"; pieces are numbered
// sequence-major, so the pieces of sequence b are piece_base_b ..
// piece_base_b + n_pieces_b - 1.  A sequence with one piece is finished by
// its CTA; one with several is combined by the merge kernel from the
// pieces' normalised partial outputs and log-sum-exps.  A sequence with no
// pages (empty, or invalid) is written by the CTA of range
// min(start_b / per, n_slots - 1).
// ---------------------------------------------------------------------------
struct SeqInfo {
    int b, start, np, n_pieces, piece_base;
    bool bad;
};

__device__ __forceinline__ int warp_incl_scan(int x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Total pages of all valid sequences (whole warp, uniform result).
__device__ __forceinline__ int total_pages(const Problem &p) {
    int acc = 0;
    for (int base = 0; base < p.B; base += 32) {
        int b = base + (threadIdx.x & 31);
        bool bad;
        int np = b < p.B ? seq_pages(p, b, &bad) : 0;
        acc += np;
    }
    return (int)__reduce_add_sync(0xffffffffu, (unsigned)acc);  // one warp reduction instruction
}

// Schedule facts for b = base + lane; run_* carry the sums of earlier chunks.
__device__ __forceinline__ SeqInfo scan_chunk(const Problem &p, int base, int per, int &run_start,
                                              int &run_piece) {
    const int lane = threadIdx.x & 31;
    SeqInfo s;
    s.b = base + lane;
    bool bad = false;
    int np = s.b < p.B ? seq_pages(p, s.b, &bad) : 0;
    int x = warp_incl_scan(np);
    s.start = run_start + x - np;
    s.np = np;
    s.n_pieces = np > 0 ? ((s.start + np - 1) / per - s.start / per + 1) : 0;
    int z = warp_incl_scan(s.n_pieces);
    s.piece_base = run_piece + z - s.n_pieces;
    run_start += __shfl_sync(0xffffffffu, x, 31);
    run_piece += __shfl_sync(0xffffffffu, z, 31);
    s.bad = bad && s.b < p.B;
    return s;
}

__device__ __forceinline__ int pages_per_slot(int total, int n_slots) {
    int per = (total + n_slots - 1) / n_slots;
    return per > 0 ? per : 1;
}

// Does range `slot` (pages [lo,hi)) own work of this sequence?
__device__ __forceinline__ bool slot_touches(const SeqInfo &s, int slot, int lo, int hi, int per,
                                             int n_slots, int B) {
    if (s.b >= B) return false;
    if (s.np > 0) return s.start < hi && s.start + s.np > lo;
    int owner = s.start / per;
    if (owner > n_slots - 1) owner = n_slots - 1;
    return owner == slot;
}

__device__ __forceinline__ SeqInfo shfl_info(const SeqInfo &s, int src) {
    SeqInfo r;
    r.b = __shfl_sync(0xffffffffu, s.b, src);
    r.start = __shfl_sync(0xffffffffu, s.start, src);
    r.np = __shfl_sync(0xffffffffu, s.np, src);
    r.n_pieces = __shfl_sync(0xffffffffu, s.n_pieces, src);
    r.piece_base = __shfl_sync(0xffffffffu, s.piece_base, src);
    r.bad = __shfl_sync(0xffffffffu, (int)s.bad, src) != 0;
    return r;
}

// One unit of CTA work: the pages [page_lo, page_hi) of sequence b.
struct Piece {
    int b;
    int page_lo, page_hi;  // page indices within the sequence
    int piece;             // global piece id (valid when !single)
    bool single;           // the whole sequence is this one piece
    bool bad_ctx;          // sequence rejected (ctx_lens invalid)
    int ctx;
};

__device__ __forceinline__ Piece make_piece(const SeqInfo &s, int slot, int lo, int hi, int per,
                                            const Problem &p) {
    Piece pc;
    pc.b = s.b;
    pc.bad_ctx = s.bad;
    pc.ctx = s.bad ? 0 : __ldg(p.ctx_lens + s.b);
    if (s.np > 0) {
        pc.page_lo = lo > s.start ? lo - s.start : 0;
        int e = hi - s.start;
        pc.page_hi = e < s.np ? e : s.np;
        pc.single = s.n_pieces == 1;
        pc.piece = s.piece_base + (slot - s.start / per);
    } else {
        pc.page_lo = pc.page_hi = 0;
        pc.single = true;
        pc.piece = -1;
    }
    return pc;
}

// Iterates the pieces of range `slot` in sequence order and calls fn(piece)
// for each.  Must be called by every thread of the CTA (each warp scans the
// schedule redundantly, so no synchronisation is needed to agree on it).
template <typename Fn>
__device__ __forceinline__ void for_each_piece(const Problem &p, int slot, Fn &&fn) {
    const int total = total_pages(p);
    const int per = pages_per_slot(total, p.n_slots);
    const int lo = slot * per;
    int hi = lo + per;
    if (hi > total) hi = total;
    int run_start = 0, run_piece = 0;
    for (int base = 0; base < p.B; base += 32) {
        SeqInfo mine = scan_chunk(p, base, per, run_start, run_piece);
        unsigned m = __ballot_sync(0xffffffffu, slot_touches(mine, slot, lo, hi, per, p.n_slots, p.B));
        while (m) {
            int src = __ffs(m) - 1;
            m &= m - 1;
            SeqInfo s = shfl_info(mine, src);
            fn(make_piece(s, slot, lo, hi, per, p));
        }
        // Later sequences all start at or after run_start; once that is past
        // this range's unclamped end, none of them (empty ones included)
        // belongs to it, except on the last range, which owns trailing empties.
        if (run_start >= lo + per && slot < p.n_slots - 1) break;
    }
}

// Piece count and first piece id of sequence b (whole warp).
__device__ __forceinline__ void pieces_of(const Problem &p, int b, int *n_pieces, int *piece_base,
                                          bool *bad) {
    const int total = total_pages(p);
    const int per = pages_per_slot(total, p.n_slots);
    int run_start = 0, run_piece = 0;
    const int chunk = b & ~31;
    for (int base = 0; base <= chunk; base += 32) {
        SeqInfo s = scan_chunk(p, base, per, run_start, run_piece);
        if (base == chunk) {
            SeqInfo t = shfl_info(s, b - chunk);
            *n_pieces = t.n_pieces;
            *piece_base = t.piece_base;
            *bad = t.bad;
        }
    }
}

__device__ __forceinline__ void store_out(void *out, int64_t idx, float v, int out_f32) {
    if (out_f32)
        static_cast<float *>(out)[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16_rn(v);
}

// Host-side launch helpers implemented per kernel family.
int launch_simt(const Problem &p, cudaStream_t stream);
int launch_append(const void *c_kv_new, const void *k_pe_new, void *kv_pages, float *kv_scale,
                  const int32_t *page_table, const int32_t *ctx_lens, int B, int T, int num_pages, int max_pages,
                  int pt_stride, int fp8, int per_tensor, int32_t *err, cudaStream_t stream);
int launch_tc(const Problem &p, cudaStream_t stream);
int launch_merge_internal(const Problem &p, cudaStream_t stream);
int launch_merge_public(const float *out_parts, const float *lse_parts, int n_parts, int64_t rows,
                        void *out, int out_f32, float *lse_out, cudaStream_t stream);
void note_cuda_error(cudaError_t e);

}  // namespace mla

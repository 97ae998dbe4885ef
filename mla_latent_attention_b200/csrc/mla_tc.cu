// tcgen05 tensor-core decode kernel for B200 (sm_100a).
//
// One CTA = one (KV range, group of 48 query rows).  Query rows are the
// heads x draft tokens of one sequence, packed together (12 heads x 3 tokens
// = 36 rows fill one group; 96 x 3 = 288 rows make six), so the padding of
// odd head counts exists only on chip.  The CTA walks its range in tiles of
// 128 cached positions (8 pages of 16).
//
// Orientation ("swap AB"): positions are the MMA M dimension (128 TMEM lanes)
// and query rows the N dimension, so
//     S^T [128 x N] = KV_tile[128 x 576] . Q^T           (scores)
//     O^T [512 x N] += V_tile^T[512 x 128] . P^T          (values, 4 blocks of 128)
// and both accumulators live in tensor memory.  With the rows as M instead, a
// 128 x 512 fp32 O alone would fill all of tensor memory.
//
// FP8 caches are consumed as stored, by kind::f8f6f4 MMAs:
//   * scores: the query is split on chip into two e4m3 parts, hi = e4m3(q/s)
//     and lo = e4m3(q/s - hi), with one power-of-two scale s per CTA.  For a
//     bf16 query hi + lo is exact (a bf16 significand has 8 bits, hi takes
//     the top 4 and the remainder fits lo).  hi and lo are stacked along N, so
//     one N = 96 MMA per K step yields both partial scores (the KV tile is
//     read once) and the softmax adds the two halves.  The per-token scale
//     multiplies S^T lane by lane.
//   * values: the weights, with the per-token value scale folded in, are
//     split the same way into hi and lo, stacked along N = 96; the epilogue
//     adds the two halves of O^T.  V is read as stored, never dequantised.
// bf16 caches use kind::f16 MMAs with N = 48 and bf16 P.
//
// Warp roles (480 threads): warp 0 issues TMA page loads, warp 1 issues the
// score MMAs and owns tensor memory, warp 14 issues the value MMAs, warps
// 2-13 run the online softmax and the epilogue.  Thread
// (warp w, lane l) owns tile position / TMEM lane 32*(w%4) + l; the softmax
// warps form three groups of four (one per TMEM lane quadrant), each group
// taking 16 of the 48 query rows.  (Fifteen warps get 128 registers per
// thread: the register file is split over four sub-partitions, each holding
// four of the warps at most.  Sixteen softmax warps of 12 rows would leave 96
// and spill.)
//
// Softmax stabiliser: per query row a running bound m2 on the log2 weight
// u = s*log2(e)*scale (+ log2 of the token's value scale for FP8), shared by
// the lanes of a row group.  It moves only when some weight exceeds it by more
// than TAU (then O^T and the row sums are rescaled), and then to DELTA above
// the new maximum, so after the first tile it rarely moves again.  Weights
// are exp2(u - m2 + C), at most 2^(TAU+C), which keeps the e4m3 weights in
// range.  Row sums are kept per lane and reduced once per piece.  The lanes
// need not agree before they write a tile's weights: each warp writes them
// with the current bound and flags the tile if one would exceed it; once
// every warp has written the tile (the same barrier the value MMAs wait on),
// a flagged tile takes a slow path in which all softmax warps agree on the
// new bounds, rescale, and rewrite the weights, and the value MMAs of that
// tile are issued only after the rewrite.  The first tile of every piece is
// flagged (no bound yet); later ones almost never are.

// Every wait is bounded: after 4e9 SM cycles (about two seconds) the CTA
// records a timeout in the error word, stops, drains its outstanding copies
// and MMAs and frees its tensor memory.
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "mla_common.cuh"
#include "tc_ptx.cuh"

namespace mla {
namespace {

constexpr int kN = 48;                 // query rows per CTA
constexpr int kTileM = 128;            // positions per tile (MMA M)
constexpr int kTilePages = kTileM / kPage;
constexpr int kRowGroups = 3;                       // softmax warp sets, one per 16 of the 48 rows
constexpr int kSoftmaxWarps = 4 * kRowGroups;       // x 4 TMEM lane quadrants
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kValueWarp = 2 + kSoftmaxWarps;      // warp 0 TMA, warp 1 score MMAs, 2..13 softmax
constexpr int kThreads = 32 * (kValueWarp + 1);     // and the value MMAs' warp
constexpr int kRpt = kN / kRowGroups;               // query rows per softmax thread
static_assert(kRpt == 16, "the row reductions and the paired score loads take 16 rows per thread");
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimit = 4000000000ull;  // SM cycles: about two seconds

// The limit of every wait in the main work: the caller's (mla_dims), else
// kWaitLimit.  The waits that drain a CTA's copies and MMAs before it exits
// always keep kWaitLimit.
__device__ __forceinline__ uint64_t wait_limit(const Problem &p) { return p.wait_limit ? p.wait_limit : kWaitLimit; }
constexpr int kDevTimeout = 4;

template <bool kFp8>
struct Cfg {
    static constexpr int kStages = kFp8 ? 2 : 1;                                   // KV stages
    static constexpr int kSBufs = kFp8 ? 1 : 2;                                    // S^T buffers
    static constexpr int kNMma = kFp8 ? 2 * kN : kN;                               // MMA N (hi|lo stacked)
    // tensor memory columns
    static constexpr uint32_t kColS1 = 64;                                         // second S^T buffer
    static constexpr uint32_t kColO = 128;
    static constexpr uint32_t kOStride = kFp8 ? 96u : 64u;                         // O block m at kColO + m*stride
    // KV stage.  The MMAs read the tile as 128-byte-wide column chunks (FP8: 4
    // chunks of 128 latent dims; bf16: 9 chunks of 64 dims, the last one the
    // RoPE part) of 128 positions, each chunk a stack of 8-position x 128 B
    // swizzle atoms.  The c_kv chunks are copied and freed in parts of kCpp
    // chunks (FP8: one part; parts of one or two chunks, which free each
    // chunk as soon as its value MMAs are done, measured slower: the smaller
    // copies cost more than the earlier start gains).  Byte offset of
    // (8-position group g, chunk c):
    //   g * kGroupStride + chunk_off(c)
    // FP8: part h holds chunks [h kCpp, (h+1) kCpp) in a region of its own; one
    //   box per (page, part) lands [half][chunk][8 rows][128 B] there, so the
    //   group stride is kCpp KB and the part's chunks are 1 KB apart; the RoPE
    //   part is a separate [128 positions][64 B] region at kRopeOff.
    // bf16: one 2 KB box per (page, chunk): chunks of [128 positions][128 B].
    static constexpr int kDimChunks = kFp8 ? 4 : 8;                               // 128-B chunks of c_kv
    static constexpr int kCpp = kFp8 ? 4 : 1;                                     // chunks per c_kv part
    static constexpr int kGroupStride = kFp8 ? kCpp * 1024 : 1024;
    static constexpr int kChunkStride = kFp8 ? 1024 : kTileM * 128;               // within a part
    static constexpr int kPartStride = kTileM * kCpp * 128;                       // c_kv part regions
    __host__ __device__ static constexpr int chunk_off(int c) {
        return (c / kCpp) * kPartStride + (c % kCpp) * kChunkStride;
    }
    static constexpr int kRopeOff = kFp8 ? 4 * 16384 : 8 * kTileM * 128;
    static constexpr int kStageBytes = kFp8 ? 4 * 16384 + kTileM * 64 : 9 * kTileM * 128;
    static constexpr int kVChunks = kDimChunks / kCpp;                            // parts holding c_kv
    static constexpr int kKvOff = 0;
    static constexpr int kScaleOff = kKvOff + kStages * kStageBytes;               // FP8: 512 B / stage
    static constexpr int kScaleBytes = kFp8 ? kTileM * 4 : 0;
    static constexpr int kQOff = (kScaleOff + kStages * kScaleBytes + 1023) & ~1023;
    // Q (MMA B operand, K-major): FP8 chunk c = [96 rows: hi 0-47, lo 48-95][128 B]; bf16 [48][128 B]
    static constexpr int kQChunk = kNMma * 128;                                    // 12288 / 6144
    static constexpr int kQRopeOff = 4 * kQChunk;                                  // FP8 RoPE chunk [96][64 B]
    static constexpr int kQBytes = kFp8 ? 4 * kQChunk + kNMma * 64 : 9 * kQChunk;
    static constexpr int kPOff = (kQOff + kQBytes + 1023) & ~1023;
    // P^T (MMA B operand, MN-major, no swizzle): groups of 16 B of rows x 128 positions
    static constexpr int kPGroupRows = kFp8 ? 16 : 8;
    static constexpr int kPBytes = (kNMma / kPGroupRows) * kTileM * 16;           // 12288 both
    static constexpr int kPLoOff = kFp8 ? (kN / 16) * kTileM * 16 : 0;             // lo rows start (group 3)
    static constexpr int kMiscOff = kPOff + 2 * kPBytes;                           // P double-buffered
    // Each stage is filled and freed in parts: the c_kv part (FP8: one part,
    // with the per-position scales; bf16: 8 chunks of 64 dims) and the RoPE
    // part, which the score MMAs alone read and so is freed first.
    static constexpr int kParts = kVChunks + 1;
    static constexpr int kRope = kVChunks;                                        // part index of the RoPE chunk
    __host__ __device__ static constexpr uint32_t part_bytes(int part) {            // per page
        return kFp8 ? (part == kRope ? 1024u : 2048u * kCpp + (part == 0 ? 64u : 0u)) : 2048u;
    }
    // exponent offset C and lazy threshold TAU of the softmax stabiliser, and
    // the headroom DELTA it is placed above a new maximum when it moves (so
    // that later, slightly larger scores do not move it again at once); the
    // largest weight stays below 2^(C + TAU) either way.
    static constexpr float kC = kFp8 ? 4.5f : 0.f;
    static constexpr float kTau = kFp8 ? 4.f : 8.f;
    static constexpr float kDelta = kFp8 ? 2.f : 0.f;
};

struct Misc {
    uint64_t part_full[2][9], part_empty[2][9];   // per KV stage and part
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], pv_done[2];  // per P buffer: weights written / value MMAs of that buffer done
    uint64_t q_full;          // the raw query rows of a piece landed
    uint64_t q_ready, o_free, drain;
    uint64_t p_redo;          // a flagged tile's weights rewritten (all softmax warps)
    uint32_t redo[2];         // per P buffer: gg + 1 when tile gg's weights must be rewritten
    uint64_t all_sync;        // all softmax warps (bounded waits, unlike bar.sync)
    uint64_t half_sync[kRowGroups];  // the four softmax warps of each row group
    uint32_t tmem_base;
    int abort;
    uint32_t stage_info[4];   // per tile mod 4: bit i page slot i loaded; bit 31 a page was invalid
    int col_lim[kN];          // positions visible to row r within this piece, 0 = none
    int col_bad[kN];
    float qscale;
    float amax[kSoftmaxWarps];
    __align__(16) float red[kRowGroups][4][kRpt];  // [row group][warp][row]
    float m2c[kN];            // per row: the stabiliser (minus C) at the end of a piece
};

template <bool kFp8>
constexpr int smem_bytes() {
    return Cfg<kFp8>::kMiscOff + (int)sizeof(Misc) + 1024;  // + alignment slack
}

__device__ __forceinline__ void cta_abort(const Problem &p, Misc &ms) {
    if (atomicExch(&ms.abort, 1) == 0) report_error(p.err, kDevTimeout, blockIdx.x);
}

__device__ __forceinline__ bool aborted(Misc &ms) { return *reinterpret_cast<volatile int *>(&ms.abort) != 0; }

// Bounded wait of a whole warp (all 32 lanes call it): every lane waits, and
// the warp goes on only if every lane saw the phase, so a lane whose limit
// runs out just before the phase completes cannot split the warp (the
// .sync.aligned tensor-memory loads that follow need all of it).
__device__ __forceinline__ bool waitb(const Problem &p, Misc &ms, uint64_t *bar, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, wait_limit(p), p.wait_limit != 0));
    if (!ok) cta_abort(p, ms);
    return ok;
}

// Barrier of a group of softmax warps: an mbarrier counting one arrival per
// warp, with a bounded wait, so that if a warp has stopped on a timeout the
// others give up too instead of hanging.
struct GroupSync {
    uint64_t *bar;
    uint32_t phase;
    __device__ explicit GroupSync(uint64_t *b) : bar(b), phase(0) {}
    __device__ __forceinline__ bool operator()(const Problem &p, Misc &ms) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar);
        const bool ok = waitb(p, ms, bar, phase & 1);
        ++phase;
        return ok;
    }
};

__device__ __forceinline__ int ntiles_of(const Piece &pc) {
    return (pc.page_hi - pc.page_lo + kTilePages - 1) / kTilePages;
}

// Reduces 16 per-lane values x[r] + off (one per row) over the warp's 32
// lanes by halving exchanges (8 + 4 + 2 + 1 + 1 shuffles instead of 16 x 5):
// the result for row r is returned in lanes 2r and 2r + 1.
template <bool kMax>
__device__ __forceinline__ float warp_reduce_rows16(const float (&x)[16], float off = 0.f) {
    const int lane = threadIdx.x & 31;
    auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
    float v8[8], v4[4], v2[2];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        v8[j] = op((b4 ? x[8 + j] : x[j]) + off, __shfl_xor_sync(0xffffffffu, (b4 ? x[j] : x[8 + j]) + off, 16));
#pragma unroll
    for (int j = 0; j < 4; ++j)
        v4[j] = op(b3 ? v8[4 + j] : v8[j], __shfl_xor_sync(0xffffffffu, b3 ? v8[j] : v8[4 + j], 8));
#pragma unroll
    for (int j = 0; j < 2; ++j)
        v2[j] = op(b2 ? v4[2 + j] : v4[j], __shfl_xor_sync(0xffffffffu, b2 ? v4[j] : v4[2 + j], 4));
    const float v1 = op(b1 ? v2[1] : v2[0], __shfl_xor_sync(0xffffffffu, b1 ? v2[0] : v2[1], 2));
    return op(v1, __shfl_xor_sync(0xffffffffu, v1, 1));
}

// ---------------------------------------------------------------------------
// warp 0: TMA producer
// ---------------------------------------------------------------------------
template <bool kFp8>
__device__ void producer(const Problem &p, const CUtensorMap *map_a, const CUtensorMap *map_b,
                         unsigned char *smem, Misc &ms, int slot) {
    using C = Cfg<kFp8>;
    const int lane = threadIdx.x & 31;
    const uint64_t pol = ptx::policy_evict_first();  // the cache is read once: first out of L2
    uint32_t g = 0;            // tiles whose copies are all armed
    uint32_t cur_parts = 0;    // parts of tile g armed so far (a stop can come mid-tile)
    bool first_piece = true;
    for_each_piece(p, slot, [&](const Piece &pc) {
        const int nt = ntiles_of(pc);
        for (int k = 0; k < nt; ++k, ++g) {
            if (aborted(ms)) return;
            // At launch every CTA wants its first tiles and its query at once;
            // the second tile waits until the query is staged, so that the
            // query's bytes are not queued behind tile copies.
            if (first_piece && k == 1 && !waitb(p, ms, &ms.q_ready, 0)) return;
            const int stage = g % C::kStages;
            const uint32_t empty_parity = ((g / C::kStages) & 1) ^ 1;
            const int pg0 = pc.page_lo + k * kTilePages;
            const int npg = min(kTilePages, pc.page_hi - pg0);
            int pid = -1;
            bool ok = false;
            if (lane < npg) {
                pid = __ldg(p.page_table + (int64_t)pc.b * p.pt_stride + pg0 + lane);
                ok = pid >= 0 && pid < p.num_pages;
            }
            const unsigned okm = __ballot_sync(0xffffffffu, ok);
            const unsigned badm = __ballot_sync(0xffffffffu, lane < npg && !ok);
            if (lane == 0) {
                if (badm) report_error(p.err, MLA_DEV_BAD_PAGE, pc.b);
                ms.stage_info[g & 3] = okm | (badm ? 0x80000000u : 0u);
            }
            const uint32_t n_ok = __popc(okm);
            unsigned char *st = smem + C::kKvOff + stage * C::kStageBytes;
            const int y = pid * kPage;
            // RoPE first (freed first, right after the previous scores), then the value chunks
            for (int q = 0; q < C::kParts; ++q) {
                const int part = q == 0 ? C::kRope : q - 1;
                if (!waitb(p, ms, &ms.part_empty[stage][part], empty_parity)) return;
                // a static per-tensor FP8 scale comes with no per-position scale copies
                const uint32_t pb = C::part_bytes(part) - (kFp8 && part == 0 && p.kv_scale_per_tensor ? 64u : 0u);
                if (lane == 0) ptx::mbar_arrive_expect_tx(&ms.part_full[stage][part], n_ok * pb);
                __syncwarp();
                cur_parts = q + 1;
                if (!ok) continue;
                uint64_t *bar = &ms.part_full[stage][part];
                if constexpr (kFp8) {
                    if (part == C::kRope) {
                        ptx::tma_load_2d_hint(st + C::kRopeOff + lane * 1024, map_b, bar, 512, y, pol);
                    } else {
                        // page slot `lane` = 8-position groups 2*lane, 2*lane+1 of the part
                        ptx::tma_load_5d_hint(st + part * C::kPartStride + lane * 2 * C::kGroupStride, map_a, bar, 0,
                                              0, part * C::kCpp, 0, pid, pol);
                        if (part == 0 && !p.kv_scale_per_tensor)
                            ptx::bulk_load_hint(smem + C::kScaleOff + stage * C::kScaleBytes + lane * 64,
                                                p.kv_scale + (int64_t)pid * kPage, 64, bar, pol);
                    }
                } else {
                    ptx::tma_load_2d_hint(st + part * C::kChunkStride + lane * 2048, map_a, bar, 64 * part, y, pol);
                }
            }
            cur_parts = 0;
        }
        first_piece = false;
    });
    // Make sure no copy is still landing when the CTA leaves, also after a
    // stop: a stage part is armed again only once its previous copy has been
    // consumed, so only the last arming of each stage part can be in flight.
    // Tiles 0..g-1 armed every part, tile g its first cur_parts parts.
    for (int s2 = 0; s2 < C::kStages; ++s2) {
        for (int qi = 0; qi < C::kParts; ++qi) {
            const int part = qi == 0 ? C::kRope : qi - 1;
            uint32_t n = g / C::kStages + ((uint32_t)s2 < g % C::kStages ? 1u : 0u);
            if (g % C::kStages == (uint32_t)s2 && (uint32_t)qi < cur_parts) ++n;
            if (n) ptx::mbar_wait(&ms.part_full[s2][part], (n - 1) & 1, kWaitLimit);
        }
    }
}

// ---------------------------------------------------------------------------
// warps 1 and 14: MMA issuers
// ---------------------------------------------------------------------------
// The score MMAs of a tile and the value MMAs of the tile before it are
// issued by two warps.  Issuing a group of MMAs blocks the issuing thread
// until most of the group has run, about a thousand cycles; with one issuer
// the value MMAs of tile k, whose completion frees the KV stage that tile
// k + 2 is copied into, waited behind that block whenever the scores of tile
// k + 1 had just been issued.  With two, each issuer waits only for what its
// own MMAs read, and the tensor pipe takes the two groups as they come.
//
// A commit tracks the MMAs of its own thread.  The KV stage part that both
// groups read is freed by the value group's commit alone: by then the scores
// of that tile have been read by the softmax, so their MMAs are done.

// Waits are made by lane 0 and broadcast, so the warp never diverges on a
// phase that completes (or a limit that expires) while it waits.
__device__ __forceinline__ bool issuer_wait(const Problem &p, Misc &ms, uint64_t *bar, uint32_t parity) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, wait_limit(p), p.wait_limit != 0) && !aborted(ms);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) cta_abort(p, ms);
    return ok != 0;
}

// every MMA this thread issued has completed before tensor memory is released
__device__ __forceinline__ void issuer_drain(Misc &ms) {
    if ((threadIdx.x & 31) == 0) ptx::mma_commit(&ms.drain);
    __syncwarp();
    ptx::mbar_wait(&ms.drain, 0, kWaitLimit);
}

// warp 1: score MMAs S^T = K Q^T of every tile, once its parts have landed
// and the score buffer is free.
template <bool kFp8>
__device__ void score_issuer(const Problem &p, unsigned char *smem, Misc &ms, int slot) {
    using C = Cfg<kFp8>;
    const int lane = threadIdx.x & 31;
    const uint32_t tmem = ms.tmem_base;
    const uint32_t kv0 = ptx::smem_u32(smem + C::kKvOff);
    const uint32_t q0 = ptx::smem_u32(smem + C::kQOff);
    constexpr uint32_t idesc_qk = kFp8 ? ptx::instr_desc(0, 0, 0, 0, kTileM, C::kNMma)
                                       : ptx::instr_desc(1, 1, 0, 0, kTileM, C::kNMma);
    // Shared-memory descriptors are built once; an MMA then only adds the
    // byte offset of its operands (>> 4) to the start-address field.
    constexpr uint64_t kStageStep = (uint64_t)(C::kStageBytes >> 4);
    const uint64_t dq_kv = ptx::smem_desc(kv0, 16, C::kGroupStride, ptx::kSwizzle128B);  // K-major 128B chunks
    const uint64_t dq_q = ptx::smem_desc(q0, 16, 1024, ptx::kSwizzle128B);
    const uint64_t dr_kv = ptx::smem_desc(kv0 + C::kRopeOff, 16, 512, ptx::kSwizzle64B);  // FP8 RoPE
    const uint64_t dr_q = ptx::smem_desc(q0 + C::kQRopeOff, 16, 512, ptx::kSwizzle64B);

    // Score MMAs reading one part of the tile (accumulate from the second MMA of the tile on).
    auto issue_qk_part = [&](uint32_t gg, int part, bool first) {
        const uint64_t so = (gg % C::kStages) * kStageStep;
        const uint32_t d = tmem + ((gg % C::kSBufs) ? C::kColS1 : 0u);
        if constexpr (kFp8) {
            // N = 96: query rows 0-47 hold hi, 48-95 hold lo
            if (part == C::kRope) {
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    ptx::mma_f8(d, dr_kv + so + 2 * ks, dr_q + 2 * ks, idesc_qk, (first && ks == 0) ? 0u : 1u);
            } else {
#pragma unroll
                for (int c = part * C::kCpp; c < (part + 1) * C::kCpp; ++c) {
                    const uint64_t a = dq_kv + so + (C::chunk_off(c) >> 4);
                    const uint64_t b = dq_q + c * (C::kQChunk >> 4);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        ptx::mma_f8(d, a + 2 * ks, b + 2 * ks, idesc_qk, (first && ks == 0) ? 0u : 1u);
                }
            }
        } else {
            const uint64_t a = dq_kv + so + part * (C::kChunkStride >> 4);
            const uint64_t b = dq_q + part * (C::kQChunk >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                ptx::mma_f16(d, a + 2 * ks, b + 2 * ks, idesc_qk, (first && ks == 0) ? 0u : 1u);
        }
    };

    uint32_t g = 0, pi = 0;
    for_each_piece(p, slot, [&](const Piece &pc) {
        const int nt = ntiles_of(pc);
        if (nt == 0 || aborted(ms)) return;
        if (!issuer_wait(p, ms, &ms.q_ready, pi & 1)) return;
        for (int k = 0; k < nt; ++k) {
            const uint32_t gq = g + k;
            const int stage = gq % C::kStages;
            if (!issuer_wait(p, ms, &ms.s_free[gq % C::kSBufs], ((gq / C::kSBufs) & 1) ^ 1)) return;
            for (int q = 0; q < C::kParts; ++q)
                if (!issuer_wait(p, ms, &ms.part_full[stage][q == 0 ? C::kRope : q - 1], (gq / C::kStages) & 1))
                    return;
            ptx::tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int q = 0; q < C::kParts; ++q) issue_qk_part(gq, q == 0 ? C::kRope : q - 1, q == 0);
                ptx::mma_commit(&ms.s_full[gq % C::kSBufs]);
                ptx::mma_commit(&ms.part_empty[stage][C::kRope]);  // RoPE is read by scores only
            }
            __syncwarp();
        }
        g += nt;
        ++pi;
    });
    issuer_drain(ms);
}

// warp 14: value MMAs O^T += V^T P^T of every tile, once all softmax warps
// have written its weights (and, for a flagged tile, rewritten them).
template <bool kFp8>
__device__ void value_issuer(const Problem &p, unsigned char *smem, Misc &ms, int slot) {
    using C = Cfg<kFp8>;
    const int lane = threadIdx.x & 31;
    const uint32_t tmem = ms.tmem_base;
    const uint32_t kv0 = ptx::smem_u32(smem + C::kKvOff);
    const uint32_t p0 = ptx::smem_u32(smem + C::kPOff);
    constexpr uint32_t idesc_pv = kFp8 ? ptx::instr_desc(0, 0, 1, 1, kTileM, C::kNMma)
                                       : ptx::instr_desc(1, 1, 1, 1, kTileM, C::kNMma);
    constexpr uint64_t kStageStep = (uint64_t)(C::kStageBytes >> 4);
    // V^T, MN-major: 128-B atoms along the dims C::kChunkStride apart, 8-position groups along K
    const uint64_t dv_kv = ptx::smem_desc(kv0, C::kChunkStride, C::kGroupStride, ptx::kSwizzle128B);
    const uint64_t dv_p = ptx::smem_desc(p0, 128, 2048, ptx::kSwizzleNone);       // P^T, MN-major

    // Value MMAs; each 128-dim block frees its value chunk(s) of the stage as it completes.
    auto issue_pv = [&](uint32_t gg, bool first) {
        const int stage = gg % C::kStages;
        const uint64_t a0 = dv_kv + stage * kStageStep;
        const uint64_t pb = dv_p + (gg & 1) * (uint64_t)(C::kPBytes >> 4);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t d = tmem + C::kColO + C::kOStride * m;
            if constexpr (kFp8) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // 32 positions (4 groups) per MMA; N = 96: P hi | P lo
                    ptx::mma_f8(d, a0 + (C::chunk_off(m) >> 4) + ks * ((4 * C::kGroupStride) >> 4),
                                pb + ks * (512 >> 4), idesc_pv, (first && ks == 0) ? 0u : 1u);
                if (m % C::kCpp == C::kCpp - 1) ptx::mma_commit(&ms.part_empty[stage][m / C::kCpp]);
            } else {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)  // 16 positions (2 groups) per MMA
                    ptx::mma_f16(d, a0 + 2 * m * (C::kChunkStride >> 4) + ks * ((2 * C::kGroupStride) >> 4),
                                 pb + ks * (256 >> 4), idesc_pv, (first && ks == 0) ? 0u : 1u);
                ptx::mma_commit(&ms.part_empty[stage][2 * m]);
                ptx::mma_commit(&ms.part_empty[stage][2 * m + 1]);
            }
        }
    };

    uint32_t g = 0, pi = 0;
    uint32_t redo_n = 0;       // rewrites of flagged tiles' weights consumed
    for_each_piece(p, slot, [&](const Piece &pc) {
        const int nt = ntiles_of(pc);
        if (nt == 0 || aborted(ms)) return;
        for (int k = 0; k < nt; ++k) {
            const uint32_t gp = g + k;
            // the epilogue of the previous piece has read O
            if (k == 0 && !issuer_wait(p, ms, &ms.o_free, (pi & 1) ^ 1)) return;
            if (!issuer_wait(p, ms, &ms.p_full[gp & 1], (gp >> 1) & 1)) return;
            // the flag was written before the last arrival on p_full
            int redo = 0;
            if (lane == 0) redo = *reinterpret_cast<volatile uint32_t *>(&ms.redo[gp & 1]) == gp + 1;
            redo = __shfl_sync(0xffffffffu, redo, 0);
            if (redo) {
                if (!issuer_wait(p, ms, &ms.p_redo, redo_n & 1)) return;
                ++redo_n;
            }
            ptx::tc_fence_after();
            if (lane == 0) {
                issue_pv(gp, k == 0);
                ptx::mma_commit(&ms.pv_done[gp & 1]);
            }
            __syncwarp();
        }
        g += nt;
        ++pi;
    });
    issuer_drain(ms);
}

// ---------------------------------------------------------------------------
// warps 2-13: query staging, online softmax, epilogue
// ---------------------------------------------------------------------------
// The 48 query rows of a group arrive raw, as two bulk copies into the query
// area: [48 rows][512] bf16 latent parts, then [48 rows][64] bf16 RoPE parts
// (a sequence's rows are contiguous in q_lat and q_pe).  One thread issues
// them when a piece starts, so they are in flight while the CTA sets up.
constexpr int kQRawRope = kN * kDl * 2;   // byte offset of the raw RoPE rows

__device__ __forceinline__ void issue_query_copy(const Problem &p, unsigned char *qs, Misc &ms, int b, int r0) {
    const int rows = min(kN, p.R - r0);
    const int64_t row0 = (int64_t)b * p.R + r0;
    ptx::fence_proxy_async_smem();  // earlier generic writes to the area come first
    ptx::mbar_arrive_expect_tx(&ms.q_full, (uint32_t)rows * (kDl + kDr) * 2);
    ptx::bulk_load(qs, p.q_lat + row0 * kDl, (uint32_t)rows * kDl * 2, &ms.q_full);
    ptx::bulk_load(qs + kQRawRope, p.q_pe + row0 * kDr, (uint32_t)rows * kDr * 2, &ms.q_full);
}

// Turns the raw rows into the score MMA's B operand in place (K-major, 128B /
// 64B swizzled chunks): every thread reads its units into registers, a
// barrier of all softmax warps separates the reads from the writes, then the
// units are written back in operand layout.  FP8: the block's largest |q|
// sets a power-of-two scale s, hi = e4m3(q/s) goes to rows 0-47 and lo =
// e4m3(q/s - hi) to rows 48-95.  A power-of-two s keeps q/s a bf16 value,
// which hi + lo represents exactly (short of e4m3 underflow far below the
// largest q).  Rows past R are zero.
template <bool kFp8>
__device__ bool stage_query(const Problem &p, unsigned char *smem, Misc &ms, int r0, int st, GroupSync &gsync) {
    using C = Cfg<kFp8>;
    unsigned char *qs = smem + C::kQOff;
    const int rows = min(kN, p.R - r0);
    if constexpr (kFp8) {
        // unit = 16 consecutive dims of one row (36 units per row, 32 latent + 4 RoPE)
        constexpr int kUnits = kN * 36;
        constexpr int kPer = (kUnits + kSoftmaxThreads - 1) / kSoftmaxThreads;  // 7
        uint4 v[kPer][2];
        // largest |q| from the bf16 bit patterns: with the sign cleared, a
        // bf16 magnitude orders like its bits, two per 32-bit word
        uint32_t mbits = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int u = st + j * kSoftmaxThreads;
            const int row = u / 36, uu = u % 36;
            v[j][0] = v[j][1] = make_uint4(0, 0, 0, 0);
            if (u < kUnits && row < rows) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    uu < 32 ? qs + row * (kDl * 2) + uu * 32 : qs + kQRawRope + row * (kDr * 2) + (uu - 32) * 32);
                v[j][0] = src[0];
                v[j][1] = src[1];
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mbits = __vmaxu2(mbits, v[j][h].x & 0x7FFF7FFFu);
                mbits = __vmaxu2(mbits, v[j][h].y & 0x7FFF7FFFu);
                mbits = __vmaxu2(mbits, v[j][h].z & 0x7FFF7FFFu);
                mbits = __vmaxu2(mbits, v[j][h].w & 0x7FFF7FFFu);
            }
        }
        // the warp's largest magnitude bits in one reduction instruction
        mbits = __reduce_max_sync(0xffffffffu, max(mbits & 0xFFFFu, mbits >> 16));
        float amax = __uint_as_float(mbits << 16);
        if ((threadIdx.x & 31) == 0) ms.amax[(threadIdx.x >> 5) - 2] = amax;
        if (!gsync(p, ms)) return false;   // also: every raw read is done
#pragma unroll
        for (int w = 0; w < kSoftmaxWarps; ++w) amax = fmaxf(amax, ms.amax[w]);
        int e2 = 0;
        if (amax > 0.f) frexpf(amax / 448.f, &e2);
        const float inv = ldexpf(1.f, -e2);
        if (st == 0) ms.qscale = ldexpf(1.f, e2);
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int u = st + j * kSoftmaxThreads;
            if (u >= kUnits) continue;
            const int row = u / 36, uu = u % 36;
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&v[j][h]);
#pragma unroll
                for (int q = 0; q < 2; ++q) {  // 4 dims -> one 32-bit word of hi and of lo
                    const float2 f0 = __bfloat1622float2(b2[2 * q]), f1 = __bfloat1622float2(b2[2 * q + 1]);
                    // q/s is exact in f16 down to its subnormals, far below lo's e4m3 range
                    const uint32_t p01 = ptx::f16x2(f0.x * inv, f0.y * inv), p23 = ptx::f16x2(f1.x * inv, f1.y * inv);
                    const uint32_t h01 = ptx::e4m3x2_from_f16x2(p01), h23 = ptx::e4m3x2_from_f16x2(p23);
                    const uint32_t l01 = ptx::e4m3x2_from_f16x2(ptx::sub_f16x2(p01, ptx::f16x2_from_e4m3x2(h01)));
                    const uint32_t l23 = ptx::e4m3x2_from_f16x2(ptx::sub_f16x2(p23, ptx::f16x2_from_e4m3x2(h23)));
                    hw[2 * h + q] = h01 | (h23 << 16);
                    lw[2 * h + q] = l01 | (l23 << 16);
                }
            }
            const uint4 hi4 = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            const uint4 lo4 = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            const int rl = row + kN;   // lo row
            if (uu < 32) {
                const int c = uu >> 3, k = uu & 7;
                *reinterpret_cast<uint4 *>(qs + c * C::kQChunk + row * 128 + ((k ^ (row & 7)) << 4)) = hi4;
                *reinterpret_cast<uint4 *>(qs + c * C::kQChunk + rl * 128 + ((k ^ (rl & 7)) << 4)) = lo4;
            } else {
                const int k = uu - 32;
                *reinterpret_cast<uint4 *>(qs + C::kQRopeOff + row * 64 + ((k ^ ((row >> 1) & 3)) << 4)) = hi4;
                *reinterpret_cast<uint4 *>(qs + C::kQRopeOff + rl * 64 + ((k ^ ((rl >> 1) & 3)) << 4)) = lo4;
            }
        }
    } else {
        constexpr int kUnits = kN * 72;  // 8 dims per unit
        constexpr int kPer = (kUnits + kSoftmaxThreads - 1) / kSoftmaxThreads;  // 9
        uint4 v[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int u = st + j * kSoftmaxThreads;
            const int row = u / 72, uu = u % 72;
            v[j] = make_uint4(0, 0, 0, 0);
            if (u < kUnits && row < rows)
                v[j] = *reinterpret_cast<const uint4 *>(uu < 64 ? qs + row * (kDl * 2) + uu * 16
                                                                : qs + kQRawRope + row * (kDr * 2) + (uu - 64) * 16);
        }
        if (!gsync(p, ms)) return false;   // every raw read is done
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int u = st + j * kSoftmaxThreads;
            if (u >= kUnits) continue;
            const int row = u / 72, uu = u % 72;
            const int c = uu >> 3, k = uu & 7;
            *reinterpret_cast<uint4 *>(qs + c * C::kQChunk + row * 128 + ((k ^ (row & 7)) << 4)) = v[j];
        }
    }
    return true;
}

// kRpt rows of one accumulator column block; for FP8 the hi and lo halves
// (48 columns apart) are added.
template <bool kFp8>
__device__ __forceinline__ void tmem_rows(uint32_t taddr, float *v) {
    if constexpr (kFp8) {
        static_assert(kRpt == 16, "the paired load takes 16 columns per half");
        float w[kRpt];
        ptx::tmem_ld16_pair(taddr, taddr + kN, v, w);
#pragma unroll
        for (int c = 0; c < kRpt; ++c) v[c] += w[c];
    } else {
        ptx::tmem_ld_cols<kRpt>(taddr, v);
    }
}

template <bool kFp8>
__device__ void softmax_role(const Problem &p, unsigned char *smem, Misc &ms, int slot, int g_idx,
                             const CUtensorMap *map_out, const CUtensorMap *map_part) {
    using C = Cfg<kFp8>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ws = warp - 2;                   // softmax warp 0 .. kSoftmaxWarps - 1
    const int h = ws >> 2;                     // row group: rows [kRpt h, kRpt (h + 1))
    const int w4 = ws & 3;                     // warp within the row group
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int i = quad * 32 + lane;            // tile position / TMEM lane
    const int st = threadIdx.x - 64;           // 0 .. kSoftmaxThreads - 1, for cooperative loops
    const int hst = w4 * 32 + lane;            // 0..127 within the row group
    const int cb = h * kRpt;
    const uint32_t tmem = ms.tmem_base + ((uint32_t)(quad * 32) << 16);
    const int r0 = g_idx * kN;
    constexpr float kEmpty = -1e30f;           // stabiliser of a row that has seen nothing yet
    uint32_t g = 0;
    GroupSync all_sync(&ms.all_sync), hsync(&ms.half_sync[h]);
    const float static_scale = kFp8 && p.kv_scale_per_tensor ? __ldg(p.kv_scale) : 1.f;

    uint32_t qn = 0;           // query copies waited for (phase of q_full)
    uint32_t q_issued = 0;     // query copies issued (thread st == 0)
    for_each_piece(p, slot, [&](const Piece &pc) {
        if (aborted(ms)) return;
        const int nt = ntiles_of(pc);
        // the query rows go out first, so they land while the piece is set up
        if (nt > 0 && st == 0) {
            issue_query_copy(p, smem + C::kQOff, ms, pc.b, r0);
            ++q_issued;
        }
        // visible positions per row, limited to this piece's pages
        if (st < kN) {
            const int r = r0 + st;
            int lim = 0, bad = 0;
            if (pc.bad_ctx) {
                bad = 1;
            } else if (r < p.R) {
                const int v = visible(p, pc.b, r / p.H, pc.ctx);
                if (v < 0) {
                    bad = 1;
                    report_error(p.err, MLA_DEV_BAD_VIS, pc.b * p.T + r / p.H);
                } else {
                    lim = min(v, pc.page_hi * kPage);
                }
            }
            ms.col_lim[st] = lim;
            ms.col_bad[st] = bad;
        }
        if (st == 0 && pc.bad_ctx && g_idx == 0) report_error(p.err, MLA_DEV_BAD_CTX, pc.b);
        if (!all_sync(p, ms)) return;
        const int rows_here = min(kN, p.R - r0);
        int min_lim = INT_MAX;  // over this row group's real rows
        for (int c = cb; c < min(cb + kRpt, rows_here); ++c) min_lim = min(min_lim, ms.col_lim[c]);
        uint32_t bad_rows = 0;  // bit c: row cb + c is invalid (its results are NaN)
#pragma unroll
        for (int c = 0; c < kRpt; ++c) bad_rows |= ms.col_bad[cb + c] ? 1u << c : 0u;

        if (nt == 0) {  // nothing to read: write the empty (or invalid) result
            for (int e = st; e < rows_here * kDl; e += kSoftmaxThreads) {
                const int c = e / kDl, d = e % kDl;
                const bool bad = ms.col_bad[c] != 0;
                store_out(p.out, ((int64_t)pc.b * p.R + r0 + c) * kDl + d, bad ? NAN : 0.f, p.out_f32);
                if (d == 0 && p.lse) p.lse[(int64_t)pc.b * p.R + r0 + c] = bad ? NAN : -INFINITY;
            }
            all_sync(p, ms);
            return;
        }

        if (!waitb(p, ms, &ms.q_full, qn & 1)) return;
        ++qn;
        if (!stage_query<kFp8>(p, smem, ms, r0, st, all_sync)) return;
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ms.q_ready);
        if (!all_sync(p, ms)) return;  // qscale visible
        const float qscale = kFp8 ? ms.qscale : 1.f;

        // m2c = stabiliser - C: weights are ex2(score - m2c)
        float m2c[kRpt], lsum[kRpt];
#pragma unroll
        for (int c = 0; c < kRpt; ++c) {
            m2c[c] = kEmpty;
            lsum[c] = 0.f;
        }
        bool piece_bad = false;
        const uint32_t g0 = g;

        // This thread's entries of the tile's weight operand P: e = ex2(s - m2c)
        // for its kRpt rows (times the token's value scale for FP8), as the
        // 32-bit words of the layout the value MMA reads (make_p), then written
        // to P buffer gg & 1 (put_p).  With add_sums the weights also enter the
        // row sums.  The conversions need no buffer, so they run before the
        // wait for one.
        constexpr int kPW = kFp8 ? kRpt / 4 : kRpt / 2;   // words per operand (hi, lo)
        auto make_p = [&](const float (&sc)[kRpt], float kvs, bool add_sums, uint32_t (&hw)[kPW],
                          uint32_t (&lw)[kPW]) {
            if constexpr (kFp8) {
                // P = hi + lo, two e4m3 operands; word w packs rows 4w..4w+3 of this
                // thread's rows.  Pairs go through f16x2: p16 = f16(P) (relative error 2^-12,
                // far below lo's 2^-9), hi = e4m3(p16), and p16 - hi is exact in
                // f16, so lo = e4m3(p16 - hi).
#pragma unroll
                for (int w = 0; w < kPW; ++w) {
                    uint32_t hp[2], lp[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int c0 = 4 * w + 2 * q;
                        const float e0 = ptx::ex2(sc[c0] - m2c[c0]), e1 = ptx::ex2(sc[c0 + 1] - m2c[c0 + 1]);
                        if (add_sums) {
                            lsum[c0] += e0;
                            lsum[c0 + 1] += e1;
                        }
                        const uint32_t p16 = ptx::f16x2(e0 * kvs, e1 * kvs);
                        hp[q] = ptx::e4m3x2_from_f16x2(p16);
                        lp[q] = ptx::e4m3x2_from_f16x2(ptx::sub_f16x2(p16, ptx::f16x2_from_e4m3x2(hp[q])));
                    }
                    hw[w] = hp[0] | (hp[1] << 16);
                    lw[w] = lp[0] | (lp[1] << 16);
                }
            } else {
                // bf16: word w packs rows 2w, 2w+1
#pragma unroll
                for (int w = 0; w < kPW; ++w) {
                    const int c0 = 2 * w;
                    const float e0 = ptx::ex2(sc[c0] - m2c[c0]), e1 = ptx::ex2(sc[c0 + 1] - m2c[c0 + 1]);
                    if (add_sums) {
                        lsum[c0] += e0;
                        lsum[c0 + 1] += e1;
                    }
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
                    hw[w] = *reinterpret_cast<uint32_t *>(&b2);
                    lw[w] = 0u;
                }
            }
        };
        auto put_p = [&](const uint32_t (&hw)[kPW], const uint32_t (&lw)[kPW], uint32_t gg) {
            unsigned char *pb = smem + C::kPOff + (gg & 1) * C::kPBytes;
            if constexpr (kFp8) {
                // P^T is [16-row groups of 16 B] x 128 positions: this thread's 16 rows
                // (cb is a multiple of 16) are one 16-B entry of hi and one of lo, so a
                // warp writes 512 contiguous bytes per store
                const int off = (cb >> 4) * 2048 + i * 16;
                *reinterpret_cast<uint4 *>(pb + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(pb + C::kPLoOff + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            } else {
                // bf16 P^T: [8-row groups of 16 B] x 128 positions: two entries
                const int off = (cb >> 3) * 2048 + i * 16;
                *reinterpret_cast<uint4 *>(pb + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(pb + off + 2048) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
        };

        for (int k = 0; k < nt; ++k) {
            const uint32_t gg = g0 + k;
            const int stage = gg % C::kStages;
            // part 0 carries the value scales; the tile's page mask was written before it
            if (!waitb(p, ms, &ms.part_full[stage][0], (gg / C::kStages) & 1)) return;
            const uint32_t info = ms.stage_info[gg & 3];
            piece_bad |= (info >> 31) != 0;
            const int pos0 = (pc.page_lo + k * kTilePages) * kPage;
            const int pos = pos0 + i;
            const bool loaded = (info >> (i / kPage)) & 1u;
            // value scale of this lane's token; 0 where the slot is not a
            // cached position (its stored scale may be anything, even NaN)
            const float kvs = !kFp8 ? 1.f
                              : !(loaded && pos < pc.ctx) ? 0.f
                              : p.kv_scale_per_tensor
                                  ? static_scale
                                  : reinterpret_cast<const float *>(smem + C::kScaleOff + stage * C::kScaleBytes)[i];
            const float factor = p.sm_scale_log2 * (kFp8 ? kvs * qscale : 1.f);
            const float lkvs = kFp8 ? __log2f(kvs) : 0.f;
            const bool fast = (info & 0xFFu) == 0xFFu && pos0 + kTileM <= min_lim;
            // u = s + lkvs exceeds the stabiliser by more than TAU iff s > m2c + (C + TAU - lkvs)
            const float kx = C::kC + C::kTau - lkvs;

            const int sb = gg % C::kSBufs;
            if (!waitb(p, ms, &ms.s_full[sb], (gg / C::kSBufs) & 1)) return;
            ptx::tc_fence_after();
            float s[kRpt];
            tmem_rows<kFp8>(tmem + (sb ? C::kColS1 : 0u) + cb, s);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ms.s_free[sb]);

            // scores in log2 units; outside the visible range -inf (the
            // per-row limits are read only for tiles that reach past one)
            if (fast) {
#pragma unroll
                for (int c = 0; c < kRpt; ++c) s[c] *= factor;
            } else {
#pragma unroll
                for (int c = 0; c < kRpt; ++c) s[c] = loaded && pos < ms.col_lim[cb + c] ? s[c] * factor : -INFINITY;
            }
            float dmax = s[0] - m2c[0];
#pragma unroll
            for (int c = 1; c < kRpt; ++c) dmax = fmaxf(dmax, s[c] - m2c[c]);
            const bool exceed = dmax > kx;
            // Optimistic stabiliser: every warp writes its weights with the
            // current stabiliser and flags the tile if one of them would be too
            // large; the tile's fate is read once every warp has written it.
            const bool wex = __any_sync(0xffffffffu, exceed);
            uint32_t hw[kPW], lw[kPW];
            // a flagged warp's weights are rewritten below, and its sums added then
            make_p(s, kvs, !wex, hw, lw);
            // P buffer gg & 1 is free once the value MMAs of tile gg - 2 are done;
            // the value warp read that tile's flag (same slot) before issuing them
            if (gg >= 2 && !waitb(p, ms, &ms.pv_done[gg & 1], ((gg - 2) >> 1) & 1)) return;
            if (wex && lane == 0) *reinterpret_cast<volatile uint32_t *>(&ms.redo[gg & 1]) = gg + 1;
            // rows past the context, and page slots this tile did not load, may
            // hold anything; their weight is 0 but 0 * NaN is NaN, so clear
            // their values before the value MMA
            if (h == 0 && !fast && (!loaded || pos >= pc.ctx)) {
                unsigned char *stg = smem + C::kKvOff + stage * C::kStageBytes;
#pragma unroll
                for (int c = 0; c < C::kDimChunks; ++c) {
                    uint4 *row = reinterpret_cast<uint4 *>(stg + (i >> 3) * C::kGroupStride + C::chunk_off(c) +
                                                           (i & 7) * 128);
#pragma unroll
                    for (int e = 0; e < 8; ++e) row[e] = make_uint4(0, 0, 0, 0);
                }
            }
            put_p(hw, lw, gg);
            if (lane == 0) ptx::mbar_arrive(&ms.p_full[gg & 1]);

            // every warp has written its weights and its flag for tile gg
            if (!waitb(p, ms, &ms.p_full[gg & 1], (gg >> 1) & 1)) return;
            if (*reinterpret_cast<volatile uint32_t *>(&ms.redo[gg & 1]) != gg + 1) continue;

            // Slow path (the first tile of a piece, then rarely): move the
            // stabiliser of the rows whose weights overflowed to DELTA above
            // their new maximum, rescale what came before, rewrite P.  The
            // value MMAs of this tile wait for it (p_redo).
            {
                const float v = warp_reduce_rows16<true>(s, lkvs);   // max over lanes of score + lkvs
                if ((lane & 1) == 0) ms.red[h][w4][lane >> 1] = v;
            }
            if (!all_sync(p, ms)) return;
            float cmax[kRpt];
#pragma unroll
            for (int c4 = 0; c4 < kRpt / 4; ++c4) {
                float4 a = reinterpret_cast<const float4 *>(ms.red[h][0])[c4];
#pragma unroll
                for (int w = 1; w < 4; ++w) {
                    const float4 t = reinterpret_cast<const float4 *>(ms.red[h][w])[c4];
                    a.x = fmaxf(a.x, t.x); a.y = fmaxf(a.y, t.y); a.z = fmaxf(a.z, t.z); a.w = fmaxf(a.w, t.w);
                }
                cmax[4 * c4] = a.x; cmax[4 * c4 + 1] = a.y; cmax[4 * c4 + 2] = a.z; cmax[4 * c4 + 3] = a.w;
            }
            float alpha[kRpt];
            bool moved = false;
#pragma unroll
            for (int c = 0; c < kRpt; ++c) {
                const float cm = cmax[c];
                const float old = m2c[c] + C::kC;
                const float mn = cm > old + C::kTau ? cm + C::kDelta : old;
                alpha[c] = mn == old ? 1.f : ptx::ex2(old - mn);
                moved |= mn != old;
                m2c[c] = mn - C::kC;
                lsum[c] *= alpha[c];     // earlier tiles, and this one for unflagged warps
            }
            if (moved && k > 0) {
                // O^T holds earlier tiles: wait for their value MMA, then rescale rows
                if (!waitb(p, ms, &ms.pv_done[(gg - 1) & 1], ((gg - 1) >> 1) & 1)) return;
                ptx::tc_fence_after();
#pragma unroll 1
                for (int m = 0; m < 4; ++m) {
#pragma unroll 1
                    for (int part = 0; part < (kFp8 ? 2 : 1); ++part) {
                        float o[kRpt];
                        const uint32_t oc = tmem + C::kColO + C::kOStride * m + part * kN + cb;
                        ptx::tmem_ld_cols<kRpt>(oc, o);
#pragma unroll
                        for (int c = 0; c < kRpt; ++c) o[c] *= alpha[c];
                        ptx::tmem_st_cols<kRpt>(oc, o);
                    }
                }
            }
            make_p(s, kvs, wex, hw, lw);
            put_p(hw, lw, gg);
            if (lane == 0) ptx::mbar_arrive(&ms.p_redo);
        }
        g = g0 + nt;

        // ---- epilogue: row sums, normalised output, log-sum-exp
        if (piece_bad) bad_rows = 0xFFFFu;
        // the last value MMAs done (a commit covers every earlier MMA too)
        if (!waitb(p, ms, &ms.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1)) return;
        ptx::tc_fence_after();
        // the warp's row sums over its 32 lanes, one row per lane pair
        {
            const float v = warp_reduce_rows16<false>(lsum);
            if ((lane & 1) == 0) ms.red[h][w4][lane >> 1] = v;
        }
        // the group's stabilisers, for the rows' log-sum-exps
        if (hst == 0) {
#pragma unroll
            for (int c = 0; c < kRpt; ++c) ms.m2c[cb + c] = m2c[c];
        }
        if (!hsync(p, ms)) return;
        // every thread forms the sums of its own rows (vector loads of the four
        // warps' parts); thread hst < kRpt of the group also forms row cb +
        // hst's log-sum-exp
        float inv_l[kRpt];
#pragma unroll
        for (int c4 = 0; c4 < kRpt / 4; ++c4) {
            float4 l = reinterpret_cast<const float4 *>(ms.red[h][0])[c4];
#pragma unroll
            for (int w = 1; w < 4; ++w) {
                const float4 t = reinterpret_cast<const float4 *>(ms.red[h][w])[c4];
                l.x += t.x; l.y += t.y; l.z += t.z; l.w += t.w;
            }
            const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = 4 * c4 + e;
                inv_l[c] = (bad_rows >> c) & 1u ? NAN : (lv[e] > 0.f ? __fdividef(1.f, lv[e]) : 0.f);
            }
        }
        float row_lse = 0.f;
        if (hst < kRpt) {
            const float l = ms.red[h][0][hst] + ms.red[h][1][hst] + ms.red[h][2][hst] + ms.red[h][3][hst];
            // ln sum_j exp(score_j) = (m2c + log2 l) * ln 2
            row_lse = (bad_rows >> hst) & 1u ? NAN : (l > 0.f ? (ms.m2c[cb + hst] + __log2f(l)) * kLn2 : -INFINITY);
        }
        // O goes out in 128-dim blocks, each row group on its own: the group's
        // threads write their dims of its 16 rows into [16][128] staging boxes
        // (in the query area, free until the next piece: 16 KB per group, so
        // all four blocks at once for bf16 boxes, two at a time for fp32),
        // and the group's first thread stores them with tensor stores; the
        // maps clip rows past the sequence's R.
        const int nrows = min(kRpt, rows_here - cb);
        const bool f32_box = pc.single && p.out_f32;   // partials are bf16
        const int per_round = f32_box ? 2 : 4;
        const int box_bytes = kRpt * 128 * (f32_box ? 4 : 2);
        unsigned char *boxes = smem + C::kQOff + h * (4 * kRpt * 128 * 2);
#pragma unroll 1
        for (int m0 = 0; m0 < 4; m0 += per_round) {
            if (m0 > 0) {  // the stores of the previous blocks have finished reading the boxes
                if (hst == 0) ptx::bulk_wait_read<0>();
                if (!hsync(p, ms)) return;
            }
#pragma unroll 1
            for (int m = m0; m < m0 + per_round; ++m) {
                unsigned char *box = boxes + (m - m0) * box_bytes;
                float o[kRpt];
                tmem_rows<kFp8>(tmem + C::kColO + C::kOStride * m + cb, o);
#pragma unroll
                for (int c = 0; c < kRpt; ++c) {
                    const float v = o[c] * inv_l[c];
                    if (f32_box)
                        reinterpret_cast<float *>(box)[c * 128 + i] = v;
                    else
                        reinterpret_cast<__nv_bfloat16 *>(box)[c * 128 + i] = __float2bfloat16_rn(v);
                }
            }
            ptx::fence_proxy_async_smem();
            if (!hsync(p, ms)) return;
            if (hst == 0 && nrows > 0) {
                for (int m = m0; m < m0 + per_round; ++m) {
                    unsigned char *box = boxes + (m - m0) * box_bytes;
                    if (pc.single)
                        ptx::tma_store_3d(map_out, box, 128 * m, r0 + cb, pc.b);
                    else
                        ptx::tma_store_3d(map_part, box, 128 * m, (int)pc.piece, r0 + cb);
                }
                ptx::bulk_commit();
            }
        }
        if (hst == 0) ptx::bulk_wait_read<0>();  // boxes read before the query area is reused
        if (hst < nrows) {
            const int64_t r = r0 + cb + hst;
            if (pc.single) {
                if (p.lse) p.lse[(int64_t)pc.b * p.R + r] = row_lse;
            } else {
                p.part_lse[r * p.max_pieces + pc.piece] = row_lse;
            }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ms.o_free);
        all_sync(p, ms);  // smem per-piece state reused next piece
    });
    // after a stop, a query copy may still be landing and an output store may
    // still be reading its staging box
    if (st == 0 && q_issued > qn) ptx::mbar_wait(&ms.q_full, (q_issued - 1) & 1, kWaitLimit);
    if (hst == 0) ptx::bulk_wait_read<0>();
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    tc_decode_kernel(const __grid_constant__ Problem p, const __grid_constant__ CUtensorMap map_a,
                     const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_out,
                     const __grid_constant__ CUtensorMap map_part) {
    using C = Cfg<kFp8>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc &ms = *reinterpret_cast<Misc *>(smem + C::kMiscOff);
    const int warp = threadIdx.x >> 5;
    const int slot = blockIdx.x / p.n_groups;
    const int g_idx = blockIdx.x % p.n_groups;
    // the merge kernel that follows may be scheduled now; it waits for this
    // grid to finish before it reads anything this grid writes
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            for (int q = 0; q < 9; ++q) {
                ptx::mbar_init(&ms.part_full[s][q], 1);
                ptx::mbar_init(&ms.part_empty[s][q], 1);
            }
            ptx::mbar_init(&ms.s_full[s], 1);
            ptx::mbar_init(&ms.s_free[s], kSoftmaxWarps);
        }
        for (int r = 0; r < kRowGroups; ++r) ptx::mbar_init(&ms.half_sync[r], 4);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&ms.p_full[b], kSoftmaxWarps);
            ptx::mbar_init(&ms.pv_done[b], 1);
        }
        ptx::mbar_init(&ms.q_ready, kSoftmaxWarps);
        ptx::mbar_init(&ms.q_full, 1);
        ptx::mbar_init(&ms.o_free, kSoftmaxWarps);
        ptx::mbar_init(&ms.drain, 2);       // one commit per MMA issuer
        ptx::mbar_init(&ms.all_sync, kSoftmaxWarps);
        ptx::mbar_init(&ms.p_redo, kSoftmaxWarps);
        ms.redo[0] = ms.redo[1] = 0;
        ms.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && threadIdx.x == 0) {
        ptx::prefetch_tensormap(&map_a);
        if (kFp8) ptx::prefetch_tensormap(&map_b);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&ms.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    if (warp == 0)
        producer<kFp8>(p, &map_a, &map_b, smem, ms, slot);
    else if (warp == 1)
        score_issuer<kFp8>(p, smem, ms, slot);
    else if (warp == kValueWarp)
        value_issuer<kFp8>(p, smem, ms, slot);
    else
        softmax_role<kFp8>(p, smem, ms, slot, g_idx, &map_out, &map_part);

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(ms.tmem_base, kTmemCols);
    }
}

// The driver's tensor-map encoder, looked up once (a function-local static is
// initialised exactly once even when several host threads call at once).
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return nullptr;
    }();
    return fn;
}

// Encoded tensor maps are remembered by everything that defines them (the
// map kind, base address and extents): encoding is host work of a few
// microseconds, and a decode step asks for the same four maps per layer at
// every step.  A map holds no reference to the memory it describes, so an
// entry stays right for any allocation at the same address and extents.
struct MapKey {
    const void *base;
    uint64_t a, b, c;
    int kind;
    bool operator==(const MapKey &o) const {
        return base == o.base && a == o.a && b == o.b && c == o.c && kind == o.kind;
    }
};

template <typename Make>
bool cached_map(const MapKey &k, CUtensorMap *out, Make &&make) {
    constexpr int kEntries = 256;
    struct Entry {
        MapKey key;
        CUtensorMap map;
        bool valid;
    };
    static Entry cache[kEntries];
    static std::mutex mu;
    uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
    h ^= (k.a + 31 * k.b + 961 * k.c + 29791 * (uint64_t)k.kind) * 0xC2B2AE3D27D4EB4Full;
    Entry &e = cache[(h >> 32) % kEntries];
    {
        std::lock_guard<std::mutex> lock(mu);
        if (e.valid && e.key == k) {
            *out = e.map;
            return true;
        }
    }
    if (!make(out)) return false;
    std::lock_guard<std::mutex> lock(mu);
    e.key = k;
    e.map = *out;
    e.valid = true;
    return true;
}

// 2-D view of the page pool: [num_pages*16 rows][576 elements], boxes of 16 rows.
bool make_kv_map(CUtensorMap *map, const void *base, int num_pages, bool fp8, uint32_t box_cols,
                 CUtensorMapSwizzle swz) {
    auto encode = get_encode_fn();
    if (!encode) return false;
    const CUtensorMapDataType dt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)num_pages * kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * (fp8 ? 1 : 2)};
    const cuuint32_t box[2] = {box_cols, (cuuint32_t)kPage};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 5-D view of the FP8 pool's c_kv bytes: {128 bytes of a chunk, 8 rows, 4
// chunks, 2 halves of a page, pages}, one box = one page's 512 latent bytes,
// landing as [half][chunk][8 rows][128 B] (the MMA's swizzled K-major atoms).
bool make_fp8_latent_map(CUtensorMap *map, const void *base, int num_pages) {
    auto encode = get_encode_fn();
    if (!encode) return false;
    const cuuint64_t dims[5] = {128, 8, 4, 2, (cuuint64_t)num_pages};
    const cuuint64_t strides[4] = {(cuuint64_t)kD, 128, (cuuint64_t)8 * kD, (cuuint64_t)kPage * kD};
    const cuuint32_t box[5] = {128, 8, (cuuint32_t)Cfg<true>::kCpp, 2, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output views for the epilogue's tensor stores, boxes of 128 dims x 16 rows
// (one softmax row group): out as [B][R][512] (bf16 or fp32), the partials
// as [R][pieces][512] bf16.
bool make_out_maps(CUtensorMap *mo, CUtensorMap *mp, const Problem &p) {
    auto encode = get_encode_fn();
    if (!encode) return false;
    const cuuint32_t estr[3] = {1, 1, 1};
    const size_t osz = p.out_f32 ? 4 : 2;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)kDl, (cuuint64_t)p.R, (cuuint64_t)p.B};
        const cuuint64_t strides[2] = {(cuuint64_t)kDl * osz, (cuuint64_t)p.R * kDl * osz};
        const cuuint32_t box[3] = {128, (cuuint32_t)kRpt, 1};
        if (encode(mo, p.out_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.out, dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    if (p.max_pieces < 1 || !p.part_o) {  // no partials: never stored through
        *mp = *mo;
        return true;
    }
    const cuuint64_t dims[3] = {(cuuint64_t)kDl, (cuuint64_t)p.max_pieces, (cuuint64_t)p.R};
    const cuuint64_t strides[2] = {(cuuint64_t)kDl * 2, (cuuint64_t)p.max_pieces * kDl * 2};
    const cuuint32_t box[3] = {128, 1, (cuuint32_t)kRpt};
    return encode(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.part_o, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kFp8>
int launch_impl(const Problem &p, cudaStream_t stream) {
    CUtensorMap ma, mb, mo, mp;
    bool ok;
    const uint64_t np = (uint64_t)p.num_pages;
    if (kFp8) {
        ok = cached_map({p.kv, np, 0, 0, 0}, &ma, [&](CUtensorMap *m) { return make_fp8_latent_map(m, p.kv, p.num_pages); }) &&
             cached_map({p.kv, np, 0, 0, 1}, &mb, [&](CUtensorMap *m) {
                 return make_kv_map(m, p.kv, p.num_pages, true, 64, CU_TENSOR_MAP_SWIZZLE_64B);
             });
    } else {
        ok = cached_map({p.kv, np, 0, 0, 2}, &ma, [&](CUtensorMap *m) {
            return make_kv_map(m, p.kv, p.num_pages, false, 64, CU_TENSOR_MAP_SWIZZLE_128B);
        });
        mb = ma;
    }
    // (make_out_maps encodes both output maps; each cached entry keeps one)
    ok = ok && cached_map({p.out, (uint64_t)p.R, (uint64_t)p.B, (uint64_t)p.out_f32, 3}, &mo, [&](CUtensorMap *m) {
             CUtensorMap unused;
             return make_out_maps(m, &unused, p);
         });
    if (ok && (p.max_pieces < 1 || !p.part_o)) {
        mp = mo;  // no partials: never stored through
    } else if (ok) {
        ok = cached_map({p.part_o, (uint64_t)p.max_pieces, (uint64_t)p.R, 0, 4}, &mp, [&](CUtensorMap *m) {
            CUtensorMap unused;
            return make_out_maps(&unused, m, p);
        });
    }
    if (!ok) return MLA_ERR_CUDA;
    const int smem = smem_bytes<kFp8>();
    // the shared-memory attribute is set once per device
    static std::atomic<uint64_t> attr_set{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    const uint64_t bit = dev < 64 ? 1ull << dev : 0;
    if (e == cudaSuccess && (!bit || !(attr_set.load() & bit))) {
        e = cudaFuncSetAttribute(tc_decode_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess && bit) attr_set.fetch_or(bit);
    }
    if (e == cudaSuccess) {
        tc_decode_kernel<kFp8><<<p.n_slots * p.n_groups, kThreads, smem, stream>>>(p, ma, mb, mo, mp);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        note_cuda_error(e);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

static_assert(smem_bytes<true>() <= 232448, "FP8 tile does not fit shared memory");
static_assert(2 * kRowGroups * kRpt * 128 * 4 <= Cfg<true>::kQBytes && 2 * kRowGroups * kRpt * 128 * 4 <= Cfg<false>::kQBytes,
              "each row group's 16 KB of epilogue staging boxes must fit the query area");
static_assert(smem_bytes<false>() <= 232448, "bf16 tile does not fit shared memory");
static_assert(Cfg<true>::kColO + 3 * Cfg<true>::kOStride + Cfg<true>::kNMma <= kTmemCols, "TMEM overflow");
static_assert(Cfg<false>::kColO + 3 * Cfg<false>::kOStride + Cfg<false>::kNMma <= kTmemCols, "TMEM overflow");

}  // namespace

int launch_tc(const Problem &p, cudaStream_t stream) {
    if (p.rows_per_group != kN) return MLA_ERR_INVALID_ARG;
    return p.kv_scale ? launch_impl<true>(p, stream) : launch_impl<false>(p, stream);
}

}  // namespace mla

// prefill_sm100.cu -- exact attention prefill on the sm_100a tensor core.
//
// What it computes: O = softmax(Q K^T * scale + mask) V and the row
// log-sum-exp, for dense batches and packed sequences, with causal and
// sliding-window masks and grouped KV heads ("What attention costs",
// "MQA and GQA", "Sliding windows and local:global layers" in samanvya.dev's
// "Attention Is the Bottleneck").
//
// How (the tiled online softmax of "FlashAttention: same math, different
// IO", arranged for B200):
//   * Persistent grid, one CTA per SM.  A work unit is 256 query rows of one
//     (sequence, query head), split into two 128-row tiles that ping-pong:
//     while the tensor core runs one tile's GEMMs, the other tile's softmax
//     warpgroup works ("FlashAttention-3": warp specialisation, ping-pong).
//     Units run heaviest first (causal: last row blocks first).
//   * Warp 8 issues TMA loads: the two Q tiles once per unit, then K_j, V_j
//     tiles (128 keys x d) into a ring of shared-memory slots, 128-byte
//     swizzled.  Only key blocks that some visible (row, key) pair needs are
//     loaded: causal and window masks skip whole tiles.
//   * Warp 9 (one thread) issues tcgen05 MMAs: S_t = Q_t K_j^T into tensor
//     memory (fp32), then O_t += P_t V_j with P_t read from tensor memory
//     where the softmax left it (bf16, aliasing S_t) -- "FlashAttention-4":
//     tensor memory takes operand traffic off shared memory.
//   * Warps 0-3 / 4-7: one thread per query row.  Each reads its S row from
//     TMEM, applies scale and mask, updates the running max m and sum l,
//     writes P = 2^(s*scale*log2e - m) back as bf16, and signals the MMA
//     warp.  The rescale of O by 2^(m_old - m_new) is skipped unless the max
//     grew by more than 8 (log2 units) in some row of the warp
//     ("FlashAttention-4": conditional rescaling); P is then at most 2^8,
//     and O and l stay consistent because both use the same reference max.
//   * The epilogue divides O by l once ("FlashAttention-2": delayed
//     normalisation) and writes O and LSE = ln2 * (m + log2 l).
#include <climits>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace prefill_impl {

constexpr int kBlockM = 128;        // rows per tile (TMEM lanes)
constexpr int kBlockN = 128;        // keys per K/V tile
constexpr int kHalf = 64;           // P is published to the MMA warp in halves
// 2 softmax warpgroups (one per Q tile, one thread per row) + 1 warpgroup
// for TMA / MMA.
constexpr int kThreads = 384;
constexpr int kSoftmaxWarps = 8;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
// Register split: launched with 384 x 168 = 64,512 registers; the softmax
// warpgroups take 216 each, the TMA/MMA warpgroup 72:
// 2 * 128 * 216 + 128 * 72 = 64,512.
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 216;
constexpr int kRegsControl = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kLaunchRegs,
              "register split");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
#ifndef FA_POLY_PERIOD
#define FA_POLY_PERIOD 8
#endif
// One score pair in kPolyPeriod takes the FMA-pipe exponential (0 = none).
constexpr int kPolyPeriod = FA_POLY_PERIOD;
#ifndef FA_POLY_F8
#define FA_POLY_F8 0
#endif
// FP8 kernel: one group of four scores in kPolyPeriodF8 takes it (0 = none).
constexpr int kPolyPeriodF8 = FA_POLY_F8;
constexpr uint32_t kTmemCols = 512;
constexpr int kPageRows = 16;                 // tokens per cache page (paged mode)
constexpr int kPagesPerTile = 128 / kPageRows;

template <int D, bool DOC = false, bool F8 = false>
struct Cfg {
    static constexpr int kElem = F8 ? 1 : 2;                       // bytes per element
    static constexpr int kBoxCols = 128 / kElem;                   // elements per 128-byte row
    static constexpr int kBoxes = D / kBoxCols;                    // TMA boxes per tile
    static constexpr int kBoxBytes = kBlockM * 128;                // 128 rows x 128 bytes
    static constexpr int kTileBytes = kBlockM * D * kElem;         // Q tile or K/V tile
    // K/V ring slots (one fewer with a document mask, for its key-id buffers;
    // FP8 tiles are half the size)
    static constexpr int kStages = F8 ? 8 : (D == 128) ? (DOC ? 4 : 5) : 6;
    static constexpr int kDocBytes = DOC ? 8 * 2 * 128 * 4 : 0;   // [warp][parity][key]
    static constexpr int kSmemBytes = 2 * kTileBytes + kStages * kTileBytes + kDocBytes + 1024;
    static constexpr uint32_t kColO = 256;                         // O_t at 256 + t*D
};

struct Params {
    void *o;
    float *lse;
    const int *cu_seqlens;
    int num_seqs, seqlen, total_tokens, max_seqlen;
    int Hq, Hkv, group;
    int causal, window;
    float scale_log2;
    int o_fp32;
    const float *sinks;   // [Hq] learned sink logits, or nullptr
    int num_mblocks;   // 256-row blocks per sequence (of max_seqlen)
    int num_units;
    // Chunked prefill over a paged cache: keys of sequence s come from its
    // pages (block_table row s, 16 tokens per page), seq_lens_k[s] of them;
    // its queries are the last L_q tokens (cu_seqlens holds the query packing).
    int paged;
    const int *block_table, *seq_lens_k;
    const uint16_t *v_cache;
    int max_pages, num_pages;
    // Document mask: one id per token (packed order); key j is visible from
    // query i only if both ids are equal.
    const int *doc;
    // FP8 operands (dense batches): E4M3 codes with scales per (sequence,
    // head, 128-token block) for Q and K, per (sequence, KV head) for V.
    const float *q_scale, *k_scale, *v_scale;
    int nblk;   // 128-token blocks per sequence
    // Sink tokens (with causal and a window): keys j < n_sink of a sequence
    // stay visible to every later query; 0 = none.
    int n_sink;
};

struct Unit {
    int seq, h, kvh;
    int tok0;   // packed index of the sequence's first token
    int L;      // sequence length
    int q0;     // first query row of the unit, local to the sequence
    int Lk;     // keys of the sequence (= L except for the paged chunked prefill)
    int off;    // key position of query row 0 (Lk - L)
    int lo[2], hi[2];  // key-block range per tile, [lo, hi)
    int lo_all, hi_all;
    // Sink tokens: tile t also takes key blocks [0, ns[t]) (ns[t] <= lo[t]);
    // the unit walks blocks [0, A) then [lo_all, hi_all), A = the tiles'
    // largest ns capped at lo_all.
    int ns[2], A;
};

template <bool PAGED, bool SINK = false>
__device__ __forceinline__ bool get_unit(int u, const Params &p, Unit &w) {
    int mb;
    if (PAGED) {
        // Chunked prefill: every row block of a chunk reads (nearly) the
        // sequence's whole cached context, which is far larger than the
        // chunk.  Units of one (sequence, KV head) -- all row blocks, all
        // query heads of the group -- are consecutive, so they run on
        // neighbouring CTAs at the same time and each page crosses HBM once
        // (the next KV head's pages follow while these are still in L2).
        const int per_kvh = p.num_mblocks * p.group;
        const int sk = u / per_kvh, r = u % per_kvh;
        w.seq = sk / p.Hkv;
        w.kvh = sk % p.Hkv;
        mb = r / p.group;
        w.h = w.kvh * p.group + r % p.group;
    } else {
        // Heaviest first: the last row blocks of every sequence and head
        // (causal: the most key blocks), then the ones before them.
        const int per_mb = p.num_seqs * p.Hq;
        mb = p.num_mblocks - 1 - u / per_mb;
        const int r = u % per_mb;
        w.seq = r / p.Hq;
        w.h = r % p.Hq;
        w.kvh = w.h / p.group;
    }
    if (p.cu_seqlens) {
        w.tok0 = __ldg(p.cu_seqlens + w.seq);
        w.L = __ldg(p.cu_seqlens + w.seq + 1) - w.tok0;
        // A sequence outside [0, total_tokens) or longer than max_seqlen
        // (offsets not ascending, or a wrong max_seqlen) is skipped by every
        // role alike and reported; nothing is read or written for it.
        if (w.tok0 < 0 || w.L < 0 || w.L > p.max_seqlen || w.tok0 > p.total_tokens - w.L) {
            report_error(kDevErrInput);
            return false;
        }
    } else {
        w.tok0 = w.seq * p.seqlen;
        w.L = p.seqlen;
    }
    w.q0 = mb * 2 * kBlockM;
    if (w.L <= 0 || w.q0 >= w.L) return false;
    w.Lk = w.L;
    w.off = 0;
    if constexpr (PAGED) {
        const int Lk = __ldg(p.seq_lens_k + w.seq);
        if (Lk < w.L || Lk > p.max_pages * kPageRows) {   // unusable lengths: skip, report
            report_error(kDevErrInput);
            return false;
        }
        w.Lk = Lk;
        w.off = Lk - w.L;
    }
    const int nkb = (w.Lk + kBlockN - 1) / kBlockN;
    w.lo_all = 1 << 30;
    w.hi_all = 0;
    for (int t = 0; t < 2; ++t) {
        const int r0 = w.q0 + t * kBlockM;
        if (r0 >= w.L) { w.lo[t] = w.hi[t] = 0; continue; }
        int lo = 0, hi = nkb;
        if (p.causal) {
            const int last = w.off + min(r0 + kBlockM - 1, w.L - 1);
            hi = min(nkb, last / kBlockN + 1);
            if (p.window > 0) lo = max(0, w.off + r0 - p.window + 1) / kBlockN;
        }
        w.lo[t] = lo;
        w.hi[t] = hi;
        w.lo_all = min(w.lo_all, lo);
        w.hi_all = max(w.hi_all, hi);
    }
    w.ns[0] = w.ns[1] = w.A = 0;
    if (SINK && !PAGED && p.n_sink > 0 && p.causal && p.window > 0) {
        const int sb = min((p.n_sink + kBlockN - 1) / kBlockN, nkb);
        w.ns[0] = (w.lo[0] < w.hi[0]) ? min(sb, w.lo[0]) : 0;
        w.ns[1] = (w.lo[1] < w.hi[1]) ? min(sb, w.lo[1]) : 0;
        w.A = min(max(w.ns[0], w.ns[1]), w.lo_all);
    }
    return true;
}

// The unit's key blocks in order: [0, A) (sink blocks), then [lo_all, hi_all).
__device__ __forceinline__ int unit_first(const Unit &w) { return w.A > 0 ? 0 : w.lo_all; }
__device__ __forceinline__ int unit_next(const Unit &w, int j) {
    return (j + 1 == w.A) ? w.lo_all : j + 1;
}

// Unit `it` of this CTA: rows of G = gridDim.x units are walked in
// alternating directions (snake order), so with units sorted by decreasing
// cost every CTA gets a similar total.
__device__ __forceinline__ int sched_unit(int it) {
    const int G = gridDim.x, b = blockIdx.x;
    return (it & 1) ? (it + 1) * G - 1 - b : it * G + b;
}

#define FOR_EACH_UNIT(u)                                                  \
    for (int it_ = 0, u = 0; it_ * (int)gridDim.x < p.num_units; ++it_)   \
        if ((u = sched_unit(it_)) < p.num_units)

struct Shared {
    uint64_t q_full[2], q_empty[2];
    uint64_t kv_full[8], kv_empty[8];
    uint64_t s_full[2], p_lo[2], p_hi[2], o_full[2], o_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// ------------------------------------------------------------- TMA producer
// Dense and packed batches: one thread issues every copy.
// FP8: one 128-byte box per tile row; V comes transposed (d rows of 128
// keys), so its tile is read at (key, 0, sequence * Hkv + KV head).
template <int D, bool DOC, bool F8, bool SINK>
__device__ void producer(const CUtensorMap *tmQ, const CUtensorMap *tmK, const CUtensorMap *tmV,
                         const Params &p, Shared &sh, uint8_t *sQ, uint8_t *sKV) {
    using C = Cfg<D, DOC, F8>;
    volatile int *abort = &sh.abort;
    uint32_t q_uses[2] = {0, 0};
    uint32_t kv_it = 0;
    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit<false, SINK>(u, p, w)) continue;
        for (int t = 0; t < 2; ++t) {
            if (w.lo[t] >= w.hi[t]) continue;
            if (!mbar_wait(&sh.q_empty[t], (q_uses[t] & 1) ^ 1, abort)) goto out;
            mbar_arrive_expect_tx(&sh.q_full[t], C::kTileBytes);
            for (int b = 0; b < C::kBoxes; ++b)
                tma_load_3d(sQ + t * C::kTileBytes + b * C::kBoxBytes, tmQ, &sh.q_full[t],
                            b * C::kBoxCols, w.h, w.tok0 + w.q0 + t * kBlockM);
            ++q_uses[t];
        }
        for (int j = SINK ? unit_first(w) : w.lo_all; j < w.hi_all;
             j = SINK ? unit_next(w, j) : j + 1) {
            for (int kv = 0; kv < 2; ++kv) {
                const int slot = kv_it % C::kStages;
                const uint32_t use = kv_it / C::kStages;
                if (!mbar_wait(&sh.kv_empty[slot], (use & 1) ^ 1, abort)) goto out;
                mbar_arrive_expect_tx(&sh.kv_full[slot], C::kTileBytes);
                if (F8 && kv) {
                    tma_load_3d(sKV + slot * C::kTileBytes, tmV, &sh.kv_full[slot], j * kBlockN,
                                0, w.seq * p.Hkv + w.kvh);
                } else {
                    for (int b = 0; b < C::kBoxes; ++b)
                        tma_load_3d(sKV + slot * C::kTileBytes + b * C::kBoxBytes, kv ? tmV : tmK,
                                    &sh.kv_full[slot], b * C::kBoxCols, w.kvh,
                                    w.tok0 + j * kBlockN);
                }
                ++kv_it;
            }
        }
    }
    return;
out:
    // Leave no copy in flight: wait for the last load issued into each slot.
    for (int s = 0; s < C::kStages; ++s) {
        if (kv_it > (uint32_t)s) {
            const uint32_t last = (kv_it - 1 - s) / C::kStages;
            mbar_drain_wait(&sh.kv_full[s], last & 1);
        }
    }
    for (int t = 0; t < 2; ++t)
        if (q_uses[t]) mbar_drain_wait(&sh.q_full[t], (q_uses[t] - 1) & 1);
}

// Chunked prefill over a paged cache: one warp.  A K or V tile is 8 cache
// pages: lane p (< 8) looks up page p of the tile in
// the block table and copies it (a 16-row box per 64 columns); pages past the
// sequence's keys are read from beyond the cache's extent, which TMA fills with
// zeros.  A page the sequence ends inside is copied for K (its tail keys are
// masked) but for V the whole warp copies its valid rows and writes zeros
// after them, because a masked key still multiplies its V row by P = 0 and
// unused slots may hold NaN.  Every kv_full phase gets two arrivals: one with
// the TMA byte count and one after the warp's own writes.
template <int D>
__device__ void producer_paged(const CUtensorMap *tmQ, const CUtensorMap *tmK, const CUtensorMap *tmV,
                         const Params &p, Shared &sh, uint8_t *sQ, uint8_t *sKV) {
    using C = Cfg<D>;
    volatile int *abort = &sh.abort;
    const int lane = lane_id();
    constexpr int kPageBytes = kPageRows * D * 2;     // one page of one KV head, all boxes
    uint32_t q_uses[2] = {0, 0};
    uint32_t kv_it = 0;
    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit<true>(u, p, w)) continue;
        for (int t = 0; t < 2; ++t) {
            if (w.lo[t] >= w.hi[t]) continue;
            if (!mbar_wait_warp(&sh.q_empty[t], (q_uses[t] & 1) ^ 1, abort)) goto out;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sh.q_full[t], C::kTileBytes);
                for (int b = 0; b < D / 64; ++b)
                    tma_load_3d(sQ + t * C::kTileBytes + b * C::kBoxBytes, tmQ, &sh.q_full[t],
                                b * 64, w.h, w.tok0 + w.q0 + t * kBlockM);
            }
            ++q_uses[t];
        }
        for (int j = w.lo_all; j < w.hi_all; ++j) {
            // paged: lane p < 8 holds page p of this key block (-1: past the keys)
            int page = -1;
            if (lane < kPagesPerTile) {
                const int pidx = j * kPagesPerTile + lane;
                if (pidx * kPageRows < w.Lk) {
                    page = __ldg(p.block_table + (size_t)w.seq * p.max_pages + pidx);
                    if (page < 0 || page >= p.num_pages) {
                        report_error(kDevErrInput);
                        page = 0;
                    }
                }
            }
            const int tail = w.Lk - j * kBlockN;          // valid keys in this tile (paged)
            const int part = (tail > 0 && tail < kBlockN && (tail % kPageRows) != 0)
                                 ? tail / kPageRows : -1;  // page the keys end inside
            for (int kv = 0; kv < 2; ++kv) {
                const int slot = kv_it % C::kStages;
                const uint32_t use = kv_it / C::kStages;
                uint8_t *dst = sKV + slot * C::kTileBytes;
                if (!mbar_wait_warp(&sh.kv_empty[slot], (use & 1) ^ 1, abort)) goto out;
                {
                    const bool manual = kv == 1 && part >= 0;
                    if (lane == 0)
                        mbar_arrive_expect_tx(&sh.kv_full[slot],
                                              C::kTileBytes - (manual ? kPageBytes : 0));
                    __syncwarp();
                    if (lane < kPagesPerTile && !(manual && lane == part)) {
                        const int row = page >= 0 ? page * kPageRows : p.num_pages * kPageRows;
                        for (int b = 0; b < D / 64; ++b)
                            tma_load_3d(dst + b * C::kBoxBytes + lane * kPageRows * 128,
                                        kv ? tmV : tmK, &sh.kv_full[slot], b * 64, w.kvh, row);
                    }
                    if (manual) {
                        // V rows of the page the keys end inside: copy the
                        // valid ones, zero the rest, in the 128-byte-swizzled
                        // layout the TMA boxes use.
                        const int vpage = __shfl_sync(0xffffffffu, page, part);
                        const int valid = tail - part * kPageRows;
                        constexpr int kChunks = kPageRows * (D / 8);   // 16-byte chunks
                        for (int idx = lane; idx < kChunks; idx += 32) {
                            const int srow = idx / (D / 8), rem = idx % (D / 8);
                            const int b = rem >> 3, c = rem & 7;
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);
                            if (srow < valid)
                                v = __ldg(reinterpret_cast<const uint4 *>(
                                    p.v_cache + ((size_t)(vpage * kPageRows + srow) * p.Hkv + w.kvh) * D +
                                    b * 64 + c * 8));
                            const int trow = part * kPageRows + srow;
                            *reinterpret_cast<uint4 *>(dst + b * C::kBoxBytes + trow * 128 +
                                                       ((c ^ (trow & 7)) << 4)) = v;
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.kv_full[slot]);
                }
                ++kv_it;
            }
        }
    }
    return;
out:
    // Leave no copy in flight: wait for the last load issued into each slot.
    if (lane == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            if (kv_it > (uint32_t)s) {
                const uint32_t last = (kv_it - 1 - s) / C::kStages;
                mbar_drain_wait(&sh.kv_full[s], last & 1);
            }
        }
        for (int t = 0; t < 2; ++t)
            if (q_uses[t]) mbar_drain_wait(&sh.q_full[t], (q_uses[t] - 1) & 1);
    }
}

// ------------------------------------------------------------ MMA issuer
template <int D, bool PAGED, bool DOC, bool F8, bool SINK>
__device__ void mma_issuer(const Params &p, Shared &sh, uint8_t *sQ, uint8_t *sKV) {
    using C = Cfg<D, DOC, F8>;
    volatile int *abort = &sh.abort;
    const uint32_t tmem = sh.tmem_base;
    const uint32_t idS = F8 ? idesc_e4m3_f32(kBlockM, kBlockN)
                            : idesc_bf16_f32(kBlockM, kBlockN, false);
    const uint32_t idPV = F8 ? idesc_e4m3_f32(kBlockM, D) : idesc_bf16_f32(kBlockM, D, true);
    const uint32_t q_addr = smem_u32(sQ), kv_addr = smem_u32(sKV);
    uint32_t q_uses[2] = {0, 0}, p_cnt[2] = {0, 0}, oe_uses[2] = {0, 0};
    uint32_t kv_it = 0;

    // S_t = Q_t K^T: d/16 MMAs of K=16; K-major, 128-byte swizzle, atoms of
    // 8 rows x 128 bytes (SBO 1024), 64 columns per TMA box.  Descriptors
    // are precomputed; a k-step adds its byte offset >> 4 to the low half.
    // (FP8: K = 32 per MMA, the same 32 bytes per k-step.)
    const uint32_t q_lo = desc_lo(q_addr, 16), kv_lo = desc_lo(kv_addr, 16);
    const uint32_t v_lo = desc_lo(kv_addr, F8 ? 16 : C::kBoxBytes);
    constexpr uint32_t kTileStep = C::kTileBytes >> 4;
    auto issue_s = [&](int t, int kslot) {
        const uint32_t qa = q_lo + t * kTileStep;
        const uint32_t ka = kv_lo + kslot * kTileStep;
        const uint32_t dt = tmem + t * kBlockN;
        #pragma unroll
        for (int ks = 0; ks < D * C::kElem / 32; ++ks) {
            const uint32_t off = ((ks >> 2) * C::kBoxBytes + (ks & 3) * 32) >> 4;
            if constexpr (F8)
                mma_ss_lo_f8(dt, qa + off, ka + off, idS, ks > 0 ? 1u : 0u);
            else
                mma_ss_lo(dt, qa + off, ka + off, idS, ks > 0 ? 1u : 0u);
        }
    };
    // O_t += P_t V: 128/16 MMAs of K=16 keys; V is MN-major (d contiguous):
    // 16 keys = two 8-row groups (SBO 1024), d split in 64-column boxes (LBO).
    // FP8: V^T is K-major (keys contiguous), 32 keys per MMA; P holds four
    // codes per TMEM column, so 64 keys are 16 columns.
    auto issue_pv_half = [&](int t, int vslot, bool first, int half) {
        const uint32_t va = v_lo + vslot * kTileStep;
        const uint32_t dt = tmem + C::kColO + t * D;
        const uint32_t pa = tmem + t * kBlockN;
        if constexpr (F8) {
            #pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int ks = half * 2 + k;
                mma_ts_lo_f8(dt, pa + ks * 8, va + ((ks * 32) >> 4), idPV,
                             (ks > 0 || !first) ? 1u : 0u);
            }
        } else {
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int ks = half * 4 + k;
                mma_ts_lo(dt, pa + half * kHalf + k * 8, va + ((ks * 2048) >> 4), idPV,
                          (ks > 0 || !first) ? 1u : 0u);
            }
        }
    };
    // P_t V in two halves of 64 keys, each issued as soon as the softmax
    // warpgroup has published that half of P.
    auto issue_pv = [&](int t, int vslot, bool &first) -> bool {
        if (!mbar_wait(&sh.p_lo[t], p_cnt[t] & 1, abort)) return false;
        if (first) {
            if (!mbar_wait(&sh.o_empty[t], (oe_uses[t] & 1) ^ 1, abort)) return false;
            ++oe_uses[t];
        }
        tc_fence_after();
        issue_pv_half(t, vslot, first, 0);
        if (!mbar_wait(&sh.p_hi[t], p_cnt[t] & 1, abort)) return false;
        tc_fence_after();
        issue_pv_half(t, vslot, false, 1);
        ++p_cnt[t];
        first = false;
        tc_commit(&sh.o_full[t]);
        return true;
    };

    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit<PAGED, SINK>(u, p, w)) continue;
        bool first_pv[2] = {true, true};
        for (int t = 0; t < 2; ++t) {
            if (w.lo[t] >= w.hi[t]) continue;
            if (!mbar_wait(&sh.q_full[t], q_uses[t] & 1, abort)) goto out;
            ++q_uses[t];
        }
        tc_fence_after();
        int prev_v = -1;
        bool last1 = false;       // (sink tokens) the previous block was one of tile 1's
        for (int j = SINK ? unit_first(w) : w.lo_all; j < w.hi_all;
             j = SINK ? unit_next(w, j) : j + 1) {
            const bool in0 = (SINK && j < w.ns[0]) || (j >= w.lo[0] && j < w.hi[0]);
            const bool in1 = (SINK && j < w.ns[1]) || (j >= w.lo[1] && j < w.hi[1]);
            const bool prev1 = SINK ? last1 : ((j - 1) >= w.lo[1] && (j - 1) < w.hi[1]);
            const int kslot = kv_it % C::kStages;
            if (!mbar_wait(&sh.kv_full[kslot], (kv_it / C::kStages) & 1, abort)) goto out;
            ++kv_it;
            const int vslot = kv_it % C::kStages;
            const uint32_t vuse = kv_it / C::kStages;
            ++kv_it;
            tc_fence_after();
            if (in0) {
                issue_s(0, kslot);
                tc_commit(&sh.s_full[0]);
            }
            if (prev1) {
                if (!issue_pv(1, prev_v, first_pv[1])) goto out;
                tc_commit(&sh.kv_empty[prev_v]);
            }
            if (in1) {
                issue_s(1, kslot);
                tc_commit(&sh.s_full[1]);
            }
            tc_commit(&sh.kv_empty[kslot]);
            if (in0 && j == w.hi[0] - 1) tc_commit(&sh.q_empty[0]);
            if (in1 && j == w.hi[1] - 1) tc_commit(&sh.q_empty[1]);
            if (!mbar_wait(&sh.kv_full[vslot], vuse & 1, abort)) goto out;
            tc_fence_after();
            if (in0) {
                if (!issue_pv(0, vslot, first_pv[0])) goto out;
            }
            if (!in1) tc_commit(&sh.kv_empty[vslot]);
            prev_v = vslot;
            if (SINK) last1 = in1;
        }
        if (SINK ? last1 : ((w.hi_all - 1) >= w.lo[1] && (w.hi_all - 1) < w.hi[1])) {
            if (!issue_pv(1, prev_v, first_pv[1])) goto out;
            tc_commit(&sh.kv_empty[prev_v]);
        }
    }
out:
    // Wait for every MMA this thread issued before TMEM is released.
    tc_commit(&sh.drain);
    mbar_drain_wait(&sh.drain, 0);
}

// Maximum of 64 scores: eight chains of 3-input max, then a combine.
__device__ __forceinline__ float row_max64(const float (&v)[kHalf]) {
    float mq[8];
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
        float a = fmax3(v[i], v[8 + i], v[16 + i]);
        a = fmax3(a, v[24 + i], v[32 + i]);
        a = fmax3(a, v[40 + i], v[48 + i]);
        mq[i] = fmaxf(a, v[56 + i]);
    }
    return fmax3(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7]));
}

// P = 2^(s*scale*log2e - m) for 64 scores, packed to bf16 pairs, with the
// running fp32 sum.  MUFU ex2 for most pairs, the FMA-pipe polynomial for one
// pair in kPolyPeriod ("software exponentials").
__device__ __forceinline__ void exp_half(const float (&v)[kHalf], float sl2, float mb,
                                         uint32_t (&pk)[kHalf / 2], uint64_t &acc) {
    const uint64_t c2 = f2pack(sl2, sl2), nm2 = f2pack(-mb, -mb);
    uint64_t a2[2] = {acc, f2pack(0.f, 0.f)};
    #pragma unroll
    for (int c = 0; c < kHalf / 2; ++c) {
        const uint64_t x = f2fma(f2pack(v[2 * c], v[2 * c + 1]), c2, nm2);
        float x0, x1, p0, p1;
        f2unpack(x, x0, x1);
        if (kPolyPeriod > 0 && (c % kPolyPeriod) == kPolyPeriod - 1) {
            exp2_poly_pair(x0, x1, p0, p1);
        } else {
            p0 = ex2(x0);
            p1 = ex2(x1);
        }
        a2[c & 1] = f2add(a2[c & 1], f2pack(p0, p1));
        pk[c] = pack_bf16(p0, p1);
    }
    acc = f2add(a2[0], a2[1]);
}

// The same for the FP8 kernel: P as E4M3 codes, four per 32-bit word (P is
// at most 2^8 under the conditional rescale, inside E4M3's range of 448).
// The running sum takes the fp32 values.
__device__ __forceinline__ void exp_half_f8(const float (&v)[kHalf], float sl2, float mb,
                                            uint32_t (&pk)[kHalf / 4], uint64_t &acc) {
    const uint64_t c2 = f2pack(sl2, sl2), nm2 = f2pack(-mb, -mb);
    uint64_t a2[2] = {acc, f2pack(0.f, 0.f)};
    #pragma unroll
    for (int c = 0; c < kHalf / 4; ++c) {
        const uint64_t x = f2fma(f2pack(v[4 * c], v[4 * c + 1]), c2, nm2);
        const uint64_t y = f2fma(f2pack(v[4 * c + 2], v[4 * c + 3]), c2, nm2);
        float x0, x1, y0, y1;
        f2unpack(x, x0, x1);
        f2unpack(y, y0, y1);
        float p0, p1, p2, p3;
        if (kPolyPeriodF8 > 0 && (c % kPolyPeriodF8) == kPolyPeriodF8 - 1) {
            exp2_poly_pair(x0, x1, p0, p1);
            exp2_poly_pair(y0, y1, p2, p3);
        } else {
            p0 = ex2(x0);
            p1 = ex2(x1);
            p2 = ex2(y0);
            p3 = ex2(y1);
        }
        a2[0] = f2add(a2[0], f2pack(p0, p1));
        a2[1] = f2add(a2[1], f2pack(p2, p3));
        pk[c] = pack_e4m3x4(p0, p1, p2, p3);
    }
    acc = f2add(a2[0], a2[1]);
}

// ---------------------------------------------------------------- softmax
template <int D, bool PAGED, bool DOC, bool F8, bool SINK>
__device__ void softmax_wg(const Params &p, Shared &sh, int *kdoc) {
    using C = Cfg<D, DOC, F8>;
    volatile int *abort = &sh.abort;
    const int warp = warp_id(), lane = lane_id();
    const int t = warp >> 2;                 // tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;    // row within the tile
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = sh.tmem_base + lanes + t * kBlockN;
    const uint32_t tO = sh.tmem_base + lanes + C::kColO + t * D;
    uint32_t s_cnt = 0, pv_cnt = 0;

    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit<PAGED, SINK>(u, p, w)) continue;
        // (selects, not w.lo[t]: a run-time index would keep the unit in
        // local memory)
        const int lo = t ? w.lo[1] : w.lo[0], hi = t ? w.hi[1] : w.hi[0];
        const int ns = SINK ? (t ? w.ns[1] : w.ns[0]) : 0;   // sink blocks before lo
        if (lo >= hi) continue;
        const int row = w.q0 + t * kBlockM + r;    // row index within the sequence
        const int rmin = w.q0 + t * kBlockM, rmax = rmin + kBlockM - 1;
        // Document mask: this row's id, and the key ids of the next block
        // (lane l holds keys 4l .. 4l+3), loaded one block ahead; ids past the
        // sequence never match (those keys are masked anyway).
        int mydoc = 0, nd[4] = {0, 0, 0, 0};
        auto load_key_docs = [&](int jb) {
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = jb * kBlockN + 4 * lane + e;
                nd[e] = (jb < hi && k < w.L) ? __ldg(p.doc + w.tok0 + k) : INT_MIN;
            }
        };
        if constexpr (DOC) {
            mydoc = (row < w.L) ? __ldg(p.doc + w.tok0 + row) : INT_MIN + 1;
            load_key_docs(lo);
        }
        // FP8: scores come out in units of q_scale * k_scale; both fold into
        // the exponent's factor, per key block.  V's scale divides O at the end.
        float sq = 1.f, sv = 1.f;
        const float *ksc = nullptr;
        if constexpr (F8) {
            sq = __ldg(p.q_scale + ((size_t)w.seq * p.Hq + w.h) * p.nblk + (w.q0 >> 7) + t);
            sv = __ldg(p.v_scale + (size_t)w.seq * p.Hkv + w.kvh);
            ksc = p.k_scale + ((size_t)w.seq * p.Hkv + w.kvh) * p.nblk;
        }
        float m_ref = -INFINITY, l = 0.f;
        const int j0 = (SINK && ns > 0) ? 0 : lo;
        for (int j = j0; j < hi; j = (SINK && j + 1 == ns) ? lo : j + 1) {
            float sl2 = p.scale_log2;
            if constexpr (F8) sl2 *= sq * __ldg(ksc + j);
            if (!mbar_wait_warp(&sh.s_full[t], s_cnt & 1, abort)) return;
            // the block's key ids, staged per warp (no cross-warp barrier)
            const int *kd = nullptr;
            if constexpr (DOC) {
                int *buf = kdoc + (warp * 2 + (s_cnt & 1)) * kBlockN;
                *reinterpret_cast<int4 *>(buf + 4 * lane) = make_int4(nd[0], nd[1], nd[2], nd[3]);
                __syncwarp();
                kd = buf;
                load_key_docs(j + 1);
            }
            ++s_cnt;
            tc_fence_after();
            const bool first = (j == j0);
            const int k0 = j * kBlockN;
            // keys of the sequence and the key position of query row 0:
            // L and 0 for dense and packed batches
            const int Lk = PAGED ? w.Lk : w.L;
            const int off = PAGED ? w.off : 0;
            const bool edge = (k0 + kBlockN > Lk) ||
                              (p.causal && k0 + kBlockN - 1 > off + rmin) ||
                              (p.window > 0 && k0 <= off + rmax - p.window);
            // visible keys of this row in the tile: c in [c_lo, c_hi); the
            // row's key position is off + row
            const int pos = off + row;
            int c_hi = Lk - k0;
            if (p.causal) c_hi = min(c_hi, pos + 1 - k0);
            const int c_lo = (p.window > 0) ? pos - p.window + 1 - k0 : 0;
            const int c_sink = SINK ? p.n_sink - k0 : INT_MIN;   // keys c < c_sink: sink tokens
            // Scores in two halves of 64 keys: the second half's TMEM load is
            // in flight while the first half is masked and reduced.
            float sA[kHalf], sB[kHalf];
            {
                uint32_t raw[kHalf];
                tmem_ld32(tS + 0, raw);
                tmem_ld32(tS + 32, raw + 32);
                tmem_wait_ld();
                #pragma unroll
                for (int c = 0; c < kHalf; ++c) sA[c] = __uint_as_float(raw[c]);
            }
            uint32_t rawB[kHalf];
            tmem_ld32(tS + 64, rawB);
            tmem_ld32(tS + 96, rawB + 32);
            if (DOC || edge) {
                #pragma unroll
                for (int c = 0; c < kHalf; ++c)
                    if (c >= c_hi || (c < c_lo && c >= c_sink) || (DOC && kd[c] != mydoc))
                        sA[c] = -INFINITY;
            }
            const float mA = row_max64(sA);
            // With the reference max unchanged (the common case under the
            // conditional rescale) the first half's P needs no block max:
            // start its exponentials while the block max is still unknown.
            float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
            uint32_t pkA[F8 ? kHalf / 4 : kHalf / 2];
            uint64_t accA = f2pack(0.f, 0.f);
            auto exp_any = [&](const float (&v)[kHalf], uint32_t (&pk)[F8 ? kHalf / 4 : kHalf / 2],
                               uint64_t &acc) {
                if constexpr (F8)
                    exp_half_f8(v, sl2, mb, pk, acc);
                else
                    exp_half(v, sl2, mb, pk, acc);
            };
            if (!first) exp_any(sA, pkA, accA);
            tmem_wait_ld();
            #pragma unroll
            for (int c = 0; c < kHalf; ++c) sB[c] = __uint_as_float(rawB[c]);
            if (DOC || edge) {
                #pragma unroll
                for (int c = 0; c < kHalf; ++c)
                    if (c + kHalf >= c_hi || (c + kHalf < c_lo && c + kHalf >= c_sink) ||
                        (DOC && kd[c + kHalf] != mydoc))
                        sB[c] = -INFINITY;
            }
            const float m_blk = fmaxf(mA, row_max64(sB)) * sl2;
            bool redo = first;
            if (first) {
                m_ref = m_blk;
            } else {
                const bool need = m_blk > m_ref + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    const float m_new = fmaxf(m_ref, m_blk);
                    const float alpha = (m_new == -INFINITY) ? 1.f : ex2(m_ref - m_new);
                    // O_t holds P V of the previous block only once that MMA is done.
                    if (!mbar_wait_warp(&sh.o_full[t], (pv_cnt - 1) & 1, abort)) return;
                    tc_fence_after();
                    // 16 columns at a time: the row's scores stay live
                    #pragma unroll 1
                    for (int c = 0; c < D; c += 16) {
                        uint32_t ov[16];
                        tmem_ld16(tO + c, ov);
                        tmem_wait_ld();
                        #pragma unroll
                        for (int e = 0; e < 16; ++e)
                            ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st16(tO + c, ov);
                    }
                    tmem_wait_st();
                    l *= alpha;
                    m_ref = m_new;
                    redo = true;
                }
            }
            if (redo) {
                mb = (m_ref == -INFINITY) ? 0.f : m_ref;
                accA = f2pack(0.f, 0.f);
                exp_any(sA, pkA, accA);
            }
            // publish P for keys 0-63 (bf16 pairs in S columns 0-31; FP8:
            // codes in columns 0-15): the MMA warp starts that half of P V
            if constexpr (F8)
                tmem_st16(tS + 0, pkA);
            else
                tmem_st32(tS + 0, pkA);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_lo[t]);
            // keys 64-127 (S columns 64-95; FP8: 16-31)
            uint32_t pkB[F8 ? kHalf / 4 : kHalf / 2];
            uint64_t accB = f2pack(0.f, 0.f);
            exp_any(sB, pkB, accB);
            if constexpr (F8)
                tmem_st16(tS + kHalf / 4, pkB);
            else
                tmem_st32(tS + kHalf, pkB);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_hi[t]);
            {
                float a0, a1, b0, b1;
                f2unpack(accA, a0, a1);
                f2unpack(accB, b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            ++pv_cnt;
        }
        // ---- epilogue: O / l, LSE
        float inv_scale_o = 1.f;
        if (!mbar_wait_warp(&sh.o_full[t], (pv_cnt - 1) & 1, abort)) return;
        tc_fence_after();
        const bool valid = row < w.L;
        if (p.sinks) {
            // Learned sink: one more denominator term 2^(z*log2e - m) of a
            // key whose value is zero; the reference max takes it in too.
            const float z2 = __ldg(p.sinks + w.h) * 1.4426950408889634f;
            const float m_new = fmaxf(m_ref, z2);
            if (m_new != -INFINITY) {
                const float a = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
                l = l * a + ex2(z2 - m_new);
                inv_scale_o = a;
                m_ref = m_new;
            }
        }
        const float inv_l = (l > 0.f) ? inv_scale_o * sv / l : 0.f;
        const size_t orow = ((size_t)(w.tok0 + row) * p.Hq + w.h) * D;
        #pragma unroll
        for (int c = 0; c < D; c += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + c, ov);
            tmem_wait_ld();
            if (valid) {
                if (p.o_fp32) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow + c);
                    #pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l,
                                             __uint_as_float(ov[4 * e + 1]) * inv_l,
                                             __uint_as_float(ov[4 * e + 2]) * inv_l,
                                             __uint_as_float(ov[4 * e + 3]) * inv_l);
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) + orow + c);
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(ov[8 * e + 0]) * inv_l, __uint_as_float(ov[8 * e + 1]) * inv_l);
                        v.y = pack_bf16(__uint_as_float(ov[8 * e + 2]) * inv_l, __uint_as_float(ov[8 * e + 3]) * inv_l);
                        v.z = pack_bf16(__uint_as_float(ov[8 * e + 4]) * inv_l, __uint_as_float(ov[8 * e + 5]) * inv_l);
                        v.w = pack_bf16(__uint_as_float(ov[8 * e + 6]) * inv_l, __uint_as_float(ov[8 * e + 7]) * inv_l);
                        dst[e] = v;
                    }
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.o_empty[t]);
        if (valid && p.lse) {
            const float lse2 = (l > 0.f) ? m_ref + __log2f(l) : -INFINITY;
            size_t idx;
            if (p.cu_seqlens)
                idx = (size_t)w.h * p.total_tokens + w.tok0 + row;
            else
                idx = ((size_t)w.seq * p.Hq + w.h) * p.seqlen + row;
            p.lse[idx] = lse2 * 0.69314718055994531f;
        }
    }
}

template <int D, bool PAGED, bool DOC, bool F8, bool SINK = false>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const Params p) {
    static_assert(!F8 || (D == 128 && !PAGED && !DOC), "FP8: dense batches, d = 128");
    static_assert(!SINK || (!PAGED && !DOC && !F8), "sink tokens: bf16 dense and packed batches");
    using C = Cfg<D, DOC, F8>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Shared sh;
    const uint32_t base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (base & 1023)) & 1023);
    uint8_t *sQ = smem;
    uint8_t *sKV = smem + 2 * C::kTileBytes;
    const int warp = warp_id();

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&sh.q_full[t], 1);
            mbar_init(&sh.q_empty[t], 1);
            mbar_init(&sh.s_full[t], 1);
            mbar_init(&sh.p_lo[t], 4);
            mbar_init(&sh.p_hi[t], 4);
            mbar_init(&sh.o_full[t], 1);
            mbar_init(&sh.o_empty[t], 4);
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&sh.kv_full[s], PAGED ? 2 : 1);
            mbar_init(&sh.kv_empty[s], 1);
        }
        mbar_init(&sh.drain, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) tmem_alloc(&sh.tmem_base, kTmemCols);
    if (warp == kWarpTma && lane_id() == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp < kSoftmaxWarps) {
        regs_increase<kRegsSoftmax>();
        softmax_wg<D, PAGED, DOC, F8, SINK>(p, sh,
                                      reinterpret_cast<int *>(sKV + C::kStages * C::kTileBytes));
    } else {
        regs_decrease<kRegsControl>();
        if (warp == kWarpTma) {
            if constexpr (PAGED)
                producer_paged<D>(&tmQ, &tmK, &tmV, p, sh, sQ, sKV);
            else if (lane_id() == 0)
                producer<D, DOC, F8, SINK>(&tmQ, &tmK, &tmV, p, sh, sQ, sKV);
        } else if (warp == kWarpMma) {
            if (lane_id() == 0) mma_issuer<D, PAGED, DOC, F8, SINK>(p, sh, sQ, sKV);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(sh.tmem_base, kTmemCols);
    }
}

// Shared memory per CTA: static (barriers, exchange buffers) + dynamic
// (Q tiles, K/V ring, 1 KiB alignment slack) within the 227 KiB opt-in limit.
static_assert(Cfg<128>::kSmemBytes + sizeof(Shared) <= 232448, "shared memory");
static_assert(Cfg<64>::kSmemBytes + sizeof(Shared) <= 232448, "shared memory");
static_assert(Cfg<128, true>::kSmemBytes + sizeof(Shared) <= 232448, "shared memory");
static_assert(Cfg<64, true>::kSmemBytes + sizeof(Shared) <= 232448, "shared memory");
static_assert(Cfg<128, false, true>::kSmemBytes + sizeof(Shared) <= 232448, "shared memory");

template <int D, bool PAGED, bool DOC, bool F8 = false, bool SINK = false>
int launch_kernel(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                  const Params &p, long long units, cudaStream_t stream) {
    using C = Cfg<D, DOC, F8>;
    // Setting the attribute is idempotent and cheap; do it on every call so
    // that any device the caller switches to is covered.
    if (cudaFuncSetAttribute(prefill_kernel<D, PAGED, DOC, F8, SINK>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
        return -5;
    const int grid = (int)(units < device_sm_count() ? units : device_sm_count());
    prefill_kernel<D, PAGED, DOC, F8, SINK><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

Params make_params(const PrefillArgs &a) {
    Params p{};
    p.o = a.o;
    p.lse = a.lse;
    p.cu_seqlens = a.cu_seqlens;
    p.num_seqs = a.num_seqs;
    p.seqlen = a.seqlen;
    p.total_tokens = a.total_tokens;
    p.max_seqlen = a.max_seqlen;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.group = a.Hq / a.Hkv;
    p.causal = a.causal;
    p.window = a.causal ? a.window : 0;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.o_fp32 = a.o_fp32;
    p.sinks = a.sinks;
    p.paged = a.paged;
    p.doc = a.doc;
    p.block_table = a.block_table;
    p.seq_lens_k = a.seq_lens_k;
    p.v_cache = static_cast<const uint16_t *>(a.v);
    p.max_pages = a.max_pages;
    p.num_pages = a.num_pages;
    p.num_mblocks = (a.max_seqlen + 2 * kBlockM - 1) / (2 * kBlockM);
    p.n_sink = a.n_sink;
    return p;
}

template <int D>
int launch_d(const PrefillArgs &a, cudaStream_t stream) {
    alignas(64) CUtensorMap tq, tk, tv;
    const uint64_t T = (uint64_t)a.total_tokens;
    // K/V: the packed tokens (dense, varlen), or the cache's num_pages * 16
    // rows read one 16-row page box at a time (paged)
    const uint64_t TK = a.paged ? (uint64_t)a.num_pages * kPageRows : T;
    const uint32_t kv_box = a.paged ? kPageRows : kBlockN;
    if (encode_tensor_map_3d(&tq, a.q, 2, D, a.Hq, T, (uint64_t)D * 2, (uint64_t)a.Hq * D * 2,
                             64, 1, kBlockM, 128) ||
        encode_tensor_map_3d(&tk, a.k, 2, D, a.Hkv, TK, (uint64_t)D * 2, (uint64_t)a.Hkv * D * 2,
                             64, 1, kv_box, 128) ||
        encode_tensor_map_3d(&tv, a.v, 2, D, a.Hkv, TK, (uint64_t)D * 2, (uint64_t)a.Hkv * D * 2,
                             64, 1, kv_box, 128))
        return -5;
    Params p = make_params(a);
    const long long units = (long long)p.num_mblocks * a.num_seqs * a.Hq;
    if (units <= 0) return 0;
    if (units > (1ll << 30)) return -2;
    p.num_units = (int)units;
    if (a.paged) return launch_kernel<D, true, false>(tq, tk, tv, p, units, stream);
    if (a.doc) return launch_kernel<D, false, true>(tq, tk, tv, p, units, stream);
    if (a.n_sink > 0 && a.causal && a.window > 0)
        return launch_kernel<D, false, false, false, true>(tq, tk, tv, p, units, stream);
    return launch_kernel<D, false, false>(tq, tk, tv, p, units, stream);
}

// FP8 operands, dense batches, d = 128: Q and K codes [B*N, H, 128] read in
// one 128-byte box per row; V^T codes [B, Hkv, 128, vt_stride] read as boxes
// of 128 keys x 128 rows of d.  Keys past N (the last block's tail) lie past
// the tensor's extent and arrive as zeros.
int launch_fp8(const PrefillArgs &a, cudaStream_t stream) {
    constexpr int D = 128;
    if (a.d != D || a.cu_seqlens || a.paged || a.doc || a.sinks) return -2;
    alignas(64) CUtensorMap tq, tk, tv;
    const uint64_t T = (uint64_t)a.total_tokens;
    if (encode_tensor_map_3d(&tq, a.q, 1, D, a.Hq, T, D, (uint64_t)a.Hq * D, 128, 1, kBlockM,
                             128) ||
        encode_tensor_map_3d(&tk, a.k, 1, D, a.Hkv, T, D, (uint64_t)a.Hkv * D, 128, 1, kBlockN,
                             128) ||
        encode_tensor_map_3d(&tv, a.v, 1, (uint64_t)a.seqlen, D, (uint64_t)a.num_seqs * a.Hkv,
                             (uint64_t)a.vt_stride, (uint64_t)D * a.vt_stride, kBlockN, D, 1, 128))
        return -5;
    Params p = make_params(a);
    p.q_scale = a.q_scale;
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.nblk = (a.seqlen + kBlockN - 1) / kBlockN;
    const long long units = (long long)p.num_mblocks * a.num_seqs * a.Hq;
    if (units <= 0) return 0;
    if (units > (1ll << 30)) return -2;
    p.num_units = (int)units;
    return launch_kernel<D, false, false, true>(tq, tk, tv, p, units, stream);
}

}  // namespace prefill_impl

int launch_prefill(const PrefillArgs &a, cudaStream_t stream) {
    if (a.d == 128) return prefill_impl::launch_d<128>(a, stream);
    if (a.d == 64) return prefill_impl::launch_d<64>(a, stream);
    return -2;
}

int launch_prefill_fp8(const PrefillArgs &a, cudaStream_t stream) {
    return prefill_impl::launch_fp8(a, stream);
}

}  // namespace fa

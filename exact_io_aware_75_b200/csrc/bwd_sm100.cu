// bwd_sm100.cu -- exact attention backward (dQ, dK, dV) on the sm_100a tensor
// core.
//
// What it computes: for O = softmax(Q K^T * scale + mask) V and an upstream
// gradient dO, the gradients of sum(dO * O) with respect to Q, K and V.  The
// attention matrix is never stored: it is recomputed from Q, K and the row
// log-sum-exp the forward saved ("FlashAttention: same math, different IO" in
// samanvya.dev's "Attention Is the Bottleneck": the backward rebuilds the
// matrix instead of keeping it, trading FLOPs for memory traffic).  With
// D_i = dO_i . O_i, for each visible (query i, key j):
//     P_ij  = 2^(S_ij * scale * log2e - LSE_i * log2e)
//     dS_ij = P_ij (dO_i . V_j - D_i)
//     dV_j += P_ij dO_i,   dK_j += scale dS_ij Q_i,   dQ_i += scale dS_ij K_j
// and grouped query heads add into their shared KV head's dK, dV.
//
// How (B200 design):
//   * bwd_prep_kernel: D = rowsum(O * dO) per (token, head), and zeroes the
//     fp32 dQ accumulator.
//   * bwd_kernel, persistent, one CTA per SM.  A work unit is one KV head's
//     block of 128 keys; K_j and V_j stay in shared memory while the unit walks
//     every (query head of the group, 64-row query tile) that sees the block.
//     dK_j and dV_j accumulate in tensor memory for the whole unit, so the GQA
//     sum over query heads costs nothing and each unit writes its rows once.
//   * Per tile, five tcgen05 GEMMs, all with the 128 keys on the TMEM lanes:
//       S^T  = K_j Q_t^T        (128 x 64, K = d)
//       dP^T = V_j dO_t^T       (128 x 64, K = d)
//       dV  += P^T dO_t         (128 x d,  K = 64; P^T read from TMEM)
//       dK  += dS^T Q_t         (128 x d,  K = 64; dS^T from shared memory)
//       dQ^T = K_j^T dS^T       (d x 64,   K = 128; lands on dP^T's columns)
//     S^T and dP^T are double-buffered in TMEM (2 x 2 x 64 columns) and dK, dV
//     take 2 x 128: the 512 columns of the SM.  Two softmax warpgroups take
//     alternate tiles, so one tile's elementwise work overlaps the next tile's
//     GEMMs.
//   * Warps 8-11 drain dQ^T from TMEM, stage it transposed in shared memory
//     and add it into the fp32 accumulator with TMA reduce-adds (the adds
//     happen in L2, 16 KB per operation); bwd_convert_kernel rounds the
//     accumulator to bf16 at the end.
//   * Warp 12 loads K_j, V_j once per unit and Q_t, dO_t per tile by TMA into
//     a 3-slot ring, with the tile's LSE (in log2 units) and D beside them.
//     Two threads issue the MMAs: warp 13 S^T and dP^T (and owns the TMEM
//     allocation), warp 14 the three gradient GEMMs, so that a tile's S^T
//     never waits behind the previous tile's gradients (which wait for that
//     tile's softmax) and the two issue streams overlap.
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace bwd_impl {

constexpr int kD = 128;          // tile width in d; a head dim of 64 is zero-padded to it
constexpr int kBlockK = 128;   // keys per unit
constexpr int kBlockQ = 64;    // queries per tile
constexpr int kPartQ = 16;     // queries per step of the elementwise pass
constexpr int kThreads = 512;
constexpr int kWarpDrain = 8;  // warps 8..11
constexpr int kWarpTma = 12;
constexpr int kWarpMma = 13;       // S^T, dP^T; TMEM allocation
constexpr int kWarpMmaGrad = 14;   // dV, dK, dQ^T
constexpr int kStages = 3;
// Register split (launched with 512 x 128 = 65,536): the two elementwise
// warpgroups hold two 16-column steps of Sᵀ and dPᵀ at a time (one being
// computed, the next in flight from TMEM).
constexpr int kRegsSoftmax = 176;
constexpr int kRegsDrain = 88;
constexpr int kRegsControl = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsDrain + 128 * kRegsControl <= kThreads * 128,
              "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // S^T of buffer b at b * 64 (P^T overwrites its first 32)
constexpr uint32_t kColDP = 128;  // dP^T of buffer b at 128 + b * 64, then the tile's dQ^T
constexpr uint32_t kColDV = 256;
constexpr uint32_t kColDK = 384;

constexpr int kKVBox = kBlockK * 64 * 2;         // 128 rows x 64 bf16 (16 KB)
constexpr int kKVTile = kBlockK * kD * 2;        // 32 KB
constexpr int kQBox = kBlockQ * 64 * 2;          // 64 rows x 64 bf16 (8 KB)
constexpr int kQTile = kBlockQ * kD * 2;         // 16 KB
constexpr int kDSBytes = kBlockK * kBlockQ * 2;  // 16 KB
constexpr int kOffK = 0;
constexpr int kOffV = kKVTile;
constexpr int kOffStage = 2 * kKVTile;           // stage s: Q_t then dO_t
constexpr int kStageBytes = 2 * kQTile;
constexpr int kOffDS = kOffStage + kStages * kStageBytes;
constexpr int kDQHalf = 32;                      // dQ rows per reduce-add
constexpr int kDQBytes = kDQHalf * kD * 4;       // 16 KB staging buffer
constexpr int kOffDQ = kOffDS + 2 * kDSBytes;    // two staging buffers
constexpr int kOffRows = kOffDQ + 2 * kDQBytes;  // stage s: lse2[64], D[64] (fp32)
constexpr int kSmemBytes = kOffRows + kStages * 2 * kBlockQ * 4 + 1024;
static_assert(kSmemBytes + 256 <= 232448, "shared memory");
constexpr int kBarDrain = 1;                     // named barrier of the dQ warps

struct Params {
    const float *lse;   // saved row log-sum-exp (natural log)
    const float *dd;    // D = rowsum(O * dO), same layout as lse
    float *dq_acc;      // [total, Hq, d] fp32
    void *dk, *dv;      // [total, Hkv, d] bf16
    const int *cu_seqlens;
    int num_seqs, seqlen, total_tokens, max_seqlen;
    int Hq, Hkv, group;
    int causal, window;
    float scale, scale_log2;
    int num_kblocks, num_units;
};

struct Unit {
    int seq, kvh, tok0, L;
    int j0, jl;        // first and last key of the block (local to the sequence)
    int t_lo, nt;      // query tiles [t_lo, t_lo + nt) of each query head
    int ntiles;        // group * nt
};

__device__ __forceinline__ bool get_unit(int u, const Params &p, Unit &w) {
    const int per = p.num_seqs * p.Hkv;
    const int jb = u / per;           // causal: low key blocks are the heaviest
    const int r = u % per;
    w.seq = r / p.Hkv;
    w.kvh = r % p.Hkv;
    if (p.cu_seqlens) {
        w.tok0 = __ldg(p.cu_seqlens + w.seq);
        w.L = __ldg(p.cu_seqlens + w.seq + 1) - w.tok0;
        // A sequence outside [0, total_tokens) or longer than max_seqlen is
        // skipped by every role alike and reported.
        if (w.tok0 < 0 || w.L < 0 || w.L > p.max_seqlen || w.tok0 > p.total_tokens - w.L) {
            report_error(kDevErrInput);
            return false;
        }
    } else {
        w.tok0 = w.seq * p.seqlen;
        w.L = p.seqlen;
    }
    w.j0 = jb * kBlockK;
    if (w.L <= 0 || w.j0 >= w.L) return false;
    w.jl = min(w.L, w.j0 + kBlockK) - 1;
    const int nq = (w.L + kBlockQ - 1) / kBlockQ;
    int lo = 0, hi = nq;
    if (p.causal) {
        lo = w.j0 / kBlockQ;                        // queries i >= j0
        if (p.window > 0) hi = min(nq, (w.jl + p.window - 1) / kBlockQ + 1);  // i < jl + W
    }
    w.t_lo = lo;
    w.nt = hi - lo;
    w.ntiles = p.group * w.nt;
    return w.nt > 0;
}

__device__ __forceinline__ void tile_of(const Unit &w, const Params &p, int k, int &h, int &q0) {
    h = w.kvh * p.group + k / w.nt;
    q0 = (w.t_lo + k % w.nt) * kBlockQ;
}

__device__ __forceinline__ size_t row_index(const Params &p, const Unit &w, int h, int i) {
    return p.cu_seqlens ? (size_t)h * p.total_tokens + w.tok0 + i
                        : ((size_t)w.seq * p.Hq + h) * p.seqlen + i;
}

__device__ __forceinline__ int sched_unit(int it) {
    const int G = gridDim.x, b = blockIdx.x;
    return (it & 1) ? (it + 1) * G - 1 - b : it * G + b;
}

#define FOR_EACH_UNIT(u)                                                  \
    for (int it_ = 0, u = 0; it_ * (int)gridDim.x < p.num_units; ++it_)   \
        if ((u = sched_unit(it_)) < p.num_units)

struct Shared {
    uint64_t kv_full, kv_empty;
    uint64_t qd_full[kStages], qd_empty[kStages];
    uint64_t s_full[2], p_full[2], dq_full[2], dq_free[2];
    uint64_t pt_free[2];     // dV of the buffer's tile done: Sᵀ's columns are free
    uint64_t ds_free[2];     // dK of the buffer's tile done: its dSᵀ buffer is free
    uint64_t acc_full, acc_free;
    uint64_t drain[2];
    uint32_t tmem_base;
    int abort;
};

// ------------------------------------------------------------- TMA producer
__device__ void producer(const CUtensorMap *tmQ, const CUtensorMap *tmK, const CUtensorMap *tmV,
                         const CUtensorMap *tmdO, const Params &p, Shared &sh, uint8_t *smem) {
    volatile int *abort = &sh.abort;
    const int lane = lane_id();
    float *rows = reinterpret_cast<float *>(smem + kOffRows);
    uint32_t uc = 0, n = 0;
    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit(u, p, w)) continue;
        if (!mbar_wait_warp(&sh.kv_empty, (uc & 1) ^ 1, abort)) goto out;
        if (lane == 0) {
            mbar_arrive_expect_tx(&sh.kv_full, 2 * kKVTile);
            for (int b = 0; b < kD / 64; ++b) {
                tma_load_3d(smem + kOffK + b * kKVBox, tmK, &sh.kv_full, b * 64, w.kvh, w.tok0 + w.j0);
                tma_load_3d(smem + kOffV + b * kKVBox, tmV, &sh.kv_full, b * 64, w.kvh, w.tok0 + w.j0);
            }
        }
        ++uc;
        for (int k = 0; k < w.ntiles; ++k, ++n) {
            const int s = n % kStages;
            if (!mbar_wait_warp(&sh.qd_empty[s], ((n / kStages) & 1) ^ 1, abort)) goto out;
            int h, q0;
            tile_of(w, p, k, h, q0);
            if (lane == 0) {
                uint8_t *st = smem + kOffStage + s * kStageBytes;
                mbar_arrive_expect_tx(&sh.qd_full[s], 2 * kQTile);
                for (int b = 0; b < kD / 64; ++b) {
                    tma_load_3d(st + b * kQBox, tmQ, &sh.qd_full[s], b * 64, h, w.tok0 + q0);
                    tma_load_3d(st + kQTile + b * kQBox, tmdO, &sh.qd_full[s], b * 64, h, w.tok0 + q0);
                }
            }
            // The tile's -LSE (log2 units) and -D; rows past the sequence get
            // LSE = +inf, so their P is exactly 0.
            float *rs = rows + s * 2 * kBlockQ;
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int rr = lane + 32 * e, i = q0 + rr;
                float l2 = INFINITY, dv = 0.f;
                if (i < w.L) {
                    const size_t idx = row_index(p, w, h, i);
                    l2 = __ldg(p.lse + idx) * 1.4426950408889634f;
                    dv = __ldg(p.dd + idx);
                }
                rs[rr] = -l2;
                rs[kBlockQ + rr] = -dv;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.qd_full[s]);
        }
    }
    return;
out:
    if (lane == 0) {
        if (uc) mbar_drain_wait(&sh.kv_full, (uc - 1) & 1);
        for (int s = 0; s < kStages; ++s)
            if (n > (uint32_t)s) mbar_drain_wait(&sh.qd_full[s], ((n - 1 - s) / kStages) & 1);
    }
}

// ----------------------------------------------------------- MMA issuers
// S^T(b) = K Q^T and dP^T(b) = V dO^T: K-major operands, d/16 steps; a step
// moves 32 bytes inside a 64-column box, 4 steps cross to the next box.  S^T
// of tile n overwrites the P^T that dV of tile n-2 reads, so it waits for
// that MMA to complete; dP^T overwrites the dQ^T of tile n-2, so it waits
// until that is drained.
__device__ void mma_issuer_s(const Params &p, Shared &sh, uint8_t *smem) {
    volatile int *abort = &sh.abort;
    const uint32_t tmem = sh.tmem_base;
    const uint32_t idS = idesc_bf16_f32_ab(kBlockK, kBlockQ, false, false);
    const uint32_t kLo = desc_lo(smem_u32(smem + kOffK), 16);
    const uint32_t vLo = desc_lo(smem_u32(smem + kOffV), 16);
    const uint32_t aStage = smem_u32(smem + kOffStage);
    uint32_t uc = 0, n = 0;
    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit(u, p, w)) continue;
        if (!mbar_wait(&sh.kv_full, uc & 1, abort)) goto out;
        ++uc;
        for (int k = 0; k < w.ntiles; ++k, ++n) {
            const int b = n & 1, s = n % kStages;
            if (!mbar_wait(&sh.qd_full[s], (n / kStages) & 1, abort)) goto out;
            if (n >= 2 && !mbar_wait(&sh.pt_free[b], ((n - 2) >> 1) & 1, abort)) goto out;
            tc_fence_after();
            const uint32_t qLo = desc_lo(aStage + s * kStageBytes, 16);
            const uint32_t dLo = qLo + (kQTile >> 4);
            #pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                const uint32_t okv = ((ks >> 2) * kKVBox + (ks & 3) * 32) >> 4;
                const uint32_t oq = ((ks >> 2) * kQBox + (ks & 3) * 32) >> 4;
                mma_ss_lo(tmem + kColS + b * kBlockQ, kLo + okv, qLo + oq, idS, ks > 0);
            }
            if (n >= 2 && !mbar_wait(&sh.dq_free[b], ((n - 2) >> 1) & 1, abort)) goto out;
            tc_fence_after();
            #pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                const uint32_t okv = ((ks >> 2) * kKVBox + (ks & 3) * 32) >> 4;
                const uint32_t oq = ((ks >> 2) * kQBox + (ks & 3) * 32) >> 4;
                mma_ss_lo(tmem + kColDP + b * kBlockQ, vLo + okv, dLo + oq, idS, ks > 0);
            }
            tc_commit(&sh.s_full[b]);
        }
        tc_commit(&sh.kv_empty);      // K_j, V_j read by this thread's MMAs
    }
out:
    tc_commit(&sh.drain[0]);
    mbar_drain_wait(&sh.drain[0], 0);
}

// dQ^T = K^T dS^T (K = 128 keys), then dV += P^T dO and dK += dS^T Q (K = 64
// queries), once the tile's softmax has published P^T (TMEM) and dS^T (shared
// memory).  dQ^T goes first so its drain, which the next dP^T on these
// columns waits for, starts early; each step is committed on its own
// barrier: dQ^T (drain may read), dV (S^T's columns free), dK (dS^T and the
// Q/dO slot free).  dO and Q are MN-major B operands (d contiguous; 16 query rows
// per step, boxes of 64 columns LBO apart); dS^T sits in shared memory as 128
// key rows of 64 queries, 128-byte swizzled: K-major A for dK, MN-major B
// for dQ^T.
__device__ void mma_issuer_grad(const Params &p, Shared &sh, uint8_t *smem) {
    volatile int *abort = &sh.abort;
    const uint32_t tmem = sh.tmem_base;
    const uint32_t idAcc = idesc_bf16_f32_ab(kBlockK, kD, false, true);
    const uint32_t idDQ = idesc_bf16_f32_ab(kD, kBlockQ, true, true);
    const uint32_t kLoMN = desc_lo(smem_u32(smem + kOffK), kKVBox);
    const uint32_t aStage = smem_u32(smem + kOffStage), aDS = smem_u32(smem + kOffDS);
    uint32_t uc = 0, m = 0;
    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit(u, p, w)) continue;
        if (!mbar_wait(&sh.kv_full, uc & 1, abort)) goto out;
        ++uc;
        for (int k = 0; k < w.ntiles; ++k, ++m) {
            const bool first = k == 0;
            const int b = m & 1, s = m % kStages;
            if (!mbar_wait(&sh.p_full[b], (m >> 1) & 1, abort)) goto out;
            if (first && uc > 1 && !mbar_wait(&sh.acc_free, (uc - 2) & 1, abort)) goto out;
            tc_fence_after();
            const uint32_t q = aStage + s * kStageBytes, dO = q + kQTile;
            const uint32_t ds = aDS + b * kDSBytes;
            const uint32_t qLoMN = desc_lo(q, kQBox), dLoMN = desc_lo(dO, kQBox);
            const uint32_t dsLoK = desc_lo(ds, 16), dsLoMN = desc_lo(ds, kDSBytes);
            #pragma unroll
            for (int ks = 0; ks < kBlockK / 16; ++ks)
                mma_ss_lo(tmem + kColDP + b * kBlockQ, kLoMN + ((ks * 2048) >> 4),
                          dsLoMN + ((ks * 2048) >> 4), idDQ, ks > 0);
            tc_commit(&sh.dq_full[b]);
            #pragma unroll
            for (int ks = 0; ks < kBlockQ / 16; ++ks)
                mma_ts_lo(tmem + kColDV, tmem + kColS + b * kBlockQ + ks * 8,
                          dLoMN + ((ks * 2048) >> 4), idAcc, (ks > 0 || !first) ? 1u : 0u);
            tc_commit(&sh.pt_free[b]);
            #pragma unroll
            for (int ks = 0; ks < kBlockQ / 16; ++ks)
                mma_ss_lo(tmem + kColDK, dsLoK + ((ks * 32) >> 4), qLoMN + ((ks * 2048) >> 4), idAcc,
                          (ks > 0 || !first) ? 1u : 0u);
            tc_commit(&sh.qd_empty[s]);
            tc_commit(&sh.ds_free[b]);
        }
        tc_commit(&sh.kv_empty);      // K_j read by dQ^T
        tc_commit(&sh.acc_full);
    }
out:
    tc_commit(&sh.drain[1]);
    mbar_drain_wait(&sh.drain[1], 0);
}

// ---------------------------------------------------- softmax-gradient warps
// The elementwise pass for one key row, in steps of 16 queries:
//   P = 2^(s * scale * log2e - LSE * log2e),  dS = P * (dP - D),
// with -LSE*log2e and -D read as broadcast float4 rows, packed f32x2 math, and
// P, dS rounded to bf16 pairs.  Each step's Sᵀ and dPᵀ columns are loaded
// while the previous step computes (two register sets of 16 + 16 values);
// Pᵀ of a step goes over the Sᵀ columns of its own queries (already read),
// dSᵀ into the step's two 16-byte chunks of the key's row (chunk index XOR
// (row & 7), the 128-byte swizzle).  EDGE: queries outside [lo_c, hi_c)
// take P = 0, as a select, so the unrolled code has no branches.
template <bool EDGE>
__device__ __forceinline__ bool grad_row(uint32_t tS, uint32_t tdP, const float4 *nl4,
                                         const float4 *nd4, uint64_t c2, int lo_c, int hi_c,
                                         uint8_t *dsb, int r, uint64_t *ds_free, uint32_t ds_par,
                                         bool wait_ds, volatile int *abort) {
    uint32_t sr[2][kPartQ], dr[2][kPartQ];
    tmem_ld16(tS, sr[0]);
    tmem_ld16(tdP, dr[0]);
    tmem_wait_ld();
    #pragma unroll
    for (int qi = 0; qi < kBlockQ / kPartQ; ++qi) {
        const int cur = qi & 1;
        if (qi + 1 < kBlockQ / kPartQ) {
            tmem_ld16(tS + (qi + 1) * kPartQ, sr[cur ^ 1]);
            tmem_ld16(tdP + (qi + 1) * kPartQ, dr[cur ^ 1]);
        }
        uint32_t pk[kPartQ / 2], dk[kPartQ / 2];
        #pragma unroll
        for (int cc = 0; cc < kPartQ; cc += 4) {
            const int c = qi * kPartQ + cc;
            const float4 nl = nl4[c >> 2], nd = nd4[c >> 2];
            float x0, x1, x2, x3;
            f2unpack(f2fma(f2pack(__uint_as_float(sr[cur][cc]), __uint_as_float(sr[cur][cc + 1])), c2,
                           f2pack(nl.x, nl.y)), x0, x1);
            f2unpack(f2fma(f2pack(__uint_as_float(sr[cur][cc + 2]), __uint_as_float(sr[cur][cc + 3])), c2,
                           f2pack(nl.z, nl.w)), x2, x3);
            float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
            if constexpr (EDGE) {
                p0 = (c + 0 >= lo_c && c + 0 < hi_c) ? p0 : 0.f;
                p1 = (c + 1 >= lo_c && c + 1 < hi_c) ? p1 : 0.f;
                p2 = (c + 2 >= lo_c && c + 2 < hi_c) ? p2 : 0.f;
                p3 = (c + 3 >= lo_c && c + 3 < hi_c) ? p3 : 0.f;
            }
            float d0, d1, d2, d3;
            f2unpack(f2mul(f2pack(p0, p1),
                           f2add(f2pack(__uint_as_float(dr[cur][cc]), __uint_as_float(dr[cur][cc + 1])),
                                 f2pack(nd.x, nd.y))), d0, d1);
            f2unpack(f2mul(f2pack(p2, p3),
                           f2add(f2pack(__uint_as_float(dr[cur][cc + 2]), __uint_as_float(dr[cur][cc + 3])),
                                 f2pack(nd.z, nd.w))), d2, d3);
            pk[cc >> 1] = pack_bf16(p0, p1);
            pk[(cc >> 1) + 1] = pack_bf16(p2, p3);
            dk[cc >> 1] = pack_bf16(d0, d1);
            dk[(cc >> 1) + 1] = pack_bf16(d2, d3);
        }
        tmem_st8(tS + qi * (kPartQ / 2), pk);
        // dK and dQ^T of tile n-2 read this dSᵀ buffer
        if (qi == 0 && wait_ds && !mbar_wait_warp(ds_free, ds_par, abort)) {
            tmem_wait_ld();     // the next step's load is in flight
            return false;
        }
        #pragma unroll
        for (int c2i = 0; c2i < 2; ++c2i) {
            const int ch = qi * 2 + c2i;
            const uint4 v = make_uint4(dk[4 * c2i], dk[4 * c2i + 1], dk[4 * c2i + 2], dk[4 * c2i + 3]);
            *reinterpret_cast<uint4 *>(dsb + ((ch ^ (r & 7)) << 4)) = v;
        }
        if (qi + 1 < kBlockQ / kPartQ) tmem_wait_ld();
    }
    return true;
}

template <int DH>
__device__ void softmax_wg(const Params &p, Shared &sh, uint8_t *smem) {
    volatile int *abort = &sh.abort;
    const int warp = warp_id(), lane = lane_id();
    const int wg = warp >> 2;                  // takes tiles n with n % 2 == wg
    const int r = (warp & 3) * 32 + lane;      // key row of the block
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = sh.tmem_base + lanes + kColS + wg * kBlockQ;
    const uint32_t tdP = sh.tmem_base + lanes + kColDP + wg * kBlockQ;
    const float *rows = reinterpret_cast<const float *>(smem + kOffRows);
    uint8_t *dsb = smem + kOffDS + wg * kDSBytes + r * 128;
    const float sl2 = p.scale_log2;
    uint32_t n = 0, uc = 0;

    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit(u, p, w)) continue;
        const int kj = w.j0 + r;                  // this thread's key
        const bool key_ok = kj < w.L;
        for (int k = 0; k < w.ntiles; ++k, ++n) {
            if ((int)(n & 1) != wg) continue;
            const int s = n % kStages;
            if (!mbar_wait_warp(&sh.s_full[wg], (n >> 1) & 1, abort)) return;
            if (!mbar_wait_warp(&sh.qd_full[s], (n / kStages) & 1, abort)) return;
            tc_fence_after();
            int h, q0;
            tile_of(w, p, k, h, q0);
            (void)h;
            const float4 *nl4 = reinterpret_cast<const float4 *>(rows + s * 2 * kBlockQ);
            const float4 *nd4 = nl4 + kBlockQ / 4;
            const int qmax = min(q0 + kBlockQ, w.L) - 1;
            const bool edge = (w.j0 + kBlockK > w.L) || (p.causal && w.jl > q0) ||
                              (p.window > 0 && w.j0 <= qmax - p.window);
            // The mask of an edge tile: the column range [lo_c, hi_c) of this
            // key's visible queries.
            int lo_c = 0, hi_c = kBlockQ;
            if (!key_ok) {
                lo_c = kBlockQ;
                hi_c = 0;
            } else if (p.causal) {
                lo_c = kj - q0;                                   // query >= key
                if (p.window > 0) hi_c = min(kBlockQ, kj + p.window - q0);   // query < key + W
            }
            const uint64_t c2 = f2pack(sl2, sl2);
            const bool ok = edge
                ? grad_row<true>(tS, tdP, nl4, nd4, c2, lo_c, hi_c, dsb, r, &sh.ds_free[wg],
                                 ((n - 2) >> 1) & 1, n >= 2, abort)
                : grad_row<false>(tS, tdP, nl4, nd4, c2, 0, 0, dsb, r, &sh.ds_free[wg],
                                  ((n - 2) >> 1) & 1, n >= 2, abort);
            if (!ok) return;
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_full[wg]);
        }
        // ---- unit end: warpgroup 0 writes dV, warpgroup 1 writes scale * dK
        if (!mbar_wait_warp(&sh.acc_full, uc & 1, abort)) return;
        ++uc;
        tc_fence_after();
        const uint32_t tAcc = sh.tmem_base + lanes + (wg ? kColDK : kColDV);
        const float mul = wg ? p.scale : 1.f;
        uint16_t *dst = static_cast<uint16_t *>(wg ? p.dk : p.dv) +
                        ((size_t)(w.tok0 + kj) * p.Hkv + w.kvh) * DH;
        #pragma unroll
        for (int c = 0; c < kD; c += 32) {
            uint32_t v[32];
            tmem_ld32(tAcc + c, v);
            tmem_wait_ld();
            if (key_ok && c < DH) {   // columns past a 64-wide head are padding
                uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    uint4 o;
                    o.x = pack_bf16(__uint_as_float(v[8 * e + 0]) * mul, __uint_as_float(v[8 * e + 1]) * mul);
                    o.y = pack_bf16(__uint_as_float(v[8 * e + 2]) * mul, __uint_as_float(v[8 * e + 3]) * mul);
                    o.z = pack_bf16(__uint_as_float(v[8 * e + 4]) * mul, __uint_as_float(v[8 * e + 5]) * mul);
                    o.w = pack_bf16(__uint_as_float(v[8 * e + 6]) * mul, __uint_as_float(v[8 * e + 7]) * mul);
                    d4[e] = o;
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.acc_free);
    }
}

// ------------------------------------------------------------- dQ drain
// dQ^T of a tile (lane = d index, column = query) is read from TMEM, scaled,
// written transposed into a shared-memory staging buffer (32 query rows x d,
// fp32) and added into the global accumulator by one TMA reduce-add per 32
// rows; two staging buffers alternate so the next rows are written while the
// previous reduce still reads.  Rows past the sequence add exact zeros (their
// P, hence dS, is 0).
template <int DH>
__device__ void dq_drain(const CUtensorMap *tmDQ, const Params &p, Shared &sh, uint8_t *smem) {
    volatile int *abort = &sh.abort;
    const int warp = warp_id(), lane = lane_id();
    const int c = (warp & 3) * 32 + lane;       // d index (TMEM lane of dQ^T)
    const bool leader = (warp == kWarpDrain && lane == 0);
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    float *stage = reinterpret_cast<float *>(smem + kOffDQ);
    uint32_t n = 0, hs = 0;
    FOR_EACH_UNIT(u) {
        Unit w;
        if (!get_unit(u, p, w)) continue;
        for (int k = 0; k < w.ntiles; ++k, ++n) {
            const int b = n & 1;
            const bool ok = mbar_wait_warp(&sh.dq_full[b], (n >> 1) & 1, abort);
            if (!named_bar_and(kBarDrain, 128, ok)) goto out;
            tc_fence_after();
            uint32_t v[64];
            const uint32_t t = sh.tmem_base + lanes + kColDP + b * kBlockQ;
            tmem_ld32(t, v);
            tmem_ld32(t + 32, v + 32);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.dq_free[b]);
            int h, q0;
            tile_of(w, p, k, h, q0);
            #pragma unroll
            for (int half = 0; half < 2; ++half, ++hs) {
                float *buf = stage + (hs & 1) * (kDQHalf * kD);
                if (leader) bulk_wait_group_read<1>();   // the reduce that used buf is done reading
                named_bar_sync(kBarDrain, 128);
                if (c < DH) {           // rows of the head dim (the reduce box is DH wide)
                    #pragma unroll
                    for (int i = 0; i < kDQHalf; ++i)
                        buf[i * DH + c] = __uint_as_float(v[half * kDQHalf + i]) * p.scale;
                }
                fence_proxy_async_smem();
                named_bar_sync(kBarDrain, 128);
                if (leader) {
                    tma_reduce_add_3d(tmDQ, buf, 0, h, w.tok0 + q0 + half * kDQHalf);
                    bulk_commit_group();
                }
            }
        }
    }
out:
    if (leader) bulk_wait_group_all();
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
           const __grid_constant__ CUtensorMap tmDQ, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ Shared sh;
    const uint32_t base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (base & 1023)) & 1023);
    const int warp = warp_id();

    if (threadIdx.x == 0) {
        mbar_init(&sh.kv_full, 1);
        mbar_init(&sh.kv_empty, 2);     // one commit from each MMA issuer
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.qd_full[s], 2);   // TMA bytes + the LSE/D rows
            mbar_init(&sh.qd_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.s_full[b], 1);
            mbar_init(&sh.p_full[b], 4);
            mbar_init(&sh.dq_full[b], 1);
            mbar_init(&sh.dq_free[b], 4);
            mbar_init(&sh.pt_free[b], 1);
            mbar_init(&sh.ds_free[b], 1);
        }
        mbar_init(&sh.acc_full, 1);
        mbar_init(&sh.acc_free, 8);
        mbar_init(&sh.drain[0], 1);
        mbar_init(&sh.drain[1], 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) tmem_alloc(&sh.tmem_base, kTmemCols);
    if (warp == kWarpTma && lane_id() == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmDQ);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp < 8) {
        regs_increase<kRegsSoftmax>();
        softmax_wg<DH>(p, sh, smem);
    } else if (warp < 12) {
        regs_decrease<kRegsDrain>();
        dq_drain<DH>(&tmDQ, p, sh, smem);
    } else {
        regs_decrease<kRegsControl>();
        if (warp == kWarpTma) {
            producer(&tmQ, &tmK, &tmV, &tmdO, p, sh, smem);
        } else if (warp == kWarpMma) {
            if (lane_id() == 0) mma_issuer_s(p, sh, smem);
        } else if (warp == kWarpMmaGrad) {
            if (lane_id() == 0) mma_issuer_grad(p, sh, smem);
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

// D = rowsum(O * dO) for every (token, query head), in the LSE layout; zeroes
// the dQ accumulator.  One warp per row of DH = 64 or 128 elements.
template <int DH>
__global__ void __launch_bounds__(256)
bwd_prep_kernel(const uint16_t *__restrict__ o, const uint16_t *__restrict__ dout,
                float *__restrict__ dd, float *__restrict__ dq_acc, int total, int Hq,
                int seqlen, int dense) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (long long)total * Hq) return;
    auto lo = [](uint32_t x) { return __uint_as_float(x << 16); };
    auto hi = [](uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); };
    float acc;
    if constexpr (DH == 128) {
        const uint2 a = reinterpret_cast<const uint2 *>(o + row * DH)[lane];
        const uint2 b = reinterpret_cast<const uint2 *>(dout + row * DH)[lane];
        acc = lo(a.x) * lo(b.x) + hi(a.x) * hi(b.x) + lo(a.y) * lo(b.y) + hi(a.y) * hi(b.y);
        reinterpret_cast<float4 *>(dq_acc + row * DH)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
        const uint32_t a = reinterpret_cast<const uint32_t *>(o + row * DH)[lane];
        const uint32_t b = reinterpret_cast<const uint32_t *>(dout + row * DH)[lane];
        acc = lo(a) * lo(b) + hi(a) * hi(b);
        reinterpret_cast<float2 *>(dq_acc + row * DH)[lane] = make_float2(0.f, 0.f);
    }
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        const long long tok = row / Hq;
        const int h = (int)(row % Hq);
        size_t idx;
        if (dense) {
            const long long bseq = tok / seqlen, i = tok % seqlen;
            idx = ((size_t)bseq * Hq + h) * seqlen + i;
        } else {
            idx = (size_t)h * total + tok;
        }
        dd[idx] = acc;
    }
}

// Gradient of a learned sink logit z_h: the sink is one more score with a
// zero value, so its dP is 0 and d Loss / d z_h = sum over the rows of head h
// of exp(z_h - LSE_i) * (0 - D_i).  One block per head; a fixed-order tree
// reduction (deterministic).
__global__ void __launch_bounds__(256)
bwd_dsink_kernel(const float *__restrict__ lse, const float *__restrict__ dd,
                 const float *__restrict__ sinks, float *__restrict__ dsinks, int num_seqs,
                 int Hq, int seqlen, int total, int dense) {
    const int h = blockIdx.x;
    const float z = sinks[h];
    float acc = 0.f;
    if (z != -INFINITY) {
        const long long rows = dense ? (long long)num_seqs * seqlen : total;
        for (long long r = threadIdx.x; r < rows; r += blockDim.x) {
            size_t idx;
            if (dense)
                idx = ((size_t)(r / seqlen) * Hq + h) * seqlen + (r % seqlen);
            else
                idx = (size_t)h * total + r;
            acc -= __expf(z - lse[idx]) * dd[idx];
        }
    }
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    __shared__ float part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += part[w];
        dsinks[h] = t;
    }
}

// dQ (bf16) = the fp32 accumulator, eight elements per thread.
__global__ void __launch_bounds__(256)
bwd_convert_kernel(const float *__restrict__ acc, uint16_t *__restrict__ dq, long long n8) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const float4 a = reinterpret_cast<const float4 *>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4 *>(acc)[2 * i + 1];
    uint4 o;
    o.x = pack_bf16(a.x, a.y);
    o.y = pack_bf16(a.z, a.w);
    o.z = pack_bf16(b.x, b.y);
    o.w = pack_bf16(b.z, b.w);
    reinterpret_cast<uint4 *>(dq)[i] = o;
}

}  // namespace bwd_impl

size_t bwd_workspace_bytes(long long total_tokens, int Hq, int d) {
    if (total_tokens < 0 || Hq <= 0 || (d != 64 && d != 128)) return 0;
    const size_t acc = (size_t)total_tokens * Hq * d * sizeof(float);
    const size_t dd = (size_t)total_tokens * Hq * sizeof(float);
    return ((acc + 255) & ~(size_t)255) + ((dd + 255) & ~(size_t)255);
}

int launch_bwd(const BwdArgs &a, cudaStream_t stream) {
    using namespace bwd_impl;
    if (a.d != 64 && a.d != 128) return -2;
    const int dh = a.d;
    const long long total = a.total_tokens;
    if (total == 0 || a.num_seqs == 0) return 0;
    const size_t acc_bytes = ((size_t)total * a.Hq * dh * sizeof(float) + 255) & ~(size_t)255;
    float *dq_acc = static_cast<float *>(a.workspace);
    float *dd = reinterpret_cast<float *>(static_cast<uint8_t *>(a.workspace) + acc_bytes);

    const long long rows = total * a.Hq;
    auto prep = dh == 128 ? bwd_prep_kernel<128> : bwd_prep_kernel<64>;
    prep<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
        static_cast<const uint16_t *>(a.o), static_cast<const uint16_t *>(a.dout), dd, dq_acc,
        (int)total, a.Hq, a.seqlen, a.cu_seqlens ? 0 : 1);
    if (cudaGetLastError() != cudaSuccess) return -5;
    if (a.sinks) {
        bwd_dsink_kernel<<<a.Hq, 256, 0, stream>>>(a.lse, dd, a.sinks, a.dsinks, a.num_seqs,
                                                   a.Hq, a.seqlen, (int)total,
                                                   a.cu_seqlens ? 0 : 1);
        if (cudaGetLastError() != cudaSuccess) return -5;
    }

    // Tensors are dh wide; tiles are kD = 128 wide, loaded as two 64-column
    // boxes.  With dh = 64 the second box lies wholly past the tensor's inner
    // extent, and TMA fills it with zeros: the padded columns add nothing to
    // S or dP, and their dK, dV, dQ columns are never written.
    alignas(64) CUtensorMap tq, tk, tv, tdo, tdq;
    const uint64_t T = (uint64_t)total;
    if (encode_tensor_map_3d(&tq, a.q, 2, dh, a.Hq, T, (uint64_t)dh * 2, (uint64_t)a.Hq * dh * 2,
                             64, 1, kBlockQ, 128) ||
        encode_tensor_map_3d(&tdo, a.dout, 2, dh, a.Hq, T, (uint64_t)dh * 2,
                             (uint64_t)a.Hq * dh * 2, 64, 1, kBlockQ, 128) ||
        encode_tensor_map_3d(&tk, a.k, 2, dh, a.Hkv, T, (uint64_t)dh * 2,
                             (uint64_t)a.Hkv * dh * 2, 64, 1, kBlockK, 128) ||
        encode_tensor_map_3d(&tv, a.v, 2, dh, a.Hkv, T, (uint64_t)dh * 2,
                             (uint64_t)a.Hkv * dh * 2, 64, 1, kBlockK, 128) ||
        encode_tensor_map_3d(&tdq, dq_acc, 4, dh, a.Hq, T, (uint64_t)dh * 4,
                             (uint64_t)a.Hq * dh * 4, dh, 1, kDQHalf, 0))
        return -5;
    Params p;
    p.lse = a.lse;
    p.dd = dd;
    p.dq_acc = dq_acc;
    p.dk = a.dk;
    p.dv = a.dv;
    p.cu_seqlens = a.cu_seqlens;
    p.num_seqs = a.num_seqs;
    p.seqlen = a.seqlen;
    p.total_tokens = (int)total;
    p.max_seqlen = a.max_seqlen;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.group = a.Hq / a.Hkv;
    p.causal = a.causal;
    p.window = a.causal ? a.window : 0;
    p.scale = a.scale;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.num_kblocks = (a.max_seqlen + kBlockK - 1) / kBlockK;
    const long long units = (long long)p.num_kblocks * a.num_seqs * a.Hkv;
    if (units > (1ll << 30)) return -2;
    p.num_units = (int)units;
    if (units > 0) {
        auto kernel = dh == 128 ? bwd_kernel<128> : bwd_kernel<64>;
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes) != cudaSuccess)
            return -5;
        const int grid = (int)(units < device_sm_count() ? units : device_sm_count());
        kernel<<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, tdo, tdq, p);
        if (cudaGetLastError() != cudaSuccess) return -5;
    }
    const long long n8 = total * a.Hq * dh / 8;
    bwd_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, stream>>>(
        dq_acc, static_cast<uint16_t *>(a.dq), n8);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace fa

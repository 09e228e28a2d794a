// decode_tc_sm100.cu -- paged split-KV decode over an FP8 (E4M3) cache with
// the dot products and P·V on the tensor core.
//
// Decode reads every cached byte once and does little arithmetic per byte
// ("Prefill and decode are different problems"), so its target is the HBM
// copy rate.  With an FP8 cache the CUDA-core kernel (decode_sm100.cu) is
// bound by its own instruction issue: per (token, KV head) it converts 2·d
// codes and runs 2·d·group fused multiply-adds.  Here both products run in
// kind::f8f6f4 on the codes exactly as the TMA copy left them:
//
//   * A tile is 128 rows = (pages of the tile) x (KV heads of the unit) x
//     16 tokens, head-major inside a page: rows 16h..16h+15 of a page are
//     KV head h.  One TMA copy per page brings the codes of all the unit's
//     KV heads (the tensor map walks d, then token rows, then heads).
//   * S = K·Q^T for all the unit's query heads at once (N = 16 or 32
//     columns; M = 128 rows): each row only keeps the columns of its own
//     KV head's query heads, so the product is block diagonal and the rest
//     is discarded.  K is the K-major A operand; Q is carried as two E4M3
//     terms (q1 = E4M3(q 2^e), q2 = E4M3(q 2^e - q1), 2^e a power of two per
//     row) stacked along N, which together hold every bf16 value exactly
//     unless its remainder falls below E4M3's normal range (2^-10 of the
//     row's largest magnitude); the softmax adds the two column groups.
//   * P·V as O^T = V^T · P^T: V^T is the MN-major A operand (d on M), P^T a
//     K-major E4M3 operand; P is zero outside the block diagonal, so one
//     chain of MMAs serves every KV head of the tile.  P is carried as two
//     E4M3 terms, P ~ hi + lo with lo = E4M3(P - hi), stacked along N:
//     relative error about 2^-8 per weight, the order of the bf16 P of the
//     prefill.
//   * Softmax: one thread per row with the tile's per-query-head maximum
//     and the conditional rescale of the prefill (threshold 8 in log2
//     units): O^T accumulates in TMEM over a unit's tiles and is rescaled
//     in place only when a query head's maximum grows past the threshold.
//
// FP8 scales: the k scale of a row's page multiplies its scores; P is
// multiplied by v_scale / vref (vref = the largest v scale of that KV head
// over the unit's pages) before it is split, and the unit's O is
// multiplied by vref / l at the end.
//
// Roles (256 threads, one CTA per SM, persistent over (sequence, head group,
// chunk) units): warps 0-3 softmax, the in-place O rescale and the unit's
// output, warp 4 TMA producer, warp 5 MMA issuer (one thread), warp 6 FP8
// scales (a ring of its own), warp 7 Q preparation.  The stages, the scales
// and every TMEM/shared buffer are handed over by mbarriers; every wait is
// bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace decode_tc_impl {

constexpr int kPage = 16;          // tokens per page
constexpr int kChunkPages = 16;    // pages per split-KV chunk (the combine's layout)
constexpr int kRows = 128;         // rows per tile
constexpr int kMaxStages = 8;
constexpr int kThreads = 256;
constexpr int kWarpProducer = 4, kWarpMma = 5, kWarpScales = 6, kWarpQ = 7;
constexpr int kScaleSlots = 4;     // scales ring (tiles ahead of the softmax)
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t kTmemCols = 256;
constexpr int kSmemLimit = 227 * 1024;

struct TcParams {
    const uint16_t *q;
    const int *block_table, *seq_lens;
    float *part_o, *part_lse;     // [S][max_chunks][Hq][D], [S][max_chunks][Hq]
    const float *k_scale, *v_scale;
    int num_seqs, num_pages, Hq, Hkv, HG, ppt, num_hg, max_pages, max_chunks, nst;
    float scale_log2;
};

// Columns of S and O per tile: the unit's query heads, padded to 16.
template <int G> constexpr int kN = G >= 4 ? 32 : 16;

// Walks this CTA's units and, inside each, its tiles of ppt pages.  Units
// are numbered sequence-major, then head group, then chunk; the CTA takes
// every gridDim.x-th unit.  All roles walk the same sequence.
struct Walk {
    int s = 0, base = 0;   // sequence scan
    int u = 0;             // unit index
    int seq = 0, hg = 0, chunk = 0, L = 0, pg0 = 0, pg1 = 0;
    int first = 0;         // first page (index within the sequence) of the tile
    int units = 0;         // units this CTA has started
    bool valid = false;

    __device__ static int pages_of(int L) { return (L + kPage - 1) / kPage; }
    __device__ static int chunks_of(int L) { return (pages_of(L) + kChunkPages - 1) / kChunkPages; }
    __device__ bool find(const TcParams &p) {
        while (s < p.num_seqs) {
            int len = __ldg(p.seq_lens + s);
            const int cap = p.max_pages * kPage;
            if (len < 0 || len > cap) {
                report_error(kDevErrInput);
                len = len < 0 ? 0 : cap;
            }
            const int nc = chunks_of(len);
            if (u < base + p.num_hg * nc) {
                const int r = u - base;
                seq = s;
                L = len;
                hg = r / nc;
                chunk = r % nc;
                pg0 = chunk * kChunkPages;
                pg1 = min(pages_of(len), pg0 + kChunkPages);
                first = pg0;
                return true;
            }
            base += p.num_hg * nc;
            ++s;
        }
        return false;
    }
    __device__ void start(const TcParams &p) {
        u = blockIdx.x;
        valid = find(p);
        units = valid ? 1 : 0;
    }
    __device__ void next_unit(const TcParams &p) {
        u += gridDim.x;
        valid = find(p);
        if (valid) ++units;
    }
    __device__ void next(const TcParams &p) {
        first += p.ppt;
        if (first >= pg1) next_unit(p);
    }
    __device__ int npg(const TcParams &p) const { return min(p.ppt, pg1 - first); }
    __device__ bool unit_first() const { return first == pg0; }
    __device__ bool unit_last(const TcParams &p) const { return first + p.ppt >= pg1; }
    __device__ int ub() const { return (units - 1) & 1; }            // per-unit buffer
    __device__ uint32_t uuse() const { return (uint32_t)(units - 1) >> 1; }
};

struct TcShared {
    uint64_t full[kMaxStages], empty[kMaxStages];
    uint64_t s_full[2], s_free[2], p_ready[2], o_ok[2], pv_done[2];
    uint64_t o_free[2];          // per unit buffer: O^T read out by the unit's epilogue
    uint64_t red_bar[2];
    uint64_t scl_full[kScaleSlots], scl_empty[kScaleSlots];
    uint64_t q_full[2], q_empty[2], l_ready[2], lred_bar[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int resc[2];                 // index of the tile whose O^T is rescaled (per tile buffer)
    // per tile: k scale [q], v scale / vref [8 + q] (q = page*HG + h), vref [16 + h]
    float scl[kScaleSlots][24];
    float qc[2][32];             // per unit buffer: score multiplier per query column
    float alpha[2][32];          // per tile buffer: O^T rescale factor per query column
    float inv_l[2][32];          // per unit buffer: vref / l per query column
    float red[2][8][8];          // per tile buffer: [half-warp][query head] partial maxima
    float redl[2][8][8];         // per unit buffer: partial sums of l
};

// Dynamic shared memory, from a 1024-byte aligned base:
//   stages  nst x [V codes | K codes], kRows x 128 bytes each (128-byte
//           swizzled rows, pages of the tile consecutive); the V codes are
//           the A operand of P·V
//   P       2 x [hi | lo]  P^T as E4M3, K-major B operand: 2N rows x 128 bytes,
//           the hi rows then the lo rows (one MMA chain with N' = 2N)
//   Q       2 x [q1 | q2]  Q as two E4M3 terms, K-major B operand: 2N rows x
//           128 bytes, the q1 rows then the q2 rows
template <int D, int G>
struct Layout {
    static_assert(D == 128, "d = 128");
    static constexpr int N = kN<G>;
    static constexpr uint32_t kRegion = kRows * D;              // codes of K (or V)
    static constexpr uint32_t kStage = 2 * kRegion;
    static constexpr uint32_t kPTerm = N * 128;                 // one E4M3 term of P^T
    static constexpr uint32_t kPBytes = 2 * kPTerm;
    static constexpr uint32_t kQBytes = 2 * N * 128;
    static constexpr uint32_t kFixed = 2 * kPBytes + 2 * kQBytes;
    __host__ __device__ static uint32_t pbuf(int nst) { return nst * kStage; }
    __host__ __device__ static uint32_t qbuf(int nst) { return pbuf(nst) + 2 * kPBytes; }
    // TMEM columns: S (2 x 2N, per tile: the q1 and the q2 products side by
    // side), O^T (2 x 2N, per unit: the hi and the lo products side by side)
    static constexpr uint32_t kColS = 0, kColO = 4 * N;
    static_assert(kColO + 4 * N <= kTmemCols, "TMEM columns");
};

// Byte offset of 16-byte chunk c of code row r in a K or V region.
template <int D>
__device__ __forceinline__ uint32_t code_off(int r, int c) {
    if constexpr (D == 128)
        return (uint32_t)r * 128 + ((uint32_t)(c ^ (r & 7)) << 4);
    else
        return (uint32_t)r * 64 + ((uint32_t)(c ^ ((r >> 1) & 3)) << 4);
}

// Four E4M3 codes (one 32-bit word, lowest index in bits 0-7) to two f16 pairs.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi) : "r"(w));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}

// Two fp32 values to a packed f16 pair (round to nearest even), lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp32 values to E4M3 codes (round to nearest even, saturating), lo in
// bits 0-7; and two E4M3 codes back to fp32 (exact).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void e4m3x2_val(uint32_t two, float &lo, float &hi) {
    asm("{\n\t.reg .b16 t, a, b;\n\t.reg .b32 h;\n\tcvt.u16.u32 t, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, t;\n\tmov.b32 {a, b}, h;\n\t"
        "cvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(two));
}

// TMEM loads of 2, 4 or 8 columns (shape 32x32b).
template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t *r) {
    if constexpr (NC == 2) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                     : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
    } else if constexpr (NC == 4) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr));
    } else if constexpr (NC == 8) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                       "=r"(r[6]), "=r"(r[7]) : "r"(taddr));
    } else {
        static_assert(NC == 16, "2, 4, 8 or 16 columns");
        tmem_ld16(taddr, r);
    }
}

// Instruction descriptors with fp32 D: kind::f16 with f16 A and B (format
// 0), and kind::f8f6f4 with E4M3 A and B (format 0); bit 15 = A MN-major.
__host__ __device__ constexpr uint32_t idesc_f32d(int M, int N, bool a_mn_major) {
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Bounded waits: the first test inline, the rest out of line (one copy per
// role R, since the roles run under different register budgets), so that
// the per-tile loops stay short in the instruction cache.
template <int R>
__device__ __noinline__ bool wait_rest(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return mbar_wait(bar, parity, abort);
}
template <int R>
__device__ __forceinline__ bool wait1(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return mbar_try_wait(smem_u32(bar), parity) || wait_rest<R>(bar, parity, abort);
}
template <int R>
__device__ __forceinline__ bool waitw(uint64_t *bar, uint32_t parity, volatile int *abort) {
    const bool ok = wait1<R>(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}
enum : int { kRoleSoftmax = 0, kRoleControl = 2 };

// ---------------------------------------------------------------- producer
// Whole warp: a unit's block-table entries are read once, one per lane; lane
// 0 issues one K and one V copy per page of each tile.
template <int D, int G>
__device__ void producer(const CUtensorMap *tmK, const CUtensorMap *tmV, const TcParams &p,
                         TcShared &sh, uint8_t *smem) {
    using Ly = Layout<D, G>;
    volatile int *abort = &sh.abort;
    const int lane = lane_id();
    const uint32_t page_bytes = 2u * D * kPage * p.HG;
    const uint32_t slot_bytes = (uint32_t)kPage * p.HG * D;   // one page of K (or V) codes
    Walk w;
    w.start(p);
    uint32_t it = 0, ph = 0;
    int cur = 0, page_lane = 0, st = 0;
    for (; w.valid; w.next(p), ++it, (++st == p.nst ? (st = 0, ph ^= 1) : 0)) {
        if (w.units != cur) {
            cur = w.units;
            const int pg = w.pg0 + lane;
            page_lane = 0;
            if (pg < w.pg1) {
                page_lane = __ldg(p.block_table + (size_t)w.seq * p.max_pages + pg);
                if (page_lane < 0 || page_lane >= p.num_pages) {
                    report_error(kDevErrInput);
                    page_lane = 0;
                }
            }
        }
        if (!waitw<kRoleControl>(&sh.empty[st], ph ^ 1, abort)) goto drain;
        {
            const int npg = w.npg(p);
            uint8_t *sV = smem + (size_t)st * Ly::kStage;
            uint8_t *sK = sV + Ly::kRegion;
            if (lane == 0) mbar_arrive_expect_tx(&sh.full[st], npg * page_bytes);
            for (int pi = 0; pi < npg; ++pi) {
                const int page = __shfl_sync(0xffffffffu, page_lane, w.first - w.pg0 + pi);
                if (lane == 0) {
                    tma_load_3d(sK + pi * slot_bytes, tmK, &sh.full[st], 0, page * kPage, w.hg * p.HG);
                    tma_load_3d(sV + pi * slot_bytes, tmV, &sh.full[st], 0, page * kPage, w.hg * p.HG);
                }
            }
        }
    }
    return;
drain:
    if (lane == 0)
        for (int s = 0; s < p.nst; ++s)
            if (it > (uint32_t)s) mbar_drain_wait(&sh.full[s], ((it - 1 - s) / p.nst) & 1);
}

// -------------------------------------------------------------- FP8 scales
// Per unit, lane l holds the 8 (page, head) k scales (l even) or v scales
// (l odd) of the unit's tile l/2, and the v lanes reduce vref (the largest v
// scale of each KV head over the unit).  Per tile, the two lanes of that
// tile store k scales, v / vref and vref into a slot of the scales ring,
// which the softmax warps release.
template <int D, int G>
__device__ void scales_warp(const TcParams &p, TcShared &sh) {
    volatile int *abort = &sh.abort;
    const int lane = lane_id();
    const int tl = lane >> 1, kind = lane & 1;
    Walk w;
    w.start(p);
    uint32_t it = 0, ph = 0;
    int cur = 0, sl = 0;
    float v[8], vref[8];
    for (; w.valid; w.next(p), ++it, (++sl == kScaleSlots ? (sl = 0, ph ^= 1) : 0)) {
        if (w.units != cur) {
            cur = w.units;
            int page[8];
            #pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int pg = w.pg0 + tl * p.ppt + q / p.HG;
                page[q] = -1;
                if (pg < w.pg1) {
                    page[q] = __ldg(p.block_table + (size_t)w.seq * p.max_pages + pg);
                    if (page[q] < 0 || page[q] >= p.num_pages) page[q] = 0;
                }
            }
            const float *src = kind ? p.v_scale : p.k_scale;
            #pragma unroll
            for (int q = 0; q < 8; ++q)
                v[q] = page[q] >= 0
                    ? __ldg(src + (size_t)page[q] * p.Hkv + w.hg * p.HG + q % p.HG)
                    : (kind ? 0.f : 1.f);
            // vref per KV head: the largest v scale over the unit (v lanes only)
            #pragma unroll
            for (int h = 0; h < 8; ++h) {
                float m = 0.f;
                #pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (kind && q % p.HG == h) m = fmaxf(m, v[q]);
                #pragma unroll
                for (int o = 2; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                vref[h] = m;
            }
            if (kind) {
                #pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float r = 0.f;
                    #pragma unroll
                    for (int h = 0; h < 8; ++h)
                        if (q % p.HG == h) r = vref[h];
                    v[q] = r > 0.f ? v[q] / r : 0.f;
                }
            }
        }
        if (!waitw<kRoleControl>(&sh.scl_empty[sl], ph ^ 1, abort)) return;
        if (tl == (w.first - w.pg0) / p.ppt) {
            #pragma unroll
            for (int q = 0; q < 8; ++q) sh.scl[sl][kind * 8 + q] = v[q];
            if (kind) {
                #pragma unroll
                for (int h = 0; h < 8; ++h) sh.scl[sl][16 + h] = vref[h];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.scl_full[sl]);
    }
}

// ------------------------------------------------------------ Q preparation
// Per unit: the unit's query heads (rows n < HG*G; the rest zero) as two
// E4M3 terms with a power-of-two row scale, written K-major with the
// 128-byte swizzle (q1 rows, then q2 rows), and the score multiplier
// scale*log2(e)*2^-e of every row.
template <int D, int G>
__device__ void q_warp(const TcParams &p, TcShared &sh, uint8_t *smem) {
    using Ly = Layout<D, G>;
    constexpr int N = Ly::N;
    constexpr int LPR = D / 8;             // lanes per row (8 elements each)
    constexpr int RPP = 32 / LPR;          // rows per pass
    volatile int *abort = &sh.abort;
    const int lane = lane_id();
    const int sub = lane % LPR, rsub = lane / LPR;
    const int nrows = p.HG * G;
    Walk w;
    w.start(p);
    for (; w.valid; w.next_unit(p)) {
        const int ub = w.ub();
        if (!waitw<kRoleControl>(&sh.q_empty[ub], (w.uuse() & 1) ^ 1, abort)) return;
        const uint32_t qb = smem_u32(smem + Ly::qbuf(p.nst) + ub * Ly::kQBytes);
        const int hq0 = w.hg * nrows;
        #pragma unroll 1
        for (int n0 = 0; n0 < N; n0 += 4 * RPP) {
            uint4 raw[4];
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int n = n0 + k * RPP + rsub;
                raw[k] = make_uint4(0, 0, 0, 0);
                if (n < nrows)
                    raw[k] = __ldg(reinterpret_cast<const uint4 *>(
                        p.q + ((size_t)w.seq * p.Hq + hq0 + n) * D) + sub);
            }
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int n = n0 + k * RPP + rsub;
                float f[8];
                const uint32_t wd[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
                float amax = 0.f;
                #pragma unroll
                for (int i = 0; i < 4; ++i) {
                    f[2 * i] = __uint_as_float(wd[i] << 16);
                    f[2 * i + 1] = __uint_as_float(wd[i] & 0xffff0000u);
                    amax = fmaxf(amax, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
                }
                #pragma unroll
                for (int m = LPR / 2; m >= 1; m >>= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
                // 2^e: the power of two that brings the row's largest magnitude
                // into [128, 256); q = (q1 + q2) 2^-e with q1 = E4M3(q 2^e) and
                // q2 = E4M3(q 2^e - q1): exact for every bf16 value whose
                // remainder is not an E4M3 subnormal (below 2^-10 of the row's max)
                int e = 0;
                if (amax > 0.f) e = min(max(127 + 7 - (int)((__float_as_uint(amax) >> 23) & 0xff), -100), 100);
                const float up = __uint_as_float((uint32_t)(127 + e) << 23);
                uint32_t c1[4], c2[4];
                #pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float x0 = f[2 * i] * up, x1 = f[2 * i + 1] * up;
                    c1[i] = e4m3x2(x0, x1);
                    float h0, h1;
                    e4m3x2_val(c1[i], h0, h1);
                    c2[i] = e4m3x2(x0 - h0, x1 - h1);
                }
                const int d0 = sub * 8;
                const uint32_t row = qb + n * 128 + ((((d0 >> 4) ^ (n & 7))) << 4) + (d0 & 15);
                asm volatile("st.shared.v2.b32 [%0], {%1, %2};"
                             ::"r"(row), "r"(c1[0] | (c1[1] << 16)), "r"(c1[2] | (c1[3] << 16)) : "memory");
                asm volatile("st.shared.v2.b32 [%0], {%1, %2};"
                             ::"r"(row + N * 128), "r"(c2[0] | (c2[1] << 16)), "r"(c2[2] | (c2[3] << 16)) : "memory");
                if (sub == 0) sh.qc[ub][n] = p.scale_log2 * __uint_as_float((uint32_t)(127 - e) << 23);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.q_full[ub]);
    }
}

// --------------------------------------------------------------- MMA issuer
// One thread.  S of the next tile is issued before P·V of the current one,
// so the softmax of tile i+1 never waits for P·V of tile i.
template <int D, int G>
__device__ void mma_issuer(const TcParams &p, TcShared &sh, uint8_t *smem) {
    using Ly = Layout<D, G>;
    constexpr int N = Ly::N;
    volatile int *abort = &sh.abort;
    const uint32_t tmem = sh.tmem_base;
    const uint32_t idS = idesc_f32d(kRows, 2 * N, false);
    const uint32_t idPV = idesc_f32d(kRows, 2 * N, true);
    const uint32_t stage0 = smem_u32(smem);
    const uint32_t pb = smem_u32(smem + Ly::pbuf(p.nst));
    const uint32_t qb = smem_u32(smem + Ly::qbuf(p.nst));

    // [S1 | S2] = K [Q1 | Q2]^T, kind::f8f6f4, 32 d per MMA: A = the K codes
    // of the stage (K-major, 128-byte swizzle, 32 bytes per step), B = the 2N
    // rows of the two E4M3 terms of Q.
    auto issue_s = [&](const Walk &w, uint32_t i, int st, uint32_t ph) -> bool {
        const int b = i & 1, ub = w.ub();
        if (w.unit_first() && !wait1<kRoleControl>(&sh.q_full[ub], w.uuse() & 1, abort)) return false;
        if (!wait1<kRoleControl>(&sh.full[st], ph, abort)) return false;
        if (i >= 2 && !wait1<kRoleControl>(&sh.s_free[b], ((i >> 1) - 1) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t k_lo = desc_lo(stage0 + st * Ly::kStage + Ly::kRegion, 16);
        const uint32_t q_lo = desc_lo(qb + ub * Ly::kQBytes, 16);
        #pragma unroll
        for (int ks = 0; ks < D / 32; ++ks)
            mma_ss_lo_f8(tmem + Ly::kColS + b * 2 * N, k_lo + ((ks * 32) >> 4),
                         q_lo + ((ks * 32) >> 4), idS, ks > 0 ? 1u : 0u);
        tc_commit(&sh.s_full[b]);
        if (w.unit_last(p)) tc_commit(&sh.q_empty[ub]);
        return true;
    };
    // [O_hi^T | O_lo^T][unit] (+)= V^T [P_hi^T | P_lo^T], kind::f8f6f4, 32 rows
    // per MMA: A = the V codes of the stage (MN-major, d on M, 128-byte
    // swizzle, 32 rows = 4096 bytes per step), B = the 2N rows of P^T
    // (K-major, 32 bytes per step).  The unit's first tile starts the
    // accumulator; the stage is released when the MMAs have read it.
    auto issue_pv = [&](bool first, int ub, uint32_t uuse, uint32_t i, int st) -> bool {
        const int b = i & 1;
        if (!wait1<kRoleControl>(&sh.o_ok[b], (i >> 1) & 1, abort)) return false;
        if (first && !wait1<kRoleControl>(&sh.o_free[ub], (uuse & 1) ^ 1, abort)) return false;
        tc_fence_after();
        const uint32_t v_lo = desc_lo(stage0 + st * Ly::kStage, 16);
        const uint32_t p_lo = desc_lo(pb + b * Ly::kPBytes, 16);
        #pragma unroll
        for (int ks = 0; ks < kRows / 32; ++ks)
            mma_ss_lo_f8(tmem + Ly::kColO + ub * 2 * N, v_lo + ((ks * 4096) >> 4),
                         p_lo + ((ks * 32) >> 4), idPV, (ks > 0 || !first) ? 1u : 0u);
        tc_commit(&sh.pv_done[b]);
        tc_commit(&sh.empty[st]);
        return true;
    };

    int pst = 0, sst = 0;
    uint32_t sph = 0;
    // w runs one tile ahead: S of tile i+1 is issued before P·V of tile i
    Walk w;
    w.start(p);
    if (w.valid) {
        if (!issue_s(w, 0, sst, sph)) goto out;
        if (++sst == p.nst) {
            sst = 0;
            sph ^= 1;
        }
        bool f0 = w.unit_first();
        int ub0 = w.ub();
        uint32_t uu0 = w.uuse();
        w.next(p);
        for (uint32_t i = 0;; ++i) {
            if (w.valid) {
                if (!issue_s(w, i + 1, sst, sph)) goto out;
                if (++sst == p.nst) {
                    sst = 0;
                    sph ^= 1;
                }
            }
            if (!issue_pv(f0, ub0, uu0, i, pst)) goto out;
            if (++pst == p.nst) pst = 0;
            if (!w.valid) break;
            f0 = w.unit_first();
            ub0 = w.ub();
            uu0 = w.uuse();
            w.next(p);
        }
    }
out:
    tc_commit(&sh.drain);
    mbar_drain_wait(&sh.drain, 0);
}

// ----------------------------------------------------------- softmax warps
// In-place rescale of this warp's 32 lanes of [O_hi^T | O_lo^T]: columns n
// and N + n times alpha[n].
template <int N>
__device__ __noinline__ void rescale_o(uint32_t to, const float *alpha) {
    #pragma unroll 1
    for (int c = 0; c < 2 * N; c += 16) {
        uint32_t ov[16];
        tmem_ld16(to + c, ov);
        tmem_wait_ld();
        #pragma unroll
        for (int k = 0; k < 16; ++k)
            ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha[(c + k) & (N - 1)]);
        tmem_st16(to + c, ov);
    }
    tmem_wait_st();
}

// A unit's normalised partial O = (O_hi + O_lo) / l: thread = d lane of O^T,
// columns n < nrows.
template <int N, int D>
__device__ __noinline__ void write_o(uint32_t to, const float *inv_l, float *dst, int nrows, int r) {
    uint32_t ov[2 * N];
    #pragma unroll
    for (int c = 0; c < 2 * N; c += 16) tmem_ld16(to + c, ov + c);
    tmem_wait_ld();
    if (r < D) {
        #pragma unroll
        for (int n = 0; n < N; ++n)
            if (n < nrows)
                dst[(size_t)n * D + r] =
                    (__uint_as_float(ov[n]) + __uint_as_float(ov[N + n])) * inv_l[n];
    }
}

// Per tile: scores of row r for its KV head's G query heads, the tile's
// maximum per query head, the conditional rescale, P^T row r; then, once
// all four warps have published, the in-place rescale of O^T when a query
// head needed one.  At a unit's last tile: l, the LSE and the normalised
// partial O (thread = d lane of O^T).
template <int D, int G>
__device__ void softmax_wg(const TcParams &p, TcShared &sh, uint8_t *smem) {
    using Ly = Layout<D, G>;
    constexpr int N = Ly::N;
    volatile int *abort = &sh.abort;
    const int warp = warp_id(), lane = lane_id();
    const int r = warp * 32 + lane;                 // tile row = TMEM lane (d for O^T)
    const int HG = p.HG;
    const int hw = r >> 4;                          // half-warp: one (page, head)
    const int h = hw % HG;                          // KV head within the group
    const int pi = r / (16 * HG);                   // page within the tile
    const int t = r & 15;
    const int cb = HG >= 2 ? ((2 * warp) % HG) * G : 0;
    const bool upper = HG >= 2 && lane >= 16;
    const bool writer = r < 16 * HG && t == 0;      // first row of head h
    const bool one_head = HG == 1;
    const uint32_t tmem = sh.tmem_base + ((uint32_t)(warp * 32) << 16);
    // P^T (K-major, 128-byte swizzle): row n = hG + j, byte r of the row
    const uint32_t pcol = smem_u32(smem + Ly::pbuf(p.nst)) + (r & 15);
    float m[G], l[G], cq[G];
    #pragma unroll
    for (int j = 0; j < G; ++j) {
        m[j] = -INFINITY;
        l[j] = 0.f;
        cq[j] = 0.f;
    }
    Walk w;
    w.start(p);
    int sl = 0, st = 0;
    uint32_t sph = 0, ph = 0;
    for (uint32_t i = 0; w.valid; w.next(p), ++i, (++sl == kScaleSlots ? (sl = 0, sph ^= 1) : 0),
                                  (++st == p.nst ? (st = 0, ph ^= 1) : 0)) {
        const int b = i & 1, ub = w.ub();
        const bool first = w.unit_first(), last = w.unit_last(p);
        if (first) {
            if (!waitw<kRoleSoftmax>(&sh.q_full[ub], w.uuse() & 1, abort)) return;
            #pragma unroll
            for (int j = 0; j < G; ++j) cq[j] = sh.qc[ub][h * G + j];
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.q_empty[ub]);
        }
        // this tile's scales
        if (!waitw<kRoleSoftmax>(&sh.scl_full[sl], sph, abort)) return;
        const bool valid = pi < w.npg(p) && (w.first + pi) * kPage + t < w.L;
        const float ks = sh.scl[sl][pi * HG + h], vr = sh.scl[sl][8 + pi * HG + h];
        const float vref = sh.scl[sl][16 + h];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.scl_empty[sl]);

        if (!waitw<kRoleSoftmax>(&sh.s_full[b], (i >> 1) & 1, abort)) return;
        tc_fence_after();
        uint32_t v[2 * G], v2[2 * G];
        tmem_ld_cols<2 * G>(tmem + Ly::kColS + b * 2 * N + cb, v);
        tmem_ld_cols<2 * G>(tmem + Ly::kColS + b * 2 * N + N + cb, v2);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.s_free[b]);

        float s[G], mx[G];
        #pragma unroll
        for (int j = 0; j < G; ++j) {
            const float sv = upper ? __uint_as_float(v[G + j]) + __uint_as_float(v2[G + j])
                                   : __uint_as_float(v[j]) + __uint_as_float(v2[j]);
            s[j] = valid ? sv * (cq[j] * ks) : -INFINITY;
            mx[j] = s[j];
        }
        #pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
            #pragma unroll
            for (int j = 0; j < G; ++j) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], o));
        }
        #pragma unroll
        for (int j = 0; j < G; ++j) {
            const float y = __shfl_xor_sync(0xffffffffu, mx[j], 16);
            if (one_head) mx[j] = fmaxf(mx[j], y);
        }
        if (p.ppt > 1) {
            // the head's rows span several warps: exchange the half-warp maxima
            if (t == 0) {
                #pragma unroll
                for (int j = 0; j < G; ++j) sh.red[b][hw][j] = mx[j];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.red_bar[b]);
            if (!waitw<kRoleSoftmax>(&sh.red_bar[b], (i >> 1) & 1, abort)) return;
            #pragma unroll
            for (int j = 0; j < G; ++j) {
                float x = -INFINITY;
                for (int q = 0; q < p.ppt; ++q) x = fmaxf(x, sh.red[b][h + q * HG][j]);
                mx[j] = x;
            }
        }
        // conditional rescale: the reference moves only when the tile's
        // maximum exceeds it by the threshold (P <= 2^8 otherwise)
        // (selects, not branches: the G heads' exponentials overlap)
        float alpha[G];
        bool resc = false;
        #pragma unroll
        for (int j = 0; j < G; ++j) {
            const bool up = !first && mx[j] > m[j] + kRescaleThreshold;
            const float a = ex2(m[j] - mx[j]);
            alpha[j] = up ? a : 1.f;
            l[j] *= alpha[j];
            m[j] = (first || up) ? mx[j] : m[j];
            resc |= up;
        }
        float pv[G];
        #pragma unroll
        for (int j = 0; j < G; ++j) {
            const float pr = ex2(s[j] - m[j]);      // 0 for rows past the sequence
            l[j] += pr;
            pv[j] = pr * vr;
        }
        // P^T[b] is free once P·V of tile i-2 has completed
        if (i >= 2 && !waitw<kRoleSoftmax>(&sh.pv_done[b], ((i >> 1) - 1) & 1, abort)) return;
        {
            // P = hi + lo, both E4M3: hi rounds P, lo rounds the remainder
            uint32_t hi[G], lo[G];
            #pragma unroll
            for (int j = 0; j < G; j += 2) {
                const float p1 = j + 1 < G ? pv[j + 1] : 0.f;
                const uint32_t c = e4m3x2(pv[j], p1);
                float h0, h1;
                e4m3x2_val(c, h0, h1);
                const uint32_t d = e4m3x2(pv[j] - h0, p1 - h1);
                hi[j] = c & 0xff;
                lo[j] = d & 0xff;
                if (j + 1 < G) {
                    hi[j + 1] = c >> 8;
                    lo[j + 1] = d >> 8;
                }
            }
            const uint32_t base = pcol + b * Ly::kPBytes;
            #pragma unroll
            for (int j = 0; j < G; ++j) {
                const int n = h * G + j;
                const uint32_t addr = base + n * 128 + ((((r >> 4) ^ n) & 7) << 4);
                asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(hi[j]) : "memory");
                asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr + Ly::kPTerm), "r"(lo[j]) : "memory");
            }
        }
        // every row of head h holds the same alpha: all lanes store it (one
        // value per address, no divergent branch)
        #pragma unroll
        for (int j = 0; j < G; ++j) sh.alpha[b][h * G + j] = alpha[j];
        if (resc) sh.resc[b] = (int)i;
        // V codes of rows past the sequence are zeroed in the stage: P is zero
        // there, and 0 * NaN would poison O (P·V reads the codes as they are)
        if (__any_sync(0xffffffffu, !valid)) {
            if (!waitw<kRoleSoftmax>(&sh.full[st], ph, abort)) return;
            if (!valid) {
                const uint32_t vrow = smem_u32(smem) + st * Ly::kStage + r * 128;
                #pragma unroll
                for (int c = 0; c < 8; ++c) sts128(vrow + c * 16, 0, 0, 0, 0);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.p_ready[b]);
        // every warp's P and rescale flags of this tile are published
        if (!waitw<kRoleSoftmax>(&sh.p_ready[b], (i >> 1) & 1, abort)) return;
        if (!first && sh.resc[b] == (int)i) {
            // rescale O^T in place: P·V of tile i-1 must have completed
            if (!waitw<kRoleSoftmax>(&sh.pv_done[b ^ 1], ((i - 1) >> 1) & 1, abort)) return;
            tc_fence_after();
            rescale_o<N>(tmem + Ly::kColO + ub * 2 * N, sh.alpha[b]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.o_ok[b]);

        if (last) {
            float ls[G];
            #pragma unroll
            for (int j = 0; j < G; ++j) ls[j] = l[j];
            #pragma unroll
            for (int o = 8; o >= 1; o >>= 1) {
                #pragma unroll
                for (int j = 0; j < G; ++j) ls[j] += __shfl_xor_sync(0xffffffffu, ls[j], o);
            }
            #pragma unroll
            for (int j = 0; j < G; ++j) {
                const float y = __shfl_xor_sync(0xffffffffu, ls[j], 16);
                if (one_head) ls[j] += y;
            }
            if (p.ppt > 1) {
                if (t == 0) {
                    #pragma unroll
                    for (int j = 0; j < G; ++j) sh.redl[ub][hw][j] = ls[j];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.lred_bar[ub]);
                if (!waitw<kRoleSoftmax>(&sh.lred_bar[ub], w.uuse() & 1, abort)) return;
                #pragma unroll
                for (int j = 0; j < G; ++j) {
                    // rows of head h in the other pages: every HG-th half-warp;
                    // for HG == 1 each warp's two halves hold the same sum
                    float x = 0.f;
                    const int step = one_head ? 2 : HG;
                    for (int q = h; q < 8; q += step) x += sh.redl[ub][q][j];
                    ls[j] = x;
                }
            }
            if (writer) {
                const size_t row0 = ((size_t)w.seq * p.max_chunks + w.chunk) * p.Hq +
                                    (size_t)w.hg * HG * G + h * G;
                #pragma unroll
                for (int j = 0; j < G; ++j) {
                    p.part_lse[row0 + j] = ls[j] > 0.f
                        ? (m[j] + __log2f(ls[j])) * 0.69314718055994531f : -INFINITY;
                    sh.inv_l[ub][h * G + j] = ls[j] > 0.f ? vref / ls[j] : 0.f;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.l_ready[ub]);
            #pragma unroll
            for (int j = 0; j < G; ++j) {
                m[j] = -INFINITY;
                l[j] = 0.f;
            }
            // the unit's partial O: wait for its last P·V and for every l
            if (!waitw<kRoleSoftmax>(&sh.pv_done[b], (i >> 1) & 1, abort)) return;
            if (!waitw<kRoleSoftmax>(&sh.l_ready[ub], w.uuse() & 1, abort)) return;
            tc_fence_after();
            const int nrows = HG * G;
            const size_t row0 = ((size_t)w.seq * p.max_chunks + w.chunk) * p.Hq +
                                (size_t)w.hg * nrows;
            write_o<N, D>(tmem + Ly::kColO + ub * 2 * N, sh.inv_l[ub], p.part_o + row0 * D, nrows, r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.o_free[ub]);
        }
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const TcParams p) {
    using Ly = Layout<D, G>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ TcShared sh;
    const uint32_t base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (base & 1023)) & 1023);
    const int warp = warp_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.nst; ++s) {
            mbar_init(&sh.full[s], 1);       // TMA bytes
            mbar_init(&sh.empty[s], 1);      // the P·V commit
        }
        for (int s = 0; s < kScaleSlots; ++s) {
            mbar_init(&sh.scl_full[s], 1);
            mbar_init(&sh.scl_empty[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.s_full[b], 1);
            mbar_init(&sh.s_free[b], 4);
            mbar_init(&sh.p_ready[b], 4);
            mbar_init(&sh.o_ok[b], 4);
            mbar_init(&sh.pv_done[b], 1);
            mbar_init(&sh.o_free[b], 4);
            sh.resc[b] = -1;
            mbar_init(&sh.red_bar[b], 4);
            mbar_init(&sh.q_full[b], 1);
            mbar_init(&sh.q_empty[b], 5);    // the MMA commit + the four softmax warps
            mbar_init(&sh.l_ready[b], 4);
            mbar_init(&sh.lred_bar[b], 4);
        }
        mbar_init(&sh.drain, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    // P^T is zero outside each KV head's block; only the block is rewritten
    {
        const uint32_t pz = smem_u32(smem + Ly::pbuf(p.nst));
        for (uint32_t off = threadIdx.x * 16; off < 2 * Ly::kPBytes; off += kThreads * 16)
            sts128(pz + off, 0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == kWarpMma) tmem_alloc(&sh.tmem_base, kTmemCols);
    if (warp == kWarpProducer && lane_id() == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp < 4) {
        softmax_wg<D, G>(p, sh, smem);
    } else {
        if (warp == kWarpProducer)
            producer<D, G>(&tmK, &tmV, p, sh, smem);
        else if (warp == kWarpMma) {
            if (lane_id() == 0) mma_issuer<D, G>(p, sh, smem);
        } else if (warp == kWarpScales)
            scales_warp<D, G>(p, sh);
        else if (warp == kWarpQ)
            q_warp<D, G>(p, sh, smem);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(sh.tmem_base, kTmemCols);
    }
}

template <int D, int G>
int launch_tc(const CUtensorMap &tk, const CUtensorMap &tv, const TcParams &p,
              cudaStream_t stream) {
    using Ly = Layout<D, G>;
    const int smem = (int)(p.nst * Ly::kStage + Ly::kFixed) + 1024;
    if (cudaFuncSetAttribute(decode_tc_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
        return -5;
    decode_tc_kernel<D, G><<<device_sm_count(), kThreads, smem, stream>>>(tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

template <int D>
int launch_tc_g(int G, const CUtensorMap &tk, const CUtensorMap &tv, const TcParams &p,
                cudaStream_t stream) {
    switch (G) {
    case 1: return launch_tc<D, 1>(tk, tv, p, stream);
    case 2: return launch_tc<D, 2>(tk, tv, p, stream);
    case 4: return launch_tc<D, 4>(tk, tv, p, stream);
    default: return launch_tc<D, 8>(tk, tv, p, stream);
    }
}

// Stages that fit beside the fixed buffers (static shared memory included).
template <int D, int G>
int stages_for() {
    using Ly = Layout<D, G>;
    const int avail = kSmemLimit - (int)sizeof(TcShared) - 1024 - (int)Ly::kFixed;
    return min(kMaxStages, avail / (int)Ly::kStage);
}

}  // namespace decode_tc_impl

bool decode_tc_supported(const DecodeArgs &a) {
    if (!a.fp8 || a.d != 128 || a.Hkv <= 0 || a.Hq % a.Hkv) return false;
    const int G = a.Hq / a.Hkv;
    return G == 1 || G == 2 || G == 4 || G == 8;
}

int launch_decode_split_tc(const DecodeArgs &a, float *part_o, float *part_lse, int max_chunks,
                           cudaStream_t stream) {
    namespace T = decode_tc_impl;
    constexpr int kPage = T::kPage;
    const int G = a.Hq / a.Hkv;
    const int N = G >= 4 ? 32 : 16;
    int HG = 1;
    for (int c = 8; c >= 1; c >>= 1)
        if (a.Hkv % c == 0 && c * G <= N) { HG = c; break; }
    alignas(64) CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)a.num_pages * kPage;
    const uint64_t s_tok = (uint64_t)a.Hkv * a.d, s_head = (uint64_t)a.d;
    const int sw = 128;
    // dims: d, token rows, KV heads (the box lands head-major: [HG][16][d])
    if (encode_tensor_map_3d(&tk, a.k_cache, 1, a.d, rows, a.Hkv, s_tok, s_head, a.d, kPage, HG, sw) ||
        encode_tensor_map_3d(&tv, a.v_cache, 1, a.d, rows, a.Hkv, s_tok, s_head, a.d, kPage, HG, sw))
        return -5;
    T::TcParams p;
    p.q = static_cast<const uint16_t *>(a.q);
    p.block_table = a.block_table;
    p.seq_lens = a.seq_lens;
    p.part_o = part_o;
    p.part_lse = part_lse;
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.num_seqs = a.num_seqs;
    p.num_pages = a.num_pages;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.HG = HG;
    p.ppt = 8 / HG;
    p.num_hg = a.Hkv / HG;
    p.max_pages = a.max_pages;
    p.max_chunks = max_chunks;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.nst = G >= 4 ? T::stages_for<128, 4>() : T::stages_for<128, 1>();
    if (p.nst < 2) return -5;
    return T::launch_tc_g<128>(G, tk, tv, p, stream);
}

}  // namespace fa

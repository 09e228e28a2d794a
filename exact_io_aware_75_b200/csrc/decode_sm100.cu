// decode_sm100.cu -- paged split-KV decode and its log-sum-exp combine.
//
// One query token per sequence attends to its whole cached context.  Decode
// does little math per byte ("Prefill and decode are different problems":
// decode is bound by reading the KV cache), so the kernel is built to stream
// the cache at HBM speed:
//   * "Flash-Decoding": every sequence's cache is cut into chunks of
//     kChunkPages pages; chunks are attended in parallel and merged with the
//     log-sum-exp rule by a second kernel.
//   * "Paging and prefix sharing": the cache is [pages, 16, Hkv, d]; a chunk
//     reads its pages through the block table.  One TMA copy brings the K
//     (or V) rows of a page for a group of KV heads -- for 8 KV heads and
//     d = 128 that is one contiguous 32 KiB page -- into a shared-memory ring
//     that a producer warp keeps several copies deep.
//   * The grid is persistent (one CTA per SM) and walks the (sequence, head
//     group, chunk) units round-robin, so long and short sequences balance
//     and the producer never drains between units.
//   * "MQA and GQA": each KV byte is read once for all the query heads that
//     share it.  A compute warp owns one KV head and up to four of its query
//     heads; lane = (token group tg, d slice ds): tokens tg, tg+4, tg+8,
//     tg+12 of each page, 8 or 16 of the d values.  Scores are summed across
//     the 8 lanes of a token group by a transposing butterfly, the running
//     max/sum per head is updated with the same conditional rescale as the
//     prefill kernel, and P V accumulates in registers.
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace decode_impl {

constexpr int kPage = 16;           // tokens per page
constexpr int kChunkPages = 16;     // pages per split-KV chunk
constexpr int kMaxComputeWarps = 8;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kSmemBudget = 200 * 1024;

struct DecodeParams {
    const uint16_t *q;
    const int *block_table, *seq_lens;
    float *part_o, *part_lse;     // [S][max_chunks][Hq][D], [S][max_chunks][Hq]
    int num_seqs, num_pages, Hq, Hkv, group, max_pages, max_chunks;
    int HG, WPK, NW, num_hg, nst;
    uint32_t box_bytes;
    float scale_log2;
    const float *k_scale, *v_scale;   // FP8 cache: [num_pages][Hkv] dequantisation scales
};

// Walks the flat unit index space (sequence-major, then head group, then
// chunk).  Returns false once past the last sequence.
struct UnitWalker {
    int s = 0, base = 0;
    __device__ __forceinline__ static int chunks_of(int L) {
        const int pages = (L + kPage - 1) / kPage;
        return (pages + kChunkPages - 1) / kChunkPages;
    }
    __device__ __forceinline__ static int clamp_len(const DecodeParams &p, int L) {
        const int cap = p.max_pages * kPage;
        if (L < 0 || L > cap) {
            report_error(kDevErrInput);
            L = L < 0 ? 0 : cap;
        }
        return L;
    }
    __device__ __forceinline__ bool find(const DecodeParams &p, int u, int &seq, int &hg,
                                         int &chunk, int &L) {
        while (s < p.num_seqs) {
            L = clamp_len(p, __ldg(p.seq_lens + s));
            const int n = p.num_hg * chunks_of(L);
            if (u < base + n) {
                const int r = u - base;
                seq = s;
                hg = r / chunks_of(L);
                chunk = r % chunks_of(L);
                return true;
            }
            base += n;
            ++s;
        }
        return false;
    }
};

struct DecShared {
    uint64_t full[8], empty[8];
    float scl[8][16];   // FP8: per stage, k scales then v scales of the head group
    int abort;
};

// Four bf16 pairs (one 16-byte load) to four packed fp32 pairs.
__device__ __forceinline__ void unpack8x2(uint4 a, uint64_t *f) {
    f[0] = f2pack(__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xffff0000u));
    f[1] = f2pack(__uint_as_float(a.y << 16), __uint_as_float(a.y & 0xffff0000u));
    f[2] = f2pack(__uint_as_float(a.z << 16), __uint_as_float(a.z & 0xffff0000u));
    f[3] = f2pack(__uint_as_float(a.w << 16), __uint_as_float(a.w & 0xffff0000u));
}

__device__ __forceinline__ void unpack8(uint4 a, float *f) {
    f[0] = __uint_as_float(a.x << 16); f[1] = __uint_as_float(a.x & 0xffff0000u);
    f[2] = __uint_as_float(a.y << 16); f[3] = __uint_as_float(a.y & 0xffff0000u);
    f[4] = __uint_as_float(a.z << 16); f[5] = __uint_as_float(a.z & 0xffff0000u);
    f[6] = __uint_as_float(a.w << 16); f[7] = __uint_as_float(a.w & 0xffff0000u);
}

// Two FP8 E4M3 codes (bits 0-7: the lower index) to a packed fp32 pair, by
// way of the hardware e4m3x2 -> f16x2 conversion and two f16 -> f32
// conversions (both exact: every E4M3 value, subnormals included, is an f16
// normal).  Measured faster here than building the fp32 words with integer
// bit placement, which loads the integer pipe the dot products also use.
__device__ __forceinline__ uint64_t e4m3x2_to_f2(uint32_t two) {
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(two));
    float lo, hi;
    asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}" : "=f"(lo), "=f"(hi) : "r"(h2));
    return f2pack(lo, hi);
}

// N FP8 codes (N = 8 or 16, loaded as one 8- or 16-byte word) to N/2 pairs.
template <int N>
__device__ __forceinline__ void unpack_e4m3(const uint8_t *src, uint64_t *f) {
    if constexpr (N == 16) {
        const uint4 a = *reinterpret_cast<const uint4 *>(src);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = e4m3x2_to_f2(w[i] & 0xffffu);
            f[2 * i + 1] = e4m3x2_to_f2(w[i] >> 16);
        }
    } else {
        const uint2 a = *reinterpret_cast<const uint2 *>(src);
        const uint32_t w[2] = {a.x, a.y};
        #pragma unroll
        for (int i = 0; i < 2; ++i) {
            f[2 * i] = e4m3x2_to_f2(w[i] & 0xffffu);
            f[2 * i + 1] = e4m3x2_to_f2(w[i] >> 16);
        }
    }
}

// Sum NV values over the 8 lanes of a token group (xor 4, 2, 1), leaving
// lane ds with the totals of flat indices [ds*NV/8, ...) (NV >= 8), or of
// index ds*NV/8 shared by a lane pair (NV == 4).
template <int NV>
__device__ __forceinline__ void group_transpose_sum(float (&v)[NV], int lane) {
    int n = NV;
    #pragma unroll
    for (int m = 4; m >= 1; m >>= 1) {
        if (n >= 2) {
            const int half = n / 2;
            const bool up = (lane & m) != 0;
            #pragma unroll
            for (int i = 0; i < NV / 2; ++i) {
                if (i < half) {
                    const float send = up ? v[i] : v[i + half];
                    const float keep = up ? v[i + half] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            n = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
        }
    }
}

// Block: warps 0-7 compute (the first NW of them work), warp 8 produces,
// warps 9-11 only complete the third warpgroup.  Registers: launched with
// 384 x 168; compute warpgroups 216 each, the producer warpgroup 72
// (2 * 128 * 216 + 128 * 72 = 64,512).
constexpr int kDecThreads = 384;
constexpr int kDecWarpProducer = 8;
constexpr int kDecWarpScales = 9;       // FP8 only
constexpr int kDecRegsCompute = 216;
constexpr int kDecRegsControl = 72;
static_assert(2 * 128 * kDecRegsCompute + 128 * kDecRegsControl <= kDecThreads * 168,
              "register split");

template <int D, int QPW, bool FP8>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const DecodeParams p) {
    constexpr int DPL = D / 8;          // d values per lane
    constexpr int NV = 4 * QPW;         // partial scores per lane per page
    constexpr int HELD = NV >= 8 ? NV / 8 : 1;
    extern __shared__ uint8_t smem_raw[];
    __shared__ DecShared sh;
    uint8_t *smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
    const int warp = warp_id(), lane = lane_id();
    volatile int *abort = &sh.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.nst; ++i) {
            mbar_init(&sh.full[i], FP8 ? 2 : 1);   // FP8: TMA bytes + the scale warp
            mbar_init(&sh.empty[i], p.NW);
        }
        sh.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp >= kMaxComputeWarps) {
        regs_decrease<kDecRegsControl>();
        if (FP8 && warp == kDecWarpScales) {
            // ------------------------------------------------ FP8 scales
            // The same page sequence as the producer: each stage gets its
            // page's k and v scales (lane l: KV head hg*HG + l), then one
            // arrival on the stage's full barrier.  Global
            // loads stall only this warp.
            UnitWalker walk;
            uint32_t it = 0;
            int seq, hg, chunk, L;
            for (int u = blockIdx.x; walk.find(p, u, seq, hg, chunk, L); u += gridDim.x) {
                const int pages = (L + kPage - 1) / kPage;
                const int pg0 = chunk * kChunkPages, pg1 = min(pages, pg0 + kChunkPages);
                for (int pg = pg0; pg < pg1; ++pg, ++it) {
                    const int st = it % p.nst;
                    if (!mbar_wait_warp(&sh.empty[st], ((it / p.nst) & 1) ^ 1, abort)) return;
                    int page = __ldg(p.block_table + (size_t)seq * p.max_pages + pg);
                    if (page < 0 || page >= p.num_pages) page = 0;
                    if (lane < p.HG) {
                        const size_t i = (size_t)page * p.Hkv + hg * p.HG + lane;
                        sh.scl[st][lane] = __ldg(p.k_scale + i);
                        sh.scl[st][8 + lane] = __ldg(p.v_scale + i);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.full[st]);
                }
            }
            return;
        }
        if (warp != kDecWarpProducer) return;
        // ------------------------------------------------------- producer
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            UnitWalker walk;
            uint32_t it = 0;
            int seq, hg, chunk, L;
            for (int u = blockIdx.x; walk.find(p, u, seq, hg, chunk, L); u += gridDim.x) {
                const int pages = (L + kPage - 1) / kPage;
                const int pg0 = chunk * kChunkPages, pg1 = min(pages, pg0 + kChunkPages);
                for (int pg = pg0; pg < pg1; ++pg) {
                    int page = __ldg(p.block_table + (size_t)seq * p.max_pages + pg);
                    if (page < 0 || page >= p.num_pages) {
                        report_error(kDevErrInput);
                        page = 0;
                    }
                    const int st = it % p.nst;
                    const uint32_t use = it / p.nst;
                    if (!mbar_wait(&sh.empty[st], (use & 1) ^ 1, abort)) goto drain;
                    mbar_arrive_expect_tx(&sh.full[st], 2 * p.box_bytes);
                    uint8_t *dst = smem + (size_t)st * 2 * p.box_bytes;
                    tma_load_3d(dst, &tmK, &sh.full[st], 0, hg * p.HG, page * kPage);
                    tma_load_3d(dst + p.box_bytes, &tmV, &sh.full[st], 0, hg * p.HG, page * kPage);
                    ++it;
                }
            }
            return;
        drain:
            for (int st = 0; st < p.nst; ++st)
                if (it > (uint32_t)st) mbar_drain_wait(&sh.full[st], ((it - 1 - st) / p.nst) & 1);
        }
        return;
    }
    regs_increase<kDecRegsCompute>();
    if (warp >= p.NW) return;

    // ------------------------------------------------------------ compute
    const int hl = warp / p.WPK;                  // KV head within the group
    const int qsub = warp % p.WPK;
    const int tg = lane >> 3, ds = lane & 7;
    UnitWalker walk;
    uint32_t it = 0;
    int seq, hg, chunk, L;
    for (int u = blockIdx.x; walk.find(p, u, seq, hg, chunk, L); u += gridDim.x) {
        const int kvh = hg * p.HG + hl;
        const int h0 = kvh * p.group + qsub * QPW;   // first query head of this warp
        // q (pre-scaled by scale*log2 e), this lane's d slice
        // fp32 pairs (packed f32x2 arithmetic halves the FMA instructions)
        uint64_t q2[QPW][DPL / 2];
        const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2);
        #pragma unroll
        for (int qh = 0; qh < QPW; ++qh) {
            // d slice of this lane: bf16 cache 8*ds + 64*b + (0..7); FP8 cache
            // DPL*ds + (0..DPL-1), one 8- or 16-byte word of codes
            const uint16_t *qp = p.q + ((size_t)seq * p.Hq + h0 + qh) * D +
                                 (FP8 ? DPL * ds : 8 * ds);
            #pragma unroll
            for (int b = 0; b < DPL / 8; ++b) {
                const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(qp + (FP8 ? 8 : 64) * b));
                unpack8x2(raw, &q2[qh][4 * b]);
            }
            #pragma unroll
            for (int i = 0; i < DPL / 2; ++i) q2[qh][i] = f2mul(q2[qh][i], sc2);
        }
        uint64_t o2[QPW][DPL / 2];
        float m_ref[QPW], l_acc[QPW];
        #pragma unroll
        for (int qh = 0; qh < QPW; ++qh) {
            m_ref[qh] = -INFINITY;
            l_acc[qh] = 0.f;
            #pragma unroll
            for (int i = 0; i < DPL / 2; ++i) o2[qh][i] = f2pack(0.f, 0.f);
        }
        const int pages = (L + kPage - 1) / kPage;
        const int pg0 = chunk * kChunkPages, pg1 = min(pages, pg0 + kChunkPages);
        for (int pg = pg0; pg < pg1; ++pg) {
            const int st = it % p.nst;
            if (!mbar_wait_warp(&sh.full[st], (it / p.nst) & 1, abort)) return;
            float ks_cur = 1.f, vs_cur = 1.f;
            if constexpr (FP8) {
                ks_cur = sh.scl[st][hl];
                vs_cur = sh.scl[st][8 + hl];
            }
            ++it;
            const uint8_t *sK = smem + (size_t)st * 2 * p.box_bytes;
            const uint8_t *sV = sK + p.box_bytes;
            const int nvalid = min(kPage, L - pg * kPage);
            // ---- scores: partial dot products over this lane's d slice
            float sc[NV];
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = tg + 4 * k;
                uint64_t kv2[DPL / 2];
                if constexpr (FP8) {
                    unpack_e4m3<DPL>(sK + (size_t)(t * p.HG + hl) * D + DPL * ds, kv2);
                } else {
                    const uint16_t *kr = reinterpret_cast<const uint16_t *>(sK) +
                                         ((size_t)(t * p.HG + hl) * D + 8 * ds);
                    #pragma unroll
                    for (int b = 0; b < DPL / 8; ++b)
                        unpack8x2(*reinterpret_cast<const uint4 *>(kr + 64 * b), &kv2[4 * b]);
                }
                #pragma unroll
                for (int qh = 0; qh < QPW; ++qh) {
                    uint64_t a0 = f2mul(q2[qh][0], kv2[0]);
                    uint64_t a1 = f2mul(q2[qh][1], kv2[1]);
                    #pragma unroll
                    for (int i = 2; i < DPL / 2; i += 2) {
                        a0 = f2fma(q2[qh][i], kv2[i], a0);
                        a1 = f2fma(q2[qh][i + 1], kv2[i + 1], a1);
                    }
                    float x0, x1, y0, y1;
                    f2unpack(a0, x0, x1);
                    f2unpack(a1, y0, y1);
                    sc[k * QPW + qh] = (x0 + x1) + (y0 + y1);
                }
            }
            group_transpose_sum<NV>(sc, lane);
            // lane holds flat indices [ds*NV/8, +HELD): token slot k = ds/2,
            // heads (ds & 1) * QPW/2 .. + HELD-1
            const int kslot = ds >> 1;
            const bool tok_ok = (tg + 4 * kslot) < nvalid;
            float s_own[HELD];
            #pragma unroll
            for (int i = 0; i < HELD; ++i) s_own[i] = tok_ok ? (FP8 ? sc[i] * ks_cur : sc[i]) : -INFINITY;
            // ---- page max per head, known to every lane
            float pmax_own[HELD];
            #pragma unroll
            for (int i = 0; i < HELD; ++i) {
                float mv = s_own[i];
                mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, 2));
                mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, 4));
                mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, 8));
                mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, 16));
                pmax_own[i] = mv;
            }
            float pmax[QPW];
            if constexpr (QPW >= 2) {
                #pragma unroll
                for (int i = 0; i < HELD; ++i) {
                    const float other = __shfl_xor_sync(0xffffffffu, pmax_own[i], 1);
                    const bool lo_half = (ds & 1) == 0;
                    pmax[i] = lo_half ? pmax_own[i] : other;
                    pmax[QPW / 2 + i] = lo_half ? other : pmax_own[i];
                }
            } else {
                pmax[0] = pmax_own[0];
            }
            // ---- conditional rescale (uniform across the warp: every lane
            // holds the same m_ref and page max for every head); one branch
            // for all heads, so the common path stays one block
            bool any_up = false;
            #pragma unroll
            for (int qh = 0; qh < QPW; ++qh) any_up |= pmax[qh] > m_ref[qh] + kRescaleThreshold;
            if (any_up) {
                #pragma unroll
                for (int qh = 0; qh < QPW; ++qh) {
                    const bool up = pmax[qh] > m_ref[qh] + kRescaleThreshold;
                    const float alpha = !up ? 1.f
                                      : (m_ref[qh] == -INFINITY) ? 0.f : ex2(m_ref[qh] - pmax[qh]);
                    m_ref[qh] = up ? pmax[qh] : m_ref[qh];
                    l_acc[qh] *= alpha;
                    const uint64_t a2 = f2pack(alpha, alpha);
                    #pragma unroll
                    for (int i = 0; i < DPL / 2; ++i) o2[qh][i] = f2mul(o2[qh][i], a2);
                }
            }
            // ---- probabilities of the held scores
            float p_own[HELD];
            #pragma unroll
            for (int i = 0; i < HELD; ++i) {
                // select, not m_ref[hq0 + i]: a run-time index would put
                // m_ref in local memory
                const float mr = (QPW >= 2 && (ds & 1)) ? m_ref[QPW / 2 + i] : m_ref[i];
                p_own[i] = ex2(s_own[i] - (mr == -INFINITY ? 0.f : mr));
            }
            // ---- gather the token group's probabilities [4 slots][QPW]
            float pr[4][QPW];
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                if constexpr (QPW >= 2) {
                    #pragma unroll
                    for (int half = 0; half < 2; ++half)
                        #pragma unroll
                        for (int i = 0; i < HELD; ++i)
                            pr[k][half * (QPW / 2) + i] =
                                __shfl_sync(0xffffffffu, p_own[i], (tg << 3) + 2 * k + half);
                } else {
                    pr[k][0] = __shfl_sync(0xffffffffu, p_own[0], (tg << 3) + 2 * k);
                }
            }
            // ---- P V over this lane's tokens (a full page in one block; the
            // sequence's last page checks each slot, since slots past
            // seq_len may hold anything)
            auto pv_slot = [&](int k) {
                const int t = tg + 4 * k;
                uint64_t vv2[DPL / 2];
                if constexpr (FP8) {
                    unpack_e4m3<DPL>(sV + (size_t)(t * p.HG + hl) * D + DPL * ds, vv2);
                } else {
                    const uint16_t *vr = reinterpret_cast<const uint16_t *>(sV) +
                                         ((size_t)(t * p.HG + hl) * D + 8 * ds);
                    #pragma unroll
                    for (int b = 0; b < DPL / 8; ++b)
                        unpack8x2(*reinterpret_cast<const uint4 *>(vr + 64 * b), &vv2[4 * b]);
                }
                #pragma unroll
                for (int qh = 0; qh < QPW; ++qh) {
                    const float pv = FP8 ? pr[k][qh] * vs_cur : pr[k][qh];
                    const uint64_t pp = f2pack(pv, pv);
                    #pragma unroll
                    for (int i = 0; i < DPL / 2; ++i) o2[qh][i] = f2fma(pp, vv2[i], o2[qh][i]);
                }
            };
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                #pragma unroll
                for (int qh = 0; qh < QPW; ++qh) l_acc[qh] += pr[k][qh];
            }
            if (nvalid == kPage) {
                #pragma unroll
                for (int k = 0; k < 4; ++k) pv_slot(k);
            } else {
                #pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (tg + 4 * k < nvalid) pv_slot(k);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.empty[st]);
        }
        // ---- merge the four token groups and write this chunk's partial
        float o[QPW][DPL];
        #pragma unroll
        for (int qh = 0; qh < QPW; ++qh) {
            l_acc[qh] += __shfl_xor_sync(0xffffffffu, l_acc[qh], 8);
            l_acc[qh] += __shfl_xor_sync(0xffffffffu, l_acc[qh], 16);
            #pragma unroll
            for (int i = 0; i < DPL / 2; ++i) f2unpack(o2[qh][i], o[qh][2 * i], o[qh][2 * i + 1]);
            #pragma unroll
            for (int i = 0; i < DPL; ++i) {
                o[qh][i] += __shfl_xor_sync(0xffffffffu, o[qh][i], 8);
                o[qh][i] += __shfl_xor_sync(0xffffffffu, o[qh][i], 16);
            }
        }
        if (tg == 0) {
            const size_t row0 = ((size_t)seq * p.max_chunks + chunk) * p.Hq + h0;
            #pragma unroll
            for (int qh = 0; qh < QPW; ++qh) {
                const float inv = l_acc[qh] > 0.f ? 1.f / l_acc[qh] : 0.f;
                float *dst = p.part_o + (row0 + qh) * D + (FP8 ? DPL * ds : 8 * ds);
                #pragma unroll
                for (int b = 0; b < DPL / 8; ++b) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + (FP8 ? 8 : 64) * b);
                    d4[0] = make_float4(o[qh][8 * b + 0] * inv, o[qh][8 * b + 1] * inv,
                                        o[qh][8 * b + 2] * inv, o[qh][8 * b + 3] * inv);
                    d4[1] = make_float4(o[qh][8 * b + 4] * inv, o[qh][8 * b + 5] * inv,
                                        o[qh][8 * b + 6] * inv, o[qh][8 * b + 7] * inv);
                }
                if (ds == 0)
                    p.part_lse[row0 + qh] = l_acc[qh] > 0.f
                        ? (m_ref[qh] + __log2f(l_acc[qh])) * 0.69314718055994531f
                        : -INFINITY;
            }
        }
    }
}

// Merge the chunks of each (sequence, head).  One block of kCombineWarps
// warps per row: the row's max LSE first, then each warp sums a strided
// subset of the chunks (several loads in flight), and the warps' partial
// sums are added in shared memory.
constexpr int kCombineWarps = 4;

template <int D>
__global__ void __launch_bounds__(32 * kCombineWarps)
decode_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse,
                      const int *__restrict__ seq_lens, uint16_t *__restrict__ o,
                      float *__restrict__ lse, const float *__restrict__ sinks,
                      int num_seqs, int Hq, int max_pages, int max_chunks) {
    constexpr int PER = D / 32;
    __shared__ float s_acc[kCombineWarps][D];
    __shared__ float s_w[kCombineWarps];
    const int row = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = row / Hq, h = row % Hq;
    int L = __ldg(seq_lens + s);
    L = max(0, min(L, max_pages * kPage));
    const int nc = ((L + kPage - 1) / kPage + kChunkPages - 1) / kChunkPages;
    const float *lse_p = part_lse + (size_t)s * max_chunks * Hq + h;
    float m = -INFINITY;
    for (int c = lane; c < nc; c += 32) m = fmaxf(m, lse_p[(size_t)c * Hq]);
    #pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    // A learned sink is one more partial: LSE z, output zero.
    const float z = sinks ? __ldg(sinks + h) : -INFINITY;
    m = fmaxf(m, z);
    float acc[PER];
    #pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float wsum = 0.f;
    if (m != -INFINITY) {
        const float *src0 = part_o + ((size_t)s * max_chunks * Hq + h) * D + lane * PER;
        #pragma unroll 4
        for (int c = warp; c < nc; c += kCombineWarps) {
            const float w = __expf(lse_p[(size_t)c * Hq] - m);
            wsum += w;
            const float4 v = *reinterpret_cast<const float4 *>(src0 + (size_t)c * Hq * D);
            acc[0] = fmaf(w, v.x, acc[0]);
            acc[1] = fmaf(w, v.y, acc[1]);
            acc[2] = fmaf(w, v.z, acc[2]);
            acc[3] = fmaf(w, v.w, acc[3]);
            if constexpr (PER == 8) {
                const float4 u = *reinterpret_cast<const float4 *>(src0 + (size_t)c * Hq * D + 4);
                acc[4] = fmaf(w, u.x, acc[4]);
                acc[5] = fmaf(w, u.y, acc[5]);
                acc[6] = fmaf(w, u.z, acc[6]);
                acc[7] = fmaf(w, u.w, acc[7]);
            }
        }
    }
    #pragma unroll
    for (int i = 0; i < PER; ++i) s_acc[warp][lane * PER + i] = acc[i];
    if (lane == 0) s_w[warp] = wsum;
    __syncthreads();
    if (warp != 0) return;
    float tw = 0.f;
    #pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) tw += s_w[w];
    if (z != -INFINITY) tw += __expf(z - m);
    const float inv = tw > 0.f ? 1.f / tw : 0.f;
    float r[PER];
    #pragma unroll
    for (int i = 0; i < PER; ++i) {
        float t = 0.f;
        #pragma unroll
        for (int w = 0; w < kCombineWarps; ++w) t += s_acc[w][lane * PER + i];
        r[i] = t * inv;
    }
    uint16_t *dst = o + ((size_t)s * Hq + h) * D + lane * PER;
    #pragma unroll
    for (int i = 0; i < PER; i += 2)
        *reinterpret_cast<uint32_t *>(dst + i) = pack_bf16(r[i], r[i + 1]);
    if (lse && lane == 0) lse[(size_t)s * Hq + h] = tw > 0.f ? m + __logf(tw) : -INFINITY;
}

struct Plan {
    int HG, WPK, NW, QPW, num_hg, nst;
    uint32_t box_bytes;
    int max_chunks;
};

bool make_plan(int Hq, int Hkv, int d, int max_pages, int elem_bytes, Plan &pl) {
    if (Hkv <= 0 || Hq % Hkv) return false;
    const int g = Hq / Hkv;
    pl.QPW = (g % 4 == 0) ? 4 : (g % 2 == 0) ? 2 : 1;
    pl.WPK = g / pl.QPW;
    if (pl.WPK > kMaxComputeWarps) return false;
    const int cap = kMaxComputeWarps / pl.WPK;
    pl.HG = 1;
    for (int c = min(cap, Hkv); c >= 1; --c)
        if (Hkv % c == 0) { pl.HG = c; break; }
    pl.NW = pl.HG * pl.WPK;
    pl.num_hg = Hkv / pl.HG;
    pl.box_bytes = (uint32_t)(kPage * pl.HG * d * elem_bytes);
    pl.nst = kSmemBudget / (2 * (int)pl.box_bytes);
    if (pl.nst > 8) pl.nst = 8;
    if (pl.nst < 2) return false;
    pl.max_chunks = (max_pages + kChunkPages - 1) / kChunkPages;
    return true;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <int D, int QPW, bool FP8>
int launch_split(const CUtensorMap &tk, const CUtensorMap &tv, const DecodeParams &p,
                 cudaStream_t stream) {
    const int smem = p.nst * 2 * (int)p.box_bytes + 128;
    if (cudaFuncSetAttribute(decode_split_kernel<D, QPW, FP8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return -5;
    decode_split_kernel<D, QPW, FP8><<<device_sm_count(), kDecThreads, smem, stream>>>(tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

template <bool FP8>
int launch_split_d(int d, int qpw, const CUtensorMap &tk, const CUtensorMap &tv,
                   const DecodeParams &p, cudaStream_t stream) {
    if (d == 128)
        return qpw == 4 ? launch_split<128, 4, FP8>(tk, tv, p, stream)
             : qpw == 2 ? launch_split<128, 2, FP8>(tk, tv, p, stream)
                        : launch_split<128, 1, FP8>(tk, tv, p, stream);
    return qpw == 4 ? launch_split<64, 4, FP8>(tk, tv, p, stream)
         : qpw == 2 ? launch_split<64, 2, FP8>(tk, tv, p, stream)
                    : launch_split<64, 1, FP8>(tk, tv, p, stream);
}

}  // namespace decode_impl

using namespace decode_impl;

size_t decode_workspace_bytes(int num_seqs, int Hq, int d, int page_size, int max_pages) {
    if (num_seqs <= 0 || Hq <= 0 || (d != 64 && d != 128) || page_size != kPage || max_pages <= 0)
        return 0;
    const size_t chunks = (size_t)((max_pages + kChunkPages - 1) / kChunkPages);
    const size_t rows = (size_t)num_seqs * chunks * Hq;
    return align256(rows * d * sizeof(float)) + align256(rows * sizeof(float));
}

int launch_decode(const DecodeArgs &a, cudaStream_t stream) {
    Plan pl;
    const int eb = a.fp8 ? 1 : 2;
    if (!make_plan(a.Hq, a.Hkv, a.d, a.max_pages, eb, pl)) return -2;
    const size_t need = decode_workspace_bytes(a.num_seqs, a.Hq, a.d, a.page_size, a.max_pages);
    if (need == 0) return -2;
    if (!a.workspace || a.workspace_bytes < need) return -4;
    if (a.num_seqs == 0) return 0;
    alignas(64) CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)a.num_pages * kPage;
    const uint64_t s1 = (uint64_t)a.d * eb, s2 = (uint64_t)a.Hkv * a.d * eb;
    if (encode_tensor_map_3d(&tk, a.k_cache, eb, a.d, a.Hkv, rows, s1, s2, a.d, pl.HG, kPage, 0) ||
        encode_tensor_map_3d(&tv, a.v_cache, eb, a.d, a.Hkv, rows, s1, s2, a.d, pl.HG, kPage, 0))
        return -5;
    DecodeParams p;
    p.q = static_cast<const uint16_t *>(a.q);
    p.block_table = a.block_table;
    p.seq_lens = a.seq_lens;
    const size_t chunk_rows = (size_t)a.num_seqs * pl.max_chunks * a.Hq;
    p.part_o = static_cast<float *>(a.workspace);
    p.part_lse = reinterpret_cast<float *>(static_cast<char *>(a.workspace) +
                                           align256(chunk_rows * a.d * sizeof(float)));
    p.num_seqs = a.num_seqs;
    p.num_pages = a.num_pages;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.group = a.Hq / a.Hkv;
    p.max_pages = a.max_pages;
    p.max_chunks = pl.max_chunks;
    p.HG = pl.HG;
    p.WPK = pl.WPK;
    p.NW = pl.NW;
    p.num_hg = pl.num_hg;
    p.nst = pl.nst;
    p.box_bytes = pl.box_bytes;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    int rc;
    if (decode_tc_supported(a))
        rc = launch_decode_split_tc(a, p.part_o, p.part_lse, pl.max_chunks, stream);
    else if (a.fp8)
        rc = launch_split_d<true>(a.d, pl.QPW, tk, tv, p, stream);
    else
        rc = launch_split_d<false>(a.d, pl.QPW, tk, tv, p, stream);
    if (rc) return rc;
    const int blocks = a.num_seqs * a.Hq;
    if (a.d == 128)
        decode_combine_kernel<128><<<blocks, 32 * kCombineWarps, 0, stream>>>(
            p.part_o, p.part_lse, a.seq_lens, static_cast<uint16_t *>(a.o), a.lse, a.sinks,
            a.num_seqs, a.Hq, a.max_pages, pl.max_chunks);
    else
        decode_combine_kernel<64><<<blocks, 32 * kCombineWarps, 0, stream>>>(
            p.part_o, p.part_lse, a.seq_lens, static_cast<uint16_t *>(a.o), a.lse, a.sinks,
            a.num_seqs, a.Hq, a.max_pages, pl.max_chunks);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace fa

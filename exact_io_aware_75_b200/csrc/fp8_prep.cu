// fp8_prep.cu -- operands of the FP8 prefill.
//
// What it computes ("FlashAttention-3" in samanvya.dev's "Attention Is the
// Bottleneck", "FlashAttention: same math, different IO": a random orthogonal
// Hadamard transform of Q and K ahead of FP8 quantisation spreads outlier
// channels over all dimensions; Ales Analytics "Attention and matrix kernels",
// "How it works": FP8 GEMMs carry a scale per block):
//   Q' = Q diag(signs) H / sqrt(d), K' = K diag(signs) H / sqrt(d), with H
//   the Sylvester Hadamard matrix and signs a random +-1 per channel given by
//   the caller, so Q' K'^T = Q K^T.  Q' and K' become E4M3 codes with one
//   scale per (batch, head, 128-token block); V (not rotated) one scale per
//   (batch, KV head), because its contraction runs over every key.  The
//   pages leave the form of a scale open: here it is the smallest power of
//   two 2^k with amax / 2^k <= 448 (448 = largest finite E4M3; k >= -126),
//   as in the OCP microscaling formats, so x / scale is an exact fp32
//   product and the code -- nearest E4M3 value, ties to even, saturating --
//   is decided on the exact value.
//
// How: HBM-bound work in two launches.
//   * fp8_rot_kernel (with a rotation): Q and K blocks on the tensor core and
//     V's block maxima, see its comment.
//   * fp8_quant_qk_kernel: one CTA per (tensor, batch, head, block) of 128
//     tokens x 128 channels.  A warp holds 16 rows, four channels per lane
//     (8-byte coalesced loads, all in flight at once), reduces the block
//     maximum, and writes the codes (128 contiguous bytes per row) and the
//     scale: Q and K without a rotation.  V blocks only record their maximum.
//   * fp8_quant_vt_kernel: one CTA per V block: the (batch, KV head) maximum
//     over its blocks, the codes, and a transpose (32-bit words through
//     shared memory, 4 x 4 bytes in registers) into the [B, Hkv, d,
//     vt_stride] layout whose rows of keys the attention kernel reads as the
//     K-major operand of P V.
#include <climits>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace fp8_impl {

constexpr int kD = 128;                        // channels (head dim)
constexpr int kBlock = 128;                    // tokens per scale block
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = kBlock / kWarps;  // 16
constexpr float kInvSqrtD = 0.08838834764831845f;   // 1 / sqrt(128)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Exponent k of a block's scale 2^k: the smallest with amax / 2^k <= 448
// (448 = 1.75 * 2^8), at least -126 so that 2^-k stays finite.  From the
// bits of amax >= 0: amax = 1.m * 2^E with E = field - 127; 1.m <= 1.75 (a
// mantissa field <= 0x600000) gives k = E - 8, else E - 7.  Sub-normal amax
// (field 0) is far below the clamp.
__device__ __forceinline__ int scale_exp(float amax) {
    const uint32_t u = __float_as_uint(amax);
    const int field = (int)(u >> 23);
    if (field == 0) return -126;
    const int k = field - 127 - ((u & 0x7FFFFFu) <= 0x600000u ? 8 : 7);
    return max(k, -126);
}

// 2^k as a float, k in [-126, 127].
__device__ __forceinline__ float pow2f(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

// Maximum over the CTA; every thread gets it.
__device__ __forceinline__ float block_max(float v, float *red) {
    #pragma unroll
    for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = red[0];
    #pragma unroll
    for (int w = 1; w < kWarps; ++w) r = fmaxf(r, red[w]);
    return r;
}

// Without a rotation: Q and K blocks scaled and quantised; V blocks: their
// maximum only.  blockIdx.x runs over the Q blocks, then K, then V, each
// (b, blk, h) with the head fastest, so CTAs running together read whole
// token rows (all heads) rather than one head's slice of many rows.  (With a rotation, fp8_rot_kernel does all of
// this.)
__global__ void __launch_bounds__(kThreads)
fp8_quant_qk_kernel(const Fp8PrepArgs a, int nblk) {
    __shared__ float red[kWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int idx = blockIdx.x;
    const int nq = a.B * a.Hq * nblk, nk = a.B * a.Hkv * nblk;
    int which, H;
    if (idx < nq) {
        which = 0;
        H = a.Hq;
    } else if (idx < nq + nk) {
        which = 1;
        H = a.Hkv;
        idx -= nq;
    } else {
        which = 2;
        H = a.Hkv;
        idx -= nq + nk;
    }
    const int h = idx % H, blk = (idx / H) % nblk, b = idx / (H * nblk);
    const int sidx = (b * H + h) * nblk + blk;   // [B, H, nblk] layout of the scales
    const uint16_t *src = static_cast<const uint16_t *>(which == 0 ? a.q : which == 1 ? a.k : a.v);
    const int n0 = blk * kBlock + warp * kRowsPerWarp;
    // all 16 row loads in flight before any arithmetic (8 bytes per lane,
    // 256 contiguous bytes per row)
    uint2 raw[kRowsPerWarp];
    #pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i)
        raw[i] = (n0 + i < a.N) ? __ldg(reinterpret_cast<const uint2 *>(
                                      src + (((size_t)b * a.N + n0 + i) * H + h) * kD) + lane)
                                : make_uint2(0u, 0u);
    float x[kRowsPerWarp][4];
    float amax = 0.f;
    #pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {              // rows past N are zeros
        x[i][0] = bf16_lo(raw[i].x);
        x[i][1] = bf16_hi(raw[i].x);
        x[i][2] = bf16_lo(raw[i].y);
        x[i][3] = bf16_hi(raw[i].y);
        #pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(x[i][e]));
    }
    amax = block_max(amax, red);
    if (which == 2) {
        if (threadIdx.x == 0) a.v_block_max[sidx] = amax;
        return;
    }
    const int kexp = amax > 0.f ? scale_exp(amax) : 0;
    const float mult = pow2f(-kexp);
    if (threadIdx.x == 0) (which == 0 ? a.q_scale : a.k_scale)[sidx] = pow2f(kexp);
    uint8_t *dst = static_cast<uint8_t *>(which == 0 ? a.q8 : a.k8);
    #pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int n = n0 + i;
        if (n < a.N)
            reinterpret_cast<uint32_t *>(dst + (((size_t)b * a.N + n) * H + h) * kD)[lane] =
                pack_e4m3x4(x[i][0] * mult, x[i][1] * mult, x[i][2] * mult, x[i][3] * mult);
    }
}

// ------------------------------------------------ rotation on the tensor core
// Q' = Q diag(signs) H is a dense 128 x 128 contraction per token: each
// 128-token block of one head is one M = N = K = 128 bf16 MMA against the
// +-1 matrix B[c][k] = signs[k] (-1)^popcount(k & c), which the CTA writes
// once into shared memory in the 128-byte-swizzled K-major layout a TMA tile
// has.  One persistent CTA per SM, warp-specialised:
//   * the last warp (one thread): TMA loads into a ring of kRotStages tiles
//     and the MMAs into two TMEM accumulators, paced by full / empty
//     mbarriers only; it writes each block's indices beside its tile, so the
//     epilogue reads them after the tile's full barrier (release / acquire);
//   * the other kRotEpiWarps warps: the epilogue, kRotCols channels of one
//     token row per thread (warps w, w + 4, .. share TMEM lanes 32 (w % 4)
//     ..): block maximum over the epilogue warps (a named barrier of their
//     own), power-of-two scale, E4M3 codes, kRotCols-byte stores.  A tile's
//     stage is released by the epilogue (not by the MMA), so a block's
//     indices stay in place until every epilogue thread has read them.
// After their Q and K blocks the same CTAs take V's blocks, reading the tile
// from shared memory for its maximum only.  fp32 accumulation of +-x terms:
// within a few ulp of the exact sums.
#ifndef FA_ROT_EPI_WARPS
#define FA_ROT_EPI_WARPS 8
#endif
constexpr int kRotEpiWarps = FA_ROT_EPI_WARPS;        // 8 or 16
constexpr int kRotCols = kD * 4 / kRotEpiWarps;        // channels per epilogue thread
static_assert(kRotEpiWarps == 8 || kRotEpiWarps == 16, "epilogue warps");
constexpr int kRotEpiThreads = kRotEpiWarps * 32;
constexpr int kRotThreads = kRotEpiThreads + 32;   // + the TMA / MMA warp
#ifndef FA_ROT_STAGES
#define FA_ROT_STAGES 4
#endif
constexpr int kRotStages = FA_ROT_STAGES;
constexpr int kRotTile = kBlock * kD * 2;          // one bf16 block: 32 KiB
constexpr int kRotBox = kBlock * 128;              // 128 rows x 64 bf16
constexpr int kRotSmem = (1 + kRotStages) * kRotTile + 1024;   // B, A ring, alignment
constexpr uint32_t kRotTmemCols = 256;             // two 128-column accumulators
constexpr int kRotEpiBar = 1;                      // named barrier of the epilogue warps

struct RotShared {
    uint64_t a_full[kRotStages], a_empty[kRotStages];
    uint64_t acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    int abort;
    int4 info[kRotStages];           // (tensor, batch, head, block) of each stage's tile
    float red[2][kRotEpiWarps];      // per-warp maxima, alternating by iteration
    float sgn[kD];
};

// Maximum of |v| over N values: eight independent chains, then a tree.
template <int N>
__device__ __forceinline__ float absmax(const float (&v)[N]) {
    float m[8];
    #pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fabsf(v[i]);
    #pragma unroll
    for (int e = 8; e < N; ++e) m[e & 7] = fmaxf(m[e & 7], fabsf(v[e]));
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])),
                 fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

__global__ void __launch_bounds__(kRotThreads, 1)
fp8_rot_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const Fp8PrepArgs a, int nblk) {
    extern __shared__ uint8_t rot_smem_raw[];
    __shared__ RotShared sh;
    const uint32_t base = smem_u32(rot_smem_raw);
    uint8_t *smem = rot_smem_raw + ((1024 - (base & 1023)) & 1023);
    uint8_t *sB = smem;
    uint8_t *sA = smem + kRotTile;                 // stage j at sA + j * kRotTile
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nq = a.B * a.Hq * nblk, nkv = a.B * a.Hkv * nblk;
    const int units = nq + 2 * nkv;                // Q blocks, K blocks, V blocks
    int my_units = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) ++my_units;
    volatile int *abort = &sh.abort;

    if (tid == 0) {
        for (int j = 0; j < kRotStages; ++j) {
            mbar_init(&sh.a_full[j], 1);
            mbar_init(&sh.a_empty[j], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sh.acc_full[j], 1);
            mbar_init(&sh.acc_empty[j], 1);
        }
        mbar_init(&sh.drain, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    if (tid < kD) sh.sgn[tid] = __ldg(a.signs + tid);
    if (warp == 0) tmem_alloc(&sh.tmem_base, kRotTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // unit -> tensor (0 Q, 1 K, 2 V), batch, head, block
    auto decode = [&](int u, int &which, int &b, int &h, int &blk) {
        which = u < nq ? 0 : (u < nq + nkv ? 1 : 2);
        const int H = which ? a.Hkv : a.Hq;
        const int v = u - (which == 0 ? 0 : (which == 1 ? nq : nq + nkv));
        h = v % H;
        blk = (v / H) % nblk;
        b = v / (H * nblk);
    };
    // A CTA's units run in increasing order, Q and K before V, so a Q or K
    // unit it is this CTA's it-th MMA: accumulator it & 1.
    auto is_qk = [&](int it) { return blockIdx.x + it * gridDim.x < nq + nkv; };
    const bool ctrl = warp == kRotEpiWarps && lane == 0;
    int issued = 0;                                // TMA loads (control thread)
    auto load = [&](int it) {
        const int st = it % kRotStages;
        int which, b, h, blk;
        decode(blockIdx.x + it * gridDim.x, which, b, h, blk);
        sh.info[st] = make_int4(which, b, h, blk);
        mbar_arrive_expect_tx(&sh.a_full[st], kRotTile);
        const CUtensorMap *m = which == 0 ? &tmQ : (which == 1 ? &tmK : &tmV);
        for (int bx = 0; bx < 2; ++bx)
            tma_load_3d(sA + st * kRotTile + bx * kRotBox, m, &sh.a_full[st], bx * 64, h,
                        b * a.N + blk * kBlock);
        ++issued;
    };
    // the first tiles' loads run while B is written
    if (ctrl) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        for (int it = 0; it < my_units && it < kRotStages; ++it) load(it);
    }
    // B: two boxes of 64 k-columns; row c, 16-byte chunk j (k = 64 box + 8 j ..)
    // at chunk position j ^ (c & 7)
    for (int ch = tid; ch < 2 * kD * 8; ch += kRotThreads) {
        const int box = ch >> 10, c = (ch >> 3) & (kD - 1), j = ch & 7;
        uint32_t w[4];
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int k0 = box * 64 + j * 8 + 2 * e, k1 = k0 + 1;
            const bool n0 = (sh.sgn[k0] < 0.f) != ((__popc(k0 & c) & 1) != 0);
            const bool n1 = (sh.sgn[k1] < 0.f) != ((__popc(k1 & c) & 1) != 0);
            w[e] = (n0 ? 0xBF80u : 0x3F80u) | ((n1 ? 0xBF80u : 0x3F80u) << 16);
        }
        *reinterpret_cast<uint4 *>(sB + box * kRotBox + c * 128 + ((j ^ (c & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
    __syncthreads();
    const uint32_t tmem = sh.tmem_base;

    if (warp == kRotEpiWarps) {
        // ---------------- control: MMAs and the loads that refill the ring.
        // Both wait on the epilogue (an accumulator, a stage), in different
        // orders, so neither blocks the other: poll and issue whichever is
        // ready, giving up after kWaitLimitCycles without progress.
        if (ctrl) {
            const uint32_t b_lo = desc_lo(smem_u32(sB), 16), a_lo = desc_lo(smem_u32(sA), 16);
            const uint32_t idesc = idesc_bf16_f32(kBlock, kD, false);
            int it_mma = 0;
            long long t_progress = clock64();
            for (uint32_t spin = 0; it_mma < my_units || issued < my_units; ++spin) {
                bool progressed = false;
                if (it_mma < my_units) {
                    const int st = it_mma % kRotStages;
                    if (!is_qk(it_mma)) {
                        ++it_mma;                  // V: no MMA
                        progressed = true;
                    } else if (mbar_test(smem_u32(&sh.acc_empty[it_mma & 1]),
                                         ((it_mma >> 1) & 1) ^ 1) &&
                               mbar_test(smem_u32(&sh.a_full[st]), (it_mma / kRotStages) & 1)) {
                        tc_fence_after();
                        const uint32_t aa = a_lo + st * (kRotTile >> 4);
                        #pragma unroll
                        for (int ks = 0; ks < kD / 16; ++ks) {
                            const uint32_t off = ((ks >> 2) * kRotBox + (ks & 3) * 32) >> 4;
                            mma_ss_lo(tmem + (it_mma & 1) * kD, aa + off, b_lo + off, idesc,
                                      ks > 0 ? 1u : 0u);
                        }
                        tc_commit(&sh.acc_full[it_mma & 1]);
                        ++it_mma;
                        progressed = true;
                    }
                }
                if (issued < my_units) {
                    // load `issued` reuses the stage of unit issued - kRotStages
                    const int prev = issued - kRotStages;
                    if (mbar_test(smem_u32(&sh.a_empty[prev % kRotStages]), (prev / kRotStages) & 1)) {
                        load(issued);
                        progressed = true;
                    }
                }
                if (progressed) {
                    t_progress = clock64();
                } else if ((spin & 63) == 0) {
                    if (*abort) break;
                    if (clock64() - t_progress > kWaitLimitCycles) {
                        *abort = 1;
                        report_error(kDevErrTimeout);
                        break;
                    }
                }
            }
            // leave no copy or MMA in flight: the last load of every stage, then
            // every MMA issued
            for (int st = 0; st < kRotStages; ++st)
                if (issued > st) mbar_drain_wait(&sh.a_full[st], ((issued - 1 - st) / kRotStages) & 1);
            tc_commit(&sh.drain);
            mbar_drain_wait(&sh.drain, 0);
        }
    } else {
        // ---------------- epilogue
        const int row = (warp & 3) * 32 + lane;    // token row of the block
        const int col0 = (warp >> 2) * kRotCols;   // first channel of this thread
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16) + col0;
        bool ok = true;
        for (int it = 0; it < my_units; ++it) {
            const int st = it % kRotStages;
            const bool qk = is_qk(it);
            ok = ok && mbar_wait(&sh.a_full[st], (it / kRotStages) & 1, abort);
            if (qk) ok = ok && mbar_wait(&sh.acc_full[it & 1], (it >> 1) & 1, abort);
            tc_fence_after();
            const int4 inf = sh.info[st];
            const int which = inf.x, b = inf.y, h = inf.z, blk = inf.w;
            const int n = blk * kBlock + row;      // this thread's token (rows past N:
            const bool valid = n < a.N;            // the next batch or zeros -- left out)
            float v[kRotCols];
            float m = 0.f;
            if (ok && qk) {
                #pragma unroll
                for (int q = 0; q < kRotCols / 32; ++q)
                    tmem_ld32(trow + (it & 1) * kD + q * 32, reinterpret_cast<uint32_t *>(v) + 32 * q);
                tmem_wait_ld();
            } else if (ok) {
                // V: this row's bf16 channels col0 .. from box col0 / 64, chunks
                // swizzled by row & 7
                const uint8_t *src = sA + st * kRotTile + (col0 / 64) * kRotBox + row * 128;
                #pragma unroll
                for (int c = 0; c < kRotCols / 8; ++c) {
                    const int ch = (col0 % 64) / 8 + c;
                    const uint4 q = *reinterpret_cast<const uint4 *>(src + ((ch ^ (row & 7)) << 4));
                    v[8 * c + 0] = bf16_lo(q.x); v[8 * c + 1] = bf16_hi(q.x);
                    v[8 * c + 2] = bf16_lo(q.y); v[8 * c + 3] = bf16_hi(q.y);
                    v[8 * c + 4] = bf16_lo(q.z); v[8 * c + 5] = bf16_hi(q.z);
                    v[8 * c + 6] = bf16_lo(q.w); v[8 * c + 7] = bf16_hi(q.w);
                }
            }
            if (ok && valid) m = absmax<kRotCols>(v);
            #pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float *red = sh.red[it & 1];
            if (lane == 0) red[warp] = m;
            // after this barrier every epilogue thread holds its values in
            // registers: the accumulator (or tile) goes back to the control
            // warp; red[] of this iteration is rewritten two iterations on
            tc_fence_before();
            ok = named_bar_and(kRotEpiBar, kRotEpiThreads, ok);
            if (!ok) break;
            if (tid == 0) {
                if (qk) mbar_arrive(&sh.acc_empty[it & 1]);
                mbar_arrive(&sh.a_empty[st]);
            }
            float r4[kRotEpiWarps / 4];
            #pragma unroll
            for (int i = 0; i < kRotEpiWarps / 4; ++i)
                r4[i] = fmaxf(fmaxf(red[4 * i], red[4 * i + 1]), fmaxf(red[4 * i + 2], red[4 * i + 3]));
            float amax = r4[0];
            #pragma unroll
            for (int i = 1; i < kRotEpiWarps / 4; ++i) amax = fmaxf(amax, r4[i]);
            if (which == 2) {
                if (tid == 0) a.v_block_max[(b * a.Hkv + h) * nblk + blk] = amax;
            } else {
                // the accumulator is H diag(signs) x; Q' = that / sqrt(128)
                const float amax_c = amax * kInvSqrtD;
                const int kexp = amax_c > 0.f ? scale_exp(amax_c) : 0;
                const float mult = kInvSqrtD * pow2f(-kexp);
                const int H = which ? a.Hkv : a.Hq;
                if (tid == 0) (which ? a.k_scale : a.q_scale)[(b * H + h) * nblk + blk] = pow2f(kexp);
                if (valid) {
                    uint32_t cw[kRotCols / 4];
                    #pragma unroll
                    for (int e = 0; e < kRotCols / 4; ++e)
                        cw[e] = pack_e4m3x4(v[4 * e] * mult, v[4 * e + 1] * mult,
                                            v[4 * e + 2] * mult, v[4 * e + 3] * mult);
                    uint4 *d4 = reinterpret_cast<uint4 *>(
                        static_cast<uint8_t *>(which ? a.k8 : a.q8) +
                        (((size_t)b * a.N + n) * H + h) * kD + col0);
                    #pragma unroll
                    for (int e = 0; e < kRotCols / 16; ++e)
                        d4[e] = make_uint4(cw[4 * e], cw[4 * e + 1], cw[4 * e + 2], cw[4 * e + 3]);
                }
            }
        }
        if (!ok) *abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kRotTmemCols);
}

// V codes, transposed: CTA (b * nblk + blk) * Hkv + h (head fastest, as
// above) writes rows c = 0..127 of (b, h) for keys blk * 128 .. + 127 (those
// below N).  The block goes through shared
// memory as 32-bit words (four channels of one token), column-swizzled by
// token / 4 so that both phases are free of bank conflicts; each lane then
// turns a 4 x 4 byte block (four tokens x four channels) around in registers
// and stores four 4-byte pieces of four V^T rows, a warp 128 bytes per row.
__global__ void __launch_bounds__(kThreads)
fp8_quant_vt_kernel(const Fp8PrepArgs a, int nblk) {
    __shared__ uint32_t sW[kBlock][kD / 4];   // [token][channel group ^ (token / 4)]
    __shared__ float red[kWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = blockIdx.x % a.Hkv, blk = (blockIdx.x / a.Hkv) % nblk;
    const int b = blockIdx.x / (a.Hkv * nblk), bh = b * a.Hkv + h;
    const int n0 = blk * kBlock;
    const uint16_t *src = static_cast<const uint16_t *>(a.v);
    // the block's rows in flight while the (b, h) maximum is reduced
    uint2 raw[kRowsPerWarp];
    #pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int n = n0 + warp * kRowsPerWarp + i;
        raw[i] = (n < a.N) ? __ldg(reinterpret_cast<const uint2 *>(
                                 src + (((size_t)b * a.N + n) * a.Hkv + h) * kD) + lane)
                           : make_uint2(0u, 0u);
    }
    float amax = 0.f;
    for (int i = threadIdx.x; i < nblk; i += kThreads)
        amax = fmaxf(amax, a.v_block_max[(size_t)bh * nblk + i]);
    amax = block_max(amax, red);
    const int kexp = amax > 0.f ? scale_exp(amax) : 0;
    const float inv = pow2f(-kexp);
    if (threadIdx.x == 0 && blk == 0) a.v_scale[bh] = pow2f(kexp);
    #pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int nl = warp * kRowsPerWarp + i;
        sW[nl][lane ^ ((nl >> 2) & 31)] =
            pack_e4m3x4(bf16_lo(raw[i].x) * inv, bf16_hi(raw[i].x) * inv,
                        bf16_lo(raw[i].y) * inv, bf16_hi(raw[i].y) * inv);
    }
    __syncthreads();
    const int nvalid = min(kBlock, a.N - n0);
    uint8_t *dst = static_cast<uint8_t *>(a.vt8) + (size_t)bh * kD * a.vt_stride + n0;
    const int t0 = 4 * lane;                    // tokens t0 .. t0 + 3 of the block
    #pragma unroll
    for (int g = 0; g < kD / 4 / kWarps; ++g) {
        const int cg = warp * (kD / 4 / kWarps) + g;   // channels 4 cg .. 4 cg + 3
        const int col = cg ^ lane;
        const uint32_t w0 = sW[t0][col], w1 = sW[t0 + 1][col];
        const uint32_t w2 = sW[t0 + 2][col], w3 = sW[t0 + 3][col];
        // byte e of word r = channel 4 cg + e of token t0 + r  ->  o[e]
        const uint32_t u0 = __byte_perm(w0, w1, 0x5140), u1 = __byte_perm(w0, w1, 0x7362);
        const uint32_t u2 = __byte_perm(w2, w3, 0x5140), u3 = __byte_perm(w2, w3, 0x7362);
        const uint32_t o[4] = {__byte_perm(u0, u2, 0x5410), __byte_perm(u0, u2, 0x7632),
                               __byte_perm(u1, u3, 0x5410), __byte_perm(u1, u3, 0x7632)};
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint8_t *row = dst + (size_t)(4 * cg + e) * a.vt_stride;
            if (t0 + 4 <= nvalid) {
                *reinterpret_cast<uint32_t *>(row + t0) = o[e];
            } else {
                for (int k = 0; k < 4; ++k)
                    if (t0 + k < nvalid) row[t0 + k] = (uint8_t)(o[e] >> (8 * k));
            }
        }
    }
}

}  // namespace fp8_impl

int launch_fp8_prepare(const Fp8PrepArgs &a, cudaStream_t stream) {
    using namespace fp8_impl;
    if (a.d != kD) return -2;
    const long long nblk = (a.N + kBlock - 1) / kBlock;
    const long long nq = (long long)a.B * a.Hq * nblk, nkv = (long long)a.B * a.Hkv * nblk;
    if (nq <= 0) return 0;
    if (nq + 2 * nkv > INT_MAX) return -2;
    if (a.signs) {
        // Q and K on the tensor core, V's block maxima in the same kernel
        alignas(64) CUtensorMap tq, tk, tv;
        const uint64_t T = (uint64_t)a.B * a.N;
        if (encode_tensor_map_3d(&tq, a.q, 2, kD, a.Hq, T, (uint64_t)kD * 2,
                                 (uint64_t)a.Hq * kD * 2, 64, 1, kBlock, 128) ||
            encode_tensor_map_3d(&tk, a.k, 2, kD, a.Hkv, T, (uint64_t)kD * 2,
                                 (uint64_t)a.Hkv * kD * 2, 64, 1, kBlock, 128) ||
            encode_tensor_map_3d(&tv, a.v, 2, kD, a.Hkv, T, (uint64_t)kD * 2,
                                 (uint64_t)a.Hkv * kD * 2, 64, 1, kBlock, 128))
            return -5;
        if (cudaFuncSetAttribute(fp8_rot_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kRotSmem) != cudaSuccess)
            return -5;
        const long long units = nq + 2 * nkv;
        const long long cap = device_sm_count();
        const int grid = (int)(units < cap ? units : cap);
        fp8_rot_kernel<<<grid, kRotThreads, kRotSmem, stream>>>(tq, tk, tv, a, (int)nblk);
    } else {
        fp8_quant_qk_kernel<<<(int)(nq + 2 * nkv), kThreads, 0, stream>>>(a, (int)nblk);
    }
    fp8_quant_vt_kernel<<<(int)nkv, kThreads, 0, stream>>>(a, (int)nblk);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace fa

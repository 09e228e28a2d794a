// fp8_prep.cu -- operands of the FP8 prefill.
//
// What it computes ("FlashAttention-3" in samanvya.dev's "Attention Is the
// Bottleneck", "FlashAttention: same math, different IO": Q and K are
// multiplied by a random orthogonal Hadamard matrix before FP8 quantisation,
// which spreads outlier channels over all dimensions; "Low precision" in the
// same post: FP8 GEMMs carry per-block scales):
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
// How: HBM-bound elementwise work, two launches.
//   * fp8_quant_qk_kernel: one CTA per (tensor, batch, head, block) of 128
//     tokens x 128 channels.  A warp holds 16 rows, four channels per lane
//     (8-byte coalesced loads), rotates each row with an in-warp fast
//     Walsh-Hadamard transform (two butterfly levels in registers, five by
//     lane shuffles), reduces the block maximum, and writes the codes (128
//     contiguous bytes per row) and the scale.  V blocks only record their
//     maximum.
//   * fp8_quant_vt_kernel: one CTA per V block: the (batch, KV head) maximum
//     over its blocks, the codes, and a transpose through shared memory into
//     the [B, Hkv, d, vt_stride] layout whose rows of keys the attention
//     kernel reads as the K-major operand of P V.
#include <climits>
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

// H x for one 128-vector held as x[e] = element 4 * lane + e: butterflies
// (a, b) -> (a + b, a - b) over index bits 0-1 in registers and bits 2-6
// across lanes.  H is the Sylvester Hadamard matrix, (i, k) entry
// (-1)^popcount(i & k).
__device__ __forceinline__ void fwht128(float (&x)[4], int lane) {
    const float a0 = x[0] + x[1], a1 = x[0] - x[1];
    const float a2 = x[2] + x[3], a3 = x[2] - x[3];
    x[0] = a0 + a2;
    x[2] = a0 - a2;
    x[1] = a1 + a3;
    x[3] = a1 - a3;
    #pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float p = __shfl_xor_sync(0xffffffffu, x[e], m);
            x[e] = upper ? p - x[e] : x[e] + p;
        }
    }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Exponent k of a block's scale 2^k: the smallest with amax / 2^k <= 448
// (448 = 0.875 * 2^9), at least -126 so that 2^-k stays finite.
__device__ __forceinline__ int scale_exp(float amax) {
    int e;
    const float f = frexpf(amax, &e);   // amax = f * 2^e, f in [0.5, 1)
    return max((f <= 0.875f) ? e - 9 : e - 8, -126);
}

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

// Q and K blocks: rotate, scale, quantise.  V blocks: their maximum only.
// blockIdx.x runs over the Q blocks, then K, then V, each (b, h, blk) with
// blk fastest.
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
    const int blk = idx % nblk, h = (idx / nblk) % H, b = idx / (nblk * H);
    const uint16_t *src = static_cast<const uint16_t *>(which == 0 ? a.q : which == 1 ? a.k : a.v);
    const bool rotate = which < 2 && a.signs != nullptr;
    float sg[4] = {1.f, 1.f, 1.f, 1.f};
    if (rotate) {
        const float4 s4 = __ldg(reinterpret_cast<const float4 *>(a.signs) + lane);
        sg[0] = s4.x; sg[1] = s4.y; sg[2] = s4.z; sg[3] = s4.w;
    }
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
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int n = n0 + i;                    // warp-uniform
        if (n < a.N) {
            x[i][0] = bf16_lo(raw[i].x);
            x[i][1] = bf16_hi(raw[i].x);
            x[i][2] = bf16_lo(raw[i].y);
            x[i][3] = bf16_hi(raw[i].y);
            if (rotate) {
                #pragma unroll
                for (int e = 0; e < 4; ++e) x[i][e] *= sg[e];
                fwht128(x[i], lane);
                #pragma unroll
                for (int e = 0; e < 4; ++e) x[i][e] *= kInvSqrtD;
            }
        } else {
            #pragma unroll
            for (int e = 0; e < 4; ++e) x[i][e] = 0.f;
        }
        #pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(x[i][e]));
    }
    amax = block_max(amax, red);
    if (which == 2) {
        if (threadIdx.x == 0) a.v_block_max[idx] = amax;
        return;
    }
    const int kexp = amax > 0.f ? scale_exp(amax) : 0;
    const float inv = ldexpf(1.f, -kexp);
    if (threadIdx.x == 0) (which == 0 ? a.q_scale : a.k_scale)[idx] = ldexpf(1.f, kexp);
    uint8_t *dst = static_cast<uint8_t *>(which == 0 ? a.q8 : a.k8);
    #pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int n = n0 + i;
        if (n < a.N)
            reinterpret_cast<uint32_t *>(dst + (((size_t)b * a.N + n) * H + h) * kD)[lane] =
                pack_e4m3x4(x[i][0] * inv, x[i][1] * inv, x[i][2] * inv, x[i][3] * inv);
    }
}

// V codes, transposed: CTA (b * Hkv + h) * nblk + blk writes rows c = 0..127
// of keys blk * 128 .. + 127 (those below N).
__global__ void __launch_bounds__(kThreads)
fp8_quant_vt_kernel(const Fp8PrepArgs a, int nblk) {
    __shared__ uint8_t sT[kD][kBlock + 1];   // [channel][token]; odd row length: no bank conflicts
    __shared__ float red[kWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int blk = blockIdx.x % nblk, bh = blockIdx.x / nblk;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
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
    const float inv = ldexpf(1.f, -kexp);
    if (threadIdx.x == 0 && blk == 0) a.v_scale[bh] = ldexpf(1.f, kexp);
    #pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int nl = warp * kRowsPerWarp + i;
        const uint32_t w = pack_e4m3x4(bf16_lo(raw[i].x) * inv, bf16_hi(raw[i].x) * inv,
                                       bf16_lo(raw[i].y) * inv, bf16_hi(raw[i].y) * inv);
        #pragma unroll
        for (int e = 0; e < 4; ++e) sT[4 * lane + e][nl] = (uint8_t)(w >> (8 * e));
    }
    __syncthreads();
    const int nvalid = min(kBlock, a.N - n0);
    uint8_t *dst = static_cast<uint8_t *>(a.vt8) + (size_t)bh * kD * a.vt_stride + n0;
    const int t0 = 4 * lane;
    #pragma unroll 4
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int c = warp * kRowsPerWarp + i;
        uint8_t *row = dst + (size_t)c * a.vt_stride;
        if (t0 + 4 <= nvalid) {
            const uint32_t w = (uint32_t)sT[c][t0] | ((uint32_t)sT[c][t0 + 1] << 8) |
                               ((uint32_t)sT[c][t0 + 2] << 16) | ((uint32_t)sT[c][t0 + 3] << 24);
            *reinterpret_cast<uint32_t *>(row + t0) = w;
        } else {
            for (int e = 0; e < 4; ++e)
                if (t0 + e < nvalid) row[t0 + e] = sT[c][t0 + e];
        }
    }
}

}  // namespace fp8_impl

int launch_fp8_prepare(const Fp8PrepArgs &a, cudaStream_t stream) {
    using namespace fp8_impl;
    if (a.d != kD) return -2;
    const long long nblk = (a.N + kBlock - 1) / kBlock;
    const long long grid_a = (long long)a.B * (a.Hq + 2 * a.Hkv) * nblk;
    const long long grid_b = (long long)a.B * a.Hkv * nblk;
    if (grid_a <= 0) return 0;
    if (grid_a > INT_MAX) return -2;
    fp8_quant_qk_kernel<<<(int)grid_a, kThreads, 0, stream>>>(a, (int)nblk);
    fp8_quant_vt_kernel<<<(int)grid_b, kThreads, 0, stream>>>(a, (int)nblk);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace fa

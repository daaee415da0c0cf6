// ln_kernel.cu -- LayerNorm (no affine) with per-chunk adaLN modulation, the step
// before the QKV projection and before the feed-forward layer of a DiT block.
//
// The wave of "Wave Forcing" (abstract) holds chunks at different denoising
// steps, so each chunk carries its own modulation: row n of the wave uses row
// n / rows_per_group of shift and scale.  y = (x - mean) / sqrt(var + eps) *
// (1 + scale) + shift, with the mean and the (biased) variance over the row,
// fp32 arithmetic and one rounding to bf16.
//
// HBM-bound: 2 bytes read and 2 written per element (the modulation tables are
// small; each block stages its rows' group in shared memory).  One warp per
// row; lane l owns the 16-byte pieces l, l + 32, ... of the row, all loaded
// before the reductions.  The kernel is instantiated for a few counts of pieces
// per lane, so that a row of C channels holds no more registers than it needs
// (occupancy sets the bytes in flight).
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

constexpr int kMaxPieces = 24;      // 16-byte pieces per lane: C <= 32 * 24 * 8 = 6144
constexpr int kRowsPerBlock = 8;

template <int kPer>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
layer_norm_modulate_kernel(const uint16_t *__restrict__ x, const float *__restrict__ shift,
                           const float *__restrict__ scale, uint16_t *__restrict__ y, long M, int C,
                           int rows_per_group, float eps)
{
    // shift and scale of the group of the block's first row, staged while the
    // row loads are in flight (a block's rows straddle two groups only at a
    // chunk boundary; such rows read their own group's rows from global memory).
    // Staged de-interleaved: the first four floats of every 8-float piece, then
    // the last four, so that a warp's 16-byte reads of one half are contiguous
    // (interleaved, lanes 32 bytes apart would take twice the wavefronts).
    extern __shared__ float4 s_mod[];            // shift lo, shift hi, scale lo, scale hi: [C/8] each
    const int lane = threadIdx.x & 31;
    const long row0 = static_cast<long>(blockIdx.x) * kRowsPerBlock;
    const long row = row0 + (threadIdx.x >> 5);
    const bool live = row < M;
    const int pieces = C / 8;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (live ? row : row0) * C);
    uint4 w[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = lane + 32 * i;
        w[i] = (live && j < pieces) ? __ldcs(src + j) : make_uint4(0u, 0u, 0u, 0u);
    }
    const long g0 = row0 / rows_per_group;
    const int q = C / 8;                         // pieces per row
    {
        const float4 *sh = reinterpret_cast<const float4 *>(shift + g0 * C);
        const float4 *sc = reinterpret_cast<const float4 *>(scale + g0 * C);
        for (int i = threadIdx.x; i < C / 4; i += 32 * kRowsPerBlock) {
            const int piece = i >> 1, half = i & 1;
            s_mod[half * q + piece] = __ldg(sh + i);
            s_mod[2 * q + half * q + piece] = __ldg(sc + i);
        }
    }
    __syncthreads();
    if (!live) return;                      // whole warps leave together
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            s += __uint_as_float(u[e] << 16) + __uint_as_float(u[e] & 0xFFFF0000u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    const float mean = s / static_cast<float>(C);
    float v = 0.0f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        if (lane + 32 * i >= pieces) break;
        const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = __uint_as_float(u[e] << 16) - mean;
            const float b = __uint_as_float(u[e] & 0xFFFF0000u) - mean;
            v = fmaf(a, a, fmaf(b, b, v));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const float rstd = rsqrtf(v / static_cast<float>(C) + eps);
    const long g = row / rows_per_group;
    const bool staged = g == g0;
    const float4 *sh4 = reinterpret_cast<const float4 *>(shift + g * C);
    const float4 *sc4 = reinterpret_cast<const float4 *>(scale + g * C);
    uint4 *dst = reinterpret_cast<uint4 *>(y + row * C);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = lane + 32 * i;
        if (j >= pieces) break;
        const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
        const float4 sa = staged ? s_mod[j] : __ldg(sh4 + 2 * j);
        const float4 sb = staged ? s_mod[q + j] : __ldg(sh4 + 2 * j + 1);
        const float4 ca = staged ? s_mod[2 * q + j] : __ldg(sc4 + 2 * j);
        const float4 cb = staged ? s_mod[3 * q + j] : __ldg(sc4 + 2 * j + 1);
        const float shv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        const float scv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = (__uint_as_float(u[e] << 16) - mean) * rstd;
            const float b = (__uint_as_float(u[e] & 0xFFFF0000u) - mean) * rstd;
            o[e] = pack_bf16x2(fmaf(a, 1.0f + scv[2 * e], shv[2 * e]),
                               fmaf(b, 1.0f + scv[2 * e + 1], shv[2 * e + 1]));
        }
        dst[j] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

int ln_max_channels() { return 32 * kMaxPieces * 8; }

cudaError_t launch_layer_norm_modulate(const uint16_t *x, const float *shift, const float *scale,
                                       uint16_t *y, long M, int C, int rows_per_group, float eps,
                                       cudaStream_t stream)
{
    if (M == 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>((M + kRowsPerBlock - 1) / kRowsPerBlock));
    const int per_lane = (C / 8 + 31) / 32;
    auto go = [&](auto kern) {
        kern<<<grid, 32 * kRowsPerBlock, 2 * C * sizeof(float), stream>>>(x, shift, scale, y, M,
                                                                           C, rows_per_group, eps);
    };
    if (per_lane <= 2)
        go(layer_norm_modulate_kernel<2>);
    else if (per_lane <= 4)
        go(layer_norm_modulate_kernel<4>);
    else if (per_lane <= 6)
        go(layer_norm_modulate_kernel<6>);
    else if (per_lane <= 8)
        go(layer_norm_modulate_kernel<8>);
    else if (per_lane <= 12)
        go(layer_norm_modulate_kernel<12>);
    else if (per_lane <= 16)
        go(layer_norm_modulate_kernel<16>);
    else if (per_lane <= 20)
        go(layer_norm_modulate_kernel<20>);
    else
        go(layer_norm_modulate_kernel<kMaxPieces>);
    return cudaGetLastError();
}

}  // namespace wf

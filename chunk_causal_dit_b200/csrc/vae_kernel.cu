// vae_kernel.cu -- the per-pixel RMSNorm + SiLU of the streaming VAE-decode stage.
//
// "Wave Forcing" (abstract) decodes the generated chunks with a pipelined VAE;
// the pages print none of its layers.  In the causal 3D-conv decoder stage built
// here each convolution's input is y = x / sqrt(mean_c x^2 + eps) * gamma
// followed by SiLU, y * sigmoid(y), over the channels of one pixel
// (channels-last [pixels][C] bf16, gamma [C] fp32, fp32 arithmetic, one rounding
// to bf16).
//
// HBM-bound (4 bytes per element; the IEEE division of SiLU made it MUFU- and
// issue-bound, 4.1 TB/s).  Half a warp per pixel: lane l of the half
// holds the 8-channel pieces l, l + 16, ... of the row in registers between the
// sum of squares and the output pass (3 pieces per lane at C = 384), so every
// lane keeps several 16-byte loads in flight; gamma is read through the
// read-only path.
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

constexpr int kWarps = 8;
constexpr int kLanesPerRow = 16;
constexpr int kRowsPerBlock = kWarps * 32 / kLanesPerRow;

template <int PPL>    // 8-channel pieces per lane (C <= 8 * 16 * PPL)
__global__ void __launch_bounds__(32 * kWarps) rms_norm_silu_kernel(const uint16_t *__restrict__ x,
                                                                    const float *__restrict__ gamma,
                                                                    uint16_t *__restrict__ y,
                                                                    long M, int C, float eps)
{
    const int sub = threadIdx.x & (kLanesPerRow - 1);
    const long row = static_cast<long>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kLanesPerRow;
    const bool live = row < M;            // both halves of a warp take part in the shuffles
    const int pieces = C / 8;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (live ? row : 0) * C);
    uint4 u[PPL];
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
        const int pc = sub + kLanesPerRow * i;
        u[i] = live && pc < pieces ? __ldcs(src + pc) : make_uint4(0u, 0u, 0u, 0u);
    }
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
        const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = __uint_as_float(w[e] << 16), b = __uint_as_float(w[e] & 0xFFFF0000u);
            ss = fmaf(a, a, fmaf(b, b, ss));
        }
    }
#pragma unroll
    for (int o = kLanesPerRow / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (!live) return;
    const float r = rsqrtf(ss / static_cast<float>(C) + eps);
    uint4 *dst = reinterpret_cast<uint4 *>(y + row * C);
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
        const int pc = sub + kLanesPerRow * i;
        if (pc >= pieces) break;
        const float4 *g4 = reinterpret_cast<const float4 *>(gamma + 8 * pc);
        const float4 ga = __ldg(g4), gb = __ldg(g4 + 1);
        const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
        const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float a = __uint_as_float(w[e] << 16) * r * g[2 * e];
            float b = __uint_as_float(w[e] & 0xFFFF0000u) * r * g[2 * e + 1];
            // SiLU as y / (1 + e^-y) with the approximate exponential and division
            // (two MUFU operations, ~2^-21 relative error); a huge e^-y gives -0
            a = __fdividef(a, 1.0f + __expf(-a));
            b = __fdividef(b, 1.0f + __expf(-b));
            o[e] = pack_bf16x2(a, b);
        }
        __stcs(dst + pc, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

}  // namespace

int rms_norm_silu_max_channels() { return 8 * kLanesPerRow * 4; }

cudaError_t launch_rms_norm_silu(const uint16_t *x, const float *gamma, uint16_t *y, long M, int C,
                                 float eps, cudaStream_t stream)
{
    if (M == 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>((M + kRowsPerBlock - 1) / kRowsPerBlock));
    const int ppl = (C / 8 + kLanesPerRow - 1) / kLanesPerRow;
    switch (ppl) {
    case 1: rms_norm_silu_kernel<1><<<grid, 32 * kWarps, 0, stream>>>(x, gamma, y, M, C, eps); break;
    case 2: rms_norm_silu_kernel<2><<<grid, 32 * kWarps, 0, stream>>>(x, gamma, y, M, C, eps); break;
    case 3: rms_norm_silu_kernel<3><<<grid, 32 * kWarps, 0, stream>>>(x, gamma, y, M, C, eps); break;
    default: rms_norm_silu_kernel<4><<<grid, 32 * kWarps, 0, stream>>>(x, gamma, y, M, C, eps); break;
    }
    return cudaGetLastError();
}

}  // namespace wf

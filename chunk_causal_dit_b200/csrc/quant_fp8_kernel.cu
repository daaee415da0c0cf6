// quant_fp8_kernel.cu -- E4M3 quantization of q_out (one scale per token and head)
// and of key-cache chunks (one scale per 128-row key tile and head), the inputs of
// the FP8 Q.K^T attention variant.
//
// The quantized Q.K^T is the B200 counterpart of the quantized attention backend
// the pages run their systems on ("Wave Forcing", abstract: SageAttention with
// W8A8 backends): scores come from 8-bit operands with per-block fp32 scales,
// while P.V stays in bf16.
//
// Rule (exact, bit-for-bit what the oracle computes): fp8_rule.cuh, applied to
// a row for Q and to a 128-row key tile of one head for K.
//
// Both kernels are HBM-bound: 2 bytes read and 1 byte written per element.
#include <cuda_bf16.h>

#include "fp8_rule.cuh"
#include "wf_check.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Rows of q [N][H][D] bf16 (row = n * H + h) -> q8 [N][H][D], scale [H][N].
// A row is D * 2 bytes = D / 8 lanes of 16 bytes; each warp takes 4 loads of
// 32 / (D / 8) rows, all issued before any reduction.
template <int D>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t *__restrict__ q,
                                                            uint8_t *__restrict__ q8,
                                                            float *__restrict__ scale, long n_rows,
                                                            int H, DeviceWords *words)
{
    constexpr int kLanesPerRow = D / 8;
    constexpr int kRowsPerLoad = 32 / kLanesPerRow;
    constexpr int kLoads = 4;
    constexpr int kRowsPerWarp = kLoads * kRowsPerLoad;
    const int lane = threadIdx.x & 31;
    const int sub = lane / kLanesPerRow;              // row within one load
    const int part = lane % kLanesPerRow;             // 16-byte piece of the row
    const long row0 = (static_cast<long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kRowsPerWarp;
    uint4 w[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const long row = row0 + i * kRowsPerLoad + sub;
        w[i] = row < n_rows ? __ldcs(reinterpret_cast<const uint4 *>(q + row * D) + part)
                            : make_uint4(0, 0, 0, 0);
    }
    const long n_tok = n_rows / H;
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const long row = row0 + i * kRowsPerLoad + sub;
        const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
        float x[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            x[2 * k] = bf16_lo(u[k]);
            x[2 * k + 1] = bf16_hi(u[k]);
        }
        float a = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) a = fmaxf(a, fabsf(x[k]));
#pragma unroll
        for (int o = kLanesPerRow / 2; o > 0; o >>= 1)
            a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        if (row < n_rows) {
            const float inv = fp8_inv(a);
            const uint2 c = make_uint2(quant4(x[0], x[1], x[2], x[3], inv),
                                       quant4(x[4], x[5], x[6], x[7], inv));
            reinterpret_cast<uint2 *>(q8 + row * D)[part] = c;
            if (part == 0) {
                const long n = row / H;
                const int h = static_cast<int>(row - n * H);
                if (WF_BOUNDS(n < n_tok && h < H, words, kSiteQuantRows))
                    scale[static_cast<long>(h) * n_tok + n] = fp8_scale(a);
            }
        }
    }
}

// One block (8 warps) per (chunk, key tile, head): the tile's rows of one head
// [R][L][H][D] bf16 -> codes in the same layout, scale [R][n_tiles][H].  A row is
// D / 8 lanes of 16 bytes; each warp loads 128 / 8 = 16 rows in kLoads loads of
// 32 / (D / 8) rows and keeps them in registers between the amax and the
// quantize passes.
template <int D>
__global__ void __launch_bounds__(256) quantize_tiles_kernel(const uint16_t *__restrict__ k,
                                                             uint8_t *__restrict__ k8,
                                                             float *__restrict__ scale,
                                                             long first_chunk, int L, int H, int R,
                                                             DeviceWords *words)
{
    constexpr int kLanesPerRow = D / 8;
    constexpr int kRowsPerLoad = 32 / kLanesPerRow;
    constexpr int kLoads = 16 / kRowsPerLoad;   // 16 rows per warp, 8 warps = 128 rows
    __shared__ float s_max[8];
    const int n_tiles = (L + 127) / 128;
    const int chunk = blockIdx.x / n_tiles;     // index within the quantized range
    const int t = blockIdx.x - chunk * n_tiles;
    const int h = blockIdx.y;
    const int slot = ring_slot(first_chunk + chunk, R);
    if (!WF_BOUNDS(slot >= 0 && slot < R && t < n_tiles && h < H, words, kSiteQuantTiles))
        return;                                  // whole block: uniform
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / kLanesPerRow, part = lane % kLanesPerRow;
    const long slot_base = static_cast<long>(slot) * L;
    const int row_base = t * 128 + warp * 16;

    uint4 w[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int r = row_base + i * kRowsPerLoad + sub;
        w[i] = r < L ? __ldcs(reinterpret_cast<const uint4 *>(k + ((slot_base + r) * H + h) * D) +
                              part)
                     : make_uint4(0, 0, 0, 0);
    }
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) a = fmaxf(a, fmaxf(fabsf(bf16_lo(u[e])), fabsf(bf16_hi(u[e]))));
    }
    a = warp_max(a);
    if (lane == 0) s_max[warp] = a;
    __syncthreads();
    a = s_max[0];
#pragma unroll
    for (int v = 1; v < 8; ++v) a = fmaxf(a, s_max[v]);
    const float inv = fp8_inv(a);
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int r = row_base + i * kRowsPerLoad + sub;
        if (r >= L) continue;
        const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
        const uint2 c = make_uint2(
            quant4(bf16_lo(u[0]), bf16_hi(u[0]), bf16_lo(u[1]), bf16_hi(u[1]), inv),
            quant4(bf16_lo(u[2]), bf16_hi(u[2]), bf16_lo(u[3]), bf16_hi(u[3]), inv));
        reinterpret_cast<uint2 *>(k8 + ((slot_base + r) * H + h) * D)[part] = c;
    }
    if (threadIdx.x == 0) scale[(static_cast<long>(slot) * n_tiles + t) * H + h] = fp8_scale(a);
}

}  // namespace

cudaError_t launch_quantize_rows(const uint16_t *q, uint8_t *q8, float *scale, long n_rows, int H,
                                 int D, cudaStream_t stream, DeviceWords *words)
{
    if (n_rows == 0) return cudaSuccess;
    const long rows_per_block = 8L * 4 * (32 / (D / 8));
    const dim3 grid(static_cast<unsigned>((n_rows + rows_per_block - 1) / rows_per_block));
    if (D == 128)
        quantize_rows_kernel<128><<<grid, 256, 0, stream>>>(q, q8, scale, n_rows, H, words);
    else
        quantize_rows_kernel<64><<<grid, 256, 0, stream>>>(q, q8, scale, n_rows, H, words);
    return cudaGetLastError();
}

cudaError_t launch_quantize_tiles(const uint16_t *k, uint8_t *k8, float *scale, long first_chunk,
                                  int n_chunks, int L, int H, int R, int D, cudaStream_t stream,
                                  DeviceWords *words)
{
    if (n_chunks == 0) return cudaSuccess;
    const int n_tiles = (L + 127) / 128;
    const dim3 grid(static_cast<unsigned>(n_chunks * n_tiles), static_cast<unsigned>(H));
    if (D == 128)
        quantize_tiles_kernel<128><<<grid, 256, 0, stream>>>(k, k8, scale, first_chunk, L, H, R,
                                                               words);
    else
        quantize_tiles_kernel<64><<<grid, 256, 0, stream>>>(k, k8, scale, first_chunk, L, H, R,
                                                              words);
    return cudaGetLastError();
}

}  // namespace wf

// ln_kernel.cu -- LayerNorm (no affine) with per-chunk adaLN modulation, the step
// before the QKV projection and before the feed-forward layer of a DiT block.
//
// The wave of "Wave Forcing" (abstract) holds chunks at different denoising
// steps, so each chunk carries its own modulation: row n of the wave uses row
// n / rows_per_group of shift and scale.  y = (x - mean) / sqrt(var + eps) *
// (1 + scale) + shift, with the mean and the (biased) variance over the row,
// fp32 arithmetic and one rounding to bf16.
//
// HBM-bound: 2 bytes read and 2 written per element; the modulation tables are
// small (one row of shift and scale per chunk) but are needed at 8 bytes per
// element.  One warp per row; lane l owns the 16-byte pieces l, l + 32, ... of
// the row, all loaded before the reductions.  Two kernels:
//   * up to 2048 channels, the rows kernel: a warp walks a contiguous range of
//     rows and keeps its lanes' modulation in registers, reloading it only when
//     the chunk changes;
//   * wider rows (whose modulation does not fit in registers): one row per warp,
//     each block staging its group's modulation in shared memory.
// Both are instantiated for a few counts of pieces per lane, so that a row of C
// channels holds no more registers than it needs (occupancy sets the bytes in
// flight), and both compute in the same order (bit-identical outputs).
#include <cuda_bf16.h>

#include <atomic>

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

// Rows kernel, for rows of at most 32 * 8 * kPer channels with kPer <= 8: each
// warp takes a contiguous range of rows and keeps its lanes' shift and
// (1 + scale) in registers while the group stays the same (a chunk's
// modulation serves thousands of rows), so the modulation costs no shared-
// memory traffic per row.  The rows themselves stream through a ring of
// kRing row buffers per warp in shared memory, filled with cp.async (each lane
// copies, and later reads back, only its own 16-byte pieces, so a lane waits
// only for its own copies: cp.async.wait_group, which the hardware completes),
// so that kRing - 1 rows per warp are in flight while one is reduced.
// Arithmetic and summation order are those of the kernel above (bit-identical
// outputs).
constexpr int kRowsWarps = 4;
constexpr int kRing = 4;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int kPer>
__global__ void __launch_bounds__(32 * kRowsWarps)
layer_norm_modulate_rows_kernel(const uint16_t *__restrict__ x, const float *__restrict__ shift,
                                const float *__restrict__ scale, uint16_t *__restrict__ y, long M,
                                int C, int rows_per_group, float eps, long rows_per_warp)
{
    // ring[warp][slot][piece i][lane]: a lane's pieces of one row, 16 bytes each
    extern __shared__ uint4 s_rows[];
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const long warp_id = static_cast<long>(blockIdx.x) * kRowsWarps + wid;
    const long r0 = warp_id * rows_per_warp;
    const long r1 = r0 + rows_per_warp < M ? r0 + rows_per_warp : M;
    if (r0 >= r1) return;                   // whole warps leave together
    const int pieces = C / 8;
    uint4 *ring = s_rows + static_cast<size_t>(wid) * kRing * kPer * 32;
    // issue the copies of `row` into ring slot `slot` (one commit group)
    auto fetch = [&](long row, int slot) {
        if (row < r1) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + row * C);
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int j = lane + 32 * i;
                if (j < pieces) cp_async16(smem_addr(ring + (slot * kPer + i) * 32 + lane), src + j);
            }
        }
        cp_async_commit();                  // possibly empty: the group count stays regular
    };
#pragma unroll
    for (int k = 0; k < kRing - 1; ++k) fetch(r0 + k, k);
    float shv[kPer][8], c1v[kPer][8];
    long g = -1;
    int slot = 0;
    for (long row = r0; row < r1; ++row) {
        fetch(row + kRing - 1, (slot + kRing - 1) % kRing);
        cp_async_wait<kRing - 1>();         // this lane's copies of `row` have landed
        uint4 cur[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int j = lane + 32 * i;
            cur[i] = j < pieces ? ring[(slot * kPer + i) * 32 + lane] : make_uint4(0u, 0u, 0u, 0u);
        }
        slot = slot + 1 == kRing ? 0 : slot + 1;
        const long gr = row / rows_per_group;
        if (gr != g) {                      // warp-uniform: rows are the warp's
            g = gr;
            const float4 *sh4 = reinterpret_cast<const float4 *>(shift + g * C);
            const float4 *sc4 = reinterpret_cast<const float4 *>(scale + g * C);
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int j = lane + 32 * i;
                float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = sa, ca = sa, cb = sa;
                if (j < pieces) {
                    sa = __ldg(sh4 + 2 * j);
                    sb = __ldg(sh4 + 2 * j + 1);
                    ca = __ldg(sc4 + 2 * j);
                    cb = __ldg(sc4 + 2 * j + 1);
                }
                const float s8[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
                const float c8[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    shv[i][e] = s8[e];
                    c1v[i][e] = 1.0f + c8[e];
                }
            }
        }
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const uint32_t u[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
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
            const uint32_t u[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
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
        uint4 *dst = reinterpret_cast<uint4 *>(y + row * C);
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int j = lane + 32 * i;
            if (j >= pieces) break;
            const uint32_t u[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = (__uint_as_float(u[e] << 16) - mean) * rstd;
                const float b = (__uint_as_float(u[e] & 0xFFFF0000u) - mean) * rstd;
                o[e] = pack_bf16x2(fmaf(a, c1v[i][2 * e], shv[i][2 * e]),
                                   fmaf(b, c1v[i][2 * e + 1], shv[i][2 * e + 1]));
            }
            __stcs(dst + j, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
    cp_async_wait<0>();                     // no copy outlives the block
}

template <int kPer>
constexpr size_t rows_smem_bytes() { return sizeof(uint4) * kRowsWarps * kRing * kPer * 32; }

// Resident blocks per SM of a rows-kernel instantiation and the SM count, once
// per device.
template <int kPer>
int rows_kernel_slots(int dev)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<int> slots[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return 0;
    int n = slots[dev].load(std::memory_order_relaxed);
    if (n < 1) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaFuncSetAttribute(layer_norm_modulate_rows_kernel<kPer>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(rows_smem_bytes<kPer>())) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, layer_norm_modulate_rows_kernel<kPer>, 32 * kRowsWarps,
                rows_smem_bytes<kPer>()) != cudaSuccess ||
            per_sm < 1) {
            (void)cudaGetLastError();
            return 0;
        }
        n = sms * per_sm;
        slots[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int kPer>
cudaError_t launch_rows(const uint16_t *x, const float *shift, const float *scale, uint16_t *y,
                        long M, int C, int rows_per_group, float eps, cudaStream_t stream)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    const int blocks = rows_kernel_slots<kPer>(dev);
    if (blocks < 1) return cudaErrorInvalidConfiguration;
    const long warps = static_cast<long>(blocks) * kRowsWarps;
    const long rows_per_warp = (M + warps - 1) / warps;
    const long need = (M + rows_per_warp - 1) / rows_per_warp;          // warps with rows
    const unsigned grid = static_cast<unsigned>((need + kRowsWarps - 1) / kRowsWarps);
    layer_norm_modulate_rows_kernel<kPer><<<grid, 32 * kRowsWarps, rows_smem_bytes<kPer>(), stream>>>(
        x, shift, scale, y, M, C, rows_per_group, eps, rows_per_warp);
    return cudaGetLastError();
}

}  // namespace

int ln_max_channels() { return 32 * kMaxPieces * 8; }

cudaError_t launch_layer_norm_modulate(const uint16_t *x, const float *shift, const float *scale,
                                       uint16_t *y, long M, int C, int rows_per_group, float eps,
                                       cudaStream_t stream)
{
    if (M == 0) return cudaSuccess;
    const int per_lane = (C / 8 + 31) / 32;
    // up to 2048 channels: the rows kernel (modulation in registers)
    if (per_lane <= 2) return launch_rows<2>(x, shift, scale, y, M, C, rows_per_group, eps, stream);
    if (per_lane <= 4) return launch_rows<4>(x, shift, scale, y, M, C, rows_per_group, eps, stream);
    if (per_lane <= 6) return launch_rows<6>(x, shift, scale, y, M, C, rows_per_group, eps, stream);
    if (per_lane <= 8) return launch_rows<8>(x, shift, scale, y, M, C, rows_per_group, eps, stream);
    const dim3 grid(static_cast<unsigned>((M + kRowsPerBlock - 1) / kRowsPerBlock));
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

// append_kernel.cu -- fused per-head Q/K RMSNorm + 3D RoPE + ring-buffer K/V append.
//
// "Wave Forcing" (abstract): Wave Parallelism delivers each layer's K/V early,
// one way, to the replicas of later chunks.  On one GPU the analogue is writing
// every wave chunk's K/V into the ring-buffer history cache in the same pass
// that normalises and rotates Q/K, so the attention kernel finds K/V in place.
//
// Memory-bound: 12*T*H*D bytes per call (read q, k, v; write q', K', V).  Each
// thread owns 8 consecutive channels (one 16-byte vector per tensor) of one
// (token, head) row; the D/8 threads of a row reduce the sum of squares with
// shuffles.  RoPE pairs (2i, 2i+1) never straddle threads.
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

__device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 pack8(const float (&y)[8])
{
    uint4 u;
    u.x = pack_bf16x2(y[0], y[1]);
    u.y = pack_bf16x2(y[2], y[3]);
    u.z = pack_bf16x2(y[4], y[5]);
    u.w = pack_bf16x2(y[6], y[7]);
    return u;
}

template <int D>
__global__ void __launch_bounds__(256) qk_norm_rope_append_kernel(const AppendParams p)
{
    constexpr int TPR = D / 8;   // threads per (token, head) row
    __shared__ float s_omega[D / 2];
    __shared__ int s_axis[D / 2];
    for (int i = threadIdx.x; i < D / 2; i += blockDim.x) {
        s_omega[i] = p.rope.omega[i];
        s_axis[i] = p.rope.axis[i];
    }
    __syncthreads();

    const long items = static_cast<long>(p.W) * p.L * p.H * TPR;
    const long it = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const unsigned mask = __ballot_sync(0xFFFFFFFFu, it < items);
    if (it >= items) return;

    const long row = it / TPR;                 // (token, head) row
    const int part = static_cast<int>(it % TPR);
    const long n = row / p.H;                  // wave token
    const int h = static_cast<int>(row - n * p.H);
    const int c = static_cast<int>(n / p.L);   // wave chunk
    const int i = static_cast<int>(n - static_cast<long>(c) * p.L);

    const long off = row * D + part * 8;
    const uint4 uq = __ldcs(reinterpret_cast<const uint4 *>(p.q + off));
    const uint4 uk = __ldcs(reinterpret_cast<const uint4 *>(p.k + off));
    const uint4 uv = __ldcs(reinterpret_cast<const uint4 *>(p.v + off));

    int pos[3];
    if (p.pos != nullptr) {
        pos[0] = __ldg(p.pos + 3 * n + 0);
        pos[1] = __ldg(p.pos + 3 * n + 1);
        pos[2] = __ldg(p.pos + 3 * n + 2);
    } else {
        const int hw = p.rope.gh * p.rope.gw;
        const int f = i / hw;
        const int rem = i - f * hw;
        const int y = rem / p.rope.gw;
        pos[0] = static_cast<int>((p.round + c) * p.rope.F + f);
        pos[1] = y;
        pos[2] = rem - y * p.rope.gw;
    }

    float xq[8], xk[8];
    unpack8(uq, xq);
    unpack8(uk, xk);
    float ssq = 0.f, ssk = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        ssq = fmaf(xq[e], xq[e], ssq);
        ssk = fmaf(xk[e], xk[e], ssk);
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) {
        ssq += __shfl_xor_sync(mask, ssq, o);
        ssk += __shfl_xor_sync(mask, ssk, o);
    }
    const float rq = rsqrtf(ssq * (1.0f / D) + p.eps);
    const float rk = rsqrtf(ssk * (1.0f / D) + p.eps);

    const float4 *gq4 = reinterpret_cast<const float4 *>(p.gamma_q + h * D + part * 8);
    const float4 *gk4 = reinterpret_cast<const float4 *>(p.gamma_k + h * D + part * 8);
    const float4 gq0 = __ldg(gq4), gq1 = __ldg(gq4 + 1);
    const float4 gk0 = __ldg(gk4), gk1 = __ldg(gk4 + 1);
    const float gq[8] = {gq0.x, gq0.y, gq0.z, gq0.w, gq1.x, gq1.y, gq1.z, gq1.w};
    const float gk[8] = {gk0.x, gk0.y, gk0.z, gk0.w, gk1.x, gk1.y, gk1.z, gk1.w};

    float yq[8], yk[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int pr = part * 4 + e;           // channel pair index
        const int ax = s_axis[pr];
        const int pv = ax == 0 ? pos[0] : (ax == 1 ? pos[1] : pos[2]);
        const float ang = static_cast<float>(pv) * s_omega[pr];
        float sn, cs;
        sincosf(ang, &sn, &cs);
        const float q0 = xq[2 * e] * rq * gq[2 * e], q1 = xq[2 * e + 1] * rq * gq[2 * e + 1];
        const float k0 = xk[2 * e] * rk * gk[2 * e], k1 = xk[2 * e + 1] * rk * gk[2 * e + 1];
        yq[2 * e] = q0 * cs - q1 * sn;
        yq[2 * e + 1] = q0 * sn + q1 * cs;
        yk[2 * e] = k0 * cs - k1 * sn;
        yk[2 * e + 1] = k0 * sn + k1 * cs;
    }

    const int slot = ring_slot(p.round + c, p.R);
    const long coff = ((static_cast<long>(slot) * p.L + i) * p.H + h) * D + part * 8;
    *reinterpret_cast<uint4 *>(p.q_out + off) = pack8(yq);
    *reinterpret_cast<uint4 *>(p.k_cache + coff) = pack8(yk);
    *reinterpret_cast<uint4 *>(p.v_cache + coff) = uv;
}

}  // namespace

cudaError_t launch_append(const AppendParams &p, int D, cudaStream_t stream)
{
    const long items = static_cast<long>(p.W) * p.L * p.H * (D / 8);
    const int threads = 256;
    const long blocks = (items + threads - 1) / threads;
    if (blocks <= 0) return cudaSuccess;
    if (D == 128)
        qk_norm_rope_append_kernel<128><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(p);
    else
        qk_norm_rope_append_kernel<64><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace wf

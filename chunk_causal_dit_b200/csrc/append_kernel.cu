// append_kernel.cu -- fused per-head Q/K RMSNorm + 3D RoPE + ring-buffer K/V append.
//
// "Wave Forcing" (abstract): Wave Parallelism delivers each layer's K/V early,
// one way, to the replicas of later chunks.  On one GPU the analogue is writing
// every wave chunk's K/V into the ring-buffer history cache in the same pass
// that normalises and rotates Q/K, so the attention kernel finds K/V in place.
//
// Memory-bound: 12*T*H*D bytes per call (read q, k, v; write q', K', V).
// A block covers kTokens consecutive tokens for a group of heads.  Thread
// (h, part) owns channels [8*part, 8*part + 8) of head h -- one 16-byte vector
// per tensor -- and issues the loads of all kTokens tokens first.
// The D/8 threads of a row reduce the sum of squares with shuffles; RoPE pairs
// (2i, 2i+1) never straddle threads.  The rotation angles depend on the token
// only, so each block computes them once per token, while its loads are in
// flight: the angle
// pos * omega in fp64, reduced to [-pi, pi] in fp64, then fp32 sincos -- so the
// fp32 error of the rotation stays a few ulps of the pair's length at any
// position.
//
// The Q8 instantiation also quantizes each (token, head) row of q' to E4M3 for
// the FP8 Q.K^T attention, in registers: the row's D / 8 threads reduce the
// amax of the bf16-rounded q' with the same shuffles as the norm, then write
// the codes and the row's scale (the rule of fp8_rule.cuh, so the bits equal
// the stand-alone row quantizer's on q_out).  q_out itself is then optional.
#include <cuda_bf16.h>

#include "fp8_rule.cuh"
#include "sm100.cuh"
#include "wf_check.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

constexpr int kTokens = 2;         // tokens per block (measured best on B200: 2 > 3 > 1 > 4 > 8)
constexpr int kMaxThreads = 512;   // threads per block (head groups split larger H)

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

template <int D, bool Q8>
__global__ void __launch_bounds__(kMaxThreads) qk_norm_rope_append_kernel(const AppendParams p,
                                                                          DeviceWords *words)
{
    constexpr int TPR = D / 8;           // threads per (token, head) row
    constexpr int NP = D / 2;            // RoPE pairs
    __shared__ float2 s_cs[kTokens][NP];   // (cos, sin) per token and pair
    __shared__ long s_off[kTokens];        // element offset of the token's row in the ring

    const long T = static_cast<long>(p.W) * p.L;
    const long n0 = static_cast<long>(blockIdx.x) * kTokens;

    // ---- loads first: they do not depend on the angles ----
    const int hl = threadIdx.x / TPR;
    const int part = threadIdx.x - hl * TPR;
    const int h = blockIdx.y * p.heads_per_block + hl;
    // the block is rounded up to whole warps; lanes past the group are idle
    const bool active = hl < p.heads_per_block && h < p.H;
    const int hh = active ? h : 0;       // inactive lanes still join the shuffles

    float gq[8], gk[8];
    {
        const float4 *gq4 = reinterpret_cast<const float4 *>(p.gamma_q + hh * D + part * 8);
        const float4 *gk4 = reinterpret_cast<const float4 *>(p.gamma_k + hh * D + part * 8);
        const float4 a = __ldg(gq4), b = __ldg(gq4 + 1), c = __ldg(gk4), d = __ldg(gk4 + 1);
        gq[0] = a.x; gq[1] = a.y; gq[2] = a.z; gq[3] = a.w;
        gq[4] = b.x; gq[5] = b.y; gq[6] = b.z; gq[7] = b.w;
        gk[0] = c.x; gk[1] = c.y; gk[2] = c.z; gk[3] = c.w;
        gk[4] = d.x; gk[5] = d.y; gk[6] = d.z; gk[7] = d.w;
    }

    uint4 uq[kTokens], uk[kTokens], uv[kTokens];
#pragma unroll
    for (int tl = 0; tl < kTokens; ++tl) {
        const long n = n0 + tl;
        if (active && n < T) {
            const long off = (n * p.H + h) * D + part * 8;
            uq[tl] = __ldcs(reinterpret_cast<const uint4 *>(p.q + off));
            uk[tl] = __ldcs(reinterpret_cast<const uint4 *>(p.k + off));
            uv[tl] = __ldcs(reinterpret_cast<const uint4 *>(p.v + off));
        } else {
            uq[tl] = uk[tl] = uv[tl] = make_uint4(0u, 0u, 0u, 0u);
        }
    }

    // ---- prologue: angles and ring rows of the block's tokens ----
    for (int i = threadIdx.x; i < kTokens * NP; i += blockDim.x) {
        const int tl = i / NP, pr = i - tl * NP;
        const long n = n0 + tl;
        if (n >= T) continue;
        const int c = static_cast<int>(n / p.L);
        const int ic = static_cast<int>(n - static_cast<long>(c) * p.L);
        const int ax = p.rope.axis[pr];
        long pos;
        if (p.pos != nullptr) {
            pos = __ldg(p.pos + 3 * n + ax);
        } else {
            const int hw = p.rope.gh * p.rope.gw;
            const int f = ic / hw;
            const int rem = ic - f * hw;
            const int y = rem / p.rope.gw;
            pos = ax == 0 ? (p.round + c) * p.rope.F + f : (ax == 1 ? y : rem - y * p.rope.gw);
        }
        const double ang = static_cast<double>(pos) * p.rope.omega[pr];
        const double k = rint(ang * 0.15915494309189535);   // 1 / (2 pi)
        const float red = static_cast<float>(fma(-k, 6.283185307179586, ang));
        float sn, cs;
        sincosf(red, &sn, &cs);
        s_cs[tl][pr] = make_float2(cs, sn);
        if (pr == 0) {
            const int slot = ring_slot(p.round + c, p.R);
            const bool in = WF_BOUNDS(slot >= 0 && slot < p.R && c < p.W && ic < p.L, words,
                                      kSiteAppend);
            s_off[tl] = in ? (static_cast<long>(slot) * p.L + ic) * p.H * D : -1;
        }
    }
    __syncthreads();

#pragma unroll
    for (int tl = 0; tl < kTokens; ++tl) {
        const long n = n0 + tl;
        if (n >= T) break;                    // uniform across the block
        float xq[8], xk[8];
        unpack8(uq[tl], xq);
        unpack8(uk[tl], xk);
        float ssq = 0.f, ssk = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            ssq = fmaf(xq[e], xq[e], ssq);
            ssk = fmaf(xk[e], xk[e], ssk);
        }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) {
            ssq += __shfl_xor_sync(0xFFFFFFFFu, ssq, o);
            ssk += __shfl_xor_sync(0xFFFFFFFFu, ssk, o);
        }
        const float rq = rsqrtf(ssq * (1.0f / D) + p.eps);
        const float rk = rsqrtf(ssk * (1.0f / D) + p.eps);
        float yq[8], yk[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 cs = s_cs[tl][part * 4 + e];
            const float q0 = xq[2 * e] * rq * gq[2 * e], q1 = xq[2 * e + 1] * rq * gq[2 * e + 1];
            const float k0 = xk[2 * e] * rk * gk[2 * e], k1 = xk[2 * e + 1] * rk * gk[2 * e + 1];
            yq[2 * e] = q0 * cs.x - q1 * cs.y;
            yq[2 * e + 1] = q0 * cs.y + q1 * cs.x;
            yk[2 * e] = k0 * cs.x - k1 * cs.y;
            yk[2 * e + 1] = k0 * cs.y + k1 * cs.x;
        }
        const uint4 q16 = pack8(yq);
        float inv = 1.0f, qs = 1.0f;
        if constexpr (Q8) {
            // amax of the row's bf16 q' over its D / 8 threads (inactive lanes hold 0)
            float a = absmax8(q16);
#pragma unroll
            for (int o = TPR / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
            inv = fp8_inv(a);
            qs = fp8_scale(a);
        }
        if (active && WF_CHECKED(s_off[tl] >= 0)) {
            const long off = (n * p.H + h) * D + part * 8;
            const long coff = s_off[tl] + static_cast<long>(h) * D + part * 8;
            if (!Q8 || p.q_out != nullptr) *reinterpret_cast<uint4 *>(p.q_out + off) = q16;
            if constexpr (Q8) {
                *reinterpret_cast<uint2 *>(p.q8 + off) = quant8(q16, inv);
                if (part == 0) p.q_scale[static_cast<long>(h) * T + n] = qs;
            }
            *reinterpret_cast<uint4 *>(p.k_cache + coff) = pack8(yk);
            *reinterpret_cast<uint4 *>(p.v_cache + coff) = uv[tl];
        }
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams &p_in, int D, cudaStream_t stream, DeviceWords *words)
{
    AppendParams p = p_in;
    const int tpr = D / 8;
    const int groups = (p.H * tpr + kMaxThreads - 1) / kMaxThreads;
    p.heads_per_block = (p.H + groups - 1) / groups;
    const int threads = (p.heads_per_block * tpr + 31) / 32 * 32;
    const long T = static_cast<long>(p.W) * p.L;
    const long bx = (T + kTokens - 1) / kTokens;
    const int by = (p.H + p.heads_per_block - 1) / p.heads_per_block;
    if (bx <= 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(by));
    const bool q8 = p.q8 != nullptr;
    if (D == 128) {
        if (q8) qk_norm_rope_append_kernel<128, true><<<grid, threads, 0, stream>>>(p, words);
        else qk_norm_rope_append_kernel<128, false><<<grid, threads, 0, stream>>>(p, words);
    } else {
        if (q8) qk_norm_rope_append_kernel<64, true><<<grid, threads, 0, stream>>>(p, words);
        else qk_norm_rope_append_kernel<64, false><<<grid, threads, 0, stream>>>(p, words);
    }
    return cudaGetLastError();
}

}  // namespace wf

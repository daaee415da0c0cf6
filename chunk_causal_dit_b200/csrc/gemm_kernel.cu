// gemm_kernel.cu -- bf16 GEMM C = A B^T on tcgen05 CTA pairs, with the epilogues of the
// DiT block fused into it.
//
// "Wave Forcing" (abstract) pushes every wave chunk through the layers of
// Wan2.1-T2V-1.3B in one pass; around the chunk-causal attention those layers
// are dense projections: the QKV projection (whose epilogue here also does the
// per-head RMSNorm, the 3D RoPE and the ring-buffer append of the wave round,
// so q/k/v never round-trip through HBM before the attention), the output
// projection and the two feed-forward layers.  A is [M][K] (activations), B is
// [N][K] (a linear layer's weight, out x in), both bf16 and K-major; the
// accumulation is fp32 in TMEM.
//
// Organisation (one cluster of two CTAs per pair of SMs, persistent):
//  * Tile = 256 rows x 256 columns per cluster; CTA rank r holds rows
//    [128r, 128r + 128) of the tile's A and rows [128r, 128r + 128) of its B
//    (columns of C).  The leader issues tcgen05.mma.cta_group::2 with M = 256,
//    N = 256, K = 16; each SM reads half of the B tile, so a stage is 32 KB per
//    SM for 512 tensor cycles of work.
//  * A ring of 64-deep K slices (one 128-byte swizzle row of bf16; 6 stages, 5
//    with the QKV epilogue's RoPE tables), filled by TMA; both CTAs' copies
//    complete on the leader's barriers, the leader's commits release the stage
//    in both CTAs.
//  * Two 256-column fp32 accumulators in TMEM (all 512 columns): the epilogue of
//    tile i reads one while the MMAs of tile i + 1 fill the other.
//  * Eight epilogue warps per CTA: warp w reads TMEM lane quarter w % 4 (the
//    lanes a warp may access) and one 128-column half of the tile; each thread
//    owns one row of C, and the warp moves its global loads and stores through
//    a staging buffer in shared memory so that they are coalesced.
//  * Tiles are dealt statically: cluster c takes tiles c, c + clusters, ...,
//    numbered with the column tile fastest, so the clusters working at one time
//    share a few row blocks of A (and all of B) in L2.
//
// Every mbarrier wait is bounded (the plan's limit); on expiry the kernel records
// kStatusTimeout, every role leaves its loop, the leader drains its copies and
// MMAs, and both CTAs meet at a cluster barrier before TMEM is freed.
#include <cuda_bf16.h>

#include <atomic>

#include "sm100.cuh"
#include "wf_check.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

constexpr int BM = 128;                    // rows of A per CTA (M = 256 per pair MMA)
constexpr int BK = 64;                     // K per stage: one 128-byte swizzle row of bf16
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);   // producer, MMA, 8 epilogue warps
constexpr uint32_t kABytes = BM * BK * 2;              // 16 KB

// Tile width BN (columns of C per tile, the MMA's N): 256 for the linear layers;
// the convolution takes 192 when the output channels are a multiple of it (384
// and 192 fill whole tiles).  Each CTA holds BN / 2 rows of B per stage.
template <int BN>
struct Tile {
    static_assert(BN == 256 || BN == 192, "tile width");
    static constexpr uint32_t kBBytes = (BN / 2) * BK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
};

template <int Epi>
struct IsConv {
    static constexpr bool value = Epi == kEpiConv || Epi == kEpiConvResidual;
};
constexpr int kTabMax = 3072;                          // float2 entries (24 KB)
constexpr uint32_t kStageRowBytes = 80;                // epilogue staging (see warp_store32)
constexpr uint32_t kWarpStageBytes = 32 * kStageRowBytes;
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kDrainLimit = 1ull << 32;

// Shared-memory plan per epilogue: the stage ring, then (QKV only) the RoPE
// (cos, sin) tables, the epilogue warps' staging buffers and the barrier block.
// (Six stages measured 1-4% faster than seven; with the tables only five fit.)
// A stage of a convolution holds the input box of 16 columns x 10 rows x 64
// channels (the 8 output rows of this CTA and one row above and below) and the
// weights of the three row taps dy = 0, 1, 2 of one (dt, dx): the MMAs of tap dy
// read the box from its row 16 dy on (a 2 KB offset, a whole number of 1024-byte
// swizzle atoms), so a box is loaded once per three taps instead of three times.
constexpr int kConvBoxRows = 10;
constexpr uint32_t kConvABytes = 16 * kConvBoxRows * BK * 2;   // 20 KB

template <int Epi, int BN>
struct Smem {
    static constexpr bool kConv = IsConv<Epi>::value;
    static constexpr uint32_t kStageBytes =
        kConv ? kConvABytes + 3 * Tile<BN>::kBBytes : Tile<BN>::kStageBytes;
    static constexpr int kStages =
        kConv ? 3 : (Epi == kEpiQkvAppend ? 5 : (BN == 192 ? 7 : 6));
    static constexpr uint32_t kTabOff = kStages * kStageBytes;
    static constexpr uint32_t kStgOff = kTabOff + (Epi == kEpiQkvAppend ? kTabMax * 8 : 0);
    static constexpr uint32_t kBarOff = kStgOff + kEpiWarps * kWarpStageBytes;
    static constexpr uint32_t kBytes = kBarOff + 256 + 1024;   // + 1024-byte alignment slack
    // barrier indices
    static constexpr int full = 0, empty = kStages, acc_full = 2 * kStages,
                         acc_empty = 2 * kStages + 2, drain = 2 * kStages + 4,
                         count = 2 * kStages + 5;
    static_assert(kBytes <= 232448, "shared memory per CTA");
    static_assert(count * 8 + 8 <= 256, "barrier block");
};

enum : uint32_t {
    kWhereProducer = 21, kWhereMmaFull = 22, kWhereMmaAcc = 23, kWhereEpi = 24, kWhereDrain = 25,
};

struct Ctl {
    volatile uint32_t *abort;
    uint32_t peer_abort;      // the other CTA's abort word (shared::cluster address)
    DeviceWords *words;
    unsigned long long limit;
};

// Bounded wait with cluster-scope acquire (phases may be completed from the peer CTA).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl &ctl,
                                         uint32_t where, bool drain = false)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    const unsigned long long limit = drain ? kDrainLimit : ctl.limit;
    while (true) {
#pragma unroll 1
        for (int k = 0; k < 32; ++k)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (!drain && *ctl.abort) return false;
        if (static_cast<unsigned long long>(clock64() - t0) > limit) {
            *ctl.abort = 1u;
            st_cluster_u32(ctl.peer_abort, 1u);     // the pair stops together
            atomicOr(&ctl.words->status, kStatusTimeout);
            atomicCAS(&ctl.words->timeout_where, 0u, where);
            return false;
        }
    }
}

// Tanh form of GELU, 0.5 x (1 + tanh(u)) with u = sqrt(2/pi) (x + 0.044715 x^3),
// evaluated through the identity 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2u)): one exp2
// and one division, and no cancellation for u < 0 (the quotient keeps its relative
// accuracy where 1 + tanh(u) would lose it).  exp(-2u) = 2^(-2u log2 e).
__device__ __forceinline__ float gelu_tanh(float x)
{
    const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
    const float e = ex2_approx(-2.8853900817779268f * u);
    return __fdividef(x, 1.0f + e);
}

__device__ __forceinline__ uint4 pack8(const float *y)
{
    uint4 u;
    u.x = pack_bf16x2(y[0], y[1]);
    u.y = pack_bf16x2(y[2], y[3]);
    u.z = pack_bf16x2(y[4], y[5]);
    u.w = pack_bf16x2(y[6], y[7]);
    return u;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float *x)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Each epilogue warp moves its 32 rows x 32 columns of bf16 through a staging
// buffer of its own in shared memory, so that global loads and stores are
// coalesced: 8 rows x 64 contiguous bytes per instruction instead of one
// 16-byte piece of each of 32 rows (measured: that pattern cost the K = 1536
// projections ~14% of their time).  Rows are 80 bytes apart (64 + 16 of
// padding), which makes the 16-byte shared stores of a warp conflict-free.

// Store: thread `lane` holds its row's 32 values packed in w; dst is that row's
// destination (nullptr: the row stores nothing).  Warp-collective.
__device__ __forceinline__ void warp_store32(uint8_t *stage, const uint4 (&w)[4], uint16_t *dst)
{
    const int lane = threadIdx.x & 31;
    uint4 *mine = reinterpret_cast<uint4 *>(stage + lane * kStageRowBytes);
#pragma unroll
    for (int j = 0; j < 4; ++j) mine[j] = w[j];
    __syncwarp();
    const unsigned long long d = reinterpret_cast<unsigned long long>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int piece = 32 * i + lane, rr = piece >> 2, part = piece & 3;
        const unsigned long long drow = __shfl_sync(0xFFFFFFFFu, d, rr);
        const uint4 v = *reinterpret_cast<const uint4 *>(stage + rr * kStageRowBytes + part * 16);
        if (drow != 0ull) reinterpret_cast<uint4 *>(drow)[part] = v;
    }
    __syncwarp();
}

// Load: src is this thread's row (nullptr: zeros); w receives the row's 32 values.
// Warp-collective.
__device__ __forceinline__ void warp_load32(uint8_t *stage, const uint16_t *src, uint4 (&w)[4])
{
    const int lane = threadIdx.x & 31;
    const unsigned long long s = reinterpret_cast<unsigned long long>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int piece = 32 * i + lane, rr = piece >> 2, part = piece & 3;
        const unsigned long long srow = __shfl_sync(0xFFFFFFFFu, s, rr);
        *reinterpret_cast<uint4 *>(stage + rr * kStageRowBytes + part * 16) =
            srow != 0ull ? __ldg(reinterpret_cast<const uint4 *>(srow) + part)
                         : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();
    const uint4 *mine = reinterpret_cast<const uint4 *>(stage + lane * kStageRowBytes);
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = mine[j];
    __syncwarp();
}

// 32 columns [c, c + 32) of one row: bias, activation / gated residual, bf16 store.
// Warp-collective (row_ok false: the row takes part but loads and stores nothing).
template <int Epi>
__device__ __forceinline__ void finish32(const GemmParams &p, const uint32_t (&r)[32], long row,
                                         bool row_ok, int c, const float *gate_row,
                                         uint8_t *stage)
{
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    if (p.bias != nullptr) {
        const float4 *b4 = reinterpret_cast<const float4 *>(p.bias + c);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 b = __ldg(b4 + j);
            v[4 * j] += b.x;
            v[4 * j + 1] += b.y;
            v[4 * j + 2] += b.z;
            v[4 * j + 3] += b.w;
        }
    }
    if constexpr (Epi == kEpiGeluTanh) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = gelu_tanh(v[i]);
    }
    if constexpr (Epi == kEpiConvResidual) {
        uint4 rw[4];
        warp_load32(stage, row_ok ? p.resid + row * p.N + c : nullptr, rw);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float x[8];
            unpack8(rw[j], x);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[8 * j + e] += x[e];
        }
    }
    if constexpr (Epi == kEpiGatedResidual) {
        uint4 rw[4];
        warp_load32(stage, row_ok ? p.resid + row * p.N + c : nullptr, rw);
        const float4 *g4 = reinterpret_cast<const float4 *>(gate_row + c);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float x[8];
            unpack8(rw[j], x);
            const float4 ga = __ldg(g4 + 2 * j), gb = __ldg(g4 + 2 * j + 1);
            const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) v[8 * j + e] = fmaf(g[e], v[8 * j + e], x[e]);
        }
    }
    uint4 w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = pack8(v + 8 * j);
    const bool st = row_ok && WF_BOUNDS(c + 32 <= p.N, p.words, kSiteGemmStore);
    warp_store32(stage, w, st ? p.c + row * p.N + c : nullptr);
}

// Linear and convolution epilogues: this thread's row (row_ok: it exists), kCols
// columns from col0 (TMEM at taddr), in pairs of 32-column chunks.
template <int Epi, int kCols>
__device__ __forceinline__ void epi_linear(const GemmParams &p, uint32_t taddr, long row,
                                           bool row_ok, int col0, uint8_t *stage)
{
    static_assert(kCols % 32 == 0, "32-column chunks");
    const float *gate_row = nullptr;
    if constexpr (Epi == kEpiGatedResidual)
        gate_row = p.gate + (row_ok ? row / p.rows_per_group : 0) * static_cast<long>(p.N);
#pragma unroll 1
    for (int h = 0; h < kCols / 64; ++h) {
        uint32_t r0[32], r1[32];
        tmem_ld32(taddr + 64 * h, r0);
        tmem_ld32(taddr + 64 * h + 32, r1);
        tmem_wait_ld();
        const int c = col0 + 64 * h;                 // warp-uniform column guards
        if (c < p.N) finish32<Epi>(p, r0, row, row_ok, c, gate_row, stage);
        if (c + 32 < p.N) finish32<Epi>(p, r1, row, row_ok, c + 32, gate_row, stage);
    }
    if constexpr (kCols % 64 != 0) {
        uint32_t r0[32];
        const int h = kCols / 64;
        tmem_ld32(taddr + 64 * h, r0);
        tmem_wait_ld();
        const int c = col0 + 64 * h;
        if (c < p.N) finish32<Epi>(p, r0, row, row_ok, c, gate_row, stage);
    }
}

// Output pixel of a convolution tile: tile t (column tile fastest, then 16-column
// and 16-row pixel tiles, then frames), CTA rank r (rows 8r .. 8r + 7 of the
// tile) and row m of the CTA's 128 rows (16 pixels per row).
struct ConvTile {
    int nb, f, y0, x0;
};

__device__ __forceinline__ ConvTile conv_tile(const GemmParams &p, int t)
{
    ConvTile c;
    c.nb = t % p.n_ntiles;
    int rest = t / p.n_ntiles;
    const int px = rest % p.n_px;
    rest /= p.n_px;
    const int py = rest % p.n_py;
    c.f = rest / p.n_py;
    c.x0 = px * 16;
    c.y0 = py * 16;
    return c;
}

// QKV epilogue: this thread's wave token `row`, 128 columns from col0, i.e. 128 / D
// heads of one of q, k, v (the column split puts q, k and v at multiples of H*D,
// which the host keeps a multiple of 128).  q and k: RMSNorm over the head with
// gain gamma, then the 3D RoPE with the (cos, sin) tables, one rounding to bf16;
// q goes to q_out [T][H][D], k and v to row ic of the ring slot of the token's
// chunk, (round + c) mod R, as the stand-alone append kernel writes them.
// A head is read from TMEM in 32-column chunks, twice for q and k (the sum of
// squares first), with the next chunk's load in flight while one is processed.
template <int D>
__device__ __forceinline__ void epi_qkv(const GemmParams &p, uint32_t taddr, long row, int col0,
                                        const float2 *tab, uint8_t *stage)
{
    constexpr int kHeads = 128 / D;
    constexpr int kChunks = D / 32;
    const int HD = p.H * D;
    const int which = col0 / HD;                 // 0 q, 1 k, 2 v (warp-uniform)
    const int h0 = (col0 - which * HD) / D;
    const long n = row < p.M ? row : 0;          // rows past M store nothing
    const int c = static_cast<int>(n / p.L);
    const int ic = static_cast<int>(n - static_cast<long>(c) * p.L);
    const bool ok = row < p.M && col0 < p.N &&
                    WF_BOUNDS(which <= 2 && h0 + kHeads <= p.H && c < p.W && ic < p.L, p.words,
                              kSiteGemmQkv);
    const int hw = p.rope.gh * p.rope.gw;
    const int f = ic / hw;
    const int rem = ic - f * hw;
    const int y = rem / p.rope.gw;
    const int x = rem - y * p.rope.gw;
    const int nt = p.rope.dt / 2, nh = p.rope.dh / 2, nw = p.rope.dw / 2;
    const int nfr = p.W * p.rope.F;
    // table index of pair pr: it + pr (t block), ih + pr (h block), iw + pr (w block)
    const int it = (c * p.rope.F + f) * nt;
    const int ih = nfr * nt + y * nh - nt;
    const int iw = nfr * nt + p.rope.gh * nh + x * nw - nt - nh;
    const int slot = ring_slot(p.round + c, p.R);
#pragma unroll 1
    for (int hh = 0; hh < kHeads; ++hh) {
        const int h = h0 + hh;
        const int col = col0 + hh * D;
        const uint32_t ta = taddr + hh * D;
        const float4 *b4 = p.bias != nullptr ? reinterpret_cast<const float4 *>(p.bias + col)
                                             : nullptr;
        uint32_t r[2][32];
        float rs = 1.0f;
        if (which < 2) {
            float ss = 0.0f;
            tmem_ld32(ta, r[0]);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < kChunks; ++j) {
                if (j + 1 < kChunks) tmem_ld32(ta + 32 * (j + 1), r[(j + 1) & 1]);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 b = b4 ? __ldg(b4 + 8 * j + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float v0 = __uint_as_float(r[j & 1][4 * q4]) + b.x;
                    const float v1 = __uint_as_float(r[j & 1][4 * q4 + 1]) + b.y;
                    const float v2 = __uint_as_float(r[j & 1][4 * q4 + 2]) + b.z;
                    const float v3 = __uint_as_float(r[j & 1][4 * q4 + 3]) + b.w;
                    ss = fmaf(v0, v0, ss);
                    ss = fmaf(v1, v1, ss);
                    ss = fmaf(v2, v2, ss);
                    ss = fmaf(v3, v3, ss);
                }
                tmem_wait_ld();
            }
            rs = rsqrtf(ss * (1.0f / D) + p.eps);
        }
        uint16_t *dst;
        if (which == 0)
            dst = p.q_out + (n * p.H + h) * D;
        else
            dst = (which == 1 ? p.k_cache : p.v_cache) +
                  ((static_cast<long>(slot) * p.L + ic) * p.H + h) * D;
        const float4 *g4 =
            reinterpret_cast<const float4 *>((which == 1 ? p.gamma_k : p.gamma_q) + h * D);
        tmem_ld32(ta, r[0]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kChunks; ++j) {
            if (j + 1 < kChunks) tmem_ld32(ta + 32 * (j + 1), r[(j + 1) & 1]);
            {
                float v[32];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 b = b4 ? __ldg(b4 + 8 * j + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[4 * q4] = __uint_as_float(r[j & 1][4 * q4]) + b.x;
                    v[4 * q4 + 1] = __uint_as_float(r[j & 1][4 * q4 + 1]) + b.y;
                    v[4 * q4 + 2] = __uint_as_float(r[j & 1][4 * q4 + 2]) + b.z;
                    v[4 * q4 + 3] = __uint_as_float(r[j & 1][4 * q4 + 3]) + b.w;
                }
                if (which < 2) {
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 g = __ldg(g4 + 8 * j + q4);
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int pl = 2 * q4 + e;           // pair within the chunk
                            const int pr = 16 * j + pl;          // pair within the head
                            const float a = v[2 * pl] * rs * (e ? g.z : g.x);
                            const float bb = v[2 * pl + 1] * rs * (e ? g.w : g.y);
                            const int ti = pr < nt ? it + pr : (pr < nt + nh ? ih + pr : iw + pr);
                            const float2 cs =
                                WF_BOUNDS(ti >= 0 && ti < p.n_tab, p.words, kSiteGemmTable)
                                    ? tab[ti] : make_float2(1.0f, 0.0f);
                            v[2 * pl] = a * cs.x - bb * cs.y;
                            v[2 * pl + 1] = a * cs.y + bb * cs.x;
                        }
                    }
                }
                uint4 w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) w[q] = pack8(v + 8 * q);
                warp_store32(stage, w, ok ? dst + 32 * j : nullptr);
            }
            tmem_wait_ld();
        }
    }
}

template <int Epi, int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ GemmParams p)
{
    using B = Smem<Epi, BN>;
    constexpr int kStages = B::kStages;
    constexpr uint32_t kStageBytes = B::kStageBytes;
    constexpr uint32_t kBBytes = Tile<BN>::kBBytes;
    constexpr bool kConv = IsConv<Epi>::value;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t sbar = sbase + B::kBarOff;
    auto bar = [&](int i) -> uint32_t { return sbar + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + B::kBarOff + 8 * B::count);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(nclusters_x());
    auto lead = [&](int i) -> uint32_t { return map_to_rank(bar(i), 0); };
    // K stages: one per 64 columns of K, or per (dt, dx, 64 input channels) of a
    // convolution (each stage covering the three row taps dy)
    const int nk = kConv ? 9 * p.n_cblk : (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B::full + s), 1);
            mbar_init(bar(B::empty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B::acc_full + b), 1);
            mbar_init(bar(B::acc_empty + b), 2 * kEpiWarps);   // both CTAs' epilogue warps
        }
        mbar_init(bar(B::drain), 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    if constexpr (Epi == kEpiQkvAppend) {
        // (cos, sin) of every (frame, t pair), (row y, h pair), (column x, w pair): the
        // angle pos * omega in fp64, reduced to [-pi, pi] in fp64, then fp32 sincos
        if (warp >= 2) {
            float2 *tab = reinterpret_cast<float2 *>(smem + B::kTabOff);
            const int nt = p.rope.dt / 2, nh = p.rope.dh / 2, nw = p.rope.dw / 2;
            const int n_t = p.W * p.rope.F * nt, n_h = p.rope.gh * nh;
            for (int i = threadIdx.x - 64; i < p.n_tab; i += 32 * kEpiWarps) {
                int pr;
                long pos;
                if (i < n_t) {
                    const int fi = i / nt;
                    pr = i - fi * nt;
                    pos = p.round * p.rope.F + fi;
                } else if (i < n_t + n_h) {
                    const int j = i - n_t, yy = j / nh;
                    pr = nt + (j - yy * nh);
                    pos = yy;
                } else {
                    const int j = i - n_t - n_h, xx = j / nw;
                    pr = nt + nh + (j - xx * nw);
                    pos = xx;
                }
                const double ang = static_cast<double>(pos) * p.rope.omega[pr];
                const double k = rint(ang * 0.15915494309189535);   // 1 / (2 pi)
                const float red = static_cast<float>(fma(-k, 6.283185307179586, ang));
                float sn, cs;
                sincosf(red, &sn, &cs);
                tab[i] = make_float2(cs, sn);
            }
        }
    }
    tc_fence_before();
    cluster_sync();                 // barriers, TMEM address and tables ready in both CTAs
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Ctl ctl{abort_flag, map_to_rank(smem_addr(const_cast<uint32_t *>(abort_flag)), rank ^ 1u),
                  p.words, p.wait_limit};

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            tma_prefetch_desc(&tmap_a);
            tma_prefetch_desc(&tmap_b);
            if (kConv && p.use_hist) tma_prefetch_desc(&tmap_h);
            uint32_t it = 0;
            const bool withheld = p.withhold != 0;   // test hook: stage 0's first fill never comes
            bool ok = true;
            for (int t = cid; ok && t < p.n_tiles; t += ncl) {
                int arow = 0, brow = 0, fr = 0, ya = 0, xa = 0;
                if constexpr (kConv) {
                    const ConvTile ct = conv_tile(p, t);
                    brow = ct.nb * BN + static_cast<int>(rank) * (BN / 2);
                    fr = ct.f;
                    ya = ct.y0 + 8 * static_cast<int>(rank);
                    xa = ct.x0;
                } else {
                    const int mb = t / p.n_ntiles, nb = t - mb * p.n_ntiles;
                    arow = mb * 2 * BM + static_cast<int>(rank) * BM;
                    brow = nb * BN + static_cast<int>(rank) * (BN / 2);
                }
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const uint32_t st = it % kStages;
                    if (!(ok = wait_bar(bar(B::empty + st), ((it / kStages) & 1u) ^ 1u, ctl,
                                        kWhereProducer)))
                        break;
                    if (withheld && it == 0) continue;
                    if (leader) mbar_arrive_expect_tx(bar(B::full + st), 2 * kStageBytes);
                    const uint32_t dst = sbase + st * kStageBytes;
                    if constexpr (kConv) {
                        // taps (dt, 0..2, dx), channels [64 cb, 64 cb + 64): A is the 16 x 10
                        // pixel box from row ya - 1, shifted by dx (rows and columns outside
                        // the frame read zeros); taps before the chunk read the history's
                        // frame tf + 2, or zeros at the start of the video
                        const int tdx = kb / p.n_cblk, cb = kb - tdx * p.n_cblk;
                        const int dt = tdx / 3, dx = tdx - 3 * dt;
                        const int tf = fr + dt - 2;
                        const bool hist = tf < 0 && p.use_hist;
                        tma_load_4d_pair(dst, hist ? &tmap_h : &tmap_a, lead(B::full + st),
                                         cb * BK, xa + dx - 1, ya - 1, hist ? tf + 2 : tf);
#pragma unroll
                        for (int dy = 0; dy < 3; ++dy)
                            tma_load_3d_pair(dst + kConvABytes + dy * kBBytes, &tmap_b,
                                             lead(B::full + st), cb * BK, dt * 9 + dy * 3 + dx,
                                             brow);
                    } else {
                        tma_load_2d_pair(dst, &tmap_a, lead(B::full + st), kb * BK, arow);
                        tma_load_2d_pair(dst + kABytes, &tmap_b, lead(B::full + st), kb * BK,
                                         brow);
                    }
                }
            }
            if (!ok && leader) {
                // both CTAs' copies complete on the leader's barriers: let the armed
                // fills land.  With the first fill of stage 0 withheld, stage 0 was
                // never filled (its next fill waits for a consumption that never came).
                for (uint32_t s = withheld ? 1u : 0u; s < static_cast<uint32_t>(kStages); ++s) {
                    const uint32_t fills = (it + kStages - 1 - s) / kStages;
                    if (fills)
                        wait_bar(bar(B::full + s), (fills - 1) & 1u, ctl, kWhereDrain, true);
                }
            }
        }
    } else if (warp == 1) {
        if (leader) {
            // ---------------- MMA issuer (leader CTA, for the pair) ----------------
            // The whole warp runs the loop and its waits (warp-uniform values), one
            // elected lane issues the MMAs and commits (as in the attention kernel:
            // a single divergent lane issues measurably fewer MMAs per cycle).
            const bool issuer = elect_one_sync();
            constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, false);
            constexpr uint32_t hi = sw128_desc_hi(1024);
            uint32_t it = 0, acc_it = 0;
            bool ok = true;
            for (int t = cid; ok && t < p.n_tiles; t += ncl, ++acc_it) {
                const uint32_t b = acc_it & 1u;
                ok = wait_bar(bar(B::acc_empty + b), ((acc_it >> 1) & 1u) ^ 1u, ctl, kWhereMmaAcc);
                if (!(ok = __all_sync(0xFFFFFFFFu, ok))) break;
                tc_fence_after();
                const uint32_t d = tmem + b * BN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const uint32_t st = it % kStages;
                    ok = wait_bar(bar(B::full + st), (it / kStages) & 1u, ctl, kWhereMmaFull);
                    if (!(ok = __all_sync(0xFFFFFFFFu, ok))) break;
                    tc_fence_after();
                    if (issuer) {
                        if constexpr (kConv) {
                            const uint32_t a0 = sbase + st * kStageBytes;
#pragma unroll
                            for (int dy = 0; dy < 3; ++dy) {
                                const uint32_t alo = sw128_desc_lo(a0 + dy * 2048, 16);
                                const uint32_t blo =
                                    sw128_desc_lo(a0 + kConvABytes + dy * kBBytes, 16);
#pragma unroll
                                for (int s = 0; s < BK / 16; ++s)
                                    umma_ss_pair(d, desc_join(alo + ((s * 32) >> 4), hi),
                                                 desc_join(blo + ((s * 32) >> 4), hi), idesc,
                                                 (kb | dy | s) ? 1u : 0u);
                            }
                        } else {
                            const uint32_t alo = sw128_desc_lo(sbase + st * kStageBytes, 16);
                            const uint32_t blo =
                                sw128_desc_lo(sbase + st * kStageBytes + kABytes, 16);
#pragma unroll
                            for (int s = 0; s < BK / 16; ++s)
                                umma_ss_pair(d, desc_join(alo + ((s * 32) >> 4), hi),
                                             desc_join(blo + ((s * 32) >> 4), hi), idesc,
                                             (kb | s) ? 1u : 0u);
                        }
                        umma_commit_pair_mc(bar(B::empty + st), 0x3);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (issuer) umma_commit_pair_mc(bar(B::acc_full + b), 0x3);
                __syncwarp();
            }
            // every MMA of the pair completes before either CTA releases TMEM
            if (issuer) umma_commit_pair_mc(bar(B::drain), 0x1);
            __syncwarp();
            wait_bar(bar(B::drain), 0u, ctl, kWhereDrain, true);
        }
    } else {
        // ---------------- epilogue: 8 warps, one row of C per thread ----------------
        const int lq = warp & 3;                   // TMEM lane quarter of this warp
        const int half = (warp - 2) >> 2;          // 128-column half of the tile
        const float2 *tab = reinterpret_cast<const float2 *>(smem + B::kTabOff);
        uint8_t *stage = smem + B::kStgOff + (warp - 2) * kWarpStageBytes;
        uint32_t acc_it = 0;
        for (int t = cid; t < p.n_tiles; t += ncl, ++acc_it) {
            const uint32_t b = acc_it & 1u;
            bool ok = wait_bar(bar(B::acc_full + b), (acc_it >> 1) & 1u, ctl, kWhereEpi);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) break;
            tc_fence_after();
            long row;
            bool row_ok;
            int nb;
            if constexpr (kConv) {
                const ConvTile ct = conv_tile(p, t);
                const int m = lq * 32 + lane;
                const int y = ct.y0 + 8 * static_cast<int>(rank) + (m >> 4);
                const int x = ct.x0 + (m & 15);
                nb = ct.nb;
                row_ok = y < p.ch && x < p.cw;
                row = (static_cast<long>(ct.f) * p.ch + y) * p.cw + x;
            } else {
                const int mb = t / p.n_ntiles;
                nb = t - mb * p.n_ntiles;
                row = static_cast<long>(mb) * 2 * BM + rank * BM + lq * 32 + lane;
                row_ok = row < p.M;
            }
            const int col0 = nb * BN + half * (BN / 2);
            const uint32_t taddr =
                tmem + (static_cast<uint32_t>(lq * 32) << 16) + b * BN + half * (BN / 2);
            if constexpr (Epi == kEpiQkvAppend)
                epi_qkv<D>(p, taddr, row, col0, tab, stage);
            else
                epi_linear<Epi, BN / 2>(p, taddr, row, row_ok, col0, stage);
            // the accumulator may be overwritten once this warp's TMEM loads are done
            // (tcgen05.wait::ld above): a relaxed arrive, so that the epilogue's global
            // stores need not drain first, as a release at cluster scope would demand
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(lead(B::acc_empty + b));
        }
    }

    // both CTAs stop sending to each other before either frees TMEM or exits
    tc_fence_before();
    __syncwarp();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

template <int Epi, int D, int BN = 256>
cudaError_t launch_gemm_t(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &mh,
                          const GemmParams &p, cudaStream_t stream)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<int> resident_pairs[kMaxDevices];
    auto kern = gemm_pair_kernel<Epi, D, BN>;
    constexpr uint32_t smem = Smem<Epi, BN>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2, 1, 1);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    // clusters of two that can be resident at once (one CTA per SM), once per device
    int resident = resident_pairs[dev].load(std::memory_order_relaxed);
    if (resident < 1) {
        if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident < 1) {
            (void)cudaGetLastError();
            return cudaErrorInvalidConfiguration;
        }
        resident_pairs[dev].store(resident, std::memory_order_relaxed);
    }
    const int n_clusters = p.n_tiles < resident ? p.n_tiles : resident;
    cfg.gridDim = dim3(2 * n_clusters, 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, ma, mb, mh, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

// Tensor maps: ma over A [M][K], mb over B [N][K], both bf16 with a 64 x 128 box and
// the 128-byte swizzle.
cudaError_t launch_gemm(const CUtensorMap &ma, const CUtensorMap &mb, const GemmParams &p, int epi,
                        cudaStream_t stream)
{
    if (p.n_tiles == 0) return cudaSuccess;
    switch (epi) {
    case kEpiStore: return launch_gemm_t<kEpiStore, 128>(ma, mb, ma, p, stream);
    case kEpiGeluTanh: return launch_gemm_t<kEpiGeluTanh, 128>(ma, mb, ma, p, stream);
    case kEpiGatedResidual: return launch_gemm_t<kEpiGatedResidual, 128>(ma, mb, ma, p, stream);
    case kEpiQkvAppend:
        return p.D == 128 ? launch_gemm_t<kEpiQkvAppend, 128>(ma, mb, ma, p, stream)
                          : launch_gemm_t<kEpiQkvAppend, 64>(ma, mb, ma, p, stream);
    default: return cudaErrorInvalidValue;
    }
}

// Causal 3x3x3 convolution as an implicit GEMM: mx over the chunk [ct][ch][cw][cin]
// and mh over its two history frames (box 64 channels x 16 columns x 10 rows x 1
// frame), mw over the weights [N][27][cin] (box 64 x 1 x BN / 2), 128-byte swizzle.
// bn: the tile width the maps were encoded for (192 or 256).
cudaError_t launch_conv(const CUtensorMap &mx, const CUtensorMap &mh, const CUtensorMap &mw,
                        const GemmParams &p, bool residual, int bn, cudaStream_t stream)
{
    if (p.n_tiles == 0) return cudaSuccess;
    if (bn == 192)
        return residual ? launch_gemm_t<kEpiConvResidual, 128, 192>(mx, mw, mh, p, stream)
                        : launch_gemm_t<kEpiConv, 128, 192>(mx, mw, mh, p, stream);
    return residual ? launch_gemm_t<kEpiConvResidual, 128, 256>(mx, mw, mh, p, stream)
                    : launch_gemm_t<kEpiConv, 128, 256>(mx, mw, mh, p, stream);
}

int gemm_tab_max() { return kTabMax; }

}  // namespace wf

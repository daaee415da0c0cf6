// attn_pair_kernel.cu -- chunk-causal wave-round attention on CTA pairs (head_dim 128).
//
// Same computation as attn_kernel.cu ("Wave Forcing", abstract: each wave chunk
// attends to the history and to wave chunks 0..c, bidirectionally inside a
// chunk), organised for two SMs per work unit:
//
//  * A cluster of two CTAs takes one unit (wave chunk c, head h, pair of 128-row
//    query tiles); CTA rank r owns query tile r of the pair.  The leader (rank 0)
//    issues tcgen05 MMAs with cta_group::2, M = 256: A (Q, or P in TMEM) comes
//    from each CTA's own rows, B is split across the two shared memories -- for
//    QK^T CTA r holds keys [64r, 64r+64) of the 128-key tile, for PV it holds
//    head-dim columns [64r, 64r+64) of V.  Each SM therefore reads 3/4 of the
//    operand bytes of a one-SM MMA of the same shape.
//  * S is double-buffered in TMEM (S0 | S1 | O, 384 of 512 columns), so QK^T of
//    key tile j+1 runs while the softmax works on tile j; P overwrites the first
//    64 columns of its S buffer and feeds PV from TMEM.
//  * Softmax: two warpgroups per CTA split each TMEM lane quarter into 16-lane
//    halves; with the 16x256b load shape a row lives in a quad of lanes (two
//    shuffles per row reduction) and 64 scores per thread.  A quarter of the
//    exponentials run on the FMA pipe (exp2_poly.h) to relieve MUFU.
//  * K/V halves stream through an 8-stage ring; each CTA's TMA copies complete
//    on the leader's barriers; the leader's commits multicast to both CTAs.
//  * Units follow a static snake order over clusters (longest first), so both
//    CTAs of a cluster walk the same sequence without exchanging anything.
//
// Every mbarrier wait is bounded; on expiry the kernel records kStatusTimeout,
// every role leaves its loop, the leader drains its copies and MMAs, and both
// CTAs meet at the final cluster barrier before freeing TMEM.
//
// Measured on B200 (Wan 1.3B 4-step wave, 12 heads x 128, chunks of 4680):
// 711 TFLOP/s against 1143 for the single-CTA kernel.  A clock64 trace shows the
// softmax at ~2900 cycles per 128 x 128 tile (twice the single kernel's cost per
// score), and with the softmax reduced to an arrival the MMA/TMA pipeline alone
// reaches 1116 TFLOP/s (single kernel: 1452).  The kernel is therefore opt-in
// (WF_ATTN_PAIR); it stays parity-tested.
#include <cuda_bf16.h>

#include <atomic>

#include "exp2_poly.h"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

constexpr int D = 128;
constexpr int BM = 128;              // query rows per CTA
constexpr int BN = 128;              // keys per key tile (64 per CTA for K)
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr unsigned long long kDrainLimit = 1ull << 32;
constexpr uint32_t kRegsLaunch = 168, kRegsSoftmax = 184, kRegsControl = 136;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl == kThreads * kRegsLaunch,
              "the register re-split must add up to the launch pool");
constexpr int kEmulatePeriod = 4;    // pair block k uses the FMA-pipe exp2 when k % 4 == 3
constexpr int kStages = 8;

constexpr uint32_t kQBytes = BM * D * 2;          // 32 KB: this CTA's 128 query rows
constexpr uint32_t kKBox = 64 * 64 * 2;           // 8 KB: 64 keys x 64 channels
constexpr uint32_t kStageBytes = 16384;           // K half (64 keys x 128) or V half (128 keys x 64)
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKVOff = kQBytes;
constexpr uint32_t kBarOff = kKVOff + kStages * kStageBytes;
constexpr uint32_t kSmemBytes = kBarOff + 512 + 1024;
constexpr uint32_t kS0 = 0, kS1 = 128, kO = 256;

struct Bars {
    static constexpr int q_full = 0, q_empty = 1, s_full = 2, p_ready = 4, o_ready = 6,
                         o_final = 7, drain = 8, kv_full = 9, kv_empty = 9 + kStages,
                         count = 9 + 2 * kStages;
};

enum : uint32_t {
    kWhereProducerQ = 1, kWhereProducerKV = 2, kWhereMmaQ = 3, kWhereMmaKV = 4,
    kWhereMmaP = 5, kWhereSoftS = 6, kWhereSoftO = 7, kWhereDrain = 8, kWhereSoftRescale = 10,
};

struct Ctl {
    volatile uint32_t *abort;
    uint32_t peer_abort;      // the other CTA's abort word (shared::cluster address)
    DeviceWords *words;
    unsigned long long limit;
};

// Bounded wait (cluster-scope acquire: phases may be completed from the peer CTA).
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

struct Unit {
    int c, h, pair, n_kt;
};

__device__ __forceinline__ Unit decode_unit(const AttnParams &p, int u)
{
    Unit r;
    const int per_c = p.H * p.n_qpairs;
    const int ci = u / per_c;
    const int rem = u - ci * per_c;
    r.c = p.W - 1 - ci;                       // longest (latest chunk) first
    r.h = rem / p.n_qpairs;
    r.pair = rem - r.h * p.n_qpairs;
    r.n_kt = (p.h_valid + r.c + 1) * p.n_ktiles;
    return r;
}

// k-th unit of this cluster in snake order over the clusters, or -1 when done;
// -2 means "no unit this round, go on" (the reversed last round is partial).
__device__ __forceinline__ int cluster_unit(int k, int n_units, int ncl, int cid)
{
    const long base = static_cast<long>(k) * ncl;
    if (base >= n_units) return -1;
    const long u = (k & 1) ? base + (ncl - 1 - cid) : base + cid;
    return u < n_units ? static_cast<int>(u) : -2;
}

__device__ __forceinline__ void issue_qk_pair(uint32_t s_tmem, uint32_t q_smem, uint32_t k_smem)
{
    constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, false);
    constexpr uint32_t hi = sw128_desc_hi(1024);
    const uint32_t qlo = sw128_desc_lo(q_smem, 16), klo = sw128_desc_lo(k_smem, 16);
#pragma unroll
    for (int s = 0; s < D / 16; ++s) {
        const uint32_t qoff = ((s >> 2) * (kQBytes / 2) + (s & 3) * 32) >> 4;
        const uint32_t koff = ((s >> 2) * kKBox + (s & 3) * 32) >> 4;
        umma_ss_pair(s_tmem, desc_join(qlo + qoff, hi), desc_join(klo + koff, hi), idesc,
                     s > 0 ? 1u : 0u);
    }
}

__device__ __forceinline__ void issue_pv_pair(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                              bool accumulate)
{
    constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, D, true);
    constexpr uint32_t hi = sw128_desc_hi(1024);
    // this CTA's V half: 128 keys x 64 channels, one 128-byte-swizzled atom wide
    const uint32_t vlo = sw128_desc_lo(v_smem, kStageBytes);
#pragma unroll
    for (int s = 0; s < BN / 16; ++s)
        umma_ts_pair(o_tmem, p_tmem + s * 8, desc_join(vlo + ((s * 2048) >> 4), hi), idesc,
                     (accumulate || s > 0) ? 1u : 0u);
}

// 2^x for a pair on the FMA pipe (see attn_kernel.cu for the derivation).
__device__ __forceinline__ void exp2_fma_pair(float x0, float x1, float &p0, float &p1)
{
    constexpr float kShift = 12582912.0f;   // 1.5 * 2^23
    x0 = fmaxf(x0, -126.0f);
    x1 = fmaxf(x1, -126.0f);
    const uint64_t x = f2_pack(x0, x1);
    const uint64_t t = f2_add(x, f2_pack(kShift, kShift));
    const uint64_t jf = f2_add(t, f2_pack(-kShift, -kShift));
    const uint64_t f = f2_fma(jf, f2_pack(-1.0f, -1.0f), x);
    uint64_t q = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
    q = f2_fma(q, f, f2_pack(kExp2C1, kExp2C1));
    q = f2_fma(q, f, f2_pack(kExp2C0, kExp2C0));
    float q0, q1, t0, t1;
    f2_unpack(q, q0, q1);
    f2_unpack(t, t0, t1);
    p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_causal_attn_pair_kernel(const __grid_constant__ CUtensorMap tmap_q,
                              const __grid_constant__ CUtensorMap tmap_k64,
                              const __grid_constant__ CUtensorMap tmap_v, const AttnParams p)
{
    constexpr int S = kStages;
    using B = Bars;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t sq = sbase + kQOff;
    const uint32_t skv = sbase + kKVOff;
    const uint32_t sbar = sbase + kBarOff;
    auto bar = [&](int i) -> uint32_t { return sbar + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBarOff + 8 * B::count);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(nclusters_x());
    auto lead = [&](int i) -> uint32_t { return map_to_rank(bar(i), 0); };

    if (threadIdx.x == 0) {
        mbar_init(bar(B::q_full), 1);
        mbar_init(bar(B::q_empty), 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B::s_full + b), 1);
            mbar_init(bar(B::p_ready + b), 2 * 8);   // 8 softmax warps in each CTA
        }
        mbar_init(bar(B::o_ready), 1);
        mbar_init(bar(B::o_final), 1);
        mbar_init(bar(B::drain), 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(bar(B::kv_full + s), 1);
            mbar_init(bar(B::kv_empty + s), 1);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc_pair(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();                 // both CTAs' barriers exist before any remote use
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Ctl ctl{abort_flag, map_to_rank(smem_addr(const_cast<uint32_t *>(abort_flag)), rank ^ 1u),
                  p.words, p.wait_limit};

    if (warp >= 8) {
        regs_dec<kRegsControl>();
        if (warp == kProducerWarp && lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k64);
            tma_prefetch_desc(&tmap_v);
            uint32_t ring = 0, q_fill = 0, q_armed = 0;   // q_armed: q_full phases armed
            bool withhold = p.withhold_q != 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int u = cluster_unit(k, p.n_units, ncl, cid);
                if (u == -1) break;
                if (u < 0) continue;
                const Unit un = decode_unit(p, u);
                if (!(ok = wait_bar(bar(B::q_empty), (q_fill & 1u) ^ 1u, ctl, kWhereProducerQ)))
                    break;
                if (withhold && leader) {
                    withhold = false;       // test hook: this q_full phase never completes
                } else {
                    if (leader) {
                        mbar_arrive_expect_tx(bar(B::q_full), 2 * kQBytes);
                        ++q_armed;
                    }
                    for (int hf = 0; hf < 2; ++hf)
                        tma_load_4d_pair(sq + hf * (kQBytes / 2), &tmap_q, lead(B::q_full), hf * 64,
                                         un.h, (2 * un.pair + static_cast<int>(rank)) * BM, un.c);
                }
                ++q_fill;
                for (int j = 0; ok && j < un.n_kt; ++j) {
                    const int b = j / p.n_ktiles;
                    const int t = j - b * p.n_ktiles;
                    const int slot = ring_slot(visible_chunk_id(p.round, p.h_valid, b), p.R);
                    for (int kv = 0; kv < 2; ++kv, ++ring) {
                        const uint32_t st = ring % S;
                        if (!(ok = wait_bar(bar(B::kv_empty + st), ((ring / S) & 1u) ^ 1u, ctl,
                                            kWhereProducerKV)))
                            break;
                        if (leader) mbar_arrive_expect_tx(bar(B::kv_full + st), 2 * kStageBytes);
                        const uint32_t dst = skv + st * kStageBytes;
                        if (kv == 0) {      // K half: this CTA's 64 keys, all 128 channels
                            for (int hf = 0; hf < 2; ++hf)
                                tma_load_4d_pair(dst + hf * kKBox, &tmap_k64, lead(B::kv_full + st),
                                                 hf * 64, un.h, t * BN + 64 * static_cast<int>(rank),
                                                 slot);
                        } else {            // V half: all 128 keys, this CTA's 64 channels
                            tma_load_4d_pair(dst, &tmap_v, lead(B::kv_full + st),
                                             64 * static_cast<int>(rank), un.h, t * BN, slot);
                        }
                    }
                }
            }
            if (!ok && leader) {
                // the copies of both CTAs complete on the leader's barriers: let them land
                if (q_armed == q_fill && q_armed)
                    wait_bar(bar(B::q_full), (q_armed - 1) & 1u, ctl, kWhereDrain, true);
                for (uint32_t s = 0; s < static_cast<uint32_t>(S); ++s) {
                    const uint32_t f = (ring + S - 1 - s) / S;   // fills of stage s
                    if (f) wait_bar(bar(B::kv_full + s), (f - 1) & 1u, ctl, kWhereDrain, true);
                }
            }
        } else if (warp == kMmaWarp && lane == 0 && leader) {
            // ---------------- MMA issuer (leader CTA, for the pair) ----------------
            uint32_t ring = 0, q_fill = 0;
            uint32_t p_phase = 0;                    // bit b: parity of p_ready + b
            auto tS = [&](int b) -> uint32_t { return tmem + (b ? kS1 : kS0); };
            const uint32_t tO = tmem + kO;
            const uint16_t both = 0x3;
            bool ok = true;
            auto stage_of = [&](uint32_t idx) -> uint32_t { return idx % S; };
            auto full = [&](uint32_t idx) -> bool {
                const bool r = wait_bar(bar(B::kv_full + idx % S), (idx / S) & 1u, ctl, kWhereMmaKV);
                tc_fence_after();
                return r;
            };
            for (int k = 0; ok; ++k) {
                const int u = cluster_unit(k, p.n_units, ncl, cid);
                if (u == -1) break;
                if (u < 0) continue;
                const Unit un = decode_unit(p, u);
                if (!(ok = wait_bar(bar(B::q_full), q_fill & 1u, ctl, kWhereMmaQ))) break;
                ++q_fill;
                tc_fence_after();
                const uint32_t base = ring;          // K_j at base + 2j, V_j at base + 2j + 1
                const int n_pre = un.n_kt < 2 ? un.n_kt : 2;
                for (int j = 0; ok && j < n_pre; ++j) {
                    const uint32_t ki = base + 2 * j;
                    if (!(ok = full(ki))) break;
                    issue_qk_pair(tS(j), sq, skv + stage_of(ki) * kStageBytes);
                    umma_commit_pair_mc(bar(B::s_full + j), both);
                    umma_commit_pair_mc(bar(B::kv_empty + stage_of(ki)), both);
                    if (j == un.n_kt - 1) umma_commit_pair_mc(bar(B::q_empty), both);
                }
                for (int j = 0; ok && j < un.n_kt; ++j) {
                    const int b = j & 1;
                    if (!(ok = wait_bar(bar(B::p_ready + b), (p_phase >> b) & 1u, ctl, kWhereMmaP)))
                        break;
                    p_phase ^= 1u << b;
                    tc_fence_after();
                    const uint32_t vi = base + 2 * j + 1;
                    if (!(ok = full(vi))) break;
                    issue_pv_pair(tO, tS(b), skv + stage_of(vi) * kStageBytes, j > 0);
                    umma_commit_pair_mc(bar(B::kv_empty + stage_of(vi)), both);
                    umma_commit_pair_mc(bar(B::o_ready), both);
                    if (j + 2 < un.n_kt) {
                        const uint32_t ki = base + 2 * (j + 2);
                        if (!(ok = full(ki))) break;
                        issue_qk_pair(tS(b), sq, skv + stage_of(ki) * kStageBytes);
                        umma_commit_pair_mc(bar(B::s_full + b), both);
                        umma_commit_pair_mc(bar(B::kv_empty + stage_of(ki)), both);
                        if (j + 2 == un.n_kt - 1) umma_commit_pair_mc(bar(B::q_empty), both);
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(bar(B::o_final), both);
                ring = base + 2 * static_cast<uint32_t>(un.n_kt);
            }
            // every MMA of the pair completes before either CTA releases TMEM
            umma_commit_pair_mc(bar(B::drain), 0x1);
            wait_bar(bar(B::drain), 0u, ctl, kWhereDrain, true);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // ---------------- softmax: two warpgroups per CTA, this CTA's 128 rows ----------------
        // In TMEM lane quarter q = warp & 3, warpgroup g takes lanes 32q + 16g .. +15;
        // thread t (t0 = t & 3, t1 = t >> 2) holds rows lane t1 and t1 + 8 of those,
        // columns 8k + 2t0 and 8k + 2t0 + 1 (16x256b load shape).
        const int g = warp >> 2;
        const int lane_base = 32 * (warp & 3) + 16 * g;
        const uint32_t lane_sel = static_cast<uint32_t>(lane_base) << 16;
        const int t0 = lane & 3, t1 = lane >> 2;
        const int row0 = lane_base + t1;            // rows of this CTA's tile: row0, row0 + 8
        const float scale = p.scale_log2;
        const uint64_t sc2 = f2_pack(scale, scale);
        const uint32_t pready_lead0 = lead(B::p_ready);   // p_ready + b: 8 bytes further
        const uint32_t tO = tmem + lane_sel + kO;
        uint32_t s_phase = 0, o_phase = 0;          // s_phase bit b: parity of s_full + b
        uint32_t pv_base = 0;                       // PVs of earlier units (o_ready phases)
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int u = cluster_unit(k, p.n_units, ncl, cid);
            if (u == -1) break;
            if (u < 0) continue;
            const Unit un = decode_unit(p, u);
            float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
            int t = 0;                              // key tile inside its chunk
            for (int j = 0; j < un.n_kt; ++j, t = (t + 1 == p.n_ktiles) ? 0 : t + 1) {
                const int b = j & 1;
                const uint32_t tS = tmem + lane_sel + (b ? kS1 : kS0);
                ok = wait_bar(bar(B::s_full + b), (s_phase >> b) & 1u, ctl, kWhereSoftS);
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) break;
                s_phase ^= 1u << b;
                tc_fence_after();
                uint32_t r[64];
                tmem_ld_16x256b_x16(tS, r);
                tmem_wait_ld();
                const int valid = t == p.n_ktiles - 1 ? p.L - t * BN : BN;
                if (valid < BN) {                   // last tile of a chunk: keys >= L
#pragma unroll
                    for (int kk = 0; kk < 16; ++kk)
#pragma unroll
                        for (int e = 0; e < 2; ++e)
                            if (8 * kk + 2 * t0 + e >= valid) {
                                r[4 * kk + e] = __float_as_uint(-INFINITY);
                                r[4 * kk + 2 + e] = __float_as_uint(-INFINITY);
                            }
                }
                float mx[2];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    float a = -INFINITY, c2 = -INFINITY;
#pragma unroll
                    for (int kk = 0; kk < 16; kk += 2) {
                        a = fmax3(a, __uint_as_float(r[4 * kk + 2 * rr]),
                                  __uint_as_float(r[4 * kk + 2 * rr + 1]));
                        c2 = fmax3(c2, __uint_as_float(r[4 * (kk + 1) + 2 * rr]),
                                   __uint_as_float(r[4 * (kk + 1) + 2 * rr + 1]));
                    }
                    a = fmaxf(a, c2);
                    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
                    mx[rr] = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
                }
                float alpha[2];
                bool need[2];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const float m_new = fmaxf(m_run[rr], mx[rr] * scale);
                    need[rr] = m_new > m_run[rr] + kRescaleThreshold;
                    alpha[rr] = need[rr] ? ex2_approx(m_run[rr] - m_new) : 1.0f;
                    if (need[rr]) {
                        l_run[rr] *= alpha[rr];
                        m_run[rr] = m_new;
                    }
                }
                if (j > 0 && __any_sync(0xFFFFFFFFu, need[0] || need[1])) {
                    // PV of the previous key tile may still run (S is double
                    // buffered): wait for it, then rescale this thread's O rows
                    const uint32_t prev = pv_base + static_cast<uint32_t>(j) - 1u;
                    ok = wait_bar(bar(B::o_ready), prev & 1u, ctl, kWhereSoftRescale);
                    ok = __all_sync(0xFFFFFFFFu, ok);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < D / 64; ++cc) {
                        uint32_t o[32];
                        tmem_ld_16x256b_x8(tO + cc * 64, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha[(e >> 1) & 1]);
                        tmem_st_16x256b_x8(tO + cc * 64, o);
                    }
                }
                const uint64_t nm0 = f2_pack(-m_run[0], -m_run[0]);
                const uint64_t nm1 = f2_pack(-m_run[1], -m_run[1]);
                uint64_t acc0 = 0ull, acc1 = 0ull;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t pk[16];
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const int kx = 8 * hf + kk;
                        float x0, x1, y0, y1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(r[4 * kx]),
                                                 __uint_as_float(r[4 * kx + 1])), sc2, nm0), x0, x1);
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(r[4 * kx + 2]),
                                                 __uint_as_float(r[4 * kx + 3])), sc2, nm1), y0, y1);
                        float p0, p1, q0, q1;
                        if ((kx % kEmulatePeriod) == kEmulatePeriod - 1) {
                            exp2_fma_pair(x0, x1, p0, p1);
                            exp2_fma_pair(y0, y1, q0, q1);
                        } else {
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                            q0 = ex2_approx(y0);
                            q1 = ex2_approx(y1);
                        }
                        acc0 = f2_add(acc0, f2_pack(p0, p1));
                        acc1 = f2_add(acc1, f2_pack(q0, q1));
                        pk[2 * kk] = pack_bf16x2(p0, p1);        // row R0, column 4kx + t0
                        pk[2 * kk + 1] = pack_bf16x2(q0, q1);    // row R1, same column
                    }
                    tmem_st_16x128b_x8(tS + 32 * hf, pk);
                }
                // publish P (and any rescale of O) to the leader's MMA thread
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(pready_lead0 + 8u * b);
                float a0, a1, b0, b1;
                f2_unpack(acc0, a0, a1);
                f2_unpack(acc1, b0, b1);
                l_run[0] += a0 + a1;                // this thread's columns; the quad
                l_run[1] += b0 + b1;                // is summed in the epilogue
            }
            if (!ok) break;
            pv_base += static_cast<uint32_t>(un.n_kt);
            // ---------------- epilogue: O / l to global, lse ----------------
            ok = wait_bar(bar(B::o_final), o_phase, ctl, kWhereSoftO);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) break;
            o_phase ^= 1u;
            tc_fence_after();
            float inv_l[2], l_tot[2];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                float l = l_run[rr];
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 1);
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 2);
                l_tot[rr] = l;
                inv_l[rr] = 1.0f / l;
            }
            const int q_row0 = (2 * un.pair + static_cast<int>(rank)) * BM + row0;
            const int q_row1 = q_row0 + 8;
            const long n0 = static_cast<long>(un.c) * p.L + q_row0;
            uint16_t *dst0 = p.o + (n0 * p.H + un.h) * D;
            uint16_t *dst1 = p.o + ((n0 + 8) * p.H + un.h) * D;
#pragma unroll 1
            for (int cc = 0; cc < D / 64; ++cc) {
                uint32_t o[32];
                tmem_ld_16x256b_x8(tO + cc * 64, o);
                tmem_wait_ld();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int col = cc * 64 + 8 * kk + 2 * t0;
                    const uint32_t w0 = pack_bf16x2(__uint_as_float(o[4 * kk]) * inv_l[0],
                                                    __uint_as_float(o[4 * kk + 1]) * inv_l[0]);
                    const uint32_t w1 = pack_bf16x2(__uint_as_float(o[4 * kk + 2]) * inv_l[1],
                                                    __uint_as_float(o[4 * kk + 3]) * inv_l[1]);
                    if (q_row0 < p.L) *reinterpret_cast<uint32_t *>(dst0 + col) = w0;
                    if (q_row1 < p.L) *reinterpret_cast<uint32_t *>(dst1 + col) = w1;
                }
            }
            if (p.lse != nullptr && t0 == 0) {
                if (q_row0 < p.L)
                    p.lse[static_cast<long>(un.h) * p.T + n0] =
                        m_run[0] * 0.6931471805599453f + logf(l_tot[0]);
                if (q_row1 < p.L)
                    p.lse[static_cast<long>(un.h) * p.T + n0 + 8] =
                        m_run[1] * 0.6931471805599453f + logf(l_tot[1]);
            }
            tc_fence_before();
        }
    }

    // both CTAs stop sending to each other before either frees TMEM or exits
    tc_fence_before();
    __syncwarp();
    cluster_sync();
    tc_fence_after();
    if (warp == kMmaWarp) {
        __syncwarp();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace

// Clusters of two that can be resident at once (one CTA per SM): fewer than
// SMs / 2 when a GPC has an odd number of SMs free.  Queried once per device.
static int max_resident_pairs(const cudaLaunchConfig_t &cfg)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaOccupancyMaxActiveClusters(&n, chunk_causal_attn_pair_kernel, &cfg) != cudaSuccess ||
        n < 1)
        return -1;
    cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Persistent launch: one cluster of two CTAs per resident pair of SMs, at most
// one cluster per work unit.  mk64 maps the key cache with a 64-row box.
cudaError_t launch_attn_pair(const CUtensorMap &mq, const CUtensorMap &mk64, const CUtensorMap &mv,
                             const AttnParams &p, cudaStream_t stream)
{
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, chunk_causal_attn_pair_kernel);
    if (e != cudaSuccess) return e;
    // the setmaxnreg split assumes exactly the launch budget
    if (fa.numRegs != static_cast<int>(kRegsLaunch)) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(chunk_causal_attn_pair_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2, 1, 1);
    const int resident = max_resident_pairs(cfg);
    if (resident < 1) {
        (void)cudaGetLastError();
        return cudaErrorInvalidConfiguration;
    }
    const int n_clusters = p.n_units < resident ? p.n_units : resident;
    cfg.gridDim = dim3(2 * n_clusters, 1, 1);
    e = cudaLaunchKernelEx(&cfg, chunk_causal_attn_pair_kernel, mq, mk64, mv, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace wf

// attn_kernel.cu -- chunk-causal wave-round attention on sm_100a tensor cores.
//
// "Wave Forcing" (abstract): with chunk-wise causal attention a chunk of the wave
// can use the chunks ahead of it, which are less noisy, while those are still
// being denoised.  For
// query chunk c the visible keys are every token of the valid history chunks
// and of wave chunks 0..c; inside a chunk attention is bidirectional.  Visible
// keys therefore form whole chunks, so masking is decided per key tile: fully
// masked tiles are never loaded, and the only element mask is "key row < L" in
// the last 128-key tile of each chunk (TMA fills the rows past L with zeros).
//
// Work unit = (wave chunk c, head h, pair of 128-row query tiles).  One CTA per
// SM pops units from a global counter.  The heads are taken in blocks of
// head_block (chosen on the host): all units of one block, longest first (cost
// (h_valid + c + 1) key chunks; greedy longest-processing-time order inside the
// block), then the next block.  The units of a block read the same key/value
// chunks of its heads at nearly the same time, and the host keeps a block's
// keys and values within half of L2, so a key tile comes from DRAM about once
// instead of once for every wave chunk that sees it.
// Warp roles (384 threads, three warpgroups):
//   warps 0-3   softmax for query tile 0 (TMEM lanes 0..127, one row per thread)
//   warps 4-7   softmax for query tile 1
//   warp  8     scheduler + TMA producer: Q tiles, then K_j, V_j into a smem ring
//   warps 9, 10 MMA issuers of query tiles 0 and 1 (whole warps, one elected
//               lane issues): S_x = Q_x K_j^T, O_x += P_x V_j.  They take turns
//               through a token, so the tensor pipe receives one fixed order
//               (QK_0 QK_1 | PV_0 QK_0 | PV_1 QK_1 | ...); two issuers on two SMSPs
//               instead of one halve the MMA-issue load that each SMSP's softmax
//               warps share
//   warp  11    idle (it only gives its registers to the softmax warpgroups)
// Registers: launched at 168 per thread; the control warpgroup drops to 104 and
// the two softmax warpgroups rise to 200 (setmaxnreg), which is exactly the
// launch pool and leaves both paths spill-free.  The host refuses to launch if the compiled kernel does not use
// 168 registers, so the increase can always be met.
// TMEM (512 columns): S0 | S1 | O0 | O1.  Softmax overwrites the first half of
// S_x with P_x (bf16 pairs) and the PV product reads P straight from TMEM.
// P is published in two halves of 64 keys: PV on the first half starts while
// the softmax still exponentiates the second.
// The two query tiles ping-pong: while one warpgroup exponentiates, the tensor
// core runs the other tile's PV and next QK^T.  Online softmax works in the
// log2 domain and rescales O only when a row maximum grows by more than 2^8.
// A fraction of the score pairs can be exponentiated on the FMA pipe
// (Cody-Waite split and a Remez polynomial, exp2_poly.h) to offload MUFU; see
// kEmulatePeriod.
//
// Every mbarrier wait is bounded (clock64 limit); on expiry the kernel records
// kStatusTimeout in the plan's status word, all roles leave their loops, wait
// for their own copies/MMAs in flight, and the CTA frees TMEM and returns.
#include <cuda_bf16.h>

#include "exp2_poly.h"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {

namespace {

constexpr int BM = 128;              // query rows per tile
constexpr int BN = 128;              // keys per tile
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
// Waits for this CTA's own copies and MMAs in flight before it releases smem
// and TMEM use this fixed limit, not the plan's (which tests may set tiny):
// those operations always complete, so the drain only has to outlast them.
constexpr unsigned long long kDrainLimit = 1ull << 32;
constexpr uint32_t kRegsLaunch = 168, kRegsSoftmax = 200, kRegsControl = 104;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl == kThreads * kRegsLaunch,
              "the register re-split must add up to the launch pool");
constexpr int kSoftmaxWarpsArrive = 8;      // sched_empty: one arrival per softmax warp
// Pair e of a 32-pair block takes the FMA-pipe exp2 when e % kEmulatePeriod ==
// kEmulatePeriod - 1 (period 3: 10 of every 32 pairs); 0 keeps every
// exponential on MUFU.  Timed on B200: with a single MMA-issuing warp, sending
// 12.5-33% of the exponentials to the FMA pipe made the kernel slower (the
// MMA-side chain set the period); with one issuer per query tile, period 3 or 4
// is 0.6-1.5% faster than MUFU alone, period 8 no faster, period 2 14% slower.
// Period 3 keeps every instantiation spill-free (period 4 spills 16 bytes).
// The polynomial's relative error (7.5e-5) is far below P's bf16 rounding.
constexpr int kEmulatePeriod = 3;

// F8: Q and K arrive as E4M3 codes (one byte per element, one 128-byte
// swizzle atom per row at D = 128) with fp32 scales; V, P and O stay as in the
// bf16 kernel.
template <int D, bool F8>
struct Cfg {
    static constexpr int kStages = D == 128 ? 4 : 8;
    static constexpr int kHalves = D / 64;                 // 128-byte column blocks (bf16)
    static constexpr uint32_t kHalfBytes = 128 * 128;      // 128 rows x 128 bytes
    static constexpr uint32_t kTileBytes = BM * D * 2;     // one bf16 tile = one K/V stage
    static constexpr uint32_t kQKTileBytes = F8 ? BM * D : kTileBytes;   // a Q or K tile
    static constexpr uint32_t kQOff = 0;
    static constexpr uint32_t kKVOff = 2 * kQKTileBytes;
    static constexpr uint32_t kBarOff = kKVOff + kStages * kTileBytes;
    static constexpr uint32_t kSmemBytes = kBarOff + 512 + 1024;
    static constexpr uint32_t kS0 = 0, kS1 = 128, kO0 = 256, kO1 = 256 + D;
};

constexpr int kIssuers = 2;    // MMA issuers: warp kMmaWarp for query tile 0, the next for tile 1

// Barrier indices inside the barrier block (8 bytes each).
template <int S>
struct Bars {
    static constexpr int q_full = 0, q_empty = 1, s_full = 2, p_ready = 4, o_final = 6,
                         drain = 8, sched_full = 9, sched_empty = 11, p_half = 13, kv_full = 15,
                         kv_empty = 15 + S, turn = 15 + 2 * S, count = 17 + 2 * S;
};

// Wait-site codes recorded in DeviceWords::timeout_where.
enum : uint32_t {
    kWhereProducerQ = 1, kWhereProducerKV = 2, kWhereMmaQ = 3, kWhereMmaKV = 4,
    kWhereMmaP = 5, kWhereSoftS = 6, kWhereSoftO = 7, kWhereDrain = 8, kWhereSched = 9,
    kWhereMmaTurn = 10,
};

struct Ctl {
    volatile uint32_t *abort;
    DeviceWords *words;
    unsigned long long limit;
};

// Bounded wait on one mbarrier phase.  Returns false on timeout or when another
// role already aborted (unless `drain`, which ignores the abort flag and waits
// up to kDrainLimit).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl &ctl,
                                         uint32_t where, bool drain = false)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    const unsigned long long limit = drain ? kDrainLimit : ctl.limit;
    while (true) {
#pragma unroll 1
        for (int k = 0; k < 32; ++k)
            if (mbar_try_wait(bar, parity)) return true;
        if (!drain && *ctl.abort) return false;
        if (static_cast<unsigned long long>(clock64() - t0) > limit) {
            *ctl.abort = 1u;
            atomicOr(&ctl.words->status, kStatusTimeout);
            atomicCAS(&ctl.words->timeout_where, 0u, where);
            return false;
        }
    }
}

struct Unit {
    int c, h, pair, n_kt;
    bool has1;                                // query tile 1 holds rows of the chunk
};

__device__ __forceinline__ Unit decode_unit(const AttnParams &p, int u)
{
    Unit r;
    // blocks of head_block heads, one after the other (the last may hold fewer);
    // inside a block the latest chunk's units (the longest) first, then by head
    // and query tile pair
    const int blk_units = p.head_block * p.W * p.n_qpairs;
    const int hb = u / blk_units;
    const int rem_b = u - hb * blk_units;
    const int gb = min(p.head_block, p.H - hb * p.head_block);
    const int per_c = gb * p.n_qpairs;
    const int ci = rem_b / per_c;
    const int rem = rem_b - ci * per_c;
    const int hi = rem / p.n_qpairs;
    r.c = p.W - 1 - ci;
    r.h = hb * p.head_block + hi;
    r.pair = rem - hi * p.n_qpairs;
    r.n_kt = (p.h_valid + r.c + 1) * p.n_ktiles;
    r.has1 = (2 * r.pair + 1) * BM < p.L;
    return r;
}

// Advance (key tile, ring slot) by one key tile: the next chunk's tile 0 after
// a chunk's last tile, in the next slot (visible chunks have consecutive ids).
__device__ __forceinline__ void next_key_tile(int &t, int &slot, const AttnParams &p)
{
    if (++t == p.n_ktiles) {
        t = 0;
        slot = slot + 1 == p.R ? 0 : slot + 1;
    }
}

// The descriptors of one operand tile differ only in the start-address field
// (low 14 bits), so they are built from a 32-bit low word and a constant high
// word: fewer live 64-bit values in the MMA-issuing thread.
template <int D, bool F8>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t q_smem, uint32_t k_smem)
{
    constexpr uint32_t hi = sw128_desc_hi(1024);
    const uint32_t qlo = sw128_desc_lo(q_smem, 16), klo = sw128_desc_lo(k_smem, 16);
    if constexpr (F8) {
        // K = 32 codes (32 bytes) per MMA: four steps along the 128-byte row
        constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
#pragma unroll
        for (int s = 0; s < D / 32; ++s) {
            const uint32_t off = (s * 32) >> 4;
            umma_ss_f8(s_tmem, desc_join(qlo + off, hi), desc_join(klo + off, hi), idesc,
                       s > 0 ? 1u : 0u);
        }
    } else {
        constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
            const uint32_t off = ((s >> 2) * Cfg<D, false>::kHalfBytes + (s & 3) * 32) >> 4;
            umma_ss(s_tmem, desc_join(qlo + off, hi), desc_join(klo + off, hi), idesc,
                    s > 0 ? 1u : 0u);
        }
    }
}

// O += P V over keys [64*half, 64*half + 64) of the tile (4 steps of 16 keys).
template <int D>
__device__ __forceinline__ void issue_pv_half(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                              int half, bool accumulate)
{
    constexpr uint32_t idesc = idesc_bf16_f32(BM, D, true);
    constexpr uint32_t hi = sw128_desc_hi(1024);
    // V tile: 16 keys per step = 2 eight-row groups of 128 bytes; the two
    // 64-channel halves of D sit kHalfBytes apart (leading byte offset).
    const uint32_t vlo = sw128_desc_lo(v_smem, Cfg<D, false>::kHalfBytes);
#pragma unroll
    for (int i = 0; i < BN / 32; ++i) {
        const int s = half * (BN / 32) + i;
        umma_ts(o_tmem, p_tmem + s * 8, desc_join(vlo + ((s * 2048) >> 4), hi), idesc,
                (accumulate || s > 0) ? 1u : 0u);
    }
}

// 2^x for a pair of scores on the FMA pipe: j = round(x) by the 1.5*2^23 shift,
// f = x - j in [-1/2, 1/2], 2^f from the Remez polynomial, then j added to the
// exponent field.  x is clamped at -126 so the exponent never wraps; inputs
// below that (masked columns, deep underflow) give 2^-126 instead of 0, which
// is below one fp32 ulp of the row sum (>= 1) and multiplies a zero V row.
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
    // the low bits of t hold j; (bits(t) << 23) == (j << 23) modulo 2^32
    p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

template <int D, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
chunk_causal_attn_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const AttnParams p)
{
    using C = Cfg<D, F8>;
    constexpr int S = C::kStages;
    using B = Bars<S>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t sq = sbase + C::kQOff;
    const uint32_t skv = sbase + C::kKVOff;
    const uint32_t sbar = sbase + C::kBarOff;
    auto bar = [&](int i) -> uint32_t { return sbar + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kBarOff + 8 * B::count);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    volatile int *sched_unit = reinterpret_cast<volatile int *>(tmem_slot + 2);   // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(bar(B::q_full), 1);
        mbar_init(bar(B::q_empty), kIssuers);
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar(B::s_full + x), 1);
            mbar_init(bar(B::p_ready + x), 128);
            mbar_init(bar(B::p_half + x), 128);
            mbar_init(bar(B::o_final + x), 1);
            mbar_init(bar(B::sched_full + x), 1);
            mbar_init(bar(B::sched_empty + x), kIssuers + kSoftmaxWarpsArrive);
            mbar_init(bar(B::turn + x), 1);
        }
        mbar_init(bar(B::drain), kIssuers);
        for (int s = 0; s < S; ++s) {
            mbar_init(bar(B::kv_full + s), 1);
            mbar_init(bar(B::kv_empty + s), kIssuers);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Ctl ctl{abort_flag, p.words, p.wait_limit};

    if (warp >= 8) {
        regs_dec<kRegsControl>();
        if (warp == kProducerWarp && lane == 0) {
            // ---------------- scheduler + TMA producer ----------------
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            uint32_t stage = 0, kv_phase = 0, q_phase = 0;
            uint32_t q_fills = 0, kv_fills = 0;   // copies issued so far
            bool withhold = p.withhold_q != 0;    // test hook: first Q copy never issued
            bool ok = true;
            for (uint32_t it = 0; ok; ++it) {
                const uint32_t sl = it & 1u, ph = (it >> 1) & 1u;
                if (!(ok = wait_bar(bar(B::sched_empty + sl), ph ^ 1u, ctl, kWhereSched))) break;
                const int u = static_cast<int>(atomicAdd(&p.words->sched_counter, 1u));
                sched_unit[sl] = u;
                mbar_arrive(bar(B::sched_full + sl));
                if (u >= p.n_units) break;
                const Unit un = decode_unit(p, u);
                if (!(ok = wait_bar(bar(B::q_empty), q_phase ^ 1u, ctl, kWhereProducerQ))) break;
                q_phase ^= 1u;
                if (withhold) {
                    // nothing will ever complete this q_full phase: the MMA
                    // thread's bounded wait must expire (tests only)
                    withhold = false;
                } else {
                    mbar_arrive_expect_tx(bar(B::q_full), (un.has1 ? 2 : 1) * C::kQKTileBytes);
                    ++q_fills;
                    for (int x = 0; x < (un.has1 ? 2 : 1); ++x) {
                        if constexpr (F8) {
                            tma_load_4d(sq + x * C::kQKTileBytes, &tmap_q, bar(B::q_full), 0,
                                        un.h, (2 * un.pair + x) * BM, un.c);
                        } else {
                            for (int hf = 0; hf < C::kHalves; ++hf)
                                tma_load_4d(sq + x * C::kQKTileBytes + hf * C::kHalfBytes, &tmap_q,
                                            bar(B::q_full), hf * 64, un.h, (2 * un.pair + x) * BM,
                                            un.c);
                        }
                    }
                }
                // key tile t of the visible chunk in ring slot `slot`: the visible
                // chunks have consecutive ids, so their slots follow each other mod R
                int t = 0, slot = ring_slot(visible_chunk_id(p.round, p.h_valid, 0), p.R);
                for (int j = 0; ok && j < un.n_kt; ++j, next_key_tile(t, slot, p)) {
                    for (int kv = 0; kv < 2; ++kv) {
                        if (!(ok = wait_bar(bar(B::kv_empty + stage), kv_phase ^ 1u, ctl,
                                            kWhereProducerKV)))
                            break;
                        const bool k_codes = F8 && kv == 0;   // E4M3 K tile: one 128-byte box
                        mbar_arrive_expect_tx(bar(B::kv_full + stage),
                                              k_codes ? C::kQKTileBytes : C::kTileBytes);
                        ++kv_fills;
                        if (k_codes) {
                            tma_load_4d(skv + stage * C::kTileBytes, &tmap_k,
                                        bar(B::kv_full + stage), 0, un.h, t * BN, slot);
                        } else {
                            const CUtensorMap *map = kv ? &tmap_v : &tmap_k;
                            for (int hf = 0; hf < C::kHalves; ++hf)
                                tma_load_4d(skv + stage * C::kTileBytes + hf * C::kHalfBytes, map,
                                            bar(B::kv_full + stage), hf * 64, un.h, t * BN, slot);
                        }
                        if (++stage == S) { stage = 0; kv_phase ^= 1u; }
                    }
                }
            }
            if (!ok) {
                // let every copy already issued land before the CTA releases smem
                if (q_fills) wait_bar(bar(B::q_full), (q_fills - 1) & 1u, ctl, kWhereDrain, true);
                for (uint32_t s = 0; s < static_cast<uint32_t>(S); ++s) {
                    const uint32_t f = (kv_fills + S - 1 - s) / S;   // fills of stage s
                    if (f) wait_bar(bar(B::kv_full + s), (f - 1) & 1u, ctl, kWhereDrain, true);
                }
            }
        } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
            // ---------------- MMA issuer of query tile x ----------------
            // The whole warp runs the loop and its waits (so the loop's values are
            // warp-uniform), and one elected lane issues every MMA, commit and
            // arrival.  Timed on B200 this issues ~15% more MMAs per cycle than a
            // single divergent lane, whose operands must be moved into uniform
            // registers one MMA at a time.
            // The issuers of the two query tiles take turns: issuer x waits on
            // turn + x and hands over by arriving on turn + (x ^ 1), so the
            // tensor pipe receives one fixed order, QK_0(0) QK_1(0) | PV_0(j)
            // QK_0(j+1) | PV_1(j) QK_1(j+1) | ...  Both wait for every K/V stage
            // and unit, and both commit every stage release (the stage and
            // q_empty barriers count two arrivals); an issuer whose tile lies
            // past the chunk's end still takes its turns.  With each issuer on
            // its own SMSP, the softmax warps that share an SMSP with one see
            // half the MMA-issue traffic (clock64 stamps: the last P arrival of
            // a tile 40-80 cycles earlier).
            const int x = warp - kMmaWarp;
            const bool leader = elect_one_sync();
            uint32_t stage = 0, kv_phase = 0, q_phase = 0, p_phase = 0, turn_phase = 0;
            const uint32_t tSx = tmem + (x ? C::kS1 : C::kS0);
            const uint32_t tOx = tmem + (x ? C::kO1 : C::kO0);
            const uint32_t sQx = sq + x * C::kQKTileBytes;
            bool ok = true;
            bool first_turn = x == 0;
            auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t where) -> bool {
                const bool r = wait_bar(b, parity, ctl, where);
                return __all_sync(0xFFFFFFFFu, r);
            };
            auto next_stage = [&](uint32_t &st) -> bool {
                st = stage;
                const bool r = wait_all(bar(B::kv_full + stage), kv_phase, kWhereMmaKV);
                if (++stage == static_cast<uint32_t>(S)) { stage = 0; kv_phase ^= 1u; }
                tc_fence_after();
                return r;
            };
            auto take_turn = [&]() -> bool {
                if (first_turn) { first_turn = false; return true; }
                const bool r = wait_all(bar(B::turn + x), turn_phase, kWhereMmaTurn);
                turn_phase ^= 1u;
                tc_fence_after();
                return r;
            };
            auto pass_turn = [&]() {
                tc_fence_before();
                __syncwarp();
                if (leader) mbar_arrive(bar(B::turn + (x ^ 1)));
                __syncwarp();
            };
            for (uint32_t it = 0; ok; ++it) {
                const uint32_t sl = it & 1u, ph = (it >> 1) & 1u;
                if (!(ok = wait_all(bar(B::sched_full + sl), ph, kWhereSched))) break;
                const int u = sched_unit[sl];
                __syncwarp();
                if (leader) mbar_arrive(bar(B::sched_empty + sl));
                if (u >= p.n_units) break;
                const Unit un = decode_unit(p, u);
                const bool mine = x == 0 || un.has1;
                if (!(ok = wait_all(bar(B::q_full), q_phase, kWhereMmaQ))) break;
                q_phase ^= 1u;
                uint32_t kst;
                if (!(ok = next_stage(kst))) break;
                if (!(ok = take_turn())) break;
                if (leader) {
                    if (mine) {
                        issue_qk<D, F8>(tSx, sQx, skv + kst * C::kTileBytes);
                        umma_commit(bar(B::s_full + x));
                    }
                    umma_commit(bar(B::kv_empty + kst));
                    if (un.n_kt == 1) umma_commit(bar(B::q_empty));
                }
                pass_turn();
                for (int j = 0; ok && j < un.n_kt; ++j) {
                    const bool more = j + 1 < un.n_kt;
                    uint32_t vst, kst2 = 0;
                    if (!(ok = next_stage(vst))) break;
                    if (more && !(ok = next_stage(kst2))) break;
                    if (!(ok = take_turn())) break;
                    if (mine) {
                        if (!(ok = wait_all(bar(B::p_half + x), p_phase, kWhereMmaP))) break;
                        tc_fence_after();
                        if (leader) issue_pv_half<D>(tOx, tSx, skv + vst * C::kTileBytes, 0, j > 0);
                        __syncwarp();
                        if (!(ok = wait_all(bar(B::p_ready + x), p_phase, kWhereMmaP))) break;
                        p_phase ^= 1u;
                        tc_fence_after();
                        if (leader) issue_pv_half<D>(tOx, tSx, skv + vst * C::kTileBytes, 1, true);
                        __syncwarp();
                    }
                    if (leader) {
                        if (more) {
                            if (mine) {
                                issue_qk<D, F8>(tSx, sQx, skv + kst2 * C::kTileBytes);
                                umma_commit(bar(B::s_full + x));
                            }
                        } else if (mine) {
                            umma_commit(bar(B::o_final + x));
                        }
                        umma_commit(bar(B::kv_empty + vst));
                        if (more) {
                            umma_commit(bar(B::kv_empty + kst2));
                            if (j + 2 == un.n_kt) umma_commit(bar(B::q_empty));
                        }
                    }
                    pass_turn();
                }
            }
            // every MMA issued by this warp's leader completes before TMEM is released
            if (leader) umma_commit(bar(B::drain));
            __syncwarp();
            wait_bar(bar(B::drain), 0u, ctl, kWhereDrain, true);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // ---------------- softmax warpgroups ----------------
        const int x = warp >> 2;                    // query tile of this warpgroup
        const int row = threadIdx.x & 127;          // TMEM lane = row of the tile
        const uint32_t lane_sel = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_sel + (x ? C::kS1 : C::kS0);
        const uint32_t tO = tmem + lane_sel + (x ? C::kO1 : C::kO0);
        const float scale0 = p.scale_log2;
        uint32_t s_phase = 0, o_phase = 0;
        bool ok = true;
        for (uint32_t it = 0; ok; ++it) {
            const uint32_t sl = it & 1u, ph = (it >> 1) & 1u;
            ok = wait_bar(bar(B::sched_full + sl), ph, ctl, kWhereSched);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) break;
            const int u = sched_unit[sl];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B::sched_empty + sl));
            if (u >= p.n_units) break;
            const Unit un = decode_unit(p, u);
            if (x == 1 && !un.has1) continue;       // the tile lies past the chunk's end
            const int q_row = (2 * un.pair + x) * BM + row;     // row inside chunk c
            // F8: the row's Q scale; a key tile's K scale is read per tile below
            float sq = 1.0f;
            if constexpr (F8)
                if (q_row < p.L) sq = p.q_scale[static_cast<long>(un.h) * p.T +
                                                static_cast<long>(un.c) * p.L + q_row];
            float m_run = -INFINITY, l_run = 0.f;
            // key tile t inside its chunk, held in ring slot `slot`
            int t = 0, slot = ring_slot(visible_chunk_id(p.round, p.h_valid, 0), p.R);
            for (int j = 0; j < un.n_kt; ++j, next_key_tile(t, slot, p)) {
                float scale = scale0;
                if constexpr (F8) {
                    // s = (q8 . k8) * sq * sk: fold both scales into the exponent scale
                    scale = scale0 * sq *
                            p.k_scale[(static_cast<long>(slot) * p.n_ktiles + t) * p.H + un.h];
                }
                const uint64_t sc2 = f2_pack(scale, scale);
                ok = wait_bar(bar(B::s_full + x), s_phase, ctl, kWhereSoftS);
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) break;
                s_phase ^= 1u;
                tc_fence_after();
                uint32_t r[4][32];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + q4 * 32, r[q4]);
                tmem_wait_ld();
                const int valid = t == p.n_ktiles - 1 ? p.L - t * BN : BN;
                if (valid < BN) {                   // last tile of a chunk: rows >= L
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (q4 * 32 + e >= valid) r[q4][e] = __float_as_uint(-INFINITY);
                }
                // row maximum: 8 independent chains of 3-input max, then a tree
                float mx8[8];
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    mx8[c] = fmaxf(__uint_as_float(r[c >> 1][(c & 1) * 16]),
                                   __uint_as_float(r[c >> 1][(c & 1) * 16 + 1]));
#pragma unroll
                for (int k = 1; k < 8; ++k)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        mx8[c] = fmax3(mx8[c], __uint_as_float(r[c >> 1][(c & 1) * 16 + 2 * k]),
                                       __uint_as_float(r[c >> 1][(c & 1) * 16 + 2 * k + 1]));
                const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                                       fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                // The row maximum only moves forward when it grew by more than
                // 2^8: otherwise exponents stay <= 2^8 against the stale maximum
                // and O keeps its scale.  (At j = 0 PV overwrites O.)
                const float m_new = fmaxf(m_run, mx * scale);
                const bool need = m_new > m_run + kRescaleThreshold;
                const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
                if (need) {
                    l_run *= alpha;
                    m_run = m_new;
                }
                if (j > 0 && __any_sync(0xFFFFFFFFu, need)) {
                    // O is quiescent here: the MMA that filled S_x(j) was issued
                    // after PV_x(j-1), and PV_x(j) waits for this warpgroup.
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld32(tO + cc * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tO + cc * 32, o);
                    }
                }
                const uint64_t nm2 = f2_pack(-m_run, -m_run);
                uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    // P columns [64*hf, 64*hf + 64) -> packed bf16 TMEM columns [32*hf, 32*hf + 32)
                    uint32_t pk[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int col = 64 * hf + 2 * e;
                        const uint64_t s2 = f2_pack(__uint_as_float(r[col >> 5][col & 31]),
                                                    __uint_as_float(r[col >> 5][(col + 1) & 31]));
                        float x0, x1, p0, p1;
                        f2_unpack(f2_fma(s2, sc2, nm2), x0, x1);
                        if (kEmulatePeriod > 0 && (e % (kEmulatePeriod > 0 ? kEmulatePeriod : 1)) ==
                                                      kEmulatePeriod - 1) {
                            exp2_fma_pair(x0, x1, p0, p1);
                        } else {
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        }
                        acc[e & 3] = f2_add(acc[e & 3], f2_pack(p0, p1));
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(tS + 32 * hf, pk);
                    // publish this half of P (and any rescale of O before it)
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar(hf == 0 ? B::p_half + x : B::p_ready + x));
                }
                float a0, a1, b0, b1;
                f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
                f2_unpack(f2_add(acc[2], acc[3]), b0, b1);
                l_run += (a0 + a1) + (b0 + b1);
            }
            if (!ok) break;
            ok = wait_bar(bar(B::o_final + x), o_phase, ctl, kWhereSoftO);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) break;
            o_phase ^= 1u;
            tc_fence_after();
            const float inv_l = 1.0f / l_run;
            const bool store = q_row < p.L;
            const long n = static_cast<long>(un.c) * p.L + q_row;
            uint16_t *dst = p.o + (n * p.H + un.h) * D;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(tO + cc * 32, o);
                tmem_wait_ld();
                uint4 w[4];
                uint32_t *wp = reinterpret_cast<uint32_t *>(w);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    wp[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                        __uint_as_float(o[2 * e + 1]) * inv_l);
                if (store) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + cc * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) d4[e] = w[e];
                }
            }
            if (store && p.lse != nullptr)
                p.lse[static_cast<long>(un.h) * p.T + n] = m_run * 0.6931471805599453f + logf(l_run);
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) {
        __syncwarp();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

template <int D, bool F8>
static cudaError_t launch_attn_d(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                 const AttnParams &p, int grid, cudaStream_t stream)
{
    const uint32_t smem = Cfg<D, F8>::kSmemBytes;
    // The setmaxnreg split assumes the kernel was compiled to exactly the
    // launch budget; any other count could leave the increase waiting.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, chunk_causal_attn_kernel<D, F8>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != static_cast<int>(kRegsLaunch)) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(chunk_causal_attn_kernel<D, F8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(&p.words->sched_counter, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    chunk_causal_attn_kernel<D, F8><<<grid, kThreads, smem, stream>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

cudaError_t launch_attn(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                        const AttnParams &p, int D, int grid, cudaStream_t stream)
{
    return D == 128 ? launch_attn_d<128, false>(mq, mk, mv, p, grid, stream)
                    : launch_attn_d<64, false>(mq, mk, mv, p, grid, stream);
}

// E4M3 Q and K (maps over the code arrays, box 128 bytes x 1 x 128 rows), bf16 V;
// head_dim 128 only.
cudaError_t launch_attn_fp8qk(const CUtensorMap &mq8, const CUtensorMap &mk8, const CUtensorMap &mv,
                              const AttnParams &p, int grid, cudaStream_t stream)
{
    return launch_attn_d<128, true>(mq8, mk8, mv, p, grid, stream);
}

}  // namespace wf

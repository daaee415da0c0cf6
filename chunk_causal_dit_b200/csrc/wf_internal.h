// wf_internal.h -- plan structure, kernel parameter blocks and the ring/visibility
// arithmetic shared by host code (wf_plan_debug_ranges, launch set-up) and the
// kernels, so that what the debug dump reports is what the kernels execute.
#pragma once
#include <cstdint>
#include <vector>
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#ifdef __CUDACC__
#define WF_HD __host__ __device__ __forceinline__
#else
#define WF_HD inline
#endif

namespace wf {

constexpr int kMaxHeadDim = 128;

// Number of history chunks visible in round r: min(Hh, r) (rounds before the
// pipeline is full see fewer).
WF_HD int history_valid(long round, int n_hist)
{
    return round < static_cast<long>(n_hist) ? static_cast<int>(round) : n_hist;
}

// Non-negative modulo for ring slots.
WF_HD int ring_slot(long chunk_id, int R)
{
    long s = chunk_id % R;
    return static_cast<int>(s < 0 ? s + R : s);
}

// Absolute id of the b-th visible key chunk (b = 0 is the oldest) in round r.
WF_HD long visible_chunk_id(long round, int h_valid, int b)
{
    return round - h_valid + b;
}

// Status bits written by kernels into the plan's device status word.
enum : uint32_t {
    kStatusTimeout = 1u,
};

// Device-resident words owned by a plan (one 256-byte allocation).
struct DeviceWords {
    uint32_t status;          // OR of kStatus* bits
    uint32_t timeout_where;   // role/barrier code of the first timeout
    uint32_t sched_counter;   // attention work-unit counter (reset before each launch)
    uint32_t pad[61];
};

struct RopeParams {
    int dt, dh, dw;           // channel widths of the t / h / w blocks
    int F, gh, gw;            // chunk geometry for derived positions (F = 0: unset)
    double omega[kMaxHeadDim / 2];  // per channel pair: theta^(-2i/d_axis)
    int8_t axis[kMaxHeadDim / 2];   // per channel pair: 0 = t, 1 = h, 2 = w
};

struct AppendParams {
    const uint16_t *q, *k, *v;
    const int32_t *pos;       // [T,3] or nullptr (derive)
    const float *gamma_q, *gamma_k;
    uint16_t *q_out, *k_cache, *v_cache;   // q_out may be nullptr when q8 is set
    uint8_t *q8;              // fused FP8 Q: E4M3 codes [T,H,D] of bf16(q'), or nullptr
    float *q_scale;           // fused FP8 Q: [H][T] per-row scales
    long round;
    int L, W, R, H;
    int heads_per_block;      // heads covered by one block (blockIdx.y picks the group)
    float eps;
    RopeParams rope;
};

struct AttnParams {
    long round;
    int L, W, R, H, T;
    int h_valid;
    int n_qpairs;             // query tile pairs per chunk: ceil(ceil(L/128)/2)
    int n_ktiles;             // key tiles per chunk: ceil(L/128)
    int n_units;              // H * W * n_qpairs
    int head_block;           // heads per block of the unit order (1..H)
    float scale_log2;         // log2(e) / sqrt(D)
    unsigned long long wait_limit;  // SM clock cycles
    int withhold_q;           // test hook: withhold each CTA's first Q-tile copy
    uint16_t *o;
    float *lse;
    DeviceWords *words;
    const float *q_scale;     // FP8 Q.K^T only: [H][T] per-row Q scales
    const float *k_scale;     // FP8 Q.K^T only: [R][n_ktiles][H] per-tile K scales
};

// Epilogues of the bf16 GEMM (the first three are WF_EPI_* of the C ABI).
enum GemmEpilogue : int {
    kEpiStore = 0,            // C = A B^T + bias
    kEpiGeluTanh = 1,         // C = gelu_tanh(A B^T + bias)
    kEpiGatedResidual = 2,    // C = resid + gate[row / rows_per_group] * (A B^T + bias)
    kEpiQkvAppend = 3,        // QKV projection: RMSNorm + RoPE on q/k, q -> q_out, k/v -> ring
    kEpiConv = 4,             // causal 3x3x3 convolution (implicit GEMM): C = conv + bias
    kEpiConvResidual = 5,     // the same plus a residual: C = resid + conv + bias
};

struct GemmParams {
    int M, N, K;
    int n_ntiles, n_tiles;    // 256-column tiles per row block; all tiles (256 x 256)
    const float *bias;        // [N] or nullptr
    uint16_t *c;              // [M][N] bf16 (linear epilogues)
    const uint16_t *resid;    // [M][N] bf16 (gated residual)
    const float *gate;        // [G][N] (gated residual)
    int rows_per_group;
    // QKV epilogue: columns [0,HD) q, [HD,2HD) k, [2HD,3HD) v; rows are wave tokens
    uint16_t *q_out, *k_cache, *v_cache;
    const float *gamma_q, *gamma_k;
    long round;
    int L, W, R, H, D;
    float eps;
    RopeParams rope;
    int n_tab;                // (cos, sin) table entries: W*F*dt/2 + gh*dh/2 + gw*dw/2
    unsigned long long wait_limit;
    int withhold;             // test hook: no CTA issues (or arms) its first stage's copies
    DeviceWords *words;
    // causal 3x3x3 convolution (kEpiConv*): output [ct][ch][cw][N] with M = ct*ch*cw
    // pixels; a K slice is one tap (dt, dy, dx) x 64 input channels
    int ct, ch, cw, cin;
    int n_cblk;               // 64-channel blocks of the input: ceil(cin / 64)
    int n_py, n_px;           // 16 x 16 pixel tiles per frame (rows, columns)
    int use_hist;             // taps before the chunk read the history map (else zeros)
};

// NVTX range around a host call of the C ABI (header-only NVTX v3: without a
// profiler attached a push/pop is a null-callback check), so that a timeline
// shows each launch under the library call that made it.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Host helpers shared by the plan API and the plan-free attention entry point
// (defined in wf_api.cu).
// 4-D TMA map over a [n3][n2][H][D] bf16 tensor, box 64 x 1 x box_rows x 1,
// 128-byte swizzle, rows past n2 read as zero.
bool encode_map(CUtensorMap *map, const void *base, int D, int H, int n2, int n2_stride_rows,
                int n3, int box_rows = 128);
// WF_OK, or the status wf_plan returns for this shape.
int check_round_shape(int chunk_tokens, int n_wave_chunks, int n_hist_chunks, int heads,
                      int head_dim);
// Heads per block of the attention's unit order (1..H) for a round with h_valid
// history chunks; k_bytes is the size of a key element (2 bf16, 1 E4M3),
// l2_bytes the device's L2 size, n_ctas the attention grid.
int attn_head_block(int H, int W, int h_valid, int L, int D, int k_bytes, long long l2_bytes,
                    int n_ctas);

}  // namespace wf

struct wf_plan_s {
    int L, W, Hh, H, D, R;
    double theta;
    double eps;
    wf::RopeParams rope;
    unsigned long long wait_limit;
    int withhold_q;           // test hook, see wf_plan_set_withhold_q
    int attn_kernel;          // WF_ATTN_* (wf_plan_set_attn_kernel)
    int device;               // -1: no device state
    int num_sms;
    long long l2_bytes;       // L2 cache size of `device`
    int head_block;           // attention unit order: heads per block, 0 = chosen per round
    std::vector<int> head_block_cache;   // attention head blocks, [fp8 keys][h_valid 0..min(Hh, 63)]; 0: not yet
    int cc_major, cc_minor;   // compute capability of `device`
    wf::DeviceWords *words;   // device memory
};

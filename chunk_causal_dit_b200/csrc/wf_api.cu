// wf_api.cu -- the C ABI of libwf.so (declared in include/wf.h): plan creation and
// validation, TMA tensor-map set-up, and the two hot-path launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "wf.h"
#include "wf_check.cuh"
#include "wf_internal.h"

namespace wf {
cudaError_t launch_append(const AppendParams &p, int D, cudaStream_t stream, DeviceWords *words);
cudaError_t launch_attn(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                        const AttnParams &p, int D, int grid, cudaStream_t stream);
cudaError_t launch_attn_pair(const CUtensorMap &mq, const CUtensorMap &mk64, const CUtensorMap &mv,
                             const AttnParams &p, cudaStream_t stream);
cudaError_t launch_attn_fp8qk(const CUtensorMap &mq8, const CUtensorMap &mk8, const CUtensorMap &mv,
                              const AttnParams &p, int grid, cudaStream_t stream);
cudaError_t launch_quantize_rows(const uint16_t *q, uint8_t *q8, float *scale, long n_rows, int H,
                                 int D, cudaStream_t stream, DeviceWords *words);
cudaError_t launch_quantize_tiles(const uint16_t *k, uint8_t *k8, float *scale, long first_chunk,
                                  int n_chunks, int L, int H, int R, int D, cudaStream_t stream,
                                  DeviceWords *words);
cudaError_t launch_gemm(const CUtensorMap &ma, const CUtensorMap &mb, const GemmParams &p, int epi,
                        cudaStream_t stream);
int gemm_tab_max();
cudaError_t launch_layer_norm_modulate(const uint16_t *x, const float *shift, const float *scale,
                                       uint16_t *y, long M, int C, int rows_per_group, float eps,
                                       cudaStream_t stream);
int ln_max_channels();
cudaError_t launch_conv(const CUtensorMap &mx, const CUtensorMap &mh, const CUtensorMap &mw,
                        const GemmParams &p, bool residual, int bn, cudaStream_t stream);
cudaError_t launch_rms_norm_silu(const uint16_t *x, const float *gamma, uint16_t *y, long M, int C,
                                 float eps, cudaStream_t stream);
int rms_norm_silu_max_channels();
}  // namespace wf

namespace wf {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

// 4-D map over a [n3][n2][H][D] bf16 tensor (slot/chunk, row, head, channel),
// box = 64 channels x 1 head x box_rows rows x 1 slot, 128-byte swizzle, OOB rows read 0.
bool encode_map(CUtensorMap *map, const void *base, int D, int H, int n2, int n2_stride_rows,
                int n3, int box_rows)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(n2), static_cast<cuuint64_t>(n3)};
    const cuuint64_t row = static_cast<cuuint64_t>(H) * D * 2;
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, row,
                                   row * static_cast<cuuint64_t>(n2_stride_rows)};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The shape rules of a wave round (wf_plan and the plan-free attention entry
// point apply the same ones): positive sizes, head_dim 64 or 128, and index
// ranges that fit the kernels' int / 40-bit arithmetic.
int check_round_shape(int chunk_tokens, int n_wave_chunks, int n_hist_chunks, int heads,
                      int head_dim)
{
    if (chunk_tokens < 1 || n_wave_chunks < 1 || n_hist_chunks < 0 || heads < 1)
        return WF_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return WF_ERR_UNSUPPORTED;
    const long long T = static_cast<long long>(chunk_tokens) * n_wave_chunks;
    const long long R = static_cast<long long>(n_hist_chunks) + n_wave_chunks;
    const long long hd = static_cast<long long>(heads) * head_dim;
    if (T * hd >= (1ll << 31) || R * chunk_tokens * hd >= (1ll << 40) || R > INT_MAX)
        return WF_ERR_INVALID_ARG;
    const long long qtiles = (chunk_tokens + 127) / 128;
    if (static_cast<long long>(heads) * n_wave_chunks * ((qtiles + 1) / 2) >= INT_MAX)
        return WF_ERR_INVALID_ARG;
    return WF_OK;
}

// Heads per block of the attention's unit order.  The units of a block of heads
// are handed out before the next block's, longest first inside the block, so
// the keys and values being read at any moment are those of one or two blocks.
// A block's visible key/value chunks (h_valid + W of them, for each of its
// heads) are kept within half of the L2 cache, so that every unit that reads
// a key tile after the first finds it in L2.  Among the counts that fit, the
// one whose schedule ends earliest is taken: each count is played through the
// kernel's dynamic schedule (each unit goes to the CTA that frees first; a
// unit costs its key tiles, 0.93 of that for a one-tile unit, plus 3 tiles of
// set-up), with ties going to the larger count.  Results do not depend on it:
// every unit computes the same rows in the same order.
int attn_head_block(int H, int W, int h_valid, int L, int D, int k_bytes, long long l2_bytes,
                    int n_ctas)
{
    const double per_head = static_cast<double>(h_valid + W) * L * D * (k_bytes + 2);
    long long g_max = H;
    if (l2_bytes > 0) {
        g_max = static_cast<long long>(0.5 * static_cast<double>(l2_bytes) / per_head);
        g_max = g_max < 1 ? 1 : (g_max > H ? H : g_max);
    }
    const int n_ktiles = (L + 127) / 128;
    const int n_qpairs = (n_ktiles + 1) / 2;
    const long long n_units = static_cast<long long>(H) * W * n_qpairs;
    constexpr int kMaxCtas = 1024;
    if (n_ctas < 1 || n_ctas > kMaxCtas || n_units * g_max > (4ll << 20))
        return static_cast<int>(g_max);
    double t[kMaxCtas];
    int best_g = static_cast<int>(g_max);
    double best = 0.0;
    for (int g = static_cast<int>(g_max); g >= 1; --g) {
        for (int i = 0; i < n_ctas; ++i) t[i] = 0.0;
        for (int hb = 0; hb < H; hb += g) {
            const int gb = H - hb < g ? H - hb : g;
            for (int c = W - 1; c >= 0; --c)
                for (int k = 0; k < gb * n_qpairs; ++k) {
                    const int pair = k % n_qpairs;
                    const bool has1 = (2 * pair + 1) * 128 < L;
                    const double d =
                        static_cast<double>(h_valid + c + 1) * n_ktiles * (has1 ? 1.0 : 0.93) + 3.0;
                    // the CTA that frees first (heap root) takes the unit
                    double v = t[0] + d;
                    int i = 0;
                    while (true) {
                        const int l = 2 * i + 1, r = l + 1;
                        int m = i;
                        double mv = v;
                        if (l < n_ctas && t[l] < mv) { m = l; mv = t[l]; }
                        if (r < n_ctas && t[r] < mv) { m = r; mv = t[r]; }
                        if (m == i) break;
                        t[i] = t[m];
                        i = m;
                    }
                    t[i] = v;
                }
        }
        double end = 0.0;
        for (int i = 0; i < n_ctas; ++i) end = t[i] > end ? t[i] : end;
        if (g == g_max || end < best * (1.0 - 2e-3)) {
            best = end;
            best_g = g;
        }
    }
    return best_g;
}

}  // namespace wf

namespace {

constexpr unsigned long long kDefaultWaitLimit = 1ull << 32;   // ~2 s of SM clock

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void fill_rope_table(wf::RopeParams &r, double theta)
{
    const int width[3] = {r.dt, r.dh, r.dw};
    int pair = 0;
    for (int a = 0; a < 3; ++a)
        for (int i = 0; i < width[a] / 2; ++i, ++pair) {
            r.omega[pair] = std::pow(theta, -2.0 * i / width[a]);
            r.axis[pair] = static_cast<int8_t>(a);
        }
}

// The same map over a [n3][n2][H][D] array of one-byte E4M3 codes: box = D bytes
// (one 128-byte swizzle row at D = 128) x 1 head x 128 rows x 1.
bool encode_map_u8(CUtensorMap *map, const void *base, int D, int H, int n2, int n3)
{
    auto enc = wf::tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(n2), static_cast<cuuint64_t>(n3)};
    const cuuint64_t row = static_cast<cuuint64_t>(H) * D;
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D), row,
                                   row * static_cast<cuuint64_t>(n2)};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(D), 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// 2-D map over a row-major [rows][cols] bf16 matrix (a GEMM operand, K = cols
// innermost): box = 64 columns x 128 rows, 128-byte swizzle, out-of-range reads 0.
bool encode_map_2d(CUtensorMap *map, const void *base, long rows, long cols)
{
    auto enc = wf::tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4-D map over a channels-last video [T][H][W][C] bf16: box = 64 channels x 16
// columns x 10 rows x 1 frame (160 pixels, one 128-byte swizzle row each: a CTA's
// 8 output rows and the rows above and below); reads outside the frame or before
// the first frame return zeros.
bool encode_map_video(CUtensorMap *map, const void *base, int T, int H, int W, int C)
{
    auto enc = wf::tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(W),
                                static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
    const cuuint64_t pix = static_cast<cuuint64_t>(C) * 2;
    const cuuint64_t strides[3] = {pix, pix * W, pix * W * H};
    const cuuint32_t box[4] = {64, 16, 10, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over conv weights [Cout][27][Cin] bf16: box = 64 channels x 1 tap x rows
// output channels.
bool encode_map_convw(CUtensorMap *map, const void *base, int Cout, int Cin, int rows)
{
    auto enc = wf::tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(Cin), 27, static_cast<cuuint64_t>(Cout)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(Cin) * 2,
                                   static_cast<cuuint64_t>(Cin) * 2 * 27};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(rows)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile counts of a GEMM (256 x 256 tiles); false if they do not fit an int.
bool gemm_tiles(long M, long N, wf::GemmParams &g)
{
    const long nt = (N + 255) / 256, mt = (M + 255) / 256;
    if (mt * nt >= INT_MAX) return false;
    g.n_ntiles = static_cast<int>(nt);
    g.n_tiles = static_cast<int>(mt * nt);
    return true;
}

int check_device(const wf_plan_s *p)
{
    if (p->device < 0 || p->words == nullptr) return WF_ERR_NO_DEVICE;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return WF_ERR_CUDA;
    if (cur != p->device) return WF_ERR_INVALID_ARG;   // plan belongs to another device
    if (p->cc_major != 10 || p->cc_minor != 0) return WF_ERR_DEVICE;   // kernels are sm_100a
    return WF_OK;
}

}  // namespace

extern "C" {

int wf_plan(int chunk_tokens, int n_wave_chunks, int n_hist_chunks, int heads, int head_dim,
            wf_plan_t *out)
{
    if (out == nullptr) return WF_ERR_INVALID_ARG;
    *out = nullptr;
    if (int st = wf::check_round_shape(chunk_tokens, n_wave_chunks, n_hist_chunks, heads, head_dim))
        return st;
    const long long R = static_cast<long long>(n_hist_chunks) + n_wave_chunks;

    wf_plan_s *p = new (std::nothrow) wf_plan_s();
    if (p == nullptr) return WF_ERR_CUDA;
    p->L = chunk_tokens;
    p->W = n_wave_chunks;
    p->Hh = n_hist_chunks;
    p->H = heads;
    p->D = head_dim;
    p->R = static_cast<int>(R);
    p->theta = 10000.0;
    p->eps = 1e-6;
    p->rope.dh = p->rope.dw = 2 * (head_dim / 6);
    p->rope.dt = head_dim - 2 * p->rope.dh;
    p->rope.F = p->rope.gh = p->rope.gw = 0;
    fill_rope_table(p->rope, p->theta);
    p->wait_limit = kDefaultWaitLimit;
    p->withhold_q = 0;
    p->attn_kernel = WF_ATTN_AUTO;
    p->device = -1;
    p->num_sms = 0;
    p->l2_bytes = 0;
    p->head_block = 0;
    try {   // h_valid = 0 .. min(Hh, 63) are kept; a longer history is rare
        p->head_block_cache.assign(2 * static_cast<size_t>(std::min(n_hist_chunks, 63) + 1), 0);
    } catch (...) {
        delete p;
        return WF_ERR_CUDA;
    }
    p->cc_major = p->cc_minor = 0;
    p->words = nullptr;

    int dev = -1;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int sms = 0, ma = 0, mi = 0, l2 = 0;
        void *w = nullptr;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&ma, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&mi, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
            cudaMalloc(&w, sizeof(wf::DeviceWords)) == cudaSuccess) {
            if (cudaMemset(w, 0, sizeof(wf::DeviceWords)) == cudaSuccess) {
                p->device = dev;
                p->num_sms = sms;
                p->l2_bytes = l2;
                p->cc_major = ma;
                p->cc_minor = mi;
                p->words = static_cast<wf::DeviceWords *>(w);
            } else {
                cudaFree(w);
            }
        }
    }
    (void)cudaGetLastError();   // a machine without a GPU leaves an error behind
    *out = p;
    return WF_OK;
}

int wf_plan_set_rope(wf_plan_t p, int frames_per_chunk, int grid_h, int grid_w, double theta)
{
    if (p == nullptr || frames_per_chunk < 1 || grid_h < 1 || grid_w < 1 || !(theta > 0.0) ||
        static_cast<long long>(frames_per_chunk) * grid_h * grid_w != p->L)
        return WF_ERR_INVALID_ARG;
    p->rope.F = frames_per_chunk;
    p->rope.gh = grid_h;
    p->rope.gw = grid_w;
    p->theta = theta;
    fill_rope_table(p->rope, theta);
    return WF_OK;
}

int wf_plan_set_rope_split(wf_plan_t p, int d_t, int d_h, int d_w)
{
    if (p == nullptr || d_t < 0 || d_h < 0 || d_w < 0 || ((d_t | d_h | d_w) & 1) ||
        d_t + d_h + d_w != p->D)
        return WF_ERR_INVALID_ARG;
    p->rope.dt = d_t;
    p->rope.dh = d_h;
    p->rope.dw = d_w;
    fill_rope_table(p->rope, p->theta);
    return WF_OK;
}

int wf_plan_set_norm_eps(wf_plan_t p, double eps)
{
    if (p == nullptr || !(eps >= 0.0)) return WF_ERR_INVALID_ARG;
    p->eps = eps;
    return WF_OK;
}

int wf_plan_set_wait_limit(wf_plan_t p, unsigned long long cycles)
{
    if (p == nullptr) return WF_ERR_INVALID_ARG;
    p->wait_limit = cycles == 0 ? kDefaultWaitLimit : cycles;
    return WF_OK;
}

int wf_plan_set_withhold_q(wf_plan_t p, int on)
{
    if (p == nullptr) return WF_ERR_INVALID_ARG;
    p->withhold_q = on ? 1 : 0;
    return WF_OK;
}

int wf_plan_set_attn_kernel(wf_plan_t p, int kind)
{
    if (p == nullptr) return WF_ERR_INVALID_ARG;
    if (kind != WF_ATTN_AUTO && kind != WF_ATTN_SINGLE && kind != WF_ATTN_PAIR)
        return WF_ERR_INVALID_ARG;
    if (kind == WF_ATTN_PAIR && p->D != 128) return WF_ERR_UNSUPPORTED;
    p->attn_kernel = kind;
    return WF_OK;
}

int wf_plan_set_head_block(wf_plan_t p, int heads)
{
    if (p == nullptr || heads < 0 || heads > p->H) return WF_ERR_INVALID_ARG;
    p->head_block = heads;
    return WF_OK;
}

namespace {

// The attention's heads per block for a round with h_valid history chunks: the
// plan's setting, else wf::attn_head_block's choice (kept per h_valid).
int plan_head_block(wf_plan_s *p, int h_valid, bool fp8_keys, int grid)
{
    if (p->head_block > 0) return p->head_block;
    const int per_key = static_cast<int>(p->head_block_cache.size() / 2);
    if (h_valid >= per_key)
        return wf::attn_head_block(p->H, p->W, h_valid, p->L, p->D, fp8_keys ? 1 : 2,
                                   p->l2_bytes, grid);
    int &slot = p->head_block_cache[(fp8_keys ? 1 : 0) * per_key + h_valid];
    if (slot <= 0)
        slot = wf::attn_head_block(p->H, p->W, h_valid, p->L, p->D, fp8_keys ? 1 : 2, p->l2_bytes,
                                   grid);
    return slot;
}

}  // namespace

int wf_plan_head_block(wf_plan_t p, long round, int fp8_keys)
{
    if (p == nullptr || round < 0) return -1;
    const int n_qpairs = ((p->L + 127) / 128 + 1) / 2;
    const int n_units = p->H * p->W * n_qpairs;
    const int grid = n_units < p->num_sms ? n_units : p->num_sms;
    return plan_head_block(p, wf::history_valid(round, p->Hh), fp8_keys != 0, grid);
}

int wf_attn_head_block(int heads, int n_wave_chunks, int h_valid, int chunk_tokens, int head_dim,
                       int key_bytes, long long l2_bytes, int n_ctas)
{
    if (heads < 1 || n_wave_chunks < 1 || h_valid < 0 || chunk_tokens < 1 || head_dim < 1 ||
        (key_bytes != 1 && key_bytes != 2))
        return -1;
    return wf::attn_head_block(heads, n_wave_chunks, h_valid, chunk_tokens, head_dim, key_bytes,
                               l2_bytes, n_ctas);
}

void wf_plan_destroy(wf_plan_t p)
{
    if (p == nullptr) return;
    if (p->words != nullptr) {
        int cur = -1;
        const bool switch_dev = cudaGetDevice(&cur) == cudaSuccess && cur != p->device;
        if (switch_dev) cudaSetDevice(p->device);
        cudaFree(p->words);
        if (switch_dev) cudaSetDevice(cur);
    }
    delete p;
}

size_t wf_cache_bytes(wf_plan_t p)
{
    if (p == nullptr) return 0;
    return static_cast<size_t>(p->R) * p->L * p->H * p->D * 2;
}

double wf_useful_flops(wf_plan_t p, long round)
{
    if (p == nullptr || round < 0) return -1.0;
    const int hv = wf::history_valid(round, p->Hh);
    double chunks = 0.0;
    for (int c = 0; c < p->W; ++c) chunks += hv + c + 1;
    return 4.0 * p->H * p->D * static_cast<double>(p->L) * p->L * chunks;
}

// The append of both entry points below (q8 == nullptr: the plain append).
static int append_common(wf_plan_t p, long round, const void *q, const void *k, const void *v,
                         const int32_t *pos_thw, const float *gamma_q, const float *gamma_k,
                         void *q_out, uint8_t *q8, float *q_scale, void *k_cache, void *v_cache,
                         void *stream)
{
    if (p == nullptr || round < 0) return WF_ERR_INVALID_ARG;
    if (!q || !k || !v || !gamma_q || !gamma_k || !k_cache || !v_cache) return WF_ERR_INVALID_ARG;
    if (q8 == nullptr && !q_out) return WF_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_out) ||
        !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(gamma_q) || !aligned16(gamma_k))
        return WF_ERR_INVALID_ARG;
    if (q8 != nullptr && (!aligned16(q8) || !q_scale || !aligned4(q_scale)))
        return WF_ERR_INVALID_ARG;
    if (pos_thw == nullptr && p->rope.F == 0) return WF_ERR_INVALID_ARG;
    if (pos_thw != nullptr && (reinterpret_cast<uintptr_t>(pos_thw) & 3u)) return WF_ERR_INVALID_ARG;
    if (pos_thw == nullptr &&
        (round + p->W) > static_cast<long>(INT_MAX / p->rope.F))
        return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;

    wf::AppendParams a;
    a.q = static_cast<const uint16_t *>(q);
    a.k = static_cast<const uint16_t *>(k);
    a.v = static_cast<const uint16_t *>(v);
    a.pos = pos_thw;
    a.gamma_q = gamma_q;
    a.gamma_k = gamma_k;
    a.q_out = static_cast<uint16_t *>(q_out);
    a.q8 = q8;
    a.q_scale = q_scale;
    a.k_cache = static_cast<uint16_t *>(k_cache);
    a.v_cache = static_cast<uint16_t *>(v_cache);
    a.round = round;
    a.L = p->L;
    a.W = p->W;
    a.R = p->R;
    a.H = p->H;
    a.eps = static_cast<float>(p->eps);
    a.rope = p->rope;
    cudaError_t e = wf::launch_append(a, p->D, static_cast<cudaStream_t>(stream), p->words);
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_qk_norm_rope_append(wf_plan_t p, long round, const void *q, const void *k, const void *v,
                           const int32_t *pos_thw, const float *gamma_q, const float *gamma_k,
                           void *q_out, void *k_cache, void *v_cache, void *stream)
{
    wf::NvtxRange nvtx_range("wf_qk_norm_rope_append");
    return append_common(p, round, q, k, v, pos_thw, gamma_q, gamma_k, q_out, nullptr, nullptr,
                         k_cache, v_cache, stream);
}

int wf_qk_norm_rope_append_fp8q(wf_plan_t p, long round, const void *q, const void *k,
                                const void *v, const int32_t *pos_thw, const float *gamma_q,
                                const float *gamma_k, void *q_out, void *q8, float *q_scale,
                                void *k_cache, void *v_cache, void *stream)
{
    wf::NvtxRange nvtx_range("wf_qk_norm_rope_append_fp8q");
    if (q8 == nullptr) return WF_ERR_INVALID_ARG;
    return append_common(p, round, q, k, v, pos_thw, gamma_q, gamma_k, q_out,
                         static_cast<uint8_t *>(q8), q_scale, k_cache, v_cache, stream);
}

int wf_chunk_causal_attn(wf_plan_t p, long round, const void *q_out, const void *k_cache,
                         const void *v_cache, void *o, float *lse, void *stream)
{
    wf::NvtxRange nvtx_range("wf_chunk_causal_attn");
    if (p == nullptr || round < 0) return WF_ERR_INVALID_ARG;
    if (!q_out || !k_cache || !v_cache || !o) return WF_ERR_INVALID_ARG;
    if (!aligned16(q_out) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;

    CUtensorMap mq, mk, mv;
    if (!wf::encode_map(&mq, q_out, p->D, p->H, p->L, p->L, p->W) ||
        !wf::encode_map(&mk, k_cache, p->D, p->H, p->L, p->L, p->R) ||
        !wf::encode_map(&mv, v_cache, p->D, p->H, p->L, p->L, p->R))
        return WF_ERR_CUDA;

    wf::AttnParams a;
    a.round = round;
    a.L = p->L;
    a.W = p->W;
    a.R = p->R;
    a.H = p->H;
    a.T = p->L * p->W;
    a.h_valid = wf::history_valid(round, p->Hh);
    a.n_ktiles = (p->L + 127) / 128;
    a.n_qpairs = (a.n_ktiles + 1) / 2;
    a.n_units = p->H * p->W * a.n_qpairs;
    a.head_block = plan_head_block(p, a.h_valid, false,
                                   a.n_units < p->num_sms ? a.n_units : p->num_sms);
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(p->D)));
    a.wait_limit = p->wait_limit;
    a.withhold_q = p->withhold_q;
    a.o = static_cast<uint16_t *>(o);
    a.lse = lse;
    a.words = p->words;
    a.q_scale = nullptr;
    a.k_scale = nullptr;
    const bool pair = p->attn_kernel == WF_ATTN_PAIR;   // AUTO: the single-CTA kernel
    cudaError_t e;
    if (pair) {
        CUtensorMap mk64;
        if (!wf::encode_map(&mk64, k_cache, p->D, p->H, p->L, p->L, p->R, 64)) return WF_ERR_CUDA;
        e = wf::launch_attn_pair(mq, mk64, mv, a, static_cast<cudaStream_t>(stream));
    } else {
        const int grid = a.n_units < p->num_sms ? a.n_units : p->num_sms;
        e = wf::launch_attn(mq, mk, mv, a, p->D, grid, static_cast<cudaStream_t>(stream));
    }
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_quantize_q_fp8(wf_plan_t p, const void *q_out, void *q8, float *q_scale, void *stream)
{
    wf::NvtxRange nvtx_range("wf_quantize_q_fp8");
    if (p == nullptr || !q_out || !q8 || !q_scale) return WF_ERR_INVALID_ARG;
    if (!aligned16(q_out) || !aligned16(q8) || !aligned4(q_scale)) return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;
    const long rows = static_cast<long>(p->L) * p->W * p->H;
    cudaError_t e = wf::launch_quantize_rows(static_cast<const uint16_t *>(q_out),
                                             static_cast<uint8_t *>(q8), q_scale, rows, p->H, p->D,
                                             static_cast<cudaStream_t>(stream), p->words);
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_quantize_k_fp8(wf_plan_t p, long first_chunk, int n_chunks, const void *k_cache,
                      void *k8_cache, float *k_scale, void *stream)
{
    wf::NvtxRange nvtx_range("wf_quantize_k_fp8");
    if (p == nullptr || first_chunk < 0 || n_chunks < 0 || n_chunks > p->R) return WF_ERR_INVALID_ARG;
    if (!k_cache || !k8_cache || !k_scale) return WF_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(k8_cache) || !aligned4(k_scale)) return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;
    cudaError_t e = wf::launch_quantize_tiles(static_cast<const uint16_t *>(k_cache),
                                              static_cast<uint8_t *>(k8_cache), k_scale, first_chunk,
                                              n_chunks, p->L, p->H, p->R, p->D,
                                              static_cast<cudaStream_t>(stream), p->words);
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_chunk_causal_attn_fp8qk(wf_plan_t p, long round, const void *q8, const float *q_scale,
                               const void *k8_cache, const float *k_scale, const void *v_cache,
                               void *o, float *lse, void *stream)
{
    wf::NvtxRange nvtx_range("wf_chunk_causal_attn_fp8qk");
    if (p == nullptr || round < 0) return WF_ERR_INVALID_ARG;
    if (p->D != 128) return WF_ERR_UNSUPPORTED;
    if (!q8 || !q_scale || !k8_cache || !k_scale || !v_cache || !o) return WF_ERR_INVALID_ARG;
    if (!aligned16(q8) || !aligned16(k8_cache) || !aligned16(v_cache) || !aligned16(o) ||
        !aligned4(q_scale) || !aligned4(k_scale) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;

    CUtensorMap mq, mk, mv;
    if (!encode_map_u8(&mq, q8, p->D, p->H, p->L, p->W) ||
        !encode_map_u8(&mk, k8_cache, p->D, p->H, p->L, p->R) ||
        !wf::encode_map(&mv, v_cache, p->D, p->H, p->L, p->L, p->R))
        return WF_ERR_CUDA;

    wf::AttnParams a;
    a.round = round;
    a.L = p->L;
    a.W = p->W;
    a.R = p->R;
    a.H = p->H;
    a.T = p->L * p->W;
    a.h_valid = wf::history_valid(round, p->Hh);
    a.n_ktiles = (p->L + 127) / 128;
    a.n_qpairs = (a.n_ktiles + 1) / 2;
    a.n_units = p->H * p->W * a.n_qpairs;
    a.head_block = plan_head_block(p, a.h_valid, true,
                                   a.n_units < p->num_sms ? a.n_units : p->num_sms);
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(p->D)));
    a.wait_limit = p->wait_limit;
    a.withhold_q = p->withhold_q;
    a.o = static_cast<uint16_t *>(o);
    a.lse = lse;
    a.words = p->words;
    a.q_scale = q_scale;
    a.k_scale = k_scale;
    const int grid = a.n_units < p->num_sms ? a.n_units : p->num_sms;
    cudaError_t e = wf::launch_attn_fp8qk(mq, mk, mv, a, grid, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_linear(wf_plan_t p, int M, int N, int K, const void *x, const void *w, const float *bias,
              int epilogue, const float *gate, const void *resid, int rows_per_group, void *y,
              void *stream)
{
    wf::NvtxRange nvtx_range("wf_linear");
    if (p == nullptr || M < 0 || N < 32 || K < 8 || N % 32 || K % 8) return WF_ERR_INVALID_ARG;
    if (epilogue < WF_EPI_STORE || epilogue > WF_EPI_GATED_RESIDUAL) return WF_ERR_INVALID_ARG;
    if (M == 0) return WF_OK;                        // nothing to compute, nothing is read
    if (!x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y) || !aligned16(bias))
        return WF_ERR_INVALID_ARG;
    if (epilogue == WF_EPI_GATED_RESIDUAL &&
        (!gate || !resid || !aligned16(gate) || !aligned16(resid) || rows_per_group < 1))
        return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;

    wf::GemmParams g{};
    g.M = M;
    g.N = N;
    g.K = K;
    if (!gemm_tiles(M, N, g)) return WF_ERR_INVALID_ARG;
    g.bias = bias;
    g.c = static_cast<uint16_t *>(y);
    g.resid = static_cast<const uint16_t *>(resid);
    g.gate = gate;
    g.rows_per_group = rows_per_group < 1 ? 1 : rows_per_group;
    g.wait_limit = p->wait_limit;
    g.withhold = p->withhold_q;
    g.words = p->words;
    CUtensorMap ma, mb;
    if (!encode_map_2d(&ma, x, M, K) || !encode_map_2d(&mb, w, N, K)) return WF_ERR_CUDA;
    cudaError_t e = wf::launch_gemm(ma, mb, g, epilogue, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_qkv_proj_norm_rope_append(wf_plan_t p, long round, int hidden, const void *x,
                                 const void *w_qkv, const float *b_qkv, const float *gamma_q,
                                 const float *gamma_k, void *q_out, void *k_cache, void *v_cache,
                                 void *stream)
{
    wf::NvtxRange nvtx_range("wf_qkv_proj_norm_rope_append");
    if (p == nullptr || round < 0 || hidden < 8 || hidden % 8) return WF_ERR_INVALID_ARG;
    if (!x || !w_qkv || !gamma_q || !gamma_k || !q_out || !k_cache || !v_cache)
        return WF_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(b_qkv) || !aligned16(gamma_q) ||
        !aligned16(gamma_k) || !aligned16(q_out) || !aligned16(k_cache) || !aligned16(v_cache))
        return WF_ERR_INVALID_ARG;
    if (p->rope.F == 0) return WF_ERR_INVALID_ARG;            // positions come from the grid
    if ((round + p->W) > static_cast<long>(INT_MAX / p->rope.F)) return WF_ERR_INVALID_ARG;
    if ((p->H * p->D) % 128) return WF_ERR_UNSUPPORTED;      // q | k | v split on 128 columns
    const long n_tab = static_cast<long>(p->W) * p->rope.F * (p->rope.dt / 2) +
                       static_cast<long>(p->rope.gh) * (p->rope.dh / 2) +
                       static_cast<long>(p->rope.gw) * (p->rope.dw / 2);
    if (n_tab > wf::gemm_tab_max()) return WF_ERR_UNSUPPORTED;
    if (int s = check_device(p)) return s;

    const long T = static_cast<long>(p->L) * p->W;
    wf::GemmParams g{};
    g.M = static_cast<int>(T);
    g.N = 3 * p->H * p->D;
    g.K = hidden;
    if (!gemm_tiles(g.M, g.N, g)) return WF_ERR_INVALID_ARG;
    g.bias = b_qkv;
    g.q_out = static_cast<uint16_t *>(q_out);
    g.k_cache = static_cast<uint16_t *>(k_cache);
    g.v_cache = static_cast<uint16_t *>(v_cache);
    g.gamma_q = gamma_q;
    g.gamma_k = gamma_k;
    g.round = round;
    g.L = p->L;
    g.W = p->W;
    g.R = p->R;
    g.H = p->H;
    g.D = p->D;
    g.eps = static_cast<float>(p->eps);
    g.rope = p->rope;
    g.n_tab = static_cast<int>(n_tab);
    g.wait_limit = p->wait_limit;
    g.withhold = p->withhold_q;
    g.words = p->words;
    CUtensorMap ma, mb;
    if (!encode_map_2d(&ma, x, T, hidden) || !encode_map_2d(&mb, w_qkv, g.N, hidden))
        return WF_ERR_CUDA;
    cudaError_t e =
        wf::launch_gemm(ma, mb, g, wf::kEpiQkvAppend, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_layer_norm_modulate(wf_plan_t p, int M, int C, const void *x, const float *shift,
                           const float *scale, int rows_per_group, void *y, void *stream)
{
    wf::NvtxRange nvtx_range("wf_layer_norm_modulate");
    if (p == nullptr || M < 0 || C < 8 || C % 8 || rows_per_group < 1) return WF_ERR_INVALID_ARG;
    if (C > wf::ln_max_channels()) return WF_ERR_UNSUPPORTED;
    if (!x || !shift || !scale || !y || !aligned16(x) || !aligned16(shift) || !aligned16(scale) ||
        !aligned16(y))
        return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;
    cudaError_t e = wf::launch_layer_norm_modulate(
        static_cast<const uint16_t *>(x), shift, scale, static_cast<uint16_t *>(y), M, C,
        rows_per_group, 1e-6f, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_causal_conv3d(wf_plan_t p, int T, int H, int W, int Cin, int Cout, const void *x,
                     const void *x_hist, const void *w, const float *bias, const void *resid,
                     void *y, void *stream)
{
    wf::NvtxRange nvtx_range("wf_causal_conv3d");
    if (p == nullptr || T < 1 || H < 1 || W < 1 || Cin < 8 || Cin % 8 || Cout < 32 || Cout % 32)
        return WF_ERR_INVALID_ARG;
    const long long M = static_cast<long long>(T) * H * W;
    if (M >= INT_MAX || static_cast<long long>(Cin) * 27 >= INT_MAX) return WF_ERR_INVALID_ARG;
    if (!x || !w || !y || !aligned16(x) || !aligned16(x_hist) || !aligned16(w) || !aligned16(y) ||
        !aligned16(bias) || !aligned16(resid))
        return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;

    const int bn = Cout % 192 == 0 ? 192 : 256;
    wf::GemmParams g{};
    g.M = static_cast<int>(M);
    g.N = Cout;
    g.K = 27 * Cin;
    g.ct = T;
    g.ch = H;
    g.cw = W;
    g.cin = Cin;
    g.n_cblk = (Cin + 63) / 64;
    g.n_py = (H + 15) / 16;
    g.n_px = (W + 15) / 16;
    g.n_ntiles = (Cout + bn - 1) / bn;
    const long long tiles = static_cast<long long>(T) * g.n_py * g.n_px * g.n_ntiles;
    if (tiles >= INT_MAX) return WF_ERR_INVALID_ARG;
    g.n_tiles = static_cast<int>(tiles);
    g.use_hist = x_hist != nullptr ? 1 : 0;
    g.bias = bias;
    g.c = static_cast<uint16_t *>(y);
    g.resid = static_cast<const uint16_t *>(resid);
    g.rows_per_group = 1;
    g.wait_limit = p->wait_limit;
    g.withhold = p->withhold_q;
    g.words = p->words;
    CUtensorMap mx, mh, mw;
    if (!encode_map_video(&mx, x, T, H, W, Cin) ||
        !encode_map_video(&mh, x_hist != nullptr ? x_hist : x, x_hist != nullptr ? 2 : T, H, W,
                          Cin) ||
        !encode_map_convw(&mw, w, Cout, Cin, bn / 2))
        return WF_ERR_CUDA;
    cudaError_t e = wf::launch_conv(mx, mh, mw, g, resid != nullptr, bn,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_rms_norm_silu(wf_plan_t p, int M, int C, const void *x, const float *gamma, void *y,
                     void *stream)
{
    wf::NvtxRange nvtx_range("wf_rms_norm_silu");
    if (p == nullptr || M < 0 || C < 8 || C % 8) return WF_ERR_INVALID_ARG;
    if (C > wf::rms_norm_silu_max_channels()) return WF_ERR_UNSUPPORTED;
    if (!x || !gamma || !y || !aligned16(x) || !aligned16(gamma) || !aligned16(y))
        return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;
    cudaError_t e = wf::launch_rms_norm_silu(static_cast<const uint16_t *>(x), gamma,
                                             static_cast<uint16_t *>(y), M, C, 1e-6f,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

int wf_sync_status(wf_plan_t p, void *stream)
{
    if (p == nullptr) return WF_ERR_INVALID_ARG;
    if (int s = check_device(p)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    wf::DeviceWords host;
    if (cudaStreamSynchronize(st) != cudaSuccess) return WF_ERR_CUDA;
    if (cudaMemcpyAsync(&host, p->words, 2 * sizeof(uint32_t), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaMemsetAsync(p->words, 0, 2 * sizeof(uint32_t), st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return WF_ERR_CUDA;
    if (host.status & wf::kStatusTimeout) return WF_ERR_TIMEOUT;
    if (host.status & wf::kStatusBounds) return WF_ERR_BOUNDS;
    return WF_OK;
}

int wf_plan_debug_ranges(wf_plan_t p, long round, int32_t *out, int cap)
{
    if (p == nullptr || round < 0 || cap < 0 || (cap > 0 && out == nullptr)) return -1;
    const int hv = wf::history_valid(round, p->Hh);
    int n = 0;
    for (int c = 0; c < p->W; ++c)
        for (int b = 0; b <= hv + c; ++b, ++n) {
            if (n >= cap) continue;
            const long id = wf::visible_chunk_id(round, hv, b);
            out[4 * n + 0] = c;
            out[4 * n + 1] = b;
            out[4 * n + 2] = static_cast<int32_t>(id);
            out[4 * n + 3] = wf::ring_slot(id, p->R);
        }
    return n;
}

const char *wf_status_string(int s)
{
    switch (s) {
    case WF_OK: return "ok";
    case WF_ERR_INVALID_ARG: return "invalid argument";
    case WF_ERR_UNSUPPORTED: return "unsupported configuration";
    case WF_ERR_CUDA: return "CUDA error";
    case WF_ERR_TIMEOUT: return "device wait timed out";
    case WF_ERR_NO_DEVICE: return "plan has no device state";
    case WF_ERR_DEVICE: return "device is not sm_100";
    case WF_ERR_BOUNDS: return "bounds check failed (debug build)";
    default: return "unknown status";
    }
}

}  // extern "C"

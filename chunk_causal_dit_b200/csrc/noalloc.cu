// noalloc.cu -- chunk-causal attention for callers that must not allocate device memory.
//
// The plan API (wf_plan) allocates a small block of device memory for the
// attention kernel's scratch: a status word, the site of a timed-out wait and
// the counter the persistent CTAs pop work units from.  Some callers cannot do
// that: a serving loop whose device memory is owned entirely by a framework's
// caching allocator or reserved up front, where a direct cudaMalloc would break
// that accounting or stall the device (cudaMalloc and cudaFree can synchronise
// it).  wf_chunk_causal_attn_noalloc serves them: it takes the shape directly
// instead of a plan and keeps the same scratch in a block compiled into this
// library (below), so it calls no cudaMalloc, no cudaFree and no allocating
// library routine.  The caller still owns every input and output buffer.
//
// The scratch block lives on every GPU that loads the library, until the
// process exits.  All calls on a device share it and it keeps the last call's
// contents; each call clears the parts that must start at zero (status, timeout
// site, work counter) on its stream before the kernel runs, so calls whose work
// overlaps on the GPU (different streams, no ordering between them) race on it
// and must not be issued.  The kernel's timeout status is recorded in the block
// but this entry point has no way to return it: use the plan API when the
// status is needed.
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <mutex>

#include "wf.h"
#include "wf_internal.h"

namespace wf {
cudaError_t launch_attn(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                        const AttnParams &p, int D, int grid, cudaStream_t stream);
}  // namespace wf

namespace {

// Fixed scratch: the attention kernel needs one DeviceWords block whatever the
// problem size, so every shape the plan API accepts fits.
constexpr size_t kNoAllocScratchBytes = 256;
static_assert(sizeof(wf::DeviceWords) <= kNoAllocScratchBytes, "scratch block too small");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host code may not use g_noalloc_scratch as an address: on the host it names a
// shadow variable, not device memory.  The device address is fetched once per
// device, with that device current, and cached here.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

int scratch_for_current_device(int dev, void **out)
{
    if (dev < 0 || dev >= kMaxDevices) return WF_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            return WF_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return WF_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 noalloc_map_encoder()
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

// Same tensor maps as the plan API: (D, H, rows, chunk-or-slot), box 64x1x128x1,
// 128-byte swizzle, rows past the extent read as zero.
bool noalloc_map(CUtensorMap *map, const void *base, int D, int H, int L, int n3)
{
    auto enc = noalloc_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(n3)};
    const cuuint64_t row = static_cast<cuuint64_t>(H) * D * 2;
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, row,
                                   row * static_cast<cuuint64_t>(L)};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int wf_chunk_causal_attn_noalloc(int chunk_tokens, int n_wave_chunks,
                                            int n_hist_chunks, int heads, int head_dim,
                                            long round, const void *q_out, const void *k_cache,
                                            const void *v_cache, void *o, float *lse,
                                            void *stream)
{
    // the plan API's shape rules
    if (chunk_tokens < 1 || n_wave_chunks < 1 || n_hist_chunks < 0 || heads < 1 || round < 0)
        return WF_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return WF_ERR_UNSUPPORTED;
    const long long T = static_cast<long long>(chunk_tokens) * n_wave_chunks;
    const long long R = static_cast<long long>(n_hist_chunks) + n_wave_chunks;
    const long long hd = static_cast<long long>(heads) * head_dim;
    if (T * hd >= (1ll << 31) || R * chunk_tokens * hd >= (1ll << 40) || R > INT_MAX)
        return WF_ERR_INVALID_ARG;
    const int n_ktiles = (chunk_tokens + 127) / 128;
    const int n_qpairs = (n_ktiles + 1) / 2;
    if (static_cast<long long>(heads) * n_wave_chunks * n_qpairs >= INT_MAX)
        return WF_ERR_INVALID_ARG;
    if (!q_out || !k_cache || !v_cache || !o) return WF_ERR_INVALID_ARG;
    if (!aligned16(q_out) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return WF_ERR_INVALID_ARG;

    int dev = -1, sms = 0, ma = 0, mi = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&ma, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&mi, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return WF_ERR_NO_DEVICE;
    }
    if (ma != 10 || mi != 0) return WF_ERR_DEVICE;
    void *scratch = nullptr;
    if (int s = scratch_for_current_device(dev, &scratch)) return s;

    CUtensorMap mq, mk, mv;
    if (!noalloc_map(&mq, q_out, head_dim, heads, chunk_tokens, n_wave_chunks) ||
        !noalloc_map(&mk, k_cache, head_dim, heads, chunk_tokens, static_cast<int>(R)) ||
        !noalloc_map(&mv, v_cache, head_dim, heads, chunk_tokens, static_cast<int>(R)))
        return WF_ERR_CUDA;

    wf::AttnParams a;
    a.round = round;
    a.L = chunk_tokens;
    a.W = n_wave_chunks;
    a.R = static_cast<int>(R);
    a.H = heads;
    a.T = static_cast<int>(T);
    a.h_valid = wf::history_valid(round, n_hist_chunks);
    a.n_ktiles = n_ktiles;
    a.n_qpairs = n_qpairs;
    a.n_units = heads * n_wave_chunks * n_qpairs;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
    a.wait_limit = 1ull << 32;
    a.withhold_q = 0;
    a.o = static_cast<uint16_t *>(o);
    a.lse = lse;
    a.words = static_cast<wf::DeviceWords *>(scratch);
    a.q_scale = nullptr;
    a.k_scale = nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // status and timeout site start at zero for this call (the work counter is
    // cleared by the launch itself)
    if (cudaMemsetAsync(scratch, 0, 2 * sizeof(uint32_t), st) != cudaSuccess) return WF_ERR_CUDA;
    const int grid = a.n_units < sms ? a.n_units : sms;
    return wf::launch_attn(mq, mk, mv, a, head_dim, grid, st) == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

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
// and wf_noalloc_sync_status reads it back (the call itself returns before the
// kernel has run, so it cannot).
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <mutex>

#include "wf.h"
#include "wf_check.cuh"
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
// shadow variable, not device memory.  The device address is looked up with
// cudaGetSymbolAddress, with the device current, and cached per device together
// with the CUDA context it belongs to.  A context that is torn down and created
// again (cudaDeviceReset, say) loads the module afresh and the array may move,
// so a call made in another context than the cached one looks the address up
// again instead of using a stale pointer.
constexpr int kMaxDevices = 64;
struct ScratchEntry {
    CUcontext ctx;
    void *addr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch[kMaxDevices] = {};

PFN_cuCtxGetCurrent_v4000 ctx_get_current()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

int scratch_for_current_device(int dev, void **out)
{
    if (dev < 0 || dev >= kMaxDevices) return WF_ERR_UNSUPPORTED;
    auto get_ctx = ctx_get_current();
    if (get_ctx == nullptr) return WF_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return WF_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchEntry &e = g_scratch[dev];
    if (ctx == nullptr || e.addr == nullptr || e.ctx != ctx) {
        // the lookup also makes the device's primary context current when no
        // context is yet, which is why the key is read again after it
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr ||
            get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
            (void)cudaGetLastError();
            return WF_ERR_CUDA;
        }
        e.ctx = ctx;
        e.addr = p;
    }
    *out = e.addr;
    return WF_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Heads per block of the attention's unit order for the last shape seen on each
// device.  The choice plays the kernel's schedule through on the host (tens to
// hundreds of microseconds at model sizes), and a serving loop repeats one shape.
struct HeadBlockEntry {
    int H, W, h_valid, L, D, l2, grid, g;
};
std::mutex g_head_block_mu;
HeadBlockEntry g_head_block[kMaxDevices] = {};

int head_block_for(int dev, int H, int W, int h_valid, int L, int D, int l2, int grid)
{
    std::lock_guard<std::mutex> lock(g_head_block_mu);
    HeadBlockEntry &e = g_head_block[dev];
    if (e.g > 0 && e.H == H && e.W == W && e.h_valid == h_valid && e.L == L && e.D == D &&
        e.l2 == l2 && e.grid == grid)
        return e.g;
    const int g = wf::attn_head_block(H, W, h_valid, L, D, 2, l2, grid);
    e = HeadBlockEntry{H, W, h_valid, L, D, l2, grid, g};
    return g;
}

}  // namespace

extern "C" int wf_chunk_causal_attn_noalloc(int chunk_tokens, int n_wave_chunks,
                                            int n_hist_chunks, int heads, int head_dim,
                                            long round, const void *q_out, const void *k_cache,
                                            const void *v_cache, void *o, float *lse,
                                            void *stream)
{
    wf::NvtxRange nvtx_range("wf_chunk_causal_attn_noalloc");
    // the plan API's shape rules
    if (round < 0) return WF_ERR_INVALID_ARG;
    if (int st = wf::check_round_shape(chunk_tokens, n_wave_chunks, n_hist_chunks, heads, head_dim))
        return st;
    const long long T = static_cast<long long>(chunk_tokens) * n_wave_chunks;
    const long long R = static_cast<long long>(n_hist_chunks) + n_wave_chunks;
    const int n_ktiles = (chunk_tokens + 127) / 128;
    const int n_qpairs = (n_ktiles + 1) / 2;
    if (!q_out || !k_cache || !v_cache || !o) return WF_ERR_INVALID_ARG;
    if (!aligned16(q_out) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return WF_ERR_INVALID_ARG;

    int dev = -1, sms = 0, ma = 0, mi = 0, l2 = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&ma, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&mi, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return WF_ERR_NO_DEVICE;
    }
    if (ma != 10 || mi != 0) return WF_ERR_DEVICE;
    void *scratch = nullptr;
    if (int s = scratch_for_current_device(dev, &scratch)) return s;

    CUtensorMap mq, mk, mv;
    if (!wf::encode_map(&mq, q_out, head_dim, heads, chunk_tokens, chunk_tokens, n_wave_chunks) ||
        !wf::encode_map(&mk, k_cache, head_dim, heads, chunk_tokens, chunk_tokens,
                        static_cast<int>(R)) ||
        !wf::encode_map(&mv, v_cache, head_dim, heads, chunk_tokens, chunk_tokens,
                        static_cast<int>(R)))
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
    const int grid = a.n_units < sms ? a.n_units : sms;
    a.head_block = head_block_for(dev, heads, n_wave_chunks, a.h_valid, chunk_tokens, head_dim, l2,
                                  grid);
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
    return wf::launch_attn(mq, mk, mv, a, head_dim, grid, st) == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

// Test hook: every 32-bit word of the current device's scratch block set to
// `word`, as a call whose bounded wait ran out leaves the status and timeout
// site set (and a work counter past the units), so that a test can show the
// next call starts clean.  Synchronous; not for use while a call runs.
extern "C" int wf_noalloc_debug_fill_scratch(unsigned int word)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return WF_ERR_NO_DEVICE;
    }
    void *scratch = nullptr;
    if (int s = scratch_for_current_device(dev, &scratch)) return s;
    uint32_t fill[kNoAllocScratchBytes / sizeof(uint32_t)];
    for (uint32_t &w : fill) w = word;
    return cudaMemcpyToSymbol(g_noalloc_scratch, fill, sizeof(fill)) == cudaSuccess ? WF_OK
                                                                                  : WF_ERR_CUDA;
}

// The status the kernel recorded in the current device's scratch block, after
// `stream` has finished: WF_ERR_TIMEOUT when a bounded wait ran out (output
// partly written), WF_ERR_BOUNDS when a bounds check of the checked build
// failed, else WF_OK.  Reads two words into host memory; clears nothing (the
// next call does).  The block is shared by every call on the device, so the
// answer covers the calls since the last one started.
extern "C" int wf_noalloc_sync_status(void *stream)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return WF_ERR_NO_DEVICE;
    }
    void *scratch = nullptr;
    if (int s = scratch_for_current_device(dev, &scratch)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t words[2] = {0u, 0u};
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpyAsync(words, scratch, sizeof(words), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return WF_ERR_CUDA;
    if (words[0] & wf::kStatusTimeout) return WF_ERR_TIMEOUT;
    if (words[0] & wf::kStatusBounds) return WF_ERR_BOUNDS;
    return WF_OK;
}

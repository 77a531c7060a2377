// recsa_decode_noalloc: decode (select + attend) for callers that cannot allocate
// device memory at the point of the call.
//
// Who needs it: code that runs where cudaMalloc is not available or not allowed,
// for example inside a stream capture in global capture mode (where allocation calls
// are rejected), in a serving loop that works inside a fixed, pre-planned memory
// budget, or in a host runtime that owns its buffers but has no allocator for the
// per-call scratch that recsa_decode expects in its workspace.  Such a caller still
// owns its inputs and outputs (KV cache, level tables built by recsa_build, q, out);
// only the scratch moves into this library.
//
// The scratch is one file-scope device array of kScratchBytes (8 MiB) that every GPU
// which loads librecsa.so keeps until the process exits.  Its device address is taken
// once per device with cudaGetSymbolAddress (host code must not use the array's name
// as a device pointer).  All calls share it, so calls that can overlap on the GPU
// race with each other.  Each call re-initialises everything it reads before reading
// it (status word, lengths, RoPE table; selections and partials are fully written
// before use), so a call never depends on what the previous call left behind.
//
// Device-side conditions (a bounded wait that gave up, a misaligned staging buffer)
// are recorded in a status word: the caller's `status_out` when given (zeroed at the
// start of the call, then written by the kernels), else a word inside the scratch
// that nobody reads.
#include <mutex>

#include "recsa_internal.cuh"

namespace recsa {

constexpr size_t kScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

static std::mutex g_scratch_mu;
static void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device (looked up on first use).
static recsa_status scratch_on_current_device(char** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return RECSA_E_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RECSA_E_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return RECSA_E_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<char*>(g_scratch_ptr[dev]);
    return RECSA_OK;
}

}  // namespace recsa

using namespace recsa;

extern "C" RECSA_API recsa_status recsa_decode_noalloc(
    const recsa_config* cfg, int64_t capacity, int32_t batch, const void* k0, const void* v0,
    const int64_t kv_strides[3], const void* levels, size_t level_bytes, const int64_t* lengths,
    const void* q, void* out, uint32_t* status_out, void* stream) {
    if (!cfg || !lengths || !q || !out) return RECSA_E_INVAL;
    if ((((uintptr_t)q) & 15u) || (((uintptr_t)out) & 15u) || (((uintptr_t)status_out) & 3u))
        return RECSA_E_INVAL;
    size_t need = 0;
    TreeView tv;
    WorkView wv;
    recsa_status st = views_for(cfg, capacity, batch, batch, k0, v0, kv_strides, levels,
                                level_bytes, nullptr, &need, &tv, &wv);
    if (st != RECSA_OK) return st;
    if (need > kScratchBytes) return RECSA_E_CAPACITY;   // shape needs more than the fixed scratch
    for (int b = 0; b < batch; ++b)
        if (lengths[b] < 0 || lengths[b] > capacity) return RECSA_E_CAPACITY;
    {
        // a level 0 in host memory takes the staged decode of recsa_decode
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, k0) != cudaSuccess) {
            cudaGetLastError();
            return RECSA_E_INVAL;
        }
        if (a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeUnregistered)
            return RECSA_E_UNSUPPORTED;
    }
    char* scratch = nullptr;
    st = scratch_on_current_device(&scratch);
    if (st != RECSA_OK) return st;
    st = views_for(cfg, capacity, batch, batch, k0, v0, kv_strides, levels, level_bytes, scratch,
                   &need, &tv, &wv);
    if (st != RECSA_OK) return st;
    if (status_out) wv.status = status_out;   // zeroed by the workspace set-up below
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = prepare_kernels(cfg->dtype, tv.D, tv.G, wv.SPL, wv.NS0, tv.C, tv.k);
    if (e == cudaSuccess) e = launch_init_workspace(tv, wv, cfg->rope_base, s);
    if (e == cudaSuccess) e = launch_set_lengths(wv, lengths, batch, s);
    if (e == cudaSuccess) {
        QueryView qv = {};
        qv.q = q;
        qv.out = out;
        qv.mode = 0;
        qv.n_per_b = 1;
        qv.q_begin = 0;
        qv.nq = batch;
        // tensor maps of the caller's tables, encoded on the host for this call
        static thread_local KVMaps maps[kMaxLevels];
        const bool mapped = uses_kv_maps(cfg->dtype, tv.D, cfg->C) &&
                            encode_kv_maps(tv, maps) == cudaSuccess;
        e = launch_select_attend(tv, wv, qv, cfg->dtype, s, nullptr, mapped ? maps : nullptr);
    }
    return e == cudaSuccess ? RECSA_OK : RECSA_E_CUDA;
}

// Internal declarations shared by the RecSA CUDA translation units (sm_100a).
#pragma once

#include <cuda.h>   // CUtensorMap only; maps are encoded through the runtime's driver entry point
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "../../include/recsa.h"

namespace recsa {

constexpr int kMaxLevels = RECSA_MAX_LEVELS;
constexpr int kThreads = 256;        // threads per CTA of the select/attend kernels
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

// Device status word values (first error wins).
enum : uint32_t { kStatusOk = 0, kStatusBadQuery = 1, kStatusCapacity = 2, kStatusTimeout = 3,
                  kStatusLayout = 4 /* a staging buffer was misaligned */,
                  kStatusBounds = 5 /* a range check of the bounds-checked build failed */ };

// Named range around each launch for profilers (NVTX; no cost without a tool).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

// Location of the tree in device memory.
struct TreeView {
    const void* k0;            // level 0 (caller's KV cache)
    const void* v0;
    void* k0w;                 // same pointers, writable (append)
    void* v0w;
    int64_t s_b, s_h, s_t;     // level-0 element strides
    char* levels;              // level tables base
    int64_t off_k[kMaxLevels]; // byte offsets of level l tables (l >= 1)
    int64_t off_v[kMaxLevels];
    int64_t rows[kMaxLevels];  // rows per (b, h) of level l (l >= 1); rows[0] = capacity
    int B, Hkv, Hq, G, D, C, k;
    int lgC;                   // log2(C) when C is a power of two, else -1
    int n_levels;              // stored levels at capacity, level 0 included
    int64_t cap;
    float scale;
    double rope_base;
    float w[RECSA_MAX_C];      // pooler logits; kernels form softmax(w[0..m-1]) in fp64
    int l0_host;               // level 0 lives in pinned host memory: plain loads and
                               // stores only (no TMA copy or bulk prefetch touches it)
};

// Parameters of the Eq.5 gated key pooler (caller-owned fp64 device arrays).
constexpr int kGatedMaxHidden = 64;
struct GatedView {
    int h;                     // MLP hidden width, 1..kGatedMaxHidden
    double tau, g, rho;
    const double* w;           // [D]
    const double* W1t;         // [2D][h]  (W1 transposed)
    const double* b1;          // [h]
    const double* W2t;         // [h][D]   (W2 transposed)
};

// Which queries a select/attend launch handles.
struct QueryView {
    const void* q;             // [Qtot][Hq][D]
    void* out;                 // [Qtot][Hq][D]
    int32_t* sel_out;          // optional [Qtot][Hkv][NL][k]
    int32_t* cnt_out;          // optional [Qtot][Hkv][NL+1]
    int mode;                  // 0: decode (t = len-1); 1: prefill (t = pos0 + i)
    int n_per_b;               // queries per sequence (1 for decode)
    int64_t pos0;
    int q_begin;               // first global query index of this wave
    int nq;                    // queries in this wave
    // optional precomputed logits of level pre_level (tensor-core prefill path):
    // pre[((qloc * Hkv + kvh) * G + g) * pre_stride + j], already scaled; used by a
    // query only when pre_level is its first scored level.  nullptr: none.
    const float* pre;
    int pre_level;
    int pre_stride;
    // decode only: the level-0 launch also re-pools the ancestors of each sequence's
    // newest token (extra CTAs after the attention CTAs)
    int walk;
    // decode with level 0 in host memory, in two launches around a gather:
    //   phase 1: levels >= 1 only (no level 0, no merge);
    //   phase 2: level 0 only, read from the staging copy l0k/l0v [nq][Hkv][C*k][D]
    //            in list order (entry j at row j), then the merge;
    //   phase 0: every level and the merge (level 0 read where it lives).
    int phase;
    const void* l0k;
    const void* l0v;
    // decode only, fused with a one-token append (non-null: [B][Hkv][D] each): the
    // token goes to position t = the current length, the walk CTAs write its rows at
    // level 0 and re-pool its ancestors, the attention CTAs take its rows from here,
    // and the last CTA of each sequence advances the length
    const void* knew;
    const void* vnew;
};

// TMA tensor maps of one level's K and V tables (bf16, d = 128): 4-d (d, row, KV
// head, sequence), box 64 dims x C rows, 128-byte swizzle.  A parent group is staged
// as two boxes (dims 0-63, 64-127) into [half][C rows][128 B] of a 1024-byte-aligned
// slot, so 8 consecutive rows fall in 8 different swizzle phases.
struct KVMaps {
    CUtensorMap k, v;
};

// Buffers of the tensor-core prefill path (inside the workspace when enabled).
struct TcView {
    uint32_t* a_hi;            // [Hkv][MB][D/32] slice images of 128 rows x 128 B
    uint32_t* a_lo;
    uint32_t* b_hi;            // [Hkv][NB][D/32] slice images of 256 rows x 128 B
    uint32_t* b_lo;
    float* logits;             // [nsub][Hkv][G][npad]
    int nsub;                  // queries per product
    int npad;                  // logits row length (multiple of 256, >= C*k)
    int MB, NB;                // M tiles (of 128 rows) and N tiles (of 256 nodes) per head
};

// Workspace carve-up.
struct WorkView {
    uint32_t* status;
    int64_t* lens;             // [B] device-side lengths
    uint32_t* done;            // [B] completion counters (append)
    const float2* rope;        // [C*k][D/2] (cos, sin)
    const double* alpha;       // [C][C]: alpha[(m-1)*C + c] = softmax(w[0..m-1])_c
    int32_t* sel;              // [Qmax][Hkv][NL][k]
    int32_t* cnt;              // [Qmax][Hkv][NL+1]
    float* part;               // [Qmax][Hkv][NSLOT][G][D+2]
    uint32_t* ucnt;            // [Qmax*Hkv] level-0 CTAs finished per unit (reset to 0)
    int nunits;                // Qmax*Hkv
    int NL, SPL, NS0, NSLOT;
    int ck;                    // C*k: rows of the RoPE table
};

// ----------------------------------------------------------------------------
// small device helpers
// ----------------------------------------------------------------------------

__device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ void set_status(uint32_t* st, uint32_t code) {
    atomicCAS(st, 0u, code);
}

// Range checks of the bounds-checked build (-DRECSA_DEBUG_BOUNDS): a row or rank index
// about to be used for a gather or a store.  A failed check records kStatusBounds (the
// caller then falls back to an index that is in range); without the flag the check
// compiles to true.
#ifdef RECSA_DEBUG_BOUNDS
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t* st) {
    if (!ok) set_status(st, kStatusBounds);
    return ok;
}
#else
__device__ __forceinline__ bool in_bounds(bool, uint32_t*) { return true; }
#endif

template <typename T> struct VecOf;
template <> struct VecOf<float> { static constexpr int N = 4; };
template <> struct VecOf<__nv_bfloat16> { static constexpr int N = 8; };

// Load 16 bytes (VecOf<T>::N elements) and widen to fp32.
template <typename T>
__device__ __forceinline__ void load16(const T* p, float* out);

template <>
__device__ __forceinline__ void load16<float>(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16* p, float* out) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(w[i] << 16);
        out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Read-only path (data not written by the running kernel).
template <typename T>
__device__ __forceinline__ void load16_nc(const T* p, float* out);
template <>
__device__ __forceinline__ void load16_nc<float>(const float* p, float* out) {
    float4 v = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
template <>
__device__ __forceinline__ void load16_nc<__nv_bfloat16>(const __nv_bfloat16* p, float* out) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(w[i] << 16);
        out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// fp64 -> storage rounding (round to nearest, ties to even), single rounding.
__device__ __forceinline__ float round_store_f32(double x) { return __double2float_rn(x); }

// fp64 -> bf16 with one correct rounding: round to odd at fp32 (24 bits, at least
// two more than bf16's 8) and then to nearest even at bf16.  Rounding to odd first
// makes the second rounding equal to a direct rounding of x (Boldo & Melquiond,
// "Emulation of FMA and correctly rounded sums: proved algorithms using rounding
// to odd", IEEE TC 2008).
__device__ __forceinline__ __nv_bfloat16 round_store_bf16(double x) {
    float f = __double2float_rz(x);
    if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
    return __float2bfloat16_rn(f);
}

template <typename T> __device__ __forceinline__ T store_round(double x);
template <> __device__ __forceinline__ float store_round<float>(double x) { return round_store_f32(x); }
template <> __device__ __forceinline__ __nv_bfloat16 store_round<__nv_bfloat16>(double x) {
    return round_store_bf16(x);
}
template <typename T> __device__ __forceinline__ T store_round_f(float x);
template <> __device__ __forceinline__ float store_round_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 store_round_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Row pointers.
template <typename T>
__device__ __forceinline__ const T* level0_row(const TreeView& tv, int b, int h, int64_t t) {
    return reinterpret_cast<const T*>(tv.k0) + (b * tv.s_b + h * tv.s_h + t * tv.s_t);
}
template <typename T>
__device__ __forceinline__ const T* level0_vrow(const TreeView& tv, int b, int h, int64_t t) {
    return reinterpret_cast<const T*>(tv.v0) + (b * tv.s_b + h * tv.s_h + t * tv.s_t);
}
template <typename T>
__device__ __forceinline__ T* level_k(const TreeView& tv, int l, int b, int h) {
    return reinterpret_cast<T*>(tv.levels + tv.off_k[l]) + ((int64_t)(b * tv.Hkv + h) * tv.rows[l]) * tv.D;
}
template <typename T>
__device__ __forceinline__ T* level_v(const TreeView& tv, int l, int b, int h) {
    return reinterpret_cast<T*>(tv.levels + tv.off_v[l]) + ((int64_t)(b * tv.Hkv + h) * tv.rows[l]) * tv.D;
}

// Query position of a (wave-local) query; returns false if it has nothing to do.
__device__ __forceinline__ bool query_pos(const QueryView& qv, const WorkView& wv, int qloc,
                                          int& b, int64_t& t, int& gq) {
    gq = qv.q_begin + qloc;
    b = gq / qv.n_per_b;
    int i = gq - b * qv.n_per_b;
    int64_t len = wv.lens[b];
    t = (qv.mode == 0) ? len - 1 : qv.pos0 + i;
    return t >= 0 && t < len;
}

// Division by the branching factor: a shift when C is a power of two.
__device__ __forceinline__ int64_t cdiv64(int64_t x, int C, int lgC) { return lgC >= 0 ? (x >> lgC) : x / C; }
__device__ __forceinline__ int cdiv(int x, int C, int lgC) { return lgC >= 0 ? (x >> lgC) : x / C; }
__device__ __forceinline__ int cmod(int x, int C, int lgC) { return lgC >= 0 ? (x & (C - 1)) : x % C; }

// a^(l) = floor(t / C^l).
__device__ __forceinline__ int64_t apow(int64_t t, int l, int C, int lgC) {
    if (lgC >= 0) {
        const int sh = l * lgC;
        return sh >= 63 ? 0 : (t >> sh);
    }
    for (int i = 0; i < l && t > 0; ++i) t /= C;
    return t;
}

// The first scored level l* of a query at position t (0 if none): the highest
// l >= 1 whose full list [0..a^(l)] has more than k entries.  Every level above it
// selects its whole list, so A^(l*) = [0..a^(l*)].
__device__ __forceinline__ int first_scored_level(int64_t t, int C, int lgC, int k) {
    int lstar = 0, l = 0;
    int64_t p = t;
    while (p > 0 && l + 1 < kMaxLevels) {
        p = cdiv64(p, C, lgC);
        ++l;
        if (p >= k) lstar = l;
    }
    return lstar;
}

// |A^(level)| for a query whose first scored level is lstar >= level (Eq.3 sizes:
// each list below l* holds the C children of the min(k, |A|) - 1 selected
// non-current nodes plus the current node's children clamped at a^(l-1)).
__device__ __forceinline__ int list_size(int64_t t, int lstar, int level, int C, int lgC, int k) {
    if (lstar == 0) return (int)(t + 1);
    int64_t al = apow(t, lstar, C, lgC);
    int nA = (int)(al + 1);
    for (int l = lstar; l > level; --l) {
        const int64_t alm1 = apow(t, l - 1, C, lgC);
        const int nS = nA < k ? nA : k;
        nA = C * (nS - 1) + (int)(alm1 - (int64_t)C * al + 1);
        al = alm1;
    }
    return nA;
}

__device__ __forceinline__ uint32_t ordered_key(float x) {
    if (x == 0.0f) x = 0.0f;   // +0 and -0 compare equal: one key
    uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Optional events recorded around one kernel (see recsa_set_profile_events).
struct ProfHook {
    int which = -100;
    cudaEvent_t start = nullptr, stop = nullptr;
};

inline void prof_mark(const ProfHook* p, int which, bool before, cudaStream_t s) {
    if (p == nullptr || p->which != which || p->start == nullptr) return;
    // inside a stream capture the record becomes an external event node of the graph
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cs);
    cudaEvent_t ev = before ? p->start : p->stop;
    if (cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, s);
}

// ----------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel on the stream is finishing.
// It must pass pdl_wait() before it reads or writes any global memory that kernel
// touches; pdl_wait() returns once that kernel has completed and its writes are
// visible.  pdl_launch_dependents() lets the next kernel start launching.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Launch attribute that allows the overlap above.
inline cudaLaunchAttribute pdl_attribute() {
    cudaLaunchAttribute a = {};
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

// ----------------------------------------------------------------------------
// TMA bulk copies into shared memory, completed on an mbarrier (no multicast)
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
// One wait on a phase of an mbarrier: the thread is suspended in hardware until the
// phase completes or about `hint_ns` nanoseconds pass (no issue slots are spent
// spinning).  Returns whether the phase completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}
// Bounded wait for a phase of an mbarrier: gives up after `polls` suspended waits
// of up to kWaitHintNs each (kWaitPolls: about one second in total), records
// kStatusTimeout and returns false.  Never waits forever.  After one wait of a CTA
// has given up, its later waits use kWaitPollsAfterFail (about 2 ms): long enough
// for copies that are merely late to land before the CTA exits, short enough that
// a unit whose copies never complete returns soon.
constexpr uint32_t kWaitHintNs = 20000;
constexpr uint32_t kWaitPolls = 50000;
constexpr uint32_t kWaitPollsAfterFail = 100;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t* status,
                                                  uint32_t polls = kWaitPolls) {
    for (uint32_t i = 0; i < polls; ++i)
        if (mbar_try_wait(bar, parity, kWaitHintNs)) return true;
    atomicCAS(status, 0u, 3u);
    return false;
}

// ----------------------------------------------------------------------------
// launchers (defined in the .cu files)
// ----------------------------------------------------------------------------
cudaError_t launch_init_workspace(const TreeView& tv, const WorkView& wv, double rope_base,
                                  cudaStream_t s);
cudaError_t launch_build(const TreeView& tv, const WorkView& wv, const int64_t* lengths,
                         int dtype, cudaStream_t s);
cudaError_t launch_append_token(const TreeView& tv, const WorkView& wv, const void* k_new,
                                const void* v_new, int dtype, cudaStream_t s,
                                const ProfHook* prof = nullptr);
cudaError_t launch_append_walk(const TreeView& tv, const WorkView& wv, int dtype, cudaStream_t s);
cudaError_t launch_append(const TreeView& tv, const WorkView& wv, const void* k_new,
                          const void* v_new, int n, int dtype, cudaStream_t s,
                          const ProfHook* prof = nullptr);
cudaError_t launch_prefill_top_tc(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                  const TcView& tc, int lt, int64_t a_max, int dtype, cudaStream_t s,
                                  const ProfHook* prof = nullptr);
cudaError_t prepare_tc_kernels(int D);
cudaError_t launch_select_attend(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                 int dtype, cudaStream_t s, const ProfHook* prof = nullptr,
                                 const KVMaps* maps = nullptr);
// Whether a tree stages its rows through swizzled tensor maps: bf16, d = 128, and
// parent groups of a multiple of 16 rows (whole tensor-core steps).
inline bool uses_kv_maps(int dtype, int D, int C) {
    return dtype == RECSA_BF16 && D == 128 && C % 16 == 0 && C <= 256;
}
// Encodes maps[l] for levels 0 .. tv.n_levels - 1 (level 0: the caller's cache).
cudaError_t encode_kv_maps(const TreeView& tv, KVMaps* maps);
cudaError_t prepare_tree_kernels(const TreeView& tv, int dtype);
cudaError_t launch_set_lengths(const WorkView& wv, const int64_t* lengths, int B, cudaStream_t s);
// The level-0 list of every decode query, copied in list order from the level-0 cache
// (host memory) into the staging buffer [nq][Hkv][C*k][D] (K and V), after a phase-1
// pass has selected level 1 (offload.cu).
cudaError_t launch_gather_level0(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                 void* stage_k, void* stage_v, int dtype, cudaStream_t s);
// Eq.5 levels 1.. with the gated key pooler: every node (add == 0) or the nodes
// covering the `add` tokens appended at the device-side lengths (gated.cu).
cudaError_t launch_gated_levels(const TreeView& tv, const WorkView& wv, const GatedView& gv,
                                int64_t add, int dtype, cudaStream_t s);
// The single-token and multi-token append helpers of tree_kernels.cu.
cudaError_t launch_append_rows(const TreeView& tv, const WorkView& wv, const void* k_new,
                               const void* v_new, int n, int dtype, cudaStream_t s);
cudaError_t launch_commit_lengths(const WorkView& wv, int B, int64_t add, int64_t cap,
                                  cudaStream_t s);
recsa_status views_for(const recsa_config* cfg, int64_t cap, int B, int Qmax, const void* k0,
                       const void* v0, const int64_t strides[3], const void* levels,
                       size_t level_bytes, char* ws, size_t* ws_bytes, TreeView* tv,
                       WorkView* wv);
cudaError_t prepare_kernels(int dtype, int D, int G, int SPL, int NS0, int C, int k);

}  // namespace recsa

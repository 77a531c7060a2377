// Tree construction (Eq.1 of "Recursive Sparse Attention", section "Tree
// Construction") and incremental append, sm_100a.
//
// A level-l node i pools its children C*i .. min(C*i+C-1, n_{l-1}-1) of level l-1:
//   K = sum_c alpha_c K_c, alpha = softmax(w) over the m present children (stand-in
//       pooler shared by all levels and heads),
//   V = (1/m) sum_c V_c.
// Sums run in fp64, one lane per dimension in child order (fused multiply-add for
// K), and are rounded once to the storage dtype; the next level pools the rounded
// values.  Build and append perform the same operations in the same order, so an
// appended tree is bitwise equal to a rebuilt one.
#include "pool.cuh"

namespace recsa {

__device__ __forceinline__ int64_t ceil_div_pow(int64_t n, int C, int l) {
    for (int i = 0; i < l; ++i) n = (n + C - 1) / C;
    return n;
}

// ----------------------------------------------------------------------------
// workspace initialisation: status, lengths, RoPE table
// ----------------------------------------------------------------------------
__global__ void init_workspace_kernel(WorkView wv, TreeView tv, int B, int D, double base) {
    const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (gid == 0) *wv.status = 0u;
    if (gid < B) { wv.lens[gid] = 0; wv.done[gid] = 0u; }
    if (blockIdx.x == 0) fill_alpha(tv.w, tv.C, const_cast<double*>(wv.alpha));
    for (int64_t i = gid; i < wv.nunits; i += (int64_t)gridDim.x * blockDim.x) wv.ucnt[i] = 0u;
    const int half = D / 2;
    const int64_t total = (int64_t)wv.ck * half;
    for (int64_t i = gid; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int p = (int)(i / half), j = (int)(i % half);
        const double theta = pow(base, -2.0 * (double)j / (double)D);
        const double ang = (double)p * theta;
        float2 cs;
        cs.x = (float)cos(ang);
        cs.y = (float)sin(ang);
        const_cast<float2*>(wv.rope)[i] = cs;
    }
}

cudaError_t launch_init_workspace(const TreeView& tv, const WorkView& wv, double rope_base,
                                  cudaStream_t s) {
    const int64_t total = (int64_t)wv.ck * (tv.D / 2);
    int blocks = (int)((total + 255) / 256);
    if (blocks < 1) blocks = 1;
    if (blocks > 4096) blocks = 4096;
    init_workspace_kernel<<<blocks, 256, 0, s>>>(wv, tv, tv.B, tv.D, rope_base);
    return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// build passes: levels s+1 and s+2 from level s, over the nodes that cover a token
// range.  add == 0: full rebuild of [0, len); add > 0: the tokens [len, len+add)
// that an append has just written (len is the old length).
// ----------------------------------------------------------------------------
struct Lengths64 { int64_t v[RECSA_MAX_BATCH]; };

__global__ void set_lengths_kernel(WorkView wv, Lengths64 L, int B) {
    const int b = threadIdx.x;
    if (b < B) wv.lens[b] = L.v[b];
    if (b == 0) __threadfence();
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 2) build_pass_kernel(TreeView tv, WorkView wv, int s, int64_t add) {
    __shared__ double alpha[RECSA_MAX_C * RECSA_MAX_C];
    for (int i = threadIdx.x; i < tv.C * tv.C; i += blockDim.x) alpha[i] = wv.alpha[i];
    __syncthreads();

    const int bh = blockIdx.y;
    const int b = bh / tv.Hkv, h = bh % tv.Hkv;
    const int C = tv.C;
    const int64_t len_old = wv.lens[b];
    const int64_t L_new = len_old + add;
    if (L_new > tv.cap || L_new <= 0) return;
    const int64_t lo = (add == 0) ? 0 : len_old;
    const int64_t hi = L_new;
    const int64_t n_s = ceil_div_pow(L_new, C, s);
    if (n_s <= 1) return;                         // level s is already the root
    const int64_t n_s1 = (n_s + C - 1) / C;
    const bool has_s2 = n_s1 > 1;
    // level-(s+2) node range covering tokens [lo, hi)
    int64_t span2 = 1;
    for (int i = 0; i < s + 2; ++i) span2 *= C;
    const int64_t p_lo = lo / span2, p_hi = (hi - 1) / span2;
    const int warp = threadIdx.x >> 5;
    const int64_t p2 = p_lo + (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
    if (p2 > p_hi) return;

    const T *sk, *sv;
    int64_t rs;
    level_rows<T>(tv, s, b, h, sk, sv, rs);
    T* k1 = level_k<T>(tv, s + 1, b, h);
    T* v1 = level_v<T>(tv, s + 1, b, h);
    const int lane = threadIdx.x & 31;
    constexpr uint32_t kRow = D * sizeof(T);
    for (int c1 = 0; c1 < C; ++c1) {
        const int64_t i1 = p2 * C + c1;
        if (i1 >= n_s1) break;
        const int m = (int)imin64(C, n_s - i1 * C);
        // rows of the parent two steps ahead go to L2 while this one is pooled
        const int64_t ia = i1 + 2;
        if (lane == 0 && c1 + 2 < C && ia < n_s1 && !(s == 0 && tv.l0_host)) {
            const int ma = (int)imin64(C, n_s - ia * C);
            if (rs == D) {
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(sk + ia * C * rs),
                             "r"(ma * kRow) : "memory");
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(sv + ia * C * rs),
                             "r"(ma * kRow) : "memory");
            }
        }
        warp_pool_node<T, D>(sk + i1 * C * rs, sv + i1 * C * rs, rs, m, alpha + (m - 1) * C,
                             k1 + i1 * D, v1 + i1 * D);
    }
    if (has_s2) {
        __syncwarp();
        T* k2 = level_k<T>(tv, s + 2, b, h);
        T* v2 = level_v<T>(tv, s + 2, b, h);
        const int m = (int)imin64(C, n_s1 - p2 * C);
        warp_pool_node<T, D>(k1 + p2 * C * D, v1 + p2 * C * D, D, m, alpha + (m - 1) * C,
                             k2 + p2 * D, v2 + p2 * D);
    }
}

// Copy n appended rows per (b, h) into level 0 at the current length.
template <typename T, int D>
__global__ void append_rows_kernel(TreeView tv, WorkView wv, const T* knew, const T* vnew, int n) {
    const int bh = blockIdx.y;
    const int b = bh / tv.Hkv, h = bh % tv.Hkv;
    const int64_t L = wv.lens[b];
    if (L + n > tv.cap) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && h == 0) set_status(wv.status, kStatusCapacity);
        return;
    }
    constexpr int VEC = VecOf<T>::N;
    constexpr int PER_ROW = D / VEC;
    const int64_t total = (int64_t)n * PER_ROW;
    T* k0 = reinterpret_cast<T*>(tv.k0w) + (b * tv.s_b + h * tv.s_h);
    T* v0 = reinterpret_cast<T*>(tv.v0w) + (b * tv.s_b + h * tv.s_h);
    const T* ks = knew + (int64_t)bh * n * D;
    const T* vs = vnew + (int64_t)bh * n * D;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / PER_ROW, c = i % PER_ROW;
        *reinterpret_cast<uint4*>(k0 + (L + r) * tv.s_t + c * VEC) =
            *reinterpret_cast<const uint4*>(ks + r * D + c * VEC);
        *reinterpret_cast<uint4*>(v0 + (L + r) * tv.s_t + c * VEC) =
            *reinterpret_cast<const uint4*>(vs + r * D + c * VEC);
    }
}

__global__ void commit_lengths_kernel(WorkView wv, int B, int64_t add, int64_t cap) {
    const int b = threadIdx.x;
    if (b < B && wv.lens[b] + add <= cap) wv.lens[b] += add;
}

// ----------------------------------------------------------------------------
// single-token append, split in two:
//   append_token_kernel writes token t = L of every (sequence, KV head) at level 0
//     and advances the length (the last CTA of a sequence does);
//   the ancestors of t are re-pooled by ancestor_walk, either in extra CTAs of the
//     next decode's level-0 kernel or by append_walk_kernel.  A decode at t reads no
//     ancestor of t: each is the current node of its level, never scored and never
//     a summary, and every other node it lists is complete.
// ----------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(64) append_token_kernel(TreeView tv, WorkView wv, const T* knew,
                                                          const T* vnew) {
    constexpr int VEC = VecOf<T>::N;
    const int bh = blockIdx.x;
    const int b = bh / tv.Hkv, h = bh % tv.Hkv;
    pdl_wait();
    const int64_t t = wv.lens[b];
    if (t + 1 > tv.cap) {
        if (h == 0 && threadIdx.x == 0) set_status(wv.status, kStatusCapacity);
        return;
    }
    T* k0 = reinterpret_cast<T*>(tv.k0w) + (b * tv.s_b + h * tv.s_h + t * tv.s_t);
    T* v0 = reinterpret_cast<T*>(tv.v0w) + (b * tv.s_b + h * tv.s_h + t * tv.s_t);
    const T* kn = knew + (int64_t)bh * D;
    const T* vn = vnew + (int64_t)bh * D;
    for (int e = threadIdx.x; e < D / VEC; e += blockDim.x) {
        *reinterpret_cast<uint4*>(k0 + e * VEC) = *reinterpret_cast<const uint4*>(kn + e * VEC);
        *reinterpret_cast<uint4*>(v0 + e * VEC) = *reinterpret_cast<const uint4*>(vn + e * VEC);
    }
    // every CTA of sequence b has read lens[b] before it counts itself here
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&wv.done[b], 1u) == (unsigned)tv.Hkv - 1) {
            wv.done[b] = 0u;
            wv.lens[b] = t + 1;
        }
    }
}

// The ancestors of each sequence's newest token t = L - 1, one CTA per (sequence,
// KV head).
template <typename T, int D>
__global__ void __launch_bounds__(256) append_walk_kernel(TreeView tv, WorkView wv) {
    extern __shared__ double walk_smem[];
    double* alpha = walk_smem;
    double* pre = walk_smem + RECSA_MAX_C * RECSA_MAX_C;
    const int b = blockIdx.x / tv.Hkv, h = blockIdx.x % tv.Hkv;
    pdl_wait();
    for (int i = threadIdx.x; i < tv.C * tv.C; i += blockDim.x) alpha[i] = wv.alpha[i];
    const int64_t t = wv.lens[b] - 1;
    __syncthreads();
    if (t < 1) return;
    ancestor_walk<T, D>(tv, b, h, t, pre, alpha, wv.status);
}

// Waits on an mbarrier that nothing arrives on, through the bounded wait of every
// kernel here: the wait gives up, records the timeout in *status and returns.
__global__ void bounded_wait_probe_kernel(uint32_t* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) mbar_init(&bar, 1);
    mbar_fence_init();
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0u, status);
}

cudaError_t launch_bounded_wait_probe(uint32_t* status, cudaStream_t s) {
    bounded_wait_probe_kernel<<<1, 32, 0, s>>>(status);
    return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// host launchers
// ----------------------------------------------------------------------------
template <typename T, int D>
static cudaError_t run_passes(const TreeView& tv, const WorkView& wv, int64_t add, cudaStream_t s) {
    NvtxRange nv(add == 0 ? "recsa build" : "recsa append levels");
    for (int src = 0; src + 1 < tv.n_levels; src += 2) {
        int64_t span2 = 1;
        for (int i = 0; i < src + 2; ++i) span2 *= tv.C;
        const int64_t tokens = (add == 0) ? tv.cap : add;
        const int64_t nodes = (tokens + span2 - 1) / span2 + 1;
        const int64_t blocks = (nodes + 7) / 8;
        dim3 grid((unsigned)blocks, (unsigned)(tv.B * tv.Hkv));
        build_pass_kernel<T, D><<<grid, 256, 0, s>>>(tv, wv, src, add);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename T, int D>
static cudaError_t build_impl(const TreeView& tv, const WorkView& wv, const int64_t* lengths,
                              cudaStream_t s) {
    Lengths64 L{};
    for (int b = 0; b < tv.B; ++b) L.v[b] = lengths[b];
    set_lengths_kernel<<<1, RECSA_MAX_BATCH, 0, s>>>(wv, L, tv.B);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return run_passes<T, D>(tv, wv, 0, s);
}


template <typename T, int D>
static cudaError_t append_impl(const TreeView& tv, const WorkView& wv, const void* k_new,
                               const void* v_new, int n, cudaStream_t s, const ProfHook* prof) {
    const int per_row = D / VecOf<T>::N;
    int64_t blocks = ((int64_t)n * per_row + 255) / 256;
    if (blocks > 1024) blocks = 1024;
    prof_mark(prof, -1, true, s);
    append_rows_kernel<T, D><<<dim3((unsigned)blocks, tv.B * tv.Hkv), 256, 0, s>>>(
        tv, wv, reinterpret_cast<const T*>(k_new), reinterpret_cast<const T*>(v_new), n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = run_passes<T, D>(tv, wv, n, s);
    if (e != cudaSuccess) return e;
    commit_lengths_kernel<<<1, RECSA_MAX_BATCH, 0, s>>>(wv, tv.B, n, tv.cap);
    prof_mark(prof, -1, false, s);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t append_token_impl(const TreeView& tv, const WorkView& wv, const void* k_new,
                                     const void* v_new, cudaStream_t s, const ProfHook* prof) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tv.B * tv.Hkv), 1, 1);
    cfg.blockDim = dim3(64, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1] = {pdl_attribute()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    NvtxRange nv("recsa append token");
    prof_mark(prof, -1, true, s);
    cudaError_t e = cudaLaunchKernelEx(&cfg, append_token_kernel<T, D>, tv, wv,
                                       reinterpret_cast<const T*>(k_new),
                                       reinterpret_cast<const T*>(v_new));
    prof_mark(prof, -1, false, s);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t append_walk_impl(const TreeView& tv, const WorkView& wv, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tv.B * tv.Hkv), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = ancestor_walk_smem(tv.n_levels, D);
    cfg.stream = s;
    cudaLaunchAttribute attr[1] = {pdl_attribute()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    NvtxRange nv("recsa ancestor walk");
    cudaError_t e = cudaLaunchKernelEx(&cfg, append_walk_kernel<T, D>, tv, wv);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

#define RECSA_DISPATCH_TD(dtype, D, FN, ...)                                              \
    do {                                                                                  \
        if ((dtype) == RECSA_BF16 && (D) == 128) return FN<__nv_bfloat16, 128>(__VA_ARGS__); \
        if ((dtype) == RECSA_BF16 && (D) == 64) return FN<__nv_bfloat16, 64>(__VA_ARGS__);   \
        if ((dtype) == RECSA_F32 && (D) == 128) return FN<float, 128>(__VA_ARGS__);          \
        if ((dtype) == RECSA_F32 && (D) == 64) return FN<float, 64>(__VA_ARGS__);            \
        return cudaErrorInvalidValue;                                                     \
    } while (0)

template <typename T, int D>
static cudaError_t prepare_tree_impl(const TreeView&) {
    return cudaFuncSetAttribute(append_walk_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)ancestor_walk_smem(kMaxLevels, D));
}

cudaError_t prepare_tree_kernels(const TreeView& tv, int dtype) {
    RECSA_DISPATCH_TD(dtype, tv.D, prepare_tree_impl, tv);
}

cudaError_t launch_set_lengths(const WorkView& wv, const int64_t* lengths, int B, cudaStream_t s) {
    Lengths64 L{};
    for (int b = 0; b < B; ++b) L.v[b] = lengths[b];
    set_lengths_kernel<<<1, RECSA_MAX_BATCH, 0, s>>>(wv, L, B);
    return cudaGetLastError();
}

cudaError_t launch_build(const TreeView& tv, const WorkView& wv, const int64_t* lengths,
                         int dtype, cudaStream_t s) {
    RECSA_DISPATCH_TD(dtype, tv.D, build_impl, tv, wv, lengths, s);
}

cudaError_t launch_append_token(const TreeView& tv, const WorkView& wv, const void* k_new,
                                const void* v_new, int dtype, cudaStream_t s, const ProfHook* prof) {
    RECSA_DISPATCH_TD(dtype, tv.D, append_token_impl, tv, wv, k_new, v_new, s, prof);
}

cudaError_t launch_append_walk(const TreeView& tv, const WorkView& wv, int dtype, cudaStream_t s) {
    RECSA_DISPATCH_TD(dtype, tv.D, append_walk_impl, tv, wv, s);
}

template <typename T, int D>
static cudaError_t append_rows_impl(const TreeView& tv, const WorkView& wv, const void* k_new,
                                   const void* v_new, int n, cudaStream_t s) {
    const int per_row = D / VecOf<T>::N;
    int64_t blocks = ((int64_t)n * per_row + 255) / 256;
    if (blocks > 1024) blocks = 1024;
    append_rows_kernel<T, D><<<dim3((unsigned)blocks, tv.B * tv.Hkv), 256, 0, s>>>(
        tv, wv, reinterpret_cast<const T*>(k_new), reinterpret_cast<const T*>(v_new), n);
    return cudaGetLastError();
}

cudaError_t launch_append_rows(const TreeView& tv, const WorkView& wv, const void* k_new,
                               const void* v_new, int n, int dtype, cudaStream_t s) {
    RECSA_DISPATCH_TD(dtype, tv.D, append_rows_impl, tv, wv, k_new, v_new, n, s);
}

cudaError_t launch_commit_lengths(const WorkView& wv, int B, int64_t add, int64_t cap,
                                  cudaStream_t s) {
    commit_lengths_kernel<<<1, RECSA_MAX_BATCH, 0, s>>>(wv, B, add, cap);
    return cudaGetLastError();
}

cudaError_t launch_append(const TreeView& tv, const WorkView& wv, const void* k_new,
                          const void* v_new, int n, int dtype, cudaStream_t s,
                          const ProfHook* prof) {
    RECSA_DISPATCH_TD(dtype, tv.D, append_impl, tv, wv, k_new, v_new, n, s, prof);
}

}  // namespace recsa

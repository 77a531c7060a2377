// Eq.5 of "Recursive Sparse Attention" (section "Pooler Distillation"): the gated key
// pooler, forward only, as an alternative to the stand-in pooler of Eq.1 ("Tree
// Construction").  For a node with present children x_1..x_m (stored keys of the
// level below):
//   mu    = mean_c x_c                                       (a vector)
//   sigma = sqrt(mean over children and dims of (x - mu)^2 + 1e-6)   (a scalar)
//   alpha = softmax_c(tau * w . (x_c - mu) / sigma)
//   p     = sum_c alpha_c x_c
//   m     = W2 SiLU(W1 [mu / rho ; (p - mu) / sigma] + b1)
//   K     = mu + g (p - mu) + sigma m
// The node's value stays Eq.1's mean of the children's values.  The readings of the
// quantities the pages leave open (sigma a scalar spread, g/tau/rho scalars, an MLP
// of hidden width h without output bias) are the ones the oracle states.
//
// Every node is pooled by one warp running gated_pool_node, in fp64 with a fixed
// order of operations, whether it comes from a full build or from an append: build
// and append give bit-identical trees.  The weights are staged in shared memory once
// per CTA (fp64; hidden width h <= kGatedMaxHidden so that W1 and W2 fit).
#include "pool.cuh"

namespace recsa {

// Shared memory of a CTA of `warps` warps: w [D], W1t [2D][h], b1 [h], W2t [h][D],
// then per warp z [2D], mu [D], pm [D], hid [h], alpha [C].
inline size_t gated_smem(int D, int h, int warps) {
    const size_t weights = (size_t)D + 2 * (size_t)D * h + h + (size_t)h * D;
    const size_t per_warp = 4 * (size_t)D + h + RECSA_MAX_C;
    return sizeof(double) * (weights + warps * per_warp);
}
// Warps per CTA: as many of 16, 8 or 4 as fit beside the weights (a node's chains
// of dependent fp64 FMAs on shared-memory operands leave each warp mostly waiting,
// so residency is what hides the latency).
inline int gated_warps(int D, int h) {
    return gated_smem(D, h, 16) <= 227 * 1024 ? 16 : gated_smem(D, h, 8) <= 227 * 1024 ? 8 : 4;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ double warp_max_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

// Element e of the lane's N consecutive dims of a row, widened exactly to fp64.
template <typename T, int N>
__device__ __forceinline__ void load_dims(const T* row, int off, double (&x)[N]) {
    float f[N];
    Dims<T, N>::load(row + off, f);
#pragma unroll
    for (int e = 0; e < N; ++e) x[e] = (double)f[e];
}

// One node: children rows sk/sv + c*rs (c < m) -> the node's K and V rounded to the
// storage dtype at dk/dv.  All lanes of the warp take part.  Lane l reads dims
// [l*N, l*N + N) of the children; the MLP's output dims are l + 32*e.
template <typename T, int D>
__device__ void gated_pool_node(const T* sk, const T* sv, int64_t rs, int m, const GatedView& gv,
                                const double* w, const double* W1t, const double* b1,
                                const double* W2t, double* z, double* mu_s, double* pm_s,
                                double* hid, double* al, T* dk, T* dv) {
    constexpr int N = D / 32;
    const int lane = threadIdx.x & 31, off = lane * N;
    const int h = gv.h;
    // 1. means of the keys and of the values, in child order
    double mu[N], vs[N];
#pragma unroll
    for (int e = 0; e < N; ++e) { mu[e] = 0.0; vs[e] = 0.0; }
    for (int c = 0; c < m; ++c) {
        double x[N], v[N];
        load_dims<T, N>(sk + c * rs, off, x);
        load_dims<T, N>(sv + c * rs, off, v);
#pragma unroll
        for (int e = 0; e < N; ++e) { mu[e] += x[e]; vs[e] += v[e]; }
    }
    const double dm = (double)m;
#pragma unroll
    for (int e = 0; e < N; ++e) mu[e] /= dm;
    // 2. each child's projection w . (x_c - mu) and the squared deviations, four
    //    children at a time so that their warp reductions overlap
    double ss = 0.0;
    for (int c0 = 0; c0 < m; c0 += 4) {
        double dw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            dw[u] = 0.0;
            if (c0 + u < m) {
                double x[N];
                load_dims<T, N>(sk + (c0 + u) * rs, off, x);
#pragma unroll
                for (int e = 0; e < N; ++e) {
                    const double dx = x[e] - mu[e];
                    dw[u] = fma(dx, w[off + e], dw[u]);
                    ss = fma(dx, dx, ss);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < 4; ++u) dw[u] += __shfl_xor_sync(kFull, dw[u], o);
        if (lane == 0)
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c0 + u < m) al[c0 + u] = dw[u];
    }
    ss = warp_sum_f64(ss);
    const double sigma = sqrt(ss / (dm * (double)D) + 1e-6);
    __syncwarp();
    // 3. softmax over the children of (tau / sigma) * projection: lane c < m (m <= 32)
    //    forms its child's logit, the maximum is a warp reduction, and
    //    exp(logit_c - max) is formed once; the sum is taken in child order
    const double ts = gv.tau / sigma;
    const double lg = lane < m ? ts * al[lane] : -INFINITY;
    const double mx = warp_max_f64(lg);
    __syncwarp();
    if (lane < m) al[lane] = exp(lg - mx);
    __syncwarp();
    double sum = 0.0;
    for (int c = 0; c < m; ++c) sum += al[c];
    // 4. p = sum_c alpha_c x_c, as (sum_c e_c x_c) / sum_c e_c: one division per dim
    double p[N];
#pragma unroll
    for (int e = 0; e < N; ++e) p[e] = 0.0;
    for (int c = 0; c < m; ++c) {
        const double a = al[c];
        double x[N];
        load_dims<T, N>(sk + c * rs, off, x);
#pragma unroll
        for (int e = 0; e < N; ++e) p[e] = fma(a, x[e], p[e]);
    }
#pragma unroll
    for (int e = 0; e < N; ++e) p[e] /= sum;
    // 5. the MLP input z = [mu / rho ; (p - mu) / sigma]; mu and p - mu kept for the end
#pragma unroll
    for (int e = 0; e < N; ++e) {
        const double pm = p[e] - mu[e];
        z[off + e] = mu[e] / gv.rho;
        z[D + off + e] = pm / sigma;
        mu_s[off + e] = mu[e];
        pm_s[off + e] = pm;
    }
    __syncwarp();
    // 6. hidden units i = lane, lane + 32: SiLU(W1 z + b1), four interleaved partial
    //    sums over the 2D inputs combined in a fixed order
    for (int i = lane; i < h; i += 32) {
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        for (int j = 0; j < 2 * D; j += 4) {
            a0 = fma(W1t[(j + 0) * h + i], z[j + 0], a0);
            a1 = fma(W1t[(j + 1) * h + i], z[j + 1], a1);
            a2 = fma(W1t[(j + 2) * h + i], z[j + 2], a2);
            a3 = fma(W1t[(j + 3) * h + i], z[j + 3], a3);
        }
        const double u = ((a0 + a1) + (a2 + a3)) + b1[i];
        hid[i] = u / (1.0 + exp(-u));
    }
    __syncwarp();
    // 7. output dims j = lane + 32 e: K = mu + g (p - mu) + sigma (W2 hid)
#pragma unroll
    for (int e = 0; e < N; ++e) {
        const int j = lane + 32 * e;
        double acc = 0.0;
        for (int i = 0; i < h; ++i) acc = fma(W2t[i * D + j], hid[i], acc);
        const double kv = mu_s[j] + gv.g * pm_s[j] + sigma * acc;
        dk[j] = store_round<T>(kv);
    }
    // the value: Eq.1's mean, stored like the stand-in pooler's
    float fv[N];
#pragma unroll
    for (int e = 0; e < N; ++e) fv[e] = (float)store_round<T>(vs[e] / dm);
    Dims<T, N>::store(dv + off, fv);
    __syncwarp();   // the warp's scratch is free for the next node
}

// One level `lvl` (>= 1) of every (sequence, KV head): the nodes covering tokens
// [L_old, L_old + add) (add > 0: an append of `add` tokens at the old device-side
// length L_old) or every node of [0, L) (add == 0).  A persistent grid: each CTA
// stages the weights once and its warps take nodes in turn.
template <typename T, int D>
__global__ void __launch_bounds__(512, 1)
    gated_level_kernel(TreeView tv, WorkView wv, GatedView gv, int lvl, int64_t add) {
    extern __shared__ __align__(16) double gsm[];
    const int h = gv.h;
    double* w = gsm;
    double* W1t = w + D;
    double* b1 = W1t + 2 * D * h;
    double* W2t = b1 + h;
    double* scratch = W2t + h * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) w[i] = gv.w[i];
    for (int i = threadIdx.x; i < 2 * D * h; i += blockDim.x) W1t[i] = gv.W1t[i];
    for (int i = threadIdx.x; i < h; i += blockDim.x) b1[i] = gv.b1[i];
    for (int i = threadIdx.x; i < h * D; i += blockDim.x) W2t[i] = gv.W2t[i];
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const int nwarp_cta = blockDim.x >> 5;
    double* z = scratch + warp * (4 * D + h + RECSA_MAX_C);
    double* mu_s = z + 2 * D;
    double* pm_s = mu_s + D;
    double* hid = pm_s + D;
    double* al = hid + h;
    const int C = tv.C;
    int64_t span = 1;   // tokens per node at level lvl
    for (int i = 0; i < lvl; ++i) span *= C;
    const int64_t span_c = span / C;   // tokens per child
    // work items: (b, h, node) over all (sequence, KV head) units, node in [p_lo, p_hi]
    const int nbh = tv.B * tv.Hkv;
    const int64_t gw = (int64_t)blockIdx.x * nwarp_cta + warp;
    const int64_t nwarps = (int64_t)gridDim.x * nwarp_cta;
    // per unit, the number of nodes to pool at this level; the units are taken in
    // order, each warp stepping through the flattened (unit, node) space
    int64_t base = 0;
    for (int bh = 0; bh < nbh; ++bh) {
        const int b = bh / tv.Hkv, hh = bh % tv.Hkv;
        const int64_t len_old = wv.lens[b];
        const int64_t L_new = len_old + add;
        int64_t cnt = 0, p_lo = 0, n_child = 0;
        if (L_new <= tv.cap && L_new > 0) {
            n_child = (L_new + span_c - 1) / span_c;   // rows of level lvl - 1
            if (n_child > 1) {
                const int64_t lo = add == 0 ? 0 : len_old;
                p_lo = lo / span;
                const int64_t p_hi = (L_new - 1) / span;
                cnt = p_hi - p_lo + 1;
            }
        }
        // this warp's items of this unit: global indices base .. base + cnt - 1
        int64_t first = gw - base;
        if (first < 0) first += ((-first + nwarps - 1) / nwarps) * nwarps;
        for (int64_t it = first; it < cnt; it += nwarps) {
            const int64_t i = p_lo + it;
            const int m = (int)imin64(C, n_child - i * C);
            const T *sk, *sv;
            int64_t rs;
            level_rows<T>(tv, lvl - 1, b, hh, sk, sv, rs);
            gated_pool_node<T, D>(sk + i * C * rs, sv + i * C * rs, rs, m, gv, w, W1t, b1, W2t,
                                  z, mu_s, pm_s, hid, al, level_k<T>(tv, lvl, b, hh) + i * D,
                                  level_v<T>(tv, lvl, b, hh) + i * D);
        }
        base += cnt;
    }
}

template <typename T, int D>
static cudaError_t gated_levels_impl(const TreeView& tv, const WorkView& wv, const GatedView& gv,
                                     int64_t add, cudaStream_t s) {
    const int warps = gated_warps(D, gv.h);
    const size_t sm = gated_smem(D, gv.h, warps);
    cudaError_t e = cudaFuncSetAttribute(gated_level_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    // an append re-pools a few nodes per unit; a build every node
    const int64_t work = add == 0 ? (int64_t)tv.B * tv.Hkv * ((tv.cap + tv.C - 1) / tv.C)
                                  : (int64_t)tv.B * tv.Hkv * (add / tv.C + 2);
    int64_t grid = (work + warps - 1) / warps;
    if (grid > nsm) grid = nsm;
    if (grid < 1) grid = 1;
    NvtxRange nv(add == 0 ? "recsa build (gated pooler)" : "recsa append levels (gated pooler)");
    for (int lvl = 1; lvl < tv.n_levels; ++lvl) {
        gated_level_kernel<T, D><<<(unsigned)grid, warps * 32, sm, s>>>(tv, wv, gv, lvl, add);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gated_levels(const TreeView& tv, const WorkView& wv, const GatedView& gv,
                                int64_t add, int dtype, cudaStream_t s) {
    if (gv.h < 1 || gv.h > kGatedMaxHidden) return cudaErrorInvalidValue;
    if (dtype == RECSA_BF16 && tv.D == 128) return gated_levels_impl<__nv_bfloat16, 128>(tv, wv, gv, add, s);
    if (dtype == RECSA_BF16 && tv.D == 64) return gated_levels_impl<__nv_bfloat16, 64>(tv, wv, gv, add, s);
    if (dtype == RECSA_F32 && tv.D == 128) return gated_levels_impl<float, 128>(tv, wv, gv, add, s);
    if (dtype == RECSA_F32 && tv.D == 64) return gated_levels_impl<float, 64>(tv, wv, gv, add, s);
    return cudaErrorInvalidValue;
}

}  // namespace recsa

// Pooling of tree nodes (Eq.1 of "Recursive Sparse Attention", section "Tree
// Construction") shared by the build, the append and the decode kernels.
//
// A level-l node i pools its children C*i .. min(C*i+C-1, n_{l-1}-1) of level l-1:
//   K = sum_c alpha_c K_c, alpha = softmax(w) over the m present children,
//   V = (1/m) sum_c V_c,
// summed in fp64, one lane per dimension in child order (fused multiply-add for
// K), and rounded once to the storage dtype.  Every caller performs the same
// operations in the same order, so a tree is bitwise the same however it was made.
#pragma once
#include "recsa_internal.cuh"

namespace recsa {

// Lanes own D/32 consecutive dimensions, so one warp instruction reads a whole
// row and every dimension is summed by one lane in child order.
template <typename T, int D>
struct PoolShape {
    static constexpr int DPL = D / 32;   // dimensions per lane
};

// DPL consecutive elements as floats (exact widening), and back.
template <typename T, int N>
struct Dims;
template <>
struct Dims<float, 4> {
    static __device__ __forceinline__ void load(const float* p, float (&x)[4]) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float (&x)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <>
struct Dims<float, 2> {
    static __device__ __forceinline__ void load(const float* p, float (&x)[2]) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x; x[1] = v.y;
    }
    static __device__ __forceinline__ void store(float* p, const float (&x)[2]) {
        *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    }
};
template <>
struct Dims<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[4]) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xffff0000u);
        x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xffff0000u);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&x)[4]) {
        uint2 v;
        v.x = (__float_as_uint(x[0]) >> 16) | (__float_as_uint(x[1]) & 0xffff0000u);
        v.y = (__float_as_uint(x[2]) >> 16) | (__float_as_uint(x[3]) & 0xffff0000u);
        *reinterpret_cast<uint2*>(p) = v;
    }
};
template <>
struct Dims<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[2]) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
        x[0] = __uint_as_float(v << 16); x[1] = __uint_as_float(v & 0xffff0000u);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&x)[2]) {
        *reinterpret_cast<uint32_t*>(p) =
            (__float_as_uint(x[0]) >> 16) | (__float_as_uint(x[1]) & 0xffff0000u);
    }
};

// One lane's DPL elements of a row as loaded (packed), widened when used, so a
// batch of rows in flight costs one register per two bf16 elements.
template <typename T, int N>
struct Packed;
template <>
struct Packed<__nv_bfloat16, 4> {
    uint2 v;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = *reinterpret_cast<const uint2*>(p); }
    __device__ __forceinline__ float get(int e) const {
        const uint32_t w = (e < 2) ? v.x : v.y;
        return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
    }
};
template <>
struct Packed<__nv_bfloat16, 2> {
    uint32_t v;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = *reinterpret_cast<const uint32_t*>(p); }
    __device__ __forceinline__ float get(int e) const {
        return __uint_as_float((e & 1) ? (v & 0xffff0000u) : (v << 16));
    }
};
template <>
struct Packed<float, 4> {
    float4 v;
    __device__ __forceinline__ void load(const float* p) { v = *reinterpret_cast<const float4*>(p); }
    __device__ __forceinline__ float get(int e) const {
        return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
    }
};
template <>
struct Packed<float, 2> {
    float2 v;
    __device__ __forceinline__ void load(const float* p) { v = *reinterpret_cast<const float2*>(p); }
    __device__ __forceinline__ float get(int e) const { return e == 0 ? v.x : v.y; }
};

// softmax(w[0..m-1]) for every m = 1..C, fp64, into alpha[(m-1)*C + c].
__device__ inline void fill_alpha(const float* w, int C, double* alpha) {
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
        int m = idx / C + 1, c = idx % C;
        double v = 0.0;
        if (c < m) {
            double mx = (double)w[0];
            for (int j = 1; j < m; ++j) mx = fmax(mx, (double)w[j]);
            double sum = 0.0;
            for (int j = 0; j < m; ++j) sum += exp((double)w[j] - mx);
            v = exp((double)w[c] - mx) / sum;
        }
        alpha[idx] = v;
    }
}

// Adds children rows [r_lo, r_hi) (row stride rs elements) of one parent to this
// lane's fp64 sums, in child order: ak += alpha_m[r] * K_r (fused), av += V_r.
// Rows are loaded B at a time ahead of the arithmetic.
template <typename T, int D, int B = 8>
__device__ __forceinline__ void pool_rows(const T* sk, const T* sv, int64_t rs, int r_lo, int r_hi,
                                          const double* alpha_m, double (&ak)[D / 32],
                                          double (&av)[D / 32]) {
    constexpr int N = PoolShape<T, D>::DPL;
    const int off = (threadIdx.x & 31) * N;
    for (int r0 = r_lo; r0 < r_hi; r0 += B) {
        Packed<T, N> kx[B], vx[B];
#pragma unroll
        for (int u = 0; u < B; ++u)
            if (r0 + u < r_hi) {
                kx[u].load(sk + (r0 + u) * rs + off);
                vx[u].load(sv + (r0 + u) * rs + off);
            }
#pragma unroll
        for (int u = 0; u < B; ++u)
            if (r0 + u < r_hi) {
                const double al = alpha_m[r0 + u];
#pragma unroll
                for (int e = 0; e < N; ++e) {
                    ak[e] = fma(al, (double)kx[u].get(e), ak[e]);
                    av[e] += (double)vx[u].get(e);
                }
            }
    }
}

// Rounds one parent's sums to storage: K = ak, V = av / m.  Returns the stored
// values widened to float in (fk, fv).
template <typename T, int D>
__device__ __forceinline__ void pool_store(const double (&ak)[D / 32], const double (&av)[D / 32],
                                           int m, T* dk, T* dv, float (&fk)[D / 32],
                                           float (&fv)[D / 32]) {
    constexpr int N = PoolShape<T, D>::DPL;
    const int off = (threadIdx.x & 31) * N;
    const double dm = (double)m;
#pragma unroll
    for (int e = 0; e < N; ++e) {
        fk[e] = (float)store_round<T>(ak[e]);
        fv[e] = (float)store_round<T>(av[e] / dm);
    }
    Dims<T, N>::store(dk + off, fk);
    Dims<T, N>::store(dv + off, fv);
}

// One warp pools the m children of one parent (the whole node).
template <typename T, int D>
__device__ __forceinline__ void warp_pool_node(const T* sk, const T* sv, int64_t rs, int m,
                                               const double* alpha_m, T* dk, T* dv) {
    constexpr int N = PoolShape<T, D>::DPL;
    double ak[N], av[N];
#pragma unroll
    for (int e = 0; e < N; ++e) { ak[e] = 0.0; av[e] = 0.0; }
    // every child row of a node in flight at once when rows pack two bf16 per word
    pool_rows<T, D, sizeof(T) == 2 ? 16 : 8>(sk, sv, rs, 0, m, alpha_m, ak, av);
    float fk[N], fv[N];
    pool_store<T, D>(ak, av, m, dk, dv, fk, fv);
}


template <typename T>
__device__ __forceinline__ void level_rows(const TreeView& tv, int l, int b, int h, const T*& k,
                                           const T*& v, int64_t& rs) {
    if (l == 0) {
        k = reinterpret_cast<const T*>(tv.k0) + (b * tv.s_b + h * tv.s_h);
        v = reinterpret_cast<const T*>(tv.v0) + (b * tv.s_b + h * tv.s_h);
        rs = tv.s_t;
    } else {
        k = level_k<T>(tv, l, b, h);
        v = level_v<T>(tv, l, b, h);
        rs = tv.D;
    }
}


// ----------------------------------------------------------------------------
// The ancestors of token t (just written at level 0) re-pooled bottom-up by one
// CTA of at least as many warps as it has levels to spread.  At level l the
// ancestor is node t / C^l, whose m = (t / C^(l-1)) mod C + 1 children are m-1
// complete nodes and, last, the ancestor at level l-1.  Warps first sum the
// complete children of every level in parallel (fp64, child order, in shared
// memory `pre`: [levels][2][D]); warp 0 then walks the levels adding the one new
// term per level.  alpha: the C x C softmax table, already in shared memory.
// ----------------------------------------------------------------------------
// RB: children rows loaded per batch (fewer registers inside a larger kernel).
template <typename T, int D, int RB = 16>
__device__ __forceinline__ void ancestor_walk(const TreeView& tv, int b, int h, int64_t t,
                                              double* pre, const double* alpha, uint32_t* status) {
    constexpr int N = PoolShape<T, D>::DPL;
    const int C = tv.C, lgC = tv.lgC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int off = lane * N;
    int nl = 0;   // levels 1..nl are pooled: level l exists while level l-1 has > 1 node
    for (int64_t x = t; x >= 1 && nl + 1 < tv.n_levels; x = cdiv64(x, C, lgC)) ++nl;
    for (int l = 1 + warp; l <= nl; l += nwarps) {
        int64_t x = t;   // ancestor index at level l-1
        for (int j = 1; j < l; ++j) x = cdiv64(x, C, lgC);
        int64_t i = cdiv64(x, C, lgC);
        int m = (int)(x - i * C) + 1;
        if (!in_bounds(i >= 0 && x < tv.rows[l - 1] && i < tv.rows[l], status)) { i = 0; m = 1; }
        const T *sk, *sv;
        int64_t rs;
        level_rows<T>(tv, l - 1, b, h, sk, sv, rs);
        double ak[N], av[N];
#pragma unroll
        for (int e = 0; e < N; ++e) { ak[e] = 0.0; av[e] = 0.0; }
        pool_rows<T, D, RB>(sk + i * C * rs, sv + i * C * rs, rs, 0, m - 1, alpha + (m - 1) * C,
                            ak, av);
#pragma unroll
        for (int e = 0; e < N; ++e) {
            pre[(2 * (l - 1)) * D + off + e] = ak[e];
            pre[(2 * (l - 1) + 1) * D + off + e] = av[e];
        }
    }
    __syncthreads();
    if (warp == 0) {
        float ck[N], cv[N];   // the newest child: the token, then each new ancestor
        const T* k0 = reinterpret_cast<const T*>(tv.k0) + (b * tv.s_b + h * tv.s_h + t * tv.s_t);
        const T* v0 = reinterpret_cast<const T*>(tv.v0) + (b * tv.s_b + h * tv.s_h + t * tv.s_t);
        Dims<T, N>::load(k0 + off, ck);
        Dims<T, N>::load(v0 + off, cv);
        int64_t x = t;
        for (int l = 1; l <= nl; ++l) {
            const int64_t i = cdiv64(x, C, lgC);
            const int m = (int)(x - i * C) + 1;
            const double al = alpha[(m - 1) * C + (m - 1)];
            double ak[N], av[N];
#pragma unroll
            for (int e = 0; e < N; ++e) {
                ak[e] = fma(al, (double)ck[e], pre[(2 * (l - 1)) * D + off + e]);
                av[e] = pre[(2 * (l - 1) + 1) * D + off + e] + (double)cv[e];
            }
            pool_store<T, D>(ak, av, m, level_k<T>(tv, l, b, h) + i * D,
                             level_v<T>(tv, l, b, h) + i * D, ck, cv);
            x = i;
        }
    }
}

// Shared memory the walk needs: `pre` for every level above 0, then alpha.
inline size_t ancestor_walk_smem(int n_levels, int D) {
    return sizeof(double) * (2 * (size_t)D * (n_levels > 1 ? n_levels - 1 : 1) + RECSA_MAX_C * RECSA_MAX_C);
}

}  // namespace recsa

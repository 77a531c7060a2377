// Level 0 in host memory ("Efficiency Results": decode at 1M and 2M tokens with the
// KV cache offloaded; "Practical Implications": the levels above 0 are under 7 % of
// the cache and stay in HBM).  A decode then runs the select/attend pass in two
// launches around this gather: after the levels >= 1 have selected S^(1), the rows of
// each query's level-0 list A^(0) = children of S^(1) (Eq.3) are copied from the
// host-resident cache into an HBM staging buffer in list order, and the level-0 pass
// reads them there.  Only the rows the query attends to cross the host link.
#include "recsa_internal.cuh"

namespace recsa {

// One CTA per (query, KV head) unit and slice of its list; 16 threads per row, 16
// bytes each, so a row's K (or V) is one 256-byte request for d = 128 bf16.  Plain
// loads from the mapped host memory (no TMA).
template <typename T, int D>
__global__ void __launch_bounds__(256) gather_level0_kernel(TreeView tv, WorkView wv, QueryView qv,
                                                            T* stage_k, T* stage_v) {
    constexpr int VEC = VecOf<T>::N;
    constexpr int TPR = D / VEC;               // threads per row
    constexpr int RPB = 256 / TPR;             // rows per CTA step
    const int unit = blockIdx.y;
    const int qloc = unit / tv.Hkv, kvh = unit % tv.Hkv;
    int b, gq;
    int64_t t;
    if (!query_pos(qv, wv, qloc, b, t, gq)) return;
    const int C = tv.C, lgC = tv.lgC, k = tv.k;
    const int lstar = first_scored_level(t, C, lgC, k);
    const int n0 = list_size(t, lstar, 0, C, lgC, k);
    const int32_t* S1 = wv.sel + (int64_t)unit * wv.NL * k;   // S^(1), current node last
    const T* k0 = reinterpret_cast<const T*>(tv.k0) + (b * tv.s_b + kvh * tv.s_h);
    const T* v0 = reinterpret_cast<const T*>(tv.v0) + (b * tv.s_b + kvh * tv.s_h);
    const int64_t so = ((int64_t)qloc * tv.Hkv + kvh) * (int64_t)wv.ck * D;
    const int tr = threadIdx.x / TPR, tc = threadIdx.x % TPR;
    for (int j = blockIdx.x * RPB + tr; j < n0; j += gridDim.x * RPB) {
        // entry j of A^(0): token j when level 0 is the first scored level, else child
        // j mod C of the (j / C)-th node of S^(1)
        int64_t tok = lstar == 0 ? (int64_t)j
                                 : (int64_t)C * S1[cdiv(j, C, lgC)] + cmod(j, C, lgC);
        if (!in_bounds(tok >= 0 && tok <= t, wv.status)) tok = 0;
        const uint4 kx = *reinterpret_cast<const uint4*>(k0 + tok * tv.s_t + tc * VEC);
        const uint4 vx = *reinterpret_cast<const uint4*>(v0 + tok * tv.s_t + tc * VEC);
        *reinterpret_cast<uint4*>(stage_k + so + (int64_t)j * D + tc * VEC) = kx;
        *reinterpret_cast<uint4*>(stage_v + so + (int64_t)j * D + tc * VEC) = vx;
    }
}

template <typename T, int D>
static cudaError_t gather_impl(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                               void* sk, void* sv, cudaStream_t s) {
    NvtxRange nv("recsa gather level 0");
    const unsigned slices = (unsigned)((wv.ck + 255) / 256);
    dim3 grid(slices < 8 ? slices : 8, (unsigned)(qv.nq * tv.Hkv));
    gather_level0_kernel<T, D><<<grid, 256, 0, s>>>(tv, wv, qv, reinterpret_cast<T*>(sk),
                                                     reinterpret_cast<T*>(sv));
    return cudaGetLastError();
}

cudaError_t launch_gather_level0(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                 void* stage_k, void* stage_v, int dtype, cudaStream_t s) {
    if (dtype == RECSA_BF16 && tv.D == 128) return gather_impl<__nv_bfloat16, 128>(tv, wv, qv, stage_k, stage_v, s);
    if (dtype == RECSA_BF16 && tv.D == 64) return gather_impl<__nv_bfloat16, 64>(tv, wv, qv, stage_k, stage_v, s);
    if (dtype == RECSA_F32 && tv.D == 128) return gather_impl<float, 128>(tv, wv, qv, stage_k, stage_v, s);
    if (dtype == RECSA_F32 && tv.D == 64) return gather_impl<float, 64>(tv, wv, qv, stage_k, stage_v, s);
    return cudaErrorInvalidValue;
}

}  // namespace recsa

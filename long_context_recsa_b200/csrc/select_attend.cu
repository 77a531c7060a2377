// Top-down selection (Eq.3, "Hierarchical Selection") with candidate-local RoPE
// ("Key Theoretical Insight") and the unified softmax over level-0 tokens and the
// summaries of unselected candidates (Eq.4, "Unified Softmax"), sm_100a.
//
// Work unit: one (query, KV head).  For each level l >= 1 a cluster of SPL CTAs
// splits the unit's candidate list A^(l) into contiguous chunks.  Each CTA
//   1. rotates the G query heads to position p_q = |A|-1 and every candidate key
//      of its chunk to its list index (cos/sin from an fp64-computed table),
//      keeping the per-head logits in shared memory (never in global memory);
//   2. picks its local top-(k-1) by (mean logit desc, index asc) with a radix
//      select, exchanges the local lists through distributed shared memory, and
//      every CTA selects the global top-(k-1) from the merged lists (the global
//      winners are a subset of the local winners);
//   3. writes S^(l) in ascending node order (rank = prefix count in list order;
//      the current node is last), and accumulates the split-softmax partial
//      (max, sum, weighted V) of its unselected candidates: the summaries.
// Entry j of the next list is node C*S[j/C] + j%C (a "slot" r*C + c), so lists
// are never materialised.  Level 0 runs the same scoring over A^(0) with every
// entry included; a combine kernel merges all partials into the output.
#include <cooperative_groups.h>

#include "recsa_internal.cuh"

namespace cg = cooperative_groups;

namespace recsa {

template <typename T, int D>
struct Shape {
    static constexpr int VEC = VecOf<T>::N;   // elements per 16-byte load
    static constexpr int KG = D / (2 * VEC);  // lanes per key (each lane: VEC rotary pairs)
    static constexpr int KPW = 32 / KG;       // keys per warp step
    static constexpr int RPL = D / VEC;       // lanes per value row
    static constexpr int RPW = 32 / RPL;      // value rows per warp step
};

// ----------------------------------------------------------------------------
// shared-memory layout of the select/attend kernels
// ----------------------------------------------------------------------------
struct Smem {
    size_t qrot, s, key, rank, flag, ulist, par, lkey, lidx, mkey, midx, hist, red, misc, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline Smem smem_layout(int G, int D, int CH, int k, int spl) {
    Smem L;
    const int K1 = k - 1 > 0 ? k - 1 : 1;
    const int RN = CH > spl * K1 ? CH : spl * K1;
    size_t o = 0;
    L.qrot = o;  o = align16(o + sizeof(float) * G * D);
    L.s = o;     o = align16(o + sizeof(float) * G * CH);
    L.key = o;   o = align16(o + sizeof(uint32_t) * CH);
    L.rank = o;  o = align16(o + sizeof(int) * RN);
    L.flag = o;  o = align16(o + sizeof(unsigned char) * CH);
    L.ulist = o; o = align16(o + sizeof(int) * CH);
    L.par = o;   o = align16(o + sizeof(int) * k);
    L.lkey = o;  o = align16(o + sizeof(uint32_t) * K1);
    L.lidx = o;  o = align16(o + sizeof(int) * K1);
    L.mkey = o;  o = align16(o + sizeof(uint32_t) * spl * K1);
    L.midx = o;  o = align16(o + sizeof(int) * spl * K1);
    L.hist = o;  o = align16(o + sizeof(uint32_t) * 256);
    L.red = o;   o = align16(o + sizeof(float) * kWarps * G * D);
    L.misc = o;  o = align16(o + sizeof(int) * 64);
    L.total = o;
    return L;
}

// ----------------------------------------------------------------------------
// block-wide primitives (kThreads threads)
// ----------------------------------------------------------------------------

// Exclusive scan of one int per thread in thread order.  scratch: kWarps+1 ints.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int tw = scratch[w];
            scratch[w] = run;
            run += tw;
        }
        scratch[kWarps] = run;
    }
    __syncthreads();
    const int off = scratch[warp] + x - v;
    total = scratch[kWarps];
    __syncthreads();
    return off;
}

// Exact top-K of n keys by (key desc, position asc).  rank[i] receives the rank of
// item i among the selected items in position order, or -1.  MSB-first radix
// select over 8-bit digits finds the threshold key T and how many items equal to T
// are needed; those are the lowest-positioned ones.
__device__ void block_topk_rank(const uint32_t* keys, int n, int K, int* rank, uint32_t* hist,
                                int* misc) {
    const int tid = threadIdx.x;
    if (K >= n || K <= 0) {
        for (int i = tid; i < n; i += kThreads) rank[i] = (K >= n) ? i : -1;
        __syncthreads();
        return;
    }
    uint32_t prefix = 0, mask = 0;
    int rem = K;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += kThreads) {
            const uint32_t kk = keys[i];
            if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            const int lane = tid;
            uint32_t cnt[8];
            uint32_t tot = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                cnt[u] = hist[255 - 8 * lane - u];
                tot += cnt[u];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            const uint32_t excl = incl - tot;
            if (excl < (uint32_t)rem && (uint32_t)rem <= incl) {
                uint32_t run = excl;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (run + cnt[u] >= (uint32_t)rem) {
                        misc[0] = 255 - 8 * lane - u;
                        misc[1] = (int)run;
                        break;
                    }
                    run += cnt[u];
                }
            }
        }
        __syncthreads();
        const int digit = misc[0], above = misc[1];
        rem -= above;
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        __syncthreads();
    }
    const uint32_t T = prefix;
    const int need_eq = rem;
    // ties: the first need_eq items equal to T (position order)
    const int ipt = (n + kThreads - 1) / kThreads;
    const int i0 = tid * ipt, i1 = min(n, i0 + ipt);
    int ceq = 0;
    for (int i = i0; i < i1; ++i) ceq += (keys[i] == T);
    int tot;
    int eq_rank = block_excl_scan(ceq, misc + 2, tot);
    int csel = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t kk = keys[i];
        bool sel = kk > T;
        if (kk == T) { sel = eq_rank < need_eq; ++eq_rank; }
        rank[i] = sel ? 1 : 0;
        csel += sel;
    }
    int r = block_excl_scan(csel, misc + 2, tot);
    for (int i = i0; i < i1; ++i) {
        if (rank[i]) rank[i] = r++;
        else rank[i] = -1;
    }
    __syncthreads();
}

// ----------------------------------------------------------------------------
// scoring: s[g][r] = scale * <R(p_q) q_g, R(j) K_node(j)>, j = j0 + r
// ----------------------------------------------------------------------------
template <typename T, int D, int G, bool WITH_KEY>
__device__ __forceinline__ void score_chunk(const T* kbase, int64_t rs, const float2* rope, int j0,
                                            int n, bool identity, const int* par, int C,
                                            float scale, const float* qrot, float* s,
                                            uint32_t* key, int CH) {
    using S = Shape<T, D>;
    constexpr int VEC = S::VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = lane % S::KG, kg = lane / S::KG;
    float qlo[G][VEC], qhi[G][VEC];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            qlo[g][v] = qrot[g * D + c * VEC + v];
            qhi[g][v] = qrot[g * D + D / 2 + c * VEC + v];
        }
    for (int base = warp * S::KPW; base < n; base += kWarps * S::KPW) {
        const int r = base + kg;
        const bool act = r < n;
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = 0.f;
        if (act) {
            const int j = j0 + r;
            const int64_t node = identity ? (int64_t)j : (int64_t)C * par[j / C] + (j % C);
            const T* row = kbase + node * rs;
            float klo[VEC], khi[VEC];
            load16_nc<T>(row + c * VEC, klo);
            load16_nc<T>(row + D / 2 + c * VEC, khi);
            const float4* cs4 = reinterpret_cast<const float4*>(rope + (int64_t)j * (D / 2) + c * VEC);
#pragma unroll
            for (int v2 = 0; v2 < VEC / 2; ++v2) {
                const float4 cs = __ldg(cs4 + v2);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int v = 2 * v2 + u;
                    const float co = u ? cs.z : cs.x, si = u ? cs.w : cs.y;
                    const float a = klo[v] * co - khi[v] * si;
                    const float bb = klo[v] * si + khi[v] * co;
#pragma unroll
                    for (int g = 0; g < G; ++g) acc[g] += qlo[g][v] * a + qhi[g][v] * bb;
                }
            }
        }
#pragma unroll
        for (int o = 1; o < S::KG; o <<= 1)
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] += __shfl_xor_sync(kFull, acc[g], o);
        if (act && c == 0) {
            float imp = 0.f;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float sv = acc[g] * scale;
                s[g * CH + r] = sv;
                imp += sv;
            }
            if (WITH_KEY) key[r] = ordered_key(imp * (1.0f / G));
        }
    }
}

// Rotate the G query heads of KV head kvh to position p_q into qrot[G][D].
template <typename T, int D, int G>
__device__ __forceinline__ void rotate_query(const T* qrow /* head kvh*G */, const float2* rope,
                                             int p_q, float* qrot) {
    for (int i = threadIdx.x; i < G * (D / 2); i += kThreads) {
        const int g = i / (D / 2), pr = i % (D / 2);
        const float x1 = (float)qrow[g * D + pr];
        const float x2 = (float)qrow[g * D + pr + D / 2];
        const float2 cs = rope[(int64_t)p_q * (D / 2) + pr];
        qrot[g * D + pr] = x1 * cs.x - x2 * cs.y;
        qrot[g * D + pr + D / 2] = x1 * cs.y + x2 * cs.x;
    }
}

// Softmax partial over the chunk entries listed in ulist (chunk-relative indices):
// m_g = max s, p = exp(s - m) (in place), l_g = sum p, o_g = sum p V.  Writes the
// partial record [G][D+2] = (o, m, l).  Empty list -> (0, -inf, 0).
template <typename T, int D, int G>
__device__ void softmax_partial(const T* vbase, int64_t rs, int j0, const int* ulist, int nu,
                                bool identity, const int* par, int C, float* s, int CH,
                                float* red, int* misc, float* outp) {
    using S = Shape<T, D>;
    constexpr int VEC = S::VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* fmisc = reinterpret_cast<float*>(misc);
    // per-head max
    float mx[G];
#pragma unroll
    for (int g = 0; g < G; ++g) mx[g] = -INFINITY;
    for (int u = threadIdx.x; u < nu; u += kThreads) {
        const int r = ulist[u];
#pragma unroll
        for (int g = 0; g < G; ++g) mx[g] = fmaxf(mx[g], s[g * CH + r]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(kFull, mx[g], o));
        if (lane == 0) red[warp * G + g] = mx[g];
    }
    __syncthreads();
    if (threadIdx.x < G) {
        float m = -INFINITY;
        for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w * G + threadIdx.x]);
        fmisc[threadIdx.x] = m;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) mx[g] = fmisc[g];
    // p = exp(s - m), per-head sums
    float sm[G];
#pragma unroll
    for (int g = 0; g < G; ++g) sm[g] = 0.f;
    for (int u = threadIdx.x; u < nu; u += kThreads) {
        const int r = ulist[u];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float p = __expf(s[g * CH + r] - mx[g]);
            s[g * CH + r] = p;
            sm[g] += p;
        }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sm[g] += __shfl_xor_sync(kFull, sm[g], o);
        if (lane == 0) red[warp * G + g] = sm[g];
    }
    __syncthreads();
    if (threadIdx.x < G) {
        float l = 0.f;
        for (int w = 0; w < kWarps; ++w) l += red[w * G + threadIdx.x];
        fmisc[G + threadIdx.x] = l;
    }
    __syncthreads();
    // o = sum p V
    const int c = lane % S::RPL, rr = lane / S::RPL;
    float acc[G][VEC];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[g][e] = 0.f;
#pragma unroll 4
    for (int base = warp * S::RPW; base < nu; base += kWarps * S::RPW) {
        const int u = base + rr;
        if (u < nu) {
            const int r = ulist[u];
            const int j = j0 + r;
            const int64_t node = identity ? (int64_t)j : (int64_t)C * par[j / C] + (j % C);
            float v[VEC];
            load16_nc<T>(vbase + node * rs + c * VEC, v);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float p = s[g * CH + r];
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[g][e] += p * v[e];
            }
        }
    }
#pragma unroll
    for (int o = S::RPL; o < 32; o <<= 1)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[g][e] += __shfl_xor_sync(kFull, acc[g][e], o);
    __syncthreads();   // red reused
    if (rr == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < VEC; ++e) red[(warp * G + g) * D + c * VEC + e] = acc[g][e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        float sum = 0.f;
        for (int w = 0; w < kWarps; ++w) sum += red[w * G * D + i];
        const int g = i / D, d = i % D;
        outp[g * (D + 2) + d] = sum;
    }
    if (threadIdx.x < G) {
        outp[threadIdx.x * (D + 2) + D] = fmisc[threadIdx.x];
        outp[threadIdx.x * (D + 2) + D + 1] = fmisc[G + threadIdx.x];
    }
}

__device__ __forceinline__ void write_empty_partial(float* outp, int G, int D) {
    for (int i = threadIdx.x; i < G * (D + 2); i += kThreads) {
        const int d = i % (D + 2);
        outp[i] = (d == D) ? -INFINITY : 0.f;
    }
}

// ----------------------------------------------------------------------------
// level l >= 1: score + RoPE + TopK + summaries (cluster of SPL CTAs per unit)
// level 0 (L0 = true): score + softmax partial over A^(0) (NS0 CTAs per unit)
// ----------------------------------------------------------------------------
template <typename T, int D, int G, bool L0>
__global__ void __launch_bounds__(kThreads) level_kernel(TreeView tv, WorkView wv, QueryView qv,
                                                         int level, int CH) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int k = tv.k, C = tv.C;
    const int K1 = k - 1;
    const int nsplit = L0 ? wv.NS0 : wv.SPL;
    const Smem SL = smem_layout(G, D, CH, k, L0 ? 1 : wv.SPL);
    float* qrot = reinterpret_cast<float*>(smem + SL.qrot);
    float* s = reinterpret_cast<float*>(smem + SL.s);
    uint32_t* key = reinterpret_cast<uint32_t*>(smem + SL.key);
    int* rank = reinterpret_cast<int*>(smem + SL.rank);
    unsigned char* flag = smem + SL.flag;
    int* ulist = reinterpret_cast<int*>(smem + SL.ulist);
    int* par = reinterpret_cast<int*>(smem + SL.par);
    uint32_t* lkey = reinterpret_cast<uint32_t*>(smem + SL.lkey);
    int* lidx = reinterpret_cast<int*>(smem + SL.lidx);
    uint32_t* mkey = reinterpret_cast<uint32_t*>(smem + SL.mkey);
    int* midx = reinterpret_cast<int*>(smem + SL.midx);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + SL.hist);
    float* red = reinterpret_cast<float*>(smem + SL.red);
    int* misc = reinterpret_cast<int*>(smem + SL.misc);

    const int unit = blockIdx.y;
    const int split = blockIdx.x;
    const int qloc = unit / tv.Hkv, kvh = unit % tv.Hkv;
    int b, gq;
    int64_t t;
    const bool valid = query_pos(qv, wv, qloc, b, t, gq);
    int64_t a[kMaxLevels];
    const int lstar = valid ? first_scored_level(t, C, k, a) : 0;
    const int NL = wv.NL;
    int32_t* cnt_ws = wv.cnt + (int64_t)unit * (NL + 1);
    int32_t* cnt_usr = qv.cnt_out ? qv.cnt_out + ((int64_t)gq * tv.Hkv + kvh) * (NL + 1) : nullptr;
    float* part = wv.part + (int64_t)unit * wv.NSLOT * G * (D + 2);

    if (!L0 && (!valid || level > lstar)) {
        // level not scored for this query: all of its list is selected
        if (split == 0) {
            for (int i = threadIdx.x; i < k; i += kThreads) {
                if (qv.sel_out) qv.sel_out[(((int64_t)gq * tv.Hkv + kvh) * NL + (level - 1)) * k + i] = -1;
            }
            if (threadIdx.x == 0) {
                cnt_ws[level] = 0;
                if (cnt_usr) cnt_usr[level] = 0;
            }
        }
        return;
    }
    if (L0 && !valid) {
        if (split == 0 && threadIdx.x == 0) {
            cnt_ws[0] = 0;
            if (cnt_usr) cnt_usr[0] = 0;
        }
        return;
    }

    const int nA = list_size(a, lstar, level, C, k);
    const bool identity = (level == lstar) || (L0 && lstar == 0);
    if (!identity) {
        const int32_t* src = wv.sel + ((int64_t)unit * NL + level) * k;   // S^(level+1)
        for (int i = threadIdx.x; i < k; i += kThreads) par[i] = src[i];
    }
    const int p_q = nA - 1;
    const T* qrow = reinterpret_cast<const T*>(qv.q) + ((int64_t)gq * tv.Hq + kvh * G) * D;
    rotate_query<T, D, G>(qrow, wv.rope, p_q, qrot);
    __syncthreads();

    const T *kbase, *vbase;
    int64_t rs;
    if (L0) {
        kbase = reinterpret_cast<const T*>(tv.k0) + (b * tv.s_b + kvh * tv.s_h);
        vbase = reinterpret_cast<const T*>(tv.v0) + (b * tv.s_b + kvh * tv.s_h);
        rs = tv.s_t;
    } else {
        kbase = level_k<T>(tv, level, b, kvh);
        vbase = level_v<T>(tv, level, b, kvh);
        rs = D;
    }
    const int chunk = (nA + nsplit - 1) / nsplit;
    const int j0 = split * chunk;
    const int j1 = min(nA, j0 + chunk);

    if (L0) {
        const int n = max(0, j1 - j0);
        score_chunk<T, D, G, false>(kbase, rs, wv.rope, j0, n, identity, par, C, tv.scale, qrot, s,
                                    key, CH);
        for (int i = threadIdx.x; i < n; i += kThreads) ulist[i] = i;
        __syncthreads();
        float* outp = part + (int64_t)(NL * wv.SPL + split) * G * (D + 2);
        if (n == 0) write_empty_partial(outp, G, D);
        else softmax_partial<T, D, G>(vbase, rs, j0, ulist, n, identity, par, C, s, CH, red, misc, outp);
        if (split == 0 && threadIdx.x == 0) {
            cnt_ws[0] = nA;
            if (cnt_usr) cnt_usr[0] = nA;
        }
        return;
    }

    int32_t* sel_ws = wv.sel + ((int64_t)unit * NL + (level - 1)) * k;
    int32_t* sel_usr = qv.sel_out ? qv.sel_out + (((int64_t)gq * tv.Hkv + kvh) * NL + (level - 1)) * k
                                  : nullptr;
    float* outp = part + (int64_t)((level - 1) * wv.SPL + split) * G * (D + 2);
    if (split == 0 && threadIdx.x == 0) {
        cnt_ws[level] = nA;
        if (cnt_usr) cnt_usr[level] = nA;
    }
    if (nA <= k) {
        // everything selected, no summaries (cannot happen below the first scored
        // level for k, C >= 2, kept for completeness)
        if (split == 0) {
            for (int i = threadIdx.x; i < k; i += kThreads) {
                int v = -1;
                if (i < nA) v = identity ? i : C * par[i / C] + (i % C);
                if (i < nA) sel_ws[i] = v;
                if (sel_usr) sel_usr[i] = v;
            }
        }
        write_empty_partial(outp, G, D);
        return;
    }

    // 1. score the chunk (the current entry nA-1 is never scored)
    const int n_sc = max(0, min(j1, nA - 1) - j0);
    score_chunk<T, D, G, true>(kbase, rs, wv.rope, j0, n_sc, identity, par, C, tv.scale, qrot, s,
                               key, CH);
    __syncthreads();

    // 2a. local top-(k-1)
    block_topk_rank(key, n_sc, K1, rank, hist, misc);
    for (int i = threadIdx.x; i < n_sc; i += kThreads) {
        const int r = rank[i];
        if (r >= 0) { lkey[r] = key[i]; lidx[r] = j0 + i; }
    }
    if (threadIdx.x == 0) misc[40] = min(n_sc, K1);
    __syncthreads();

    // 2b. exchange local lists across the cluster, merge in list order
    cg::cluster_group cluster = cg::this_cluster();
    const int csize = (int)cluster.num_blocks();
    const int crank = (int)cluster.block_rank();
    cluster.sync();
    int M = 0, off_self = 0;
    for (int r = 0; r < csize; ++r) {
        const int* rn = cluster.map_shared_rank(misc + 40, r);
        const int nr = *rn;
        if (r == crank) off_self = M;
        const uint32_t* rk = cluster.map_shared_rank(lkey, r);
        const int* ri = cluster.map_shared_rank(lidx, r);
        for (int i = threadIdx.x; i < nr; i += kThreads) {
            mkey[M + i] = rk[i];
            midx[M + i] = ri[i];
        }
        M += nr;
    }
    cluster.sync();   // every CTA has finished reading remote lists

    // 2c. global top-(k-1) over the merged lists; ranks in list order
    block_topk_rank(mkey, M, K1, rank, hist, misc);
    for (int i = threadIdx.x; i < n_sc; i += kThreads) flag[i] = 0;
    __syncthreads();
    const int n_self = misc[40];
    for (int i = threadIdx.x; i < n_self; i += kThreads) {
        const int r = rank[off_self + i];
        if (r >= 0) {
            const int j = midx[off_self + i];
            const int node = identity ? j : C * par[j / C] + (j % C);
            sel_ws[r] = node;
            if (sel_usr) sel_usr[r] = node;
            flag[j - j0] = 1;
        }
    }
    if (crank == 0 && threadIdx.x == 0) {
        sel_ws[K1] = (int)a[level];
        if (sel_usr) sel_usr[K1] = (int)a[level];
    }
    __syncthreads();

    // 3. summaries: unselected scored entries of this chunk
    int cu = 0;
    const int ipt = (n_sc + kThreads - 1) / kThreads;
    const int i0 = threadIdx.x * ipt, i1 = min(n_sc, i0 + ipt);
    for (int i = i0; i < i1; ++i) cu += (flag[i] == 0);
    int nu;
    int off = block_excl_scan(cu, misc + 2, nu);
    for (int i = i0; i < i1; ++i)
        if (flag[i] == 0) ulist[off++] = i;
    __syncthreads();
    if (nu == 0) write_empty_partial(outp, G, D);
    else softmax_partial<T, D, G>(vbase, rs, j0, ulist, nu, identity, par, C, s, CH, red, misc, outp);
}

// ----------------------------------------------------------------------------
// combine: log-sum-exp merge of every valid partial into the output
// ----------------------------------------------------------------------------
template <typename T, int D, int G>
__global__ void combine_kernel(TreeView tv, WorkView wv, QueryView qv) {
    const int unit = blockIdx.x;
    const int qloc = unit / tv.Hkv, kvh = unit % tv.Hkv;
    int b, gq;
    int64_t t;
    const bool valid = query_pos(qv, wv, qloc, b, t, gq);
    T* out = reinterpret_cast<T*>(qv.out) + ((int64_t)gq * tv.Hq + kvh * G) * D;
    if (!valid) {
        for (int i = threadIdx.x; i < G * D; i += blockDim.x) out[i] = store_round_f<T>(0.f);
        if (qv.mode == 1 && threadIdx.x == 0) set_status(wv.status, kStatusBadQuery);
        return;
    }
    int64_t a[kMaxLevels];
    const int lstar = first_scored_level(t, tv.C, tv.k, a);
    const float* P = wv.part + (int64_t)unit * wv.NSLOT * G * (D + 2);
    const int n_lvl_slots = lstar * wv.SPL;
    const int s0 = wv.NL * wv.SPL;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, d = i % D;
        float M = -INFINITY;
        for (int sl = 0; sl < n_lvl_slots; ++sl) M = fmaxf(M, P[(sl * G + g) * (D + 2) + D]);
        for (int sl = s0; sl < s0 + wv.NS0; ++sl) M = fmaxf(M, P[(sl * G + g) * (D + 2) + D]);
        float L = 0.f, O = 0.f;
        for (int sl = 0; sl < n_lvl_slots + wv.NS0; ++sl) {
            const int slot = sl < n_lvl_slots ? sl : s0 + (sl - n_lvl_slots);
            const float* rec = P + (slot * G + g) * (D + 2);
            const float l = rec[D + 1];
            if (l > 0.f) {
                const float w = __expf(rec[D] - M);
                L += w * l;
                O += w * rec[d];
            }
        }
        out[i] = store_round_f<T>(L > 0.f ? O / L : 0.f);
    }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
template <typename T, int D, int G>
static cudaError_t prepare_impl(int SPL, int NS0, int C, int k) {
    const int ck = C * k;
    const int CH = (ck + SPL - 1) / SPL;
    const int CH0 = (ck + NS0 - 1) / NS0;
    const size_t sm = smem_layout(G, D, CH, k, SPL).total;
    const size_t sm0 = smem_layout(G, D, CH0, k, 1).total;
    if (sm > 227 * 1024 || sm0 > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(level_kernel<T, D, G, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    if (SPL > 8) {
        e = cudaFuncSetAttribute(level_kernel<T, D, G, false>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    return cudaFuncSetAttribute(level_kernel<T, D, G, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm0);
}

template <typename T, int D, int G>
static cudaError_t select_attend_impl(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                      cudaStream_t s, const ProfHook* prof) {
    const int ck = tv.C * tv.k;
    const int CH = (ck + wv.SPL - 1) / wv.SPL;
    const int CH0 = (ck + wv.NS0 - 1) / wv.NS0;
    const size_t sm = smem_layout(G, D, CH, tv.k, wv.SPL).total;
    const size_t sm0 = smem_layout(G, D, CH0, tv.k, 1).total;
    const unsigned units = (unsigned)(qv.nq * tv.Hkv);
    for (int level = wv.NL; level >= 1; --level) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)wv.SPL, units, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = sm;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)wv.SPL;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        prof_mark(prof, level, true, s);
        cudaError_t e = cudaLaunchKernelEx(&cfg, level_kernel<T, D, G, false>, tv, wv, qv, level, CH);
        prof_mark(prof, level, false, s);
        if (e != cudaSuccess) return e;
    }
    prof_mark(prof, 0, true, s);
    level_kernel<T, D, G, true><<<dim3((unsigned)wv.NS0, units), kThreads, sm0, s>>>(tv, wv, qv, 0, CH0);
    prof_mark(prof, 0, false, s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prof_mark(prof, -2, true, s);
    combine_kernel<T, D, G><<<units, 128, 0, s>>>(tv, wv, qv);
    prof_mark(prof, -2, false, s);
    return cudaGetLastError();
}

#define RECSA_DISPATCH_TDG(dtype, D, G, FN, ...)                                          \
    do {                                                                                  \
        if ((dtype) == RECSA_BF16 && (D) == 128) {                                        \
            if ((G) == 1) return FN<__nv_bfloat16, 128, 1>(__VA_ARGS__);                  \
            if ((G) == 2) return FN<__nv_bfloat16, 128, 2>(__VA_ARGS__);                  \
            if ((G) == 4) return FN<__nv_bfloat16, 128, 4>(__VA_ARGS__);                  \
            if ((G) == 8) return FN<__nv_bfloat16, 128, 8>(__VA_ARGS__);                  \
        }                                                                                 \
        if ((dtype) == RECSA_BF16 && (D) == 64) {                                         \
            if ((G) == 1) return FN<__nv_bfloat16, 64, 1>(__VA_ARGS__);                   \
            if ((G) == 2) return FN<__nv_bfloat16, 64, 2>(__VA_ARGS__);                   \
            if ((G) == 4) return FN<__nv_bfloat16, 64, 4>(__VA_ARGS__);                   \
            if ((G) == 8) return FN<__nv_bfloat16, 64, 8>(__VA_ARGS__);                   \
        }                                                                                 \
        if ((dtype) == RECSA_F32 && (D) == 128) {                                         \
            if ((G) == 1) return FN<float, 128, 1>(__VA_ARGS__);                          \
            if ((G) == 2) return FN<float, 128, 2>(__VA_ARGS__);                          \
            if ((G) == 4) return FN<float, 128, 4>(__VA_ARGS__);                          \
            if ((G) == 8) return FN<float, 128, 8>(__VA_ARGS__);                          \
        }                                                                                 \
        if ((dtype) == RECSA_F32 && (D) == 64) {                                          \
            if ((G) == 1) return FN<float, 64, 1>(__VA_ARGS__);                           \
            if ((G) == 2) return FN<float, 64, 2>(__VA_ARGS__);                           \
            if ((G) == 4) return FN<float, 64, 4>(__VA_ARGS__);                           \
            if ((G) == 8) return FN<float, 64, 8>(__VA_ARGS__);                           \
        }                                                                                 \
        return cudaErrorInvalidValue;                                                     \
    } while (0)

cudaError_t prepare_kernels(int dtype, int D, int G, int SPL, int NS0, int C, int k) {
    RECSA_DISPATCH_TDG(dtype, D, G, prepare_impl, SPL, NS0, C, k);
}

cudaError_t launch_select_attend(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                 int dtype, cudaStream_t s, const ProfHook* prof) {
    RECSA_DISPATCH_TDG(dtype, tv.D, tv.G, select_attend_impl, tv, wv, qv, s, prof);
}

size_t select_smem_bytes(int G, int D, int C, int k, int spl) {
    const int ck = C * k;
    return smem_layout(G, D, (ck + spl - 1) / spl, k, spl).total;
}

}  // namespace recsa

// Top-down selection (Eq.3, "Hierarchical Selection") with candidate-local RoPE
// ("Key Theoretical Insight") and the unified softmax over level-0 tokens and the
// summaries of unselected candidates (Eq.4, "Unified Softmax"), sm_100a.
//
// Work unit: one (query, KV head).  For each level l >= 1 a cluster of SPL CTAs
// splits the unit's candidate list A^(l) into contiguous chunks of whole parent
// groups (C entries).  Each CTA
//   1. scores its chunk: the G query heads are rotated once per parent group
//      and every key by its child offset (slot-based rotation splitting, below);
//      per-head logits stay in shared memory, never in global memory;
//   2. exchanges the chunk's importance keys (mean logit, order-preserving
//      uint32) with the other CTAs of the cluster through distributed shared
//      memory, so that every CTA holds all |A|-1 keys in list order, and runs an
//      exact radix select of the top k-1 (ties to the lower list position, which
//      is the lower node index because lists are ascending);
//   3. writes its part of S^(l) (rank = number of selected entries before it;
//      the current node is last) and accumulates the split-softmax partial
//      (max, sum, weighted V) of its unselected entries: the summaries.
// Entry j of the next list is node C*S[j/C] + j%C, so lists are never
// materialised.  Level 0 scores A^(0) the same way with every entry included; the
// last level-0 CTA of a unit merges all partials of the unit into the output.
//
// Slot-based rotation splitting: entry j = C*r + c sits at candidate-local
// position j and the query at p_q = |A|-1, and
//     <R(p_q) q, R(j) K> = <R(p_q - C r) q, R(c) K>,
// so the query is rotated once per parent group r and each key only by one of C
// fixed rotations R(0..C-1), staged in shared memory.
#include <cooperative_groups.h>

#include "pool.cuh"

namespace cg = cooperative_groups;

namespace recsa {

template <typename T, int D>
struct Shape {
    static constexpr int VEC = VecOf<T>::N;   // elements per 16-byte load
    // scoring: LPK lanes per key, each owning PPL consecutive rotary pairs (CPL
    // couples of two pairs) of the low and of the high half of the key
    static constexpr int LPK = 16;
    static constexpr int PPL = D / 2 / LPK;
    static constexpr int CPL = PPL / 2;
    static constexpr int KPW = 32 / LPK;      // keys per warp step
    static constexpr int RPL = D / VEC;       // lanes per value row
    static constexpr int RPW = 32 / RPL;      // value rows per warp step
};

// PPL consecutive elements (a multiple of 2) as CPL fp32 pairs.
template <typename T, int PPL>
struct PairLoad;
template <>
struct PairLoad<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void get(const unsigned char* p, float2 (&o)[2]) {
        const uint2 w = *reinterpret_cast<const uint2*>(p);
        o[0] = make_float2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u));
        o[1] = make_float2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
    }
};
template <>
struct PairLoad<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void get(const unsigned char* p, float2 (&o)[1]) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        o[0] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
};
template <>
struct PairLoad<float, 4> {
    static __device__ __forceinline__ void get(const unsigned char* p, float2 (&o)[2]) {
        const float4 w = *reinterpret_cast<const float4*>(p);
        o[0] = make_float2(w.x, w.y);
        o[1] = make_float2(w.z, w.w);
    }
};
template <>
struct PairLoad<float, 2> {
    static __device__ __forceinline__ void get(const unsigned char* p, float2 (&o)[1]) {
        o[0] = *reinterpret_cast<const float2*>(p);
    }
};

// Rows of bf16 keys and values with d = 128 can be staged by TMA tensor copies
// with 128-byte swizzle (the SW kernels): a parent group of C rows (C a multiple of
// 16) fills its slot as [half][C rows][128 B], half 0 holding dims 0-63 and half 1
// dims 64-127, and the 16-byte chunk j of row r stored at chunk j ^ (r mod 8).  The
// rows of an 8-row tile then fall in 8 different bank groups for ldmatrix.
template <typename T, int D>
constexpr bool kSwzCapable = false;
template <>
constexpr bool kSwzCapable<__nv_bfloat16, 128> = true;

// Byte offset of 16-byte chunk `chunk` (0..7) of half `half` of row `row` in a slot.
__device__ __forceinline__ uint32_t swz_off(int half, int row, int chunk, int C) {
    return (uint32_t)(half * C * 128 + row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ----------------------------------------------------------------------------
// shared-memory layout of the select/attend kernels
// ----------------------------------------------------------------------------
struct Smem {
    size_t qsm, rc4, s, key, nodes, flag, par, mkey, hist, gs, misc, geo, bars, ring, red, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Words of the cluster selection's global histogram held by each of `csize` CTAs
// (a multiple of 4, so a 16-byte group of words has one owner).
__host__ __device__ inline int gs_words(int csize) {
    return ((1024 + csize - 1) / csize + 3) & ~3;
}
constexpr int kSelCand = 384;   // candidates of the cluster selection's boundary bin

// CH: entries per CTA chunk; NA: largest list (C*k), 0 at level 0 (no selection);
// gsw: the CTA's slice of the cluster histogram (0 at level 0); ring_bytes: the
// warps' staging slots.  The reduction buffer reuses the ring once every block has
// been consumed.  mkey holds the exchanged keys of the heavy-tie path, or the
// published and gathered candidates of the cluster selection.
__host__ __device__ inline Smem smem_layout(int G, int D, int CH, int k, int C, int NA, int gsw,
                                            int nslot, int ring_bytes) {
    Smem L;
    size_t o = 0;
    L.qsm = o;   o = align16(o + sizeof(float) * G * D);
    L.rc4 = o;   o = align16(o + sizeof(float2) * C * (D / 2));
    L.s = o;     o = align16(o + sizeof(float) * G * CH);
    L.key = o;   o = align16(o + sizeof(uint32_t) * CH);
    L.nodes = o; o = align16(o + sizeof(int) * CH);
    L.flag = o;  o = align16(o + sizeof(unsigned char) * CH);
    L.par = o;   o = align16(o + sizeof(int) * 3 * k);   // S^(l) in buffer l mod 3
    const int mk = NA > 0 && NA < 4 * kSelCand ? 4 * kSelCand : NA;
    L.mkey = o;  o = align16(o + sizeof(uint32_t) * mk);
    L.hist = o;  o = align16(o + sizeof(uint32_t) * 1024);   // >= kSelBins / 2, radix 512
    L.gs = o;    o = align16(o + sizeof(uint32_t) * gsw);
    L.misc = o;  o = align16(o + sizeof(int) * 128);
    L.geo = o;   o = align16(o + sizeof(int) * 4 * kMaxLevels);   // per-level list geometry
    L.bars = o;  o = align16(o + sizeof(uint64_t) * kWarps * 2);
    o = (o + 1023) & ~size_t(1023);   // swizzled slots need 1024-byte alignment
    L.ring = o;
    L.red = o;
    // the value reduction, or the merge's weights, (m, l) and one slot column
    size_t red_bytes = sizeof(float) * kWarps * G * (D + 1);
    const size_t merge_bytes = sizeof(float) * (size_t)(3 * G + 1) * nslot;
    if (merge_bytes > red_bytes) red_bytes = merge_bytes;
    o += (size_t)ring_bytes > red_bytes ? (size_t)ring_bytes : red_bytes;
    L.total = o;
    return L;
}

// misc slots
enum { kMiscDigit = 0, kMiscAbove = 1, kMiscCount = 2, kMiscScan = 4 /* kWarps+1 */,
       kMiscFloat = 16 /* 2*G floats */, kMiscLast = 40, kMiscN = 41,
       // cluster selection: published counts, gathered counts (one per CTA), scalars
       kMiscPubC = 48, kMiscPubA = 49, kMiscTk = 53, kMiscTj = 54, kMiscGC = 64 /* 16 */,
       kMiscGA = 80 /* 16 */,
       kMiscWA = 104 /* kWarps: keys above the boundary bin per slice */,
       kMiscBase = 112 /* kWarps: first rank of each slice */,
       kMiscFailed = 100 /* a bounded wait of this CTA gave up */ };

// Split cluster barrier: arrive (release) and, later, wait (acquire); every thread
// of every CTA of the cluster takes both, in this order.
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
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
    if (threadIdx.x < 32) {
        const int w = threadIdx.x < kWarps ? scratch[threadIdx.x] : 0;
        int inc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, inc, o);
            if (threadIdx.x >= o) inc += y;
        }
        if (threadIdx.x < kWarps) scratch[threadIdx.x] = inc - w;
        if (threadIdx.x == kWarps - 1) scratch[kWarps] = inc;
    }
    __syncthreads();
    const int off = scratch[warp] + x - v;
    total = scratch[kWarps];
    __syncthreads();
    return off;
}

// Exact threshold of the top K of n keys (0 < K < n): T is the K-th largest key,
// need_eq how many keys equal to T belong to the top K, cnt_eq how many keys equal
// T.  MSB-first radix select over 8-bit digits; histogram updates are aggregated
// per warp (__match_any_sync) because the leading digits of float keys fall into
// a few bins.  hist: 512 words (two alternating 256-bin histograms).
__device__ void block_threshold(const uint32_t* keys, int n, int K, uint32_t* hist, int* misc,
                                uint32_t& T, int& need_eq, int& cnt_eq, int stride = 1) {
    const int tid = threadIdx.x, lane = tid & 31;
    for (int i = tid; i < 512; i += kThreads) hist[i] = 0u;
    __syncthreads();
    uint32_t prefix = 0, mask = 0;
    int rem = K, cnt = 0;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        uint32_t* h = hist + (pass & 1) * 256;
        uint32_t* hn = hist + ((pass + 1) & 1) * 256;
        for (int i0 = 0; i0 < n; i0 += kThreads) {
            const int i = i0 + tid;
            const uint32_t kk = i < n ? keys[i * stride] : 0u;
            const bool in = i < n && (kk & mask) == prefix;
            const uint32_t dig = in ? ((kk >> shift) & 255u) : 256u;
            const unsigned same = __match_any_sync(kFull, dig);
            if (in && lane == __ffs(same) - 1) atomicAdd(&h[dig], (uint32_t)__popc(same));
        }
        if (pass > 0)
            for (int i = tid; i < 256; i += kThreads) hn[i] = 0u;   // last read by the previous scan
        __syncthreads();
        if (tid < 32) {
            uint32_t c8[8];
            uint32_t tot = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                c8[u] = h[255 - 8 * lane - u];
                tot += c8[u];
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
                    if (run + c8[u] >= (uint32_t)rem) {
                        misc[kMiscDigit] = 255 - 8 * lane - u;
                        misc[kMiscAbove] = (int)run;
                        misc[kMiscCount] = (int)c8[u];
                        break;
                    }
                    run += c8[u];
                }
            }
        }
        __syncthreads();
        const int digit = misc[kMiscDigit];
        rem -= misc[kMiscAbove];
        cnt = misc[kMiscCount];
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
    }
    __syncthreads();
    T = prefix;
    need_eq = rem;
    cnt_eq = cnt;
}

// Selection ranks of n keys in list order given the threshold: selected = key > T,
// or key == T among the first need_eq such keys.  Calls fn(i, rank) for every
// selected item i in [lo, hi).  Returns the number of selected items.
template <typename Fn>
__device__ int block_select_ranks(const uint32_t* keys, int n, uint32_t T, int need_eq, int cnt_eq,
                                  int lo, int hi, int* misc, Fn fn, int stride = 1) {
    const int ipt = (n + kThreads - 1) / kThreads;
    const int i0 = threadIdx.x * ipt, i1 = min(n, i0 + ipt);
    const bool all_eq = (cnt_eq == need_eq);
    int eq_rank = 0, tot;
    if (!all_eq) {
        int ceq = 0;
        for (int i = i0; i < i1; ++i) ceq += (keys[i * stride] == T);
        eq_rank = block_excl_scan(ceq, misc + kMiscScan, tot);
    }
    int csel = 0;
    {
        int er = eq_rank;
        for (int i = i0; i < i1; ++i) {
            const uint32_t kk = keys[i * stride];
            bool sel = kk > T;
            if (kk == T) { sel = all_eq || er < need_eq; ++er; }
            csel += sel;
        }
    }
    int r = block_excl_scan(csel, misc + kMiscScan, tot);
    {
        int er = eq_rank;
        for (int i = i0; i < i1; ++i) {
            const uint32_t kk = keys[i * stride];
            bool sel = kk > T;
            if (kk == T) { sel = all_eq || er < need_eq; ++er; }
            if (sel) {
                if (i >= lo && i < hi) fn(i, r);
                ++r;
            }
        }
    }
    return tot;
}

// Same ranks for a list of at most 16 * kThreads keys: each thread takes a run of
// a multiple of 4 consecutive keys, read once with 16-byte loads into registers
// (runs may read up to 15 words past n; those words are never counted).
template <typename Fn>
__device__ void block_select_ranks_short(const uint32_t* keys, int n, uint32_t T, int need_eq,
                                         int cnt_eq, int lo, int hi, int* misc, Fn fn) {
    constexpr int MAXI = 16;
    const int ipt = (((n + kThreads - 1) / kThreads) + 3) & ~3;
    const int i0 = threadIdx.x * ipt;
    uint32_t kv[MAXI];
#pragma unroll
    for (int u = 0; u < MAXI; u += 4) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (u < ipt && i0 + u < n) w = *reinterpret_cast<const uint4*>(keys + i0 + u);
        kv[u] = w.x; kv[u + 1] = w.y; kv[u + 2] = w.z; kv[u + 3] = w.w;
    }
    const bool all_eq = (cnt_eq == need_eq);
    int tot, eq_rank = 0;
    if (!all_eq) {
        int ceq = 0;
#pragma unroll
        for (int u = 0; u < MAXI; ++u) ceq += (u < ipt && i0 + u < n && kv[u] == T);
        eq_rank = block_excl_scan(ceq, misc + kMiscScan, tot);
    }
    uint32_t selm = 0;
    int er = eq_rank;
#pragma unroll
    for (int u = 0; u < MAXI; ++u) {
        if (u < ipt && i0 + u < n) {
            bool sel = kv[u] > T;
            if (kv[u] == T) { sel = all_eq || er < need_eq; ++er; }
            selm |= (uint32_t)sel << u;
        }
    }
    int r = block_excl_scan(__popc(selm), misc + kMiscScan, tot);
    while (selm) {
        const int u = __ffs(selm) - 1;
        selm &= selm - 1;
        const int i = i0 + u;
        if (i >= lo && i < hi) fn(i, r);
        ++r;
    }
}

// Exact top-K (0 < K < M) of the M keys of mkey in list order; calls mark(j, rank)
// for every selected list position j in [lo, hi), rank = its position among the
// selected in list order.  One pass histograms the leading kSelBits bits of every
// key (two 16-bit bin counts per word); a suffix count over the bins finds the bin
// that holds the K-th largest key.  The keys of that bin (usually about a hundred)
// are ranked exactly against each other (key descending, position ascending); the
// one ranked K - above - 1 is the threshold T.  The ranks in list order then follow
// from T.  A bin larger than kSelCand keys (heavy ties) uses the radix select.
// hist: kSelBins / 2 words.
constexpr int kSelBits = 11;
constexpr int kSelBins = 1 << kSelBits;
enum { kMiscCand = 3, kMiscT = 13, kMiscNeedEq = 14, kMiscCntEq = 15 };

// Given each thread's BPT bin counts in descending bin order (thread t owns bins
// kSelBins-1-BPT*t-u), finds the bin holding the K-th largest key: misc[kMiscDigit]
// = the bin, misc[kMiscAbove] = keys in higher bins, misc[kMiscCount] = its keys.
template <int BPT>
__device__ __forceinline__ void find_boundary_bin(const uint32_t (&cnt8)[BPT], int K, int* misc) {
    int tot = 0;
#pragma unroll
    for (int u = 0; u < BPT; ++u) tot += (int)cnt8[u];
    int all;
    const int excl = block_excl_scan(tot, misc + kMiscScan, all);
    if (excl < K && K <= excl + tot) {
        int run = excl;
#pragma unroll
        for (int u = 0; u < BPT; ++u) {
            if (run + (int)cnt8[u] >= K) {
                misc[kMiscDigit] = kSelBins - 1 - BPT * (int)threadIdx.x - u;
                misc[kMiscAbove] = run;
                misc[kMiscCount] = (int)cnt8[u];
                break;
            }
            run += (int)cnt8[u];
        }
    }
    __syncthreads();
}

template <typename Fn>
__device__ void select_topk(uint32_t* mkey, int M, int K, uint32_t* hist, int* misc, int lo, int hi,
                            Fn mark) {
    constexpr int SH = 32 - kSelBits;
    constexpr int BPT = kSelBins / kThreads;   // bins per thread
    const int tid = threadIdx.x;
    for (int i = tid; i < kSelBins / 2; i += kThreads) hist[i] = 0u;
    if (tid == 0) misc[kMiscCand] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < M; i0 += kThreads) {
        const int i = i0 + tid;
        if (i < M) {
            const uint32_t dig = mkey[i] >> SH;
            atomicAdd(&hist[dig >> 1], 1u << (16 * (dig & 1)));
        }
    }
    __syncthreads();
    // thread t owns bins kSelBins-1-BPT*t-u, u = 0..BPT-1 (descending key order)
    uint32_t cnt8[BPT];
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
        const int bin = kSelBins - 1 - BPT * tid - u;
        cnt8[u] = (hist[bin >> 1] >> (16 * (bin & 1))) & 0xFFFFu;
    }
    find_boundary_bin<BPT>(cnt8, K, misc);
    const uint32_t bd = (uint32_t)misc[kMiscDigit];
    const int need = K - misc[kMiscAbove];   // keys to take from bin bd: 1..cnt
    const int cnt = misc[kMiscCount];
    uint32_t T;
    int need_eq, cnt_eq;
    if (cnt <= kSelCand) {
        // the bin's (key, position) pairs, in any order, into the free histogram
        // two passes without atomics: each warp counts the bin's keys in its slice of
        // the list, then writes them after the counts of the warps before it
        uint2* cand = reinterpret_cast<uint2*>(hist);
        const int lane = tid & 31, warp = tid >> 5;
        const int per = (((M + kWarps - 1) / kWarps) + 31) & ~31;
        const int w0 = warp * per, w1 = min(M, w0 + per);
        int wcnt = 0;
        for (int i = w0 + lane; i - lane < w1; i += 32) {
            const bool in = i < w1 && (mkey[i] >> SH) == bd;
            wcnt += __popc(__ballot_sync(kFull, in));
        }
        if (lane == 0) misc[kMiscScan + warp] = wcnt;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; ++w) base += misc[kMiscScan + w];
        for (int i = w0 + lane; i - lane < w1; i += 32) {
            const uint32_t kk = i < w1 ? mkey[i] : 0u;
            const bool in = i < w1 && (kk >> SH) == bd;
            const unsigned bal = __ballot_sync(kFull, in);
            if (in) cand[base + __popc(bal & ((1u << lane) - 1u))] = make_uint2(kk, (uint32_t)i);
            base += __popc(bal);
        }
        __syncthreads();
        for (int c = tid; c < cnt; c += kThreads) {
            const uint2 me = cand[c];
            int gt = 0, eq = 0, eq_before = 0;
            int j = 0;
            for (; j + 8 <= cnt; j += 8) {   // eight loads in flight per step
                uint4 o[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) o[u] = *reinterpret_cast<const uint4*>(cand + j + 2 * u);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    gt += (o[u].x > me.x) + (o[u].z > me.x);
                    eq += (o[u].x == me.x) + (o[u].z == me.x);
                    eq_before += ((o[u].x == me.x) & (o[u].y < me.y)) + ((o[u].z == me.x) & (o[u].w < me.y));
                }
            }
            for (; j < cnt; ++j) {
                const uint2 o = cand[j];
                gt += o.x > me.x;
                eq += o.x == me.x;
                eq_before += (o.x == me.x) & (o.y < me.y);
            }
            if (gt + eq_before == need - 1) {
                misc[kMiscT] = (int)me.x;
                misc[kMiscNeedEq] = need - gt;
                misc[kMiscCntEq] = eq;
            }
        }
        __syncthreads();
        T = (uint32_t)misc[kMiscT];
        need_eq = misc[kMiscNeedEq];
        cnt_eq = misc[kMiscCntEq];
    } else {
        block_threshold(mkey, M, K, hist, misc, T, need_eq, cnt_eq);
    }
    if (M <= 16 * kThreads)
        block_select_ranks_short(mkey, M, T, need_eq, cnt_eq, lo, hi, misc, mark);
    else
        block_select_ranks(mkey, M, T, need_eq, cnt_eq, lo, hi, misc, mark);
}

// ----------------------------------------------------------------------------
// Exact top-K (0 < K < M) over a cluster.  The M keys of a list are spread over the
// csize CTAs of the cluster: CTA r holds, in its `key` array, the n_loc keys of
// the contiguous slice that starts at list position j0 = r * chunk.  Every CTA
// finds the same threshold (T, jT), the K-th entry in the order (key descending,
// list position ascending); entry j is selected when key > T, or key == T and
// j <= jT.  mark(j, rank) is called for this CTA's selected entries, rank = the
// entry's position among all selected entries in list order.
//  1. Each CTA histograms the leading kSelBits bits of its keys (lh, zeroed by the
//     caller) and adds its non-zero words into the global histogram, whose words
//     are spread over the CTAs (gsw words each, zeroed by the caller before a
//     cluster arrive that the caller's wait completed): distributed shared memory
//     atomics.  A cluster barrier follows.
//  2. Every CTA reads the global histogram (one 16-byte remote load per thread) and
//     finds the bin bd holding the K-th key with warp scans.  A bin of more than
//     kSelCand keys (heavy ties) returns false here, in every CTA alike, and the
//     caller runs the exchange-and-select path instead.
//  3. Each warp takes a slice of the CTA's keys in list order, publishes the (key,
//     position) pairs of its keys in bd and counts its keys above bd; after a
//     second barrier every CTA gathers all candidates and their counts.  The
//     caller arrives on the cluster barrier once its remote reads and its stores
//     of S are done, and waits on it at the end of the level.
//  4. Warp 0 finds the threshold from a 256-bin histogram of the candidates' next 8
//     key bits and an exact rank of the few candidates in the boundary sub-bin,
//     and the rank at which each slice starts: the selected entries of the CTAs
//     before this one (their counts above bd plus their selected candidates) and
//     of the slices before it.
//  5. Each warp ranks its slice's selected entries with ballots.
// ----------------------------------------------------------------------------
template <typename Fn>
__device__ bool cluster_select(const uint32_t* key, int n_loc, int j0, int K, int csize, int crank,
                               int gsw, uint32_t* lh, uint32_t* gs, uint2* pub, uint2* all,
                               int* misc, Fn mark) {
    constexpr int SH = 32 - kSelBits;
    constexpr int BPT = kSelBins / kThreads;
    constexpr int W = kSelBins / 2;   // histogram words, two 16-bit counts each
    static_assert(W == 4 * kThreads && kThreads == 256, "one 16-byte word group per thread");
    cg::cluster_group cluster = cg::this_cluster();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // 1. local histogram, then its non-zero words into their owners' slices
    for (int i = tid; i < n_loc; i += kThreads) {
        const uint32_t dig = key[i] >> SH;
        atomicAdd(&lh[dig >> 1], 1u << (16 * (dig & 1)));
    }
    __syncthreads();
    {
        const uint4 w = *reinterpret_cast<const uint4*>(lh + 4 * tid);
        if (w.x | w.y | w.z | w.w) {
            uint32_t* dst = cluster.map_shared_rank(gs, (4 * tid) / gsw) + (4 * tid) % gsw;
            if (w.x) atomicAdd(dst, w.x);
            if (w.y) atomicAdd(dst + 1, w.y);
            if (w.z) atomicAdd(dst + 2, w.z);
            if (w.w) atomicAdd(dst + 3, w.w);
        }
    }
    cluster.sync();

    // 2. the global histogram: thread t owns bins kSelBins-1-BPT*t-u, the words
    //    from W-4-4t (bin b: word b/2, high half when b is odd).  Keys above a
    //    thread's bins: a warp scan plus the totals of the warps before it.
    {
        const int w0 = W - 4 - 4 * tid;
        const uint4 w = *reinterpret_cast<const uint4*>(cluster.map_shared_rank(gs, w0 / gsw) + w0 % gsw);
        const uint32_t ws[4] = {w.w, w.z, w.y, w.x};
        uint32_t cnt8[BPT];
        int tot = 0;
#pragma unroll
        for (int u = 0; u < BPT; ++u) {
            cnt8[u] = (ws[u >> 1] >> (16 * (1 - (u & 1)))) & 0xFFFFu;
            tot += (int)cnt8[u];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) misc[kMiscScan + warp] = incl;
        __syncthreads();
        int run = incl - tot;
        for (int ww = 0; ww < warp; ++ww) run += misc[kMiscScan + ww];
        if (run < K && K <= run + tot) {
#pragma unroll
            for (int u = 0; u < BPT; ++u) {
                if (run < K && K <= run + (int)cnt8[u]) {
                    misc[kMiscDigit] = kSelBins - 1 - BPT * tid - u;
                    misc[kMiscAbove] = run;
                    misc[kMiscCount] = (int)cnt8[u];
                }
                run += (int)cnt8[u];
            }
        }
        __syncthreads();
    }
    const uint32_t bd = (uint32_t)misc[kMiscDigit];
    const int cnt = misc[kMiscCount];
    if (cnt > kSelCand) return false;
    const int need = K - misc[kMiscAbove];   // 1..cnt
    const unsigned lt = (1u << lane) - 1u;

    // 3. this CTA's candidates and its count above bd, for the other CTAs; each warp
    //    takes a slice of the keys in list order and counts its keys above bd
    const int per = (((n_loc + kWarps - 1) / kWarps) + 31) & ~31;
    const int s0 = warp * per, s1 = min(n_loc, s0 + per);
    {
        int wab = 0;
        for (int i = s0 + lane; i - lane < s1; i += 32) {
            const bool v = i < s1;
            const uint32_t kk = v ? key[i] : 0u;
            const uint32_t dig = kk >> SH;
            const bool in = v && dig == bd;
            wab += __popc(__ballot_sync(kFull, v && dig > bd));
            const unsigned bal = __ballot_sync(kFull, in);
            if (bal) {
                int base = 0;
                if (lane == 0) base = atomicAdd(&misc[kMiscPubC], __popc(bal));
                base = __shfl_sync(kFull, base, 0);
                if (in) pub[base + __popc(bal & lt)] = make_uint2(kk, (uint32_t)(j0 + i));
            }
        }
        if (lane == 0) {
            misc[kMiscWA + warp] = wab;
            if (wab) atomicAdd(&misc[kMiscPubA], wab);
        }
    }
    cluster.sync();
    if (tid < csize) {
        const int* rm = cluster.map_shared_rank(misc, tid);
        misc[kMiscGC + tid] = rm[kMiscPubC];
        misc[kMiscGA + tid] = rm[kMiscPubA];
    }
    uint32_t* sub = lh;   // free since step 1: sub-bin counts, then the members
    sub[tid] = 0u;
    __syncthreads();
    // 4. every CTA's candidates, with a histogram of their next 8 key bits
    for (int idx = tid; idx < cnt; idx += kThreads) {
        int r = 0, off = 0;
        while (r < csize - 1 && idx >= off + misc[kMiscGC + r]) off += misc[kMiscGC + r++];
        const uint2 c = cluster.map_shared_rank(pub, r)[idx - off];
        all[idx] = c;
        atomicAdd(&sub[(c.x >> (SH - 8)) & 255u], 1u);
    }
    __syncthreads();

    // 5. warp 0: the threshold (the sub-bin holding the need-th candidate, then an
    //    exact rank of its members) and the rank at which each warp's slice starts
    // (rolled loops over the candidates in shared memory: this code runs once per
    // level in one warp, and its instructions often arrive cold)
    if (warp == 0) {
        // lane l holds sub-bins [8l, 8l + 8); higher lanes hold higher keys
        const uint4 h0 = *reinterpret_cast<const uint4*>(sub + 8 * lane);
        const uint4 h1 = *reinterpret_cast<const uint4*>(sub + 8 * lane + 4);
        const uint32_t h8[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
        uint32_t t8 = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) t8 += h8[u];
        uint32_t suf = t8;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(kFull, suf, o);
            if (lane + o < 32) suf += y;
        }
        uint32_t srun = suf - t8;
        const unsigned hit = __ballot_sync(kFull, srun < (uint32_t)need && (uint32_t)need <= suf);
        const int src = hit ? __ffs(hit) - 1 : 0;
        int sbl = 0, sba = 0;
        bool found = false;
#pragma unroll
        for (int u = 7; u >= 0; --u) {
            if (!found) {
                if (srun + h8[u] >= (uint32_t)need) { found = true; sbl = 8 * lane + u; sba = (int)srun; }
                else srun += h8[u];
            }
        }
        const uint32_t sb = (uint32_t)__shfl_sync(kFull, sbl, src);
        const int need2 = need - __shfl_sync(kFull, sba, src);
        __syncwarp();   // the sub-bin counts are read: their words take the members
        uint2* memb = reinterpret_cast<uint2*>(sub);
        int nm = 0;
#pragma unroll 1
        for (int i0 = 0; i0 < cnt; i0 += 32) {
            const int idx = i0 + lane;
            const uint2 c = idx < cnt ? all[idx] : make_uint2(0u, 0u);
            const bool in = idx < cnt && ((c.x >> (SH - 8)) & 255u) == sb;
            const unsigned bal = __ballot_sync(kFull, in);
            if (in) memb[nm + __popc(bal & lt)] = c;
            nm += __popc(bal);
        }
        __syncwarp();
        uint32_t Tk = 0u, Tj = 0u;
#pragma unroll 1
        for (int mi = lane; mi - lane < nm; mi += 32) {
            const uint2 me = mi < nm ? memb[mi] : make_uint2(0u, 0u);
            int gt = 0;
            for (int o = 0; o < nm; ++o) {
                const uint2 xo = memb[o];
                gt += (xo.x > me.x || (xo.x == me.x && xo.y < me.y)) ? 1 : 0;
            }
            const unsigned hb = __ballot_sync(kFull, mi < nm && gt == need2 - 1);
            if (hb) {
                const int sl = __ffs(hb) - 1;
                Tk = __shfl_sync(kFull, me.x, sl);
                Tj = __shfl_sync(kFull, me.y, sl);
            }
        }
        // selected candidates before this CTA, and in each slice of this CTA (added
        // into kMiscWA, which holds each slice's keys above bd)
        int before = 0;
#pragma unroll 1
        for (int idx = lane; idx < cnt; idx += 32) {
            const uint2 c = all[idx];
            const bool sel = c.x > Tk || (c.x == Tk && c.y <= Tj);
            const int li = (int)c.y - j0;
            before += (sel && li < 0) ? 1 : 0;
            if (sel && li >= 0 && li < n_loc) atomicAdd(&misc[kMiscWA + li / per], 1);
        }
        before = (int)__reduce_add_sync(kFull, (unsigned)before);
        const int above_before =
            (int)__reduce_add_sync(kFull, (unsigned)(lane < crank ? misc[kMiscGA + lane] : 0));
        __syncwarp();
        if (lane == 0) {
            int base = above_before + before;
            for (int ww = 0; ww < kWarps; ++ww) {
                misc[kMiscBase + ww] = base;
                base += misc[kMiscWA + ww];
            }
            misc[kMiscTk] = (int)Tk;
            misc[kMiscTj] = (int)Tj;
        }
    }
    __syncthreads();
    const uint32_t T = (uint32_t)misc[kMiscTk], jT = (uint32_t)misc[kMiscTj];

    // 6. this warp's selected entries, ranked in list order
    int r = misc[kMiscBase + warp];
    for (int i = s0 + lane; i - lane < s1; i += 32) {
        const bool v = i < s1;
        const uint32_t kk = v ? key[i] : 0u;
        const bool sel = v && (kk > T || (kk == T && (uint32_t)(j0 + i) <= jT));
        const unsigned bal = __ballot_sync(kFull, sel);
        if (sel) mark(j0 + i, r + __popc(bal & lt));
        r += __popc(bal);
    }
    return true;
}

// ----------------------------------------------------------------------------
// L2 prefetch: a bulk asynchronous request that holds no registers or shared
// memory; the rows are in L2 when the loads reach them.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}


// 16 loaded bytes as VEC/2 fp32 pairs (elements 2i, 2i+1).
template <typename T>
__device__ __forceinline__ void unpack_pairs(const uint4& w, float2* out);
template <>
__device__ __forceinline__ void unpack_pairs<float>(const uint4& w, float2* out) {
    out[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
    out[1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
}
template <>
__device__ __forceinline__ void unpack_pairs<__nv_bfloat16>(const uint4& w, float2* out) {
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        out[i] = make_float2(__uint_as_float(x[i] << 16), __uint_as_float(x[i] & 0xffff0000u));
}

// Reduce-scatter of N register values over the KG lanes (a power of two) of a
// key group: afterwards v[0 .. N/KG) of lane c8 hold the group sums of original
// indices [c8*N/KG, (c8+1)*N/KG).  Each stage halves the live values: lanes whose
// stage bit is set keep the upper half and send the lower one.
template <int N, int KG>
__device__ __forceinline__ void reduce_scatter(float (&v)[N], int c8) {
#pragma unroll
    for (int o = KG / 2, n = N; o >= 1; o >>= 1, n >>= 1) {
        const bool up = (c8 & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float lo = v[i], hi = v[i + n / 2];
            const float send = up ? lo : hi;
            const float keep = up ? hi : lo;
            v[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
    }
}

// ----------------------------------------------------------------------------
// Per-warp ring of parent-group blocks (C rows of K or V) staged in shared memory
// by TMA bulk copies.  Block q of a warp goes to slot q % nsw; a slot is re-armed
// only after the warp has consumed its previous block, so each warp keeps nsw
// blocks in flight without holding registers.
// ----------------------------------------------------------------------------
struct WarpRing {
    unsigned char* slots;
    uint64_t* bars;
    int nsw, slot_bytes;
    uint32_t* status;
    volatile int* failed;   // CTA-wide: set once any wait of the CTA has given up
};

// Issue block q: rows [first, first + cnt) of a table with row stride rs.  One lane.
template <typename T, int D>
__device__ __forceinline__ void ring_issue(const WarpRing& R, int q, const T* base, int64_t rs,
                                           int64_t first, int cnt) {
    constexpr uint32_t kRow = D * sizeof(T);
    const int s = q % R.nsw;
    unsigned char* dst = R.slots + (size_t)s * R.slot_bytes;
    mbar_expect_tx(&R.bars[s], (uint32_t)cnt * kRow);
    if (rs == D) {
        bulk_g2s(dst, base + first * D, (uint32_t)cnt * kRow, &R.bars[s]);
    } else {
        for (int r = 0; r < cnt; ++r) bulk_g2s(dst + r * kRow, base + (first + r) * rs, kRow, &R.bars[s]);
    }
}

// Issue block q from a tensor map: the C rows from `first` of KV head h of sequence
// b as two swizzled boxes (dims 0-63 and 64-127).  Rows past the table arrive as
// zeros; the full box is always delivered.  One lane.
__device__ __forceinline__ void ring_issue_map(const WarpRing& R, int q, const CUtensorMap* map,
                                               int64_t first, int h, int b, int C) {
    const int s = q % R.nsw;
    unsigned char* dst = R.slots + (size_t)s * R.slot_bytes;
    mbar_expect_tx(&R.bars[s], (uint32_t)C * 256u);
#pragma unroll
    for (int half = 0; half < 2; ++half)
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
            "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst + half * C * 128)),
            "l"(reinterpret_cast<uint64_t>(map)), "r"(half * 64), "r"((int)first), "r"(h), "r"(b),
            "r"(smem_u32(&R.bars[s]))
            : "memory");
}

// Wait (bounded) for block q; all lanes of the warp.  Once a wait of the CTA has
// given up (the status word holds the timeout), later waits are short: the unit's
// output is then garbage anyway, and the CTA must reach its exit soon rather than
// spend a full limit on every remaining block.
__device__ __forceinline__ const unsigned char* ring_wait(const WarpRing& R, int q) {
    const int s = q % R.nsw;
    const uint32_t polls = *R.failed ? kWaitPollsAfterFail : kWaitPolls;
    if (!mbar_wait_bounded(&R.bars[s], (uint32_t)((q / R.nsw) & 1), R.status, polls)) *R.failed = 1;
    return R.slots + (size_t)s * R.slot_bytes;
}

// ----------------------------------------------------------------------------
// Scores of one parent group staged in shared memory: row c of blk is the key of
// list entry jb + c (c < nch).  s[g][r] = scale * <R(p_q - jb) q_g, R(c) K>, the
// order-preserving key of the mean over heads, and the node index first + c,
// at r = jb - j0 + c.  LPK lanes share a key, each rotating and multiplying its
// PPL pairs of both halves with packed fp32x2 arithmetic; the U keys of a lane
// are computed branch-free so their chains interleave, and the partial dot
// products are combined by a reduce-scatter over the LPK lanes.
// ----------------------------------------------------------------------------
template <typename T, int D, int G, bool WITH_KEY, bool SW>
__device__ __forceinline__ void score_parent(const unsigned char* blk, int C, int jb,
                                             const float4 (&qcs)[Shape<T, D>::CPL], int j0, int nch,
                                             int64_t first, const float4* rc4, const float* qsm,
                                             float scale, float* s, uint32_t* key, int* nodes,
                                             int CH) {
    using S = Shape<T, D>;
    constexpr int LPK = S::LPK, PPL = S::PPL, CPL = S::CPL, KPW = S::KPW, H = D / 2;
    constexpr int kRow = D * (int)sizeof(T);
    constexpr int kHalf = H * (int)sizeof(T);
    constexpr int U = 4;                       // keys per lane per batch
    constexpr int NV = U * G;                  // values reduced over a key's lanes
    constexpr int R = NV / LPK;                // values per lane after reduce-scatter
    constexpr bool RS = (NV % LPK == 0) && (R >= 1) && (G % (R > 0 ? R : 1) == 0);
    const int lane = threadIdx.x & 31;
    const int cl = lane % LPK, kg = lane / LPK;
    const int off = cl * PPL * (int)sizeof(T);   // byte offset of the lane's pairs in a half
    // the query heads rotated by R(p_q - jb), the lane's couples only; qcs holds the
    // lane's couples of that rotation, loaded by the caller a group ahead
    float2 qlo[G][CPL], qhi[G][CPL];
    {
        const float4* q4 = reinterpret_cast<const float4*>(qsm) + cl * CPL;
#pragma unroll
        for (int w = 0; w < CPL; ++w) {
            const float4 cs = qcs[w];   // (cos v, sin v, cos v+1, sin v+1)
            const float2 co = make_float2(cs.x, cs.z);
            const float2 si = make_float2(cs.y, cs.w);
            const float2 ns = make_float2(-cs.y, -cs.w);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float4 xq = q4[g * (H / 2) + w];   // (low v, low v+1, high v, high v+1)
                const float2 x1 = make_float2(xq.x, xq.y);
                const float2 x2 = make_float2(xq.z, xq.w);
                qlo[g][w] = __ffma2_rn(x2, ns, __fmul2_rn(x1, co));
                qhi[g][w] = __ffma2_rn(x1, si, __fmul2_rn(x2, co));
            }
        }
    }
    // swizzled slots: row cb + u*KPW + kg (cb a multiple of KPW*U = 8, so the row's
    // swizzle phase is u*KPW + kg) keeps the lane's chunk cl/2 at chunk
    // (cl/2 ^ kg) ^ (u*KPW); the slot always holds C rows, so rows past nch are read
    // too and their results dropped
    static_assert(!SW || (KPW == 2 && U == 4), "swizzle phases of the scoring rows");
    const uint32_t ch0 = (uint32_t)((cl >> 1) ^ kg);
    const uint32_t rb0 = (uint32_t)kg * 128u + (uint32_t)(cl & 1) * 8u;
    for (int cb = 0; cb < nch; cb += KPW * U) {
        float v[NV];
        // a key past the group reads row 0 (always staged); its value is never stored
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = cb + u * KPW + kg;
            const int cr = SW ? c : (c < nch ? c : 0);
            float2 kl[CPL], kh[CPL];
            if constexpr (SW) {
                // the lane's 8 bytes: half of 16-byte chunk cl / 2 of each half row
                const unsigned char* row =
                    blk + (uint32_t)cb * 128u + rb0 + (uint32_t)(u * KPW) * 128u + ((ch0 ^ (uint32_t)(u * KPW)) << 4);
                PairLoad<T, PPL>::get(row, kl);
                PairLoad<T, PPL>::get(row + C * 128, kh);
            } else {
                const unsigned char* row = blk + cr * kRow;
                PairLoad<T, PPL>::get(row + off, kl);
                PairLoad<T, PPL>::get(row + kHalf + off, kh);
            }
            const float4* rc = rc4 + cr * (H / 2) + cl;
            float2 acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < CPL; ++w) {
                const float4 cs = rc[w * LPK];   // (cos v, cos v+1, sin v, sin v+1) of c * theta
                const float2 co = make_float2(cs.x, cs.y);
                const float2 si = make_float2(cs.z, cs.w);
                const float2 ns = make_float2(-cs.z, -cs.w);
                const float2 ka = __ffma2_rn(kh[w], ns, __fmul2_rn(kl[w], co));
                const float2 kb = __ffma2_rn(kl[w], si, __fmul2_rn(kh[w], co));
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    acc[g] = __ffma2_rn(qlo[g][w], ka, acc[g]);
                    acc[g] = __ffma2_rn(qhi[g][w], kb, acc[g]);
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) v[u * G + g] = acc[g].x + acc[g].y;
        }
        if constexpr (RS) {
            reduce_scatter<NV, LPK>(v, cl);
            const int u = (cl * R) / G, g0 = (cl * R) % G;
            const int c = cb + u * KPW + kg;
            float imp = 0.f;
#pragma unroll
            for (int i = 0; i < R; ++i) imp += v[i];
#pragma unroll
            for (int o = 1; o < G / R; o <<= 1) imp += __shfl_xor_sync(kFull, imp, o);
            if (c < nch) {
                const int r = jb - j0 + c;
#pragma unroll
                for (int i = 0; i < R; ++i) s[(g0 + i) * CH + r] = v[i] * scale;
                if (g0 == 0) {
                    nodes[r] = (int)(first + c);
                    if (WITH_KEY) key[r] = ordered_key(imp * scale * (1.0f / G));
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < NV; ++i)
#pragma unroll
                for (int o = 1; o < LPK; o <<= 1) v[i] += __shfl_xor_sync(kFull, v[i], o);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = cb + u * KPW + kg;
                if (c < nch && cl == 0) {
                    const int r = jb - j0 + c;
                    float imp = 0.f;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        s[g * CH + r] = v[u * G + g] * scale;
                        imp += v[u * G + g];
                    }
                    nodes[r] = (int)(first + c);
                    if (WITH_KEY) key[r] = ordered_key(imp * scale * (1.0f / G));
                }
            }
        }
    }
}

// Unrotated query heads of one KV head (fp32, as couples: float4 (low v, low v+1,
// high v, high v+1) of pairs v, v+1 at [g][v/2]) and the C child rotations R(c) into
// shared memory.  R(c) is stored per pair couple (v, v+1) as (cos v, cos v+1,
// sin v, sin v+1); couple w of the lane that owns couples [CPL*l, CPL*l + CPL)
// sits at c * (D/4) + w * LPK + l, so the LPK lanes of one key read consecutive
// 16-byte words.  Every global load of the thread is issued before its first
// shared-memory store, so the loads overlap instead of waiting one by one.
template <typename T, int D, int G>
__device__ __forceinline__ void stage_query(const T* qrow, const float2* rope, int C, float* qsm,
                                            float4* rc4) {
    using S = Shape<T, D>;
    constexpr int QN = (G * D + kThreads - 1) / kThreads;
    constexpr int RN = (RECSA_MAX_C * (D / 4) + kThreads - 1) / kThreads;
    const int nr = C * (D / 4);
    float qv[QN];
    float2 ra[RN], rb[RN];
#pragma unroll
    for (int u = 0; u < QN; ++u) {
        const int i = threadIdx.x + u * kThreads;
        qv[u] = i < G * D ? (float)qrow[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < RN; ++u) {
        const int i = threadIdx.x + u * kThreads;
        ra[u] = rb[u] = make_float2(0.f, 0.f);
        if (i < nr) {
            ra[u] = rope[2 * i];
            rb[u] = rope[2 * i + 1];
        }
    }
#pragma unroll
    for (int u = 0; u < QN; ++u) {
        // dim d of head g at couple d/2 (low half) or (d-H)/2 (high half) of head g:
        // float4 (low v, low v+1, high v, high v+1)
        const int i = threadIdx.x + u * kThreads;
        const int g = i / D, d = i % D, hi = d >= D / 2, dd = hi ? d - D / 2 : d;
        if (i < G * D) qsm[(g * (D / 4) + dd / 2) * 4 + 2 * hi + (dd & 1)] = qv[u];
    }
#pragma unroll
    for (int u = 0; u < RN; ++u) {
        const int i = threadIdx.x + u * kThreads;
        if (i < nr) {
            const int c = i / (D / 4), f = i % (D / 4);
            rc4[c * (D / 4) + (f % S::CPL) * S::LPK + f / S::CPL] =
                make_float4(ra[u].x, rb[u].x, ra[u].y, rb[u].y);
        }
    }
}

// Softmax weights of the included chunk entries (entry i < n with flag[i] == 0,
// or every entry when flag is null): m_g = max s, s <- exp(s - m) in place, and
// this thread's part of l_g = sum exp.  fm[0..G) receives m.
template <int G>
__device__ __forceinline__ void softmax_weights(float* s, int n, const unsigned char* flag, int CH,
                                                float* red, float* fm, float* lsum) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float mx[G];
#pragma unroll
    for (int g = 0; g < G; ++g) mx[g] = -INFINITY;
    for (int i = threadIdx.x; i < n; i += kThreads)
        if (!flag || flag[i] == 0)
#pragma unroll
            for (int g = 0; g < G; ++g) mx[g] = fmaxf(mx[g], s[g * CH + i]);
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
        fm[threadIdx.x] = m;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        mx[g] = fm[g];
        lsum[g] = 0.f;
    }
    for (int i = threadIdx.x; i < n; i += kThreads)
        if (!flag || flag[i] == 0)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float p = __expf(s[g * CH + i] - mx[g]);
                s[g * CH + i] = p;
                lsum[g] += p;
            }
    __syncthreads();
}

// o_g += p_g * V for the rows of one staged parent group: row c of blk is the
// value of entry jb + c (c < nrow), left out when flagged (selected).  Branch-free
// so the unrolled rows pipeline their loads: a row past the group reads row 0 and,
// like a flagged row, gets weight 0.
template <typename T, int D, int G>
__device__ __forceinline__ void accum_parent(const unsigned char* blk, int jb, int j0, int nrow,
                                             const unsigned char* flag, const float* s, int CH,
                                             float2 (&acc)[G][VecOf<T>::N / 2]) {
    using S = Shape<T, D>;
    constexpr int V2 = S::VEC / 2;
    constexpr int kRow = D * (int)sizeof(T);
    const int lane = threadIdx.x & 31;
    const int c = lane % S::RPL, rr = lane / S::RPL;
#pragma unroll 4
    for (int cb = 0; cb < nrow; cb += S::RPW) {
        const int cr0 = cb + rr;
        const bool in_group = cr0 < nrow;
        const int cr = in_group ? cr0 : 0;
        const int r = jb - j0 + cr;
        const bool inc = in_group && (!flag || flag[r] == 0);
        float2 v[V2];
        unpack_pairs<T>(*reinterpret_cast<const uint4*>(blk + cr * kRow + c * 16), v);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float p = inc ? s[g * CH + r] : 0.f;
            const float2 p2 = make_float2(p, p);
#pragma unroll
            for (int e = 0; e < V2; ++e) acc[g][e] = __ffma2_rn(p2, v[e], acc[g][e]);
        }
    }
}

// Second half of a partial: each warp has written its o rows to red[warp][g][0..D);
// its l partials go to red[warp][g][D], then the warps are summed into the record
// [G][D+2] = (o, m, l).
template <int D, int G>
__device__ __forceinline__ void partial_tail(float* lsum, const float* fm, float* red, float* outp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lsum[g] += __shfl_xor_sync(kFull, lsum[g], o);
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) red[(warp * G + g) * (D + 1) + D] = lsum[g];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * (D + 1); i += kThreads) {
        float sum = 0.f;
        for (int w = 0; w < kWarps; ++w) sum += red[w * G * (D + 1) + i];
        const int g = i / (D + 1), d = i % (D + 1);
        if (d < D) outp[g * (D + 2) + d] = sum;
        else outp[g * (D + 2) + D + 1] = sum;
    }
    if (threadIdx.x < G) outp[threadIdx.x * (D + 2) + D] = fm[threadIdx.x];
}

// Cross-lane and cross-warp reduction of the value accumulators and l partials
// into the partial record [G][D+2] = (o, m, l).  red must be free.
template <typename T, int D, int G>
__device__ __forceinline__ void finish_partial(float2 (&acc)[G][VecOf<T>::N / 2], float* lsum,
                                               const float* fm, float* red, float* outp) {
    using S = Shape<T, D>;
    constexpr int VEC = S::VEC, V2 = VEC / 2;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = lane % S::RPL, rr = lane / S::RPL;
#pragma unroll
    for (int o = S::RPL; o < 32; o <<= 1)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < V2; ++e) {
                acc[g][e].x += __shfl_xor_sync(kFull, acc[g][e].x, o);
                acc[g][e].y += __shfl_xor_sync(kFull, acc[g][e].y, o);
            }
    if (rr == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < V2; ++e) {
                red[(warp * G + g) * (D + 1) + c * VEC + 2 * e] = acc[g][e].x;
                red[(warp * G + g) * (D + 1) + c * VEC + 2 * e + 1] = acc[g][e].y;
            }
    }
    partial_tail<D, G>(lsum, fm, red, outp);
}

// ---- value accumulation on the tensor cores (SW kernels: bf16, d = 128) ----
// o^T[d][g] += sum_r V[r][d] p_g[r] as mma.sync m16n8k16 products with fp32
// accumulation: M = the D value dims (D/16 tiles), N = 8 query-head columns (G used,
// the rest zero), K = 16 rows of the group per step.  A = V^T comes straight from
// the swizzled slot by ldmatrix.trans; B = the weights, split into a bf16 high part
// and a bf16 remainder so that together they carry 16 significant bits (two
// products), which keeps the accumulated output as close to an fp32 product as the
// scalar path's.  acc[mt][0..3] holds (dim mt*16 + lane/4, heads 2*(lane%4), +1)
// and (dim + 8, same heads).
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// The weights of rows k0 + 2t, +1 (b0) and k0 + 2t + 8, +9 (b1) for head lane/4 as
// bf16 high parts and remainders; zero for rows past nrow, flagged rows, and head
// columns >= G.
template <int G>
__device__ __forceinline__ void weight_frags(const float* s, const unsigned char* flag, int CH,
                                             int rb, int k0, int nrow, uint32_t (&bh)[2],
                                             uint32_t (&bl)[2]) {
    const int lane = threadIdx.x & 31;
    const int gi = lane >> 2, tg = lane & 3;
    bh[0] = bh[1] = bl[0] = bl[1] = 0u;
    if (gi < G) {
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = k0 + 2 * tg + (i & 1) + (i >> 1) * 8;
            const int r = rb + c;
            const bool inc = c < nrow && (!flag || flag[r] == 0);
            p[i] = inc ? s[gi * CH + r] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(p[2 * j], p[2 * j + 1]);
            const float2 hf = __bfloat1622float2(h);
            bh[j] = *reinterpret_cast<const uint32_t*>(&h);
            bl[j] = pack_bf16x2(p[2 * j] - hf.x, p[2 * j + 1] - hf.y);
        }
    }
}

template <int D, int G>
__device__ __forceinline__ void accum_parent_mma(const unsigned char* blk, int C, int jb, int j0,
                                                 int nrow, const unsigned char* flag,
                                                 const float* s, int CH, float (&acc)[D / 16][4]) {
    const int lane = threadIdx.x & 31;
    const int tg = lane & 3;
    const uint32_t base = smem_u32(blk);
    // ldmatrix.x4: lanes 8j..8j+7 address the rows of 8x8 tile j = (rows + 8 (j >> 1),
    // dims + 8 (j & 1)) of the 16 x 16 step, so registers 0..3 are the A fragment
    const int lrow = (lane & 7) + ((lane >> 4) << 3);
    const int ldim = ((lane >> 3) & 1) * 8;
    for (int k0 = 0; k0 < C; k0 += 16) {
        uint32_t bh[2], bl[2];
        weight_frags<G>(s, flag, CH, jb - j0, k0, nrow, bh, bl);
        // rows past nrow hold other nodes' rows or stale data: their V elements are
        // masked to zero so that a weight of zero never meets a non-finite value
        uint32_t m01 = 0xffffffffu, m89 = 0xffffffffu;
        if (k0 + 16 > nrow) {
            const int c = k0 + 2 * tg;
            m01 = (c < nrow ? 0x0000ffffu : 0u) | (c + 1 < nrow ? 0xffff0000u : 0u);
            m89 = (c + 8 < nrow ? 0x0000ffffu : 0u) | (c + 9 < nrow ? 0xffff0000u : 0u);
        }
        const int row = k0 + lrow;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            const int d0 = mt * 16 + ldim;
            const uint32_t addr = base + swz_off(d0 >> 6, row, (d0 & 63) >> 3, C);
            uint32_t a0, a1, a2, a3;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                         : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                         : "r"(addr)
                         : "memory");
            a0 &= m01;
            a1 &= m01;
            a2 &= m89;
            a3 &= m89;
            mma_bf16_16816(acc[mt], a0, a1, a2, a3, bh[0], bh[1]);
            mma_bf16_16816(acc[mt], a0, a1, a2, a3, bl[0], bl[1]);
        }
    }
}

// Writes each warp's tensor-core accumulators to red[warp][g][d] and finishes the
// partial record.
template <int D, int G>
__device__ __forceinline__ void finish_partial_mma(float (&acc)[D / 16][4], float* lsum,
                                                   const float* fm, float* red, float* outp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gi = lane >> 2, tg = lane & 3;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int g = 2 * tg + j;
        if (g < G) {
            float* row = red + (warp * G + g) * (D + 1);
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                row[mt * 16 + gi] = acc[mt][j];
                row[mt * 16 + gi + 8] = acc[mt][2 + j];
            }
        }
    }
    partial_tail<D, G>(lsum, fm, red, outp);
}

__device__ __forceinline__ void write_empty_partial(float* outp, int G, int D) {
    for (int i = threadIdx.x; i < G * (D + 2); i += kThreads) {
        const int d = i % (D + 2);
        outp[i] = (d == D) ? -INFINITY : 0.f;
    }
}

// Log-sum-exp merge of a unit's partials into its G output heads, output elements
// [e0, e1) of the G*D.  Partials of other CTAs are read through L2 (ld.global.cg),
// all of a slice's loads issued together into shared memory (buf, nbuf floats:
// weights, (m, l) of every slot and head, then the staged values) so they cost one
// latency rather than one per slot; the sums run over the slots in slot order.
template <typename T, int D, int G>
__device__ void combine_unit(const float* P, int lstar, int SPL, int NS0, int NL, T* out,
                             float* buf, int nbuf, float* Lsh /* G */, int e0, int e1) {
    const int nls = lstar * SPL;
    const int ns = nls + NS0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* wsh = buf;            // [G][ns] weights
    float* mm = buf + G * ns;    // [G][ns] m
    float* ll = mm + G * ns;     // [G][ns] l
    float* vals = ll + G * ns;   // [ns][E] staged values
    auto slot_of = [&](int i) { return i < nls ? i : NL * SPL + (i - nls); };
    const int cap = (nbuf - 3 * G * ns) / ns;   // output elements staged per round
    // (m, l) of every slot and head, then the first round of values.  The code runs
    // once per launch (its instructions are fetched cold), so it stays short: no
    // division per element, and KB loads of a thread in flight before their stores.
    constexpr int KB = 8;
    const int E0 = min(cap, e1 - e0);
    for (int x = threadIdx.x; x < ns * G; x += kThreads) {
        const int i = x / G, g = x % G;
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(P + (slot_of(i) * G + g) * (D + 2) + D));
        mm[g * ns + i] = ml.x;
        ll[g * ns + i] = ml.y;
    }
    // thread -> column e0 + c of slots i0, i0 + di, ... (when E0 divides kThreads)
    const bool cols = kThreads % E0 == 0;
    const int c = cols ? threadIdx.x % E0 : 0, i0 = cols ? threadIdx.x / E0 : 0;
    const int di = cols ? kThreads / E0 : 1;
    const float* colp = P + ((e0 + c) / D) * (D + 2) + (e0 + c) % D;
    if (cols) {
        for (int ib = i0; ib < ns; ib += KB * di) {
            float v[KB];
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const int i = ib + u * di;
                v[u] = i < ns ? __ldcg(colp + slot_of(i) * G * (D + 2)) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < KB; ++u)
                if (ib + u * di < ns) vals[(ib + u * di) * E0 + c] = v[u];
        }
    } else {
        for (int y = threadIdx.x; y < ns * E0; y += kThreads) {
            const int i = y / E0, e = e0 + y % E0;
            vals[y] = __ldcg(P + (slot_of(i) * G + e / D) * (D + 2) + e % D);
        }
    }
    __syncthreads();
    for (int g = warp; g < G; g += kWarps) {
        float M = -INFINITY;
        for (int i = lane; i < ns; i += 32) M = fmaxf(M, mm[g * ns + i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
        float L = 0.f;
        for (int i = lane; i < ns; i += 32) {
            const float l = ll[g * ns + i];
            const float w = l > 0.f ? __expf(mm[g * ns + i] - M) : 0.f;
            wsh[g * ns + i] = w;
            L += w * l;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(kFull, L, o);
        if (lane == 0) Lsh[g] = L;
    }
    for (int c0 = e0; c0 < e1; c0 += cap) {
        const int E = min(cap, e1 - c0);
        __syncthreads();   // the previous round's reads (and the weights) are done
        if (c0 > e0)
            for (int x = threadIdx.x; x < ns * E; x += kThreads) {
                const int i = x / E, e = c0 + x % E;
                vals[x] = __ldcg(P + (slot_of(i) * G + e / D) * (D + 2) + e % D);
            }
        __syncthreads();
        for (int x = threadIdx.x; x < E; x += kThreads) {
            const int e = c0 + x, g = e / D;
            float O = 0.f;
            for (int i = 0; i < ns; ++i) O += wsh[g * ns + i] * vals[i * E + x];
            const float L = Lsh[g];
            out[e] = store_round_f<T>(L > 0.f ? O / L : 0.f);
        }
    }
}


// ----------------------------------------------------------------------------
// One select/attend pass: every level of a unit in one kernel.  A unit (query, KV
// head) is one cluster of SPL CTAs that walks the levels top-down:
//   level l >= 1: score + RoPE + TopK + summaries; the CTAs' parts of S^(l) are
//                 in place for level l-1 after a cluster barrier;
//   level 0:      score + softmax partial over A^(0);
// then a cluster barrier and the log-sum-exp merge of every partial of the unit,
// each CTA writing a slice of the G output heads.  Units never wait on each
// other, so a unit's next level starts as soon as its own selection is done, and
// the code of the scoring, selection and value loops serves all levels.
// Each warp takes every kWarps-th parent group of its CTA's chunk; its K blocks
// and then its V blocks stream through its ring (block numbering continues
// across levels, so the mbarrier phases do too), so V loads overlap the
// selection.  SW kernels (bf16, d = 128, C a multiple of 16) stage the groups
// through the swizzled tensor maps of each level and accumulate values on the
// tensor cores; the others use plain bulk copies and fp32 FMAs.
// CTAs past the units' clusters (blockIdx.y >= units, decode only) re-pool the
// ancestors of each sequence's newest token; nothing in the pass reads them.
// ----------------------------------------------------------------------------
constexpr int kMapLevels = 8;   // levels whose tensor maps a launch carries
struct PassMaps {
    KVMaps m[kMapLevels];
};

// Fused append: every CTA that reads lens[b] (the sequence's attention CTAs and its
// walk CTAs, Hkv * (csize + 1) in all) counts itself once it has; the last one stores
// the new length t + 1.  One thread per CTA, after a CTA barrier that follows the
// reads.
__device__ __forceinline__ void fused_count(const TreeView& tv, const WorkView& wv, int b,
                                            int64_t t, int csize) {
    __threadfence();
    if (atomicAdd(&wv.done[b], 1u) == (unsigned)(tv.Hkv * (csize + 1)) - 1u) {
        wv.done[b] = 0u;
        wv.lens[b] = t + 1;
    }
}

// Fused append: row r of a staged block (C rows, plain or swizzled) replaced by the
// new token's row; lanes 0..D*esize/16-1 each store 16 bytes.  The stores are fenced
// against the slot's next tensor copy.
template <typename T, int D, bool SW>
__device__ __forceinline__ void patch_row(unsigned char* blk, int r, int C, const T* row) {
    constexpr int NCH = D * (int)sizeof(T) / 16;
    const int lane = threadIdx.x & 31;
    if (lane < NCH) {
        const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned char*>(row) + 16 * lane);
        uint32_t off;
        if constexpr (SW) off = swz_off(lane >> 3, r, lane & 7, C);
        else off = (uint32_t)(r * D * (int)sizeof(T) + 16 * lane);
        *reinterpret_cast<uint4*>(blk + off) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
}

// FU: the decode fused with a one-token append (a separate instantiation, so that the
// other launches carry none of its checks)
template <typename T, int D, int G, bool SW, bool FU>
__global__ void __launch_bounds__(kThreads, 2)
    pass_kernel(TreeView tv, WorkView wv, QueryView qv, const __grid_constant__ PassMaps maps,
                int CH, int NA, int nsw) {
    static_assert(!SW || kSwzCapable<T, D>, "swizzled staging is bf16, d = 128 only");
    extern __shared__ __align__(1024) unsigned char smem[];
    const int units = qv.nq * tv.Hkv;
    if ((int)blockIdx.y >= units) {
        const int ci = ((int)blockIdx.y - units) * (int)gridDim.x + (int)blockIdx.x;
        if (ci >= tv.B * tv.Hkv) return;
        double* alpha = reinterpret_cast<double*>(smem);
        double* pre = alpha + RECSA_MAX_C * RECSA_MAX_C;
        pdl_wait();
        for (int i = threadIdx.x; i < tv.C * tv.C; i += kThreads) alpha[i] = wv.alpha[i];
        const int b = ci / tv.Hkv, h = ci % tv.Hkv;
        const bool fused = FU && qv.knew != nullptr;
        const int64_t t = fused ? wv.lens[b] : wv.lens[b] - 1;
        if (fused && t < tv.cap) {
            // the new token's rows at level 0, read back by this CTA's walk
            constexpr int VEC = VecOf<T>::N;
            const int64_t o = b * tv.s_b + h * tv.s_h + t * tv.s_t;
            const T* kn = reinterpret_cast<const T*>(qv.knew) + ((int64_t)b * tv.Hkv + h) * D;
            const T* vn = reinterpret_cast<const T*>(qv.vnew) + ((int64_t)b * tv.Hkv + h) * D;
            for (int e = threadIdx.x; e < D / VEC; e += kThreads) {
                *reinterpret_cast<uint4*>(reinterpret_cast<T*>(tv.k0w) + o + e * VEC) =
                    *reinterpret_cast<const uint4*>(kn + e * VEC);
                *reinterpret_cast<uint4*>(reinterpret_cast<T*>(tv.v0w) + o + e * VEC) =
                    *reinterpret_cast<const uint4*>(vn + e * VEC);
            }
        }
        __syncthreads();
        if (fused && threadIdx.x == 0) fused_count(tv, wv, b, t, (int)gridDim.x);
        if (t >= 1 && t < tv.cap) ancestor_walk<T, D, 4>(tv, b, h, t, pre, alpha, wv.status);
        return;
    }
    constexpr int kRow = D * (int)sizeof(T);
    constexpr int V2 = VecOf<T>::N / 2;
    const int k = tv.k, C = tv.C, lgC = tv.lgC, K1 = k - 1, NL = wv.NL;
    const int nsplit = wv.SPL;   // == NS0
    const int slot_bytes = C * kRow;
    const int gsw = gs_words(nsplit);
    const Smem SL = smem_layout(G, D, CH, k, C, NA, gsw, wv.NSLOT, kWarps * nsw * slot_bytes);
    float* qsm = reinterpret_cast<float*>(smem + SL.qsm);
    float4* rc4 = reinterpret_cast<float4*>(smem + SL.rc4);
    float* s = reinterpret_cast<float*>(smem + SL.s);
    uint32_t* key = reinterpret_cast<uint32_t*>(smem + SL.key);
    int* nodes = reinterpret_cast<int*>(smem + SL.nodes);
    unsigned char* flag = smem + SL.flag;
    // S^(l), as far as this CTA needs it, in buffer l mod 3: at a level the CTA reads
    // its parents S^(level+1) while the cluster's CTAs store S^(level) into the next
    // buffer, and a CTA that runs one level ahead stores S^(level-1) into the third
    int* pbuf = reinterpret_cast<int*>(smem + SL.par);
    uint32_t* mkey = reinterpret_cast<uint32_t*>(smem + SL.mkey);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + SL.hist);
    uint32_t* gs = reinterpret_cast<uint32_t*>(smem + SL.gs);
    int* misc = reinterpret_cast<int*>(smem + SL.misc);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL.bars);
    unsigned char* ring = smem + SL.ring;
    float* red = reinterpret_cast<float*>(smem + SL.red);   // reuses the ring between levels
    float* fm = reinterpret_cast<float*>(misc + kMiscFloat);
    if constexpr (SW) {
        // the swizzle pattern assumes 1024-byte aligned slots; every CTA of the launch
        // sees the same base, so all of them return here together
        if (smem_u32(ring) & 1023u) {
            if (threadIdx.x == 0) set_status(wv.status, kStatusLayout);
            return;
        }
    }

    const int unit = blockIdx.y;
    const int split = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qloc = unit / tv.Hkv, kvh = unit % tv.Hkv;
    const int gq = qv.q_begin + qloc;
    const int b = gq / qv.n_per_b;
    cg::cluster_group cluster = cg::this_cluster();
    const int csize = (int)cluster.num_blocks();
    const int crank = (int)cluster.block_rank();
    const T* qrow = reinterpret_cast<const T*>(qv.q) + ((int64_t)gq * tv.Hq + kvh * G) * D;
    if (threadIdx.x == 0) misc[kMiscFailed] = 0;
    if (threadIdx.x < kWarps * nsw) mbar_init(&bars[threadIdx.x], 1);
    mbar_fence_init();
    if constexpr (SW) {
        // the levels' tensor-map descriptors into the descriptor cache
        if (threadIdx.x < 2 * kMapLevels && threadIdx.x / 2 <= NL) {
            const KVMaps& m = maps.m[threadIdx.x / 2];
            asm volatile("prefetch.tensormap [%0];" ::"l"(
                             reinterpret_cast<uint64_t>((threadIdx.x & 1) ? &m.v : &m.k))
                         : "memory");
        }
    }
    if (threadIdx.x == 0) {
        // while the kernel before (an append) may still run, this CTA's share of the
        // RoPE table and, in a decode, its chunk of the first scored level go
        // towards L2: those rows do not change in an append, only the list length
        // may grow by one, so a length read before the wait is enough of a hint
        // (the range is clamped to the tables)
        const int nct = (int)(gridDim.x * units);
        const int ci = unit * (int)gridDim.x + split;
        const int per = (wv.ck + nct - 1) / nct;
        const int r0 = ci * per, r1 = min(wv.ck, r0 + per);
        if (r1 > r0)
            prefetch_l2(wv.rope + (int64_t)r0 * (D / 2), (uint32_t)(r1 - r0) * (D / 2) * sizeof(float2));
        if (qv.mode == 0) {
            const int64_t th = *reinterpret_cast<const volatile int64_t*>(wv.lens + b);
            const int lh = th >= 1 ? first_scored_level(th, C, lgC, k) : 0;
            if (lh >= 1) {
                const int nAh = list_size(th, lh, lh, C, lgC, k);
                const int ch = ((cdiv(nAh + C - 1, C, lgC) + nsplit - 1) / nsplit) * C;
                const int a = split * ch;
                const int e = (int)imin64(imin64(nAh, a + ch + C), tv.rows[lh]);
                if (e > a) {
                    prefetch_l2(level_k<T>(tv, lh, b, kvh) + (int64_t)a * D, (uint32_t)(e - a) * kRow);
                    prefetch_l2(level_v<T>(tv, lh, b, kvh) + (int64_t)a * D, (uint32_t)(e - a) * kRow);
                }
            }
        }
    }
    // Nothing before this wait reads global memory that an earlier kernel may have
    // written (only L2 prefetch hints go out above): the kernel just before may be
    // the caller's own, writing q.
    pdl_wait();
    const int64_t len = wv.lens[b];
    stage_query<T, D, G>(qrow, wv.rope, C, qsm, rc4);
    const bool fused = FU && qv.knew != nullptr;   // decode fused with a one-token append
    const int64_t t = (qv.mode == 0) ? (fused ? len : len - 1) : qv.pos0 + (gq - b * qv.n_per_b);
    const bool valid = t >= 0 && t < (fused ? tv.cap : len);
    const int lstar = valid ? first_scored_level(t, C, lgC, k) : 0;
    // the list geometry of every level, one thread per level (each a chain of
    // dependent integer steps): |A^(l)|, the entries per CTA, and the parents per
    // CTA of the level below
    int* geo = reinterpret_cast<int*>(smem + SL.geo);
    if (valid && threadIdx.x <= lstar) {
        const int l = threadIdx.x;
        const int nA_l = list_size(t, lstar, l, C, lgC, k);
        const int npar_l = cdiv(nA_l + C - 1, C, lgC);
        geo[4 * l] = nA_l;
        geo[4 * l + 1] = ((npar_l + nsplit - 1) / nsplit) * C;
        if (l >= 1) {
            const int nA_m = list_size(t, lstar, l - 1, C, lgC, k);
            geo[4 * l + 2] = (cdiv(nA_m + C - 1, C, lgC) + nsplit - 1) / nsplit;
        }
    }
    int32_t* cnt_ws = wv.cnt + (int64_t)unit * (NL + 1);
    int32_t* cnt_usr = qv.cnt_out ? qv.cnt_out + ((int64_t)gq * tv.Hkv + kvh) * (NL + 1) : nullptr;
    float* part = wv.part + (int64_t)unit * wv.NSLOT * G * (D + 2);
    T* out = reinterpret_cast<T*>(qv.out) + ((int64_t)gq * tv.Hq + kvh * G) * D;
    __syncthreads();
    if (fused && threadIdx.x == 0) fused_count(tv, wv, b, t, csize);
    // fused append: the new token (entry |A^(0)|-1, the level-0 list's last) is staged
    // from these rows instead of the cache, which its walk CTA is writing meanwhile
    const T* knew_row = fused ? reinterpret_cast<const T*>(qv.knew) + ((int64_t)b * tv.Hkv + kvh) * D : nullptr;
    const T* vnew_row = fused ? reinterpret_cast<const T*>(qv.vnew) + ((int64_t)b * tv.Hkv + kvh) * D : nullptr;

    if (!valid) {
        // nothing to attend (empty sequence, or a prefill row beyond the length):
        // every level unscored, a zero output
        if (split == 0) {
            for (int l = 1; l <= NL; ++l) {
                if (qv.sel_out)
                    for (int i = threadIdx.x; i < k; i += kThreads)
                        qv.sel_out[(((int64_t)gq * tv.Hkv + kvh) * NL + (l - 1)) * k + i] = -1;
                if (threadIdx.x == 0) {
                    cnt_ws[l] = 0;
                    if (cnt_usr) cnt_usr[l] = 0;
                }
            }
            for (int i = threadIdx.x; i < G * D; i += kThreads) out[i] = store_round_f<T>(0.f);
            if (threadIdx.x == 0) {
                cnt_ws[0] = 0;
                if (cnt_usr) cnt_usr[0] = 0;
                if (qv.mode == 1) set_status(wv.status, kStatusBadQuery);
            }
        }
        pdl_launch_dependents();
        return;
    }

    int qbase = 0;   // blocks this warp has taken from its ring so far
    for (int level = NL; level >= 0; --level) {
        const bool L0 = level == 0;
        if (level > lstar) continue;   // not scored: recorded after the pass
        if (qv.phase == 2 && !L0) continue;   // levels >= 1 were done by the phase-1 launch
        if (qv.phase == 1 && L0) break;       // level 0 and the merge: the phase-2 launch
        // Below the first scored level no barrier is needed here: every CTA of the
        // cluster stored its part of S^(level+1) into the other CTAs' buffers, and
        // zeroed its slice of the selection's global histogram, before the cluster
        // arrive that the level above waited on at its end.
        const int* par = pbuf + ((level + 1) % 3) * k;
        int* par_next = pbuf + (level % 3) * k;
        const bool first = level == lstar;
        if (!L0) {
            // this CTA's own histogram and counters (peers read the counters only
            // after the selection's second barrier)
            for (int i = threadIdx.x; i < kSelBins / 2; i += kThreads) hist[i] = 0u;
            if (threadIdx.x == 0) misc[kMiscPubC] = misc[kMiscPubA] = 0;
            if (first) {
                // the global histogram's slices start at zero in every CTA before any
                // CTA adds into them (waited on after the scores)
                for (int i = threadIdx.x; i < gsw; i += kThreads) gs[i] = 0u;
                __syncthreads();
                cluster_arrive();
            }
        } else {
            pdl_launch_dependents();   // the next kernel may start launching
        }
        const int nA = geo[4 * level];
        // phase 2 reads level 0 from the staging copy, where entry j is row j
        const bool identity = level == lstar || qv.phase == 2;
        const int chunk = geo[4 * level + 1];
        const int j0 = split * chunk;
        const int j1 = min(nA, j0 + chunk);
        const T *kbase, *vbase;
        int64_t rs;
        if (L0 && qv.phase == 2) {
            const int64_t so = ((int64_t)qloc * tv.Hkv + kvh) * (int64_t)wv.ck * D;
            kbase = reinterpret_cast<const T*>(qv.l0k) + so;
            vbase = reinterpret_cast<const T*>(qv.l0v) + so;
            rs = D;
        } else if (L0) {
            kbase = reinterpret_cast<const T*>(tv.k0) + (b * tv.s_b + kvh * tv.s_h);
            vbase = reinterpret_cast<const T*>(tv.v0) + (b * tv.s_b + kvh * tv.s_h);
            rs = tv.s_t;
        } else {
            kbase = level_k<T>(tv, level, b, kvh);
            vbase = level_v<T>(tv, level, b, kvh);
            rs = D;
        }
        const int p_q = nA - 1;
        // scored entries: all of A^(0); at levels >= 1 all but the current entry nA-1
        const int n_sc = L0 ? max(0, j1 - j0) : max(0, min(j1, nA - 1) - j0);
        if (split == 0 && threadIdx.x == 0) {
            cnt_ws[level] = nA;
            if (cnt_usr) cnt_usr[level] = nA;
        }
        int32_t* sel_ws = L0 ? nullptr : wv.sel + ((int64_t)unit * NL + (level - 1)) * k;
        int32_t* sel_usr = (L0 || !qv.sel_out)
                               ? nullptr
                               : qv.sel_out + (((int64_t)gq * tv.Hkv + kvh) * NL + (level - 1)) * k;
        float* outp = part + (int64_t)((L0 ? NL * wv.SPL : (level - 1) * wv.SPL) + split) * G * (D + 2);
        // parents per CTA at the next level: parent rank r goes to CTA r / ppc_next
        const int ppc_next = L0 ? 1 : geo[4 * level + 2];
        if (!L0 && nA <= k) {
            // everything selected, no summaries (not reachable below the first scored
            // level when k, C >= 2; kept for completeness)
            if (split == 0) {
                for (int i = threadIdx.x; i < k; i += kThreads) {
                    int v = -1;
                    if (i < nA) v = identity ? i : C * par[cdiv(i, C, lgC)] + cmod(i, C, lgC);
                    if (i < nA) {
                        sel_ws[i] = v;
                        cluster.map_shared_rank(par_next, i / ppc_next)[i] = v;
                    }
                    if (sel_usr) sel_usr[i] = v;
                }
            }
            write_empty_partial(outp, G, D);
            if (first) cluster_wait();   // the arrive at the level's start
            for (int i = threadIdx.x; i < gsw; i += kThreads) gs[i] = 0u;
            __syncthreads();
            cluster_arrive();   // S^(level) stored, the slice zeroed for the level below
            cluster_wait();
            continue;
        }

        // ---- the warp's parent groups and their blocks (K then V) ----
        const int P = (j1 > j0) ? cdiv(j1 - j0 + C - 1, C, lgC) : 0;
        const int nw = warp < P ? (P - warp + kWarps - 1) / kWarps : 0;
        // logits already computed for this level (tensor-core prefill): no K blocks
        const bool pre = !L0 && qv.pre != nullptr && level == qv.pre_level && identity;
        const int nk = pre ? 0 : nw;   // blocks [0, nk) are K, [nk, nk + nw) are V
        const WarpRing R{ring + (size_t)warp * nsw * slot_bytes, bars + warp * nsw, nsw,
                         slot_bytes, wv.status, misc + kMiscFailed};
        // rows of the table this level reads (the staging copy in phase 2)
        const int64_t trows = L0 ? (qv.phase == 2 ? (int64_t)wv.ck : tv.cap) : tv.rows[level];
        auto group_first = [&](int jb) -> int64_t {
            const int64_t f = identity ? (int64_t)jb : (int64_t)C * par[cdiv(jb, C, lgC)];
            return in_bounds(f >= 0 && f < trows && jb >= 0 && jb < nA, wv.status) ? f : 0;
        };
        const KVMaps* lmap = &maps.m[level < kMapLevels ? level : 0];
        auto issue = [&](int q) {
            const int i = q < nk ? q : q - nk;
            const int jb = j0 + (warp + kWarps * i) * C;
            if constexpr (SW)
                ring_issue_map(R, qbase + q, q < nk ? &lmap->k : &lmap->v, group_first(jb), kvh, b, C);
            else
                ring_issue<T, D>(R, qbase + q, q < nk ? kbase : vbase, rs, group_first(jb),
                                 min(C, j1 - jb));
        };
        if (lane == 0)
            for (int q = 0; q < nsw && q < nk + nw; ++q) issue(q);

        // 1. scores of the chunk
        if (pre) {
            // the query's list is [0..a_t] (identity): entry j is node j
            const float* prow = qv.pre + (int64_t)(qloc * tv.Hkv + kvh) * G * qv.pre_stride;
            for (int i = 0; i < nw; ++i) {
                const int jb = j0 + (warp + kWarps * i) * C;
                const int nch = min(C, j0 + n_sc - jb);
                for (int c = lane; c < nch; c += 32) {
                    const int r = jb - j0 + c;
                    float imp = 0.f;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float v = __ldcg(prow + (int64_t)g * qv.pre_stride + jb + c);
                        s[g * CH + r] = v;
                        imp += v;
                    }
                    nodes[r] = jb + c;
                    key[r] = ordered_key(imp * (1.0f / G));
                }
            }
            __syncwarp();
        } else {
            // the rotation R(p_q - jb) of each group, the lane's couples, loaded one
            // group ahead into registers
            constexpr int CPL = Shape<T, D>::CPL;
            const int qoff = (lane % Shape<T, D>::LPK) * Shape<T, D>::PPL;
            float4 qcs[CPL];
            auto load_qcs = [&](int jb_, float4 (&o)[CPL]) {
                const float4* r = reinterpret_cast<const float4*>(wv.rope + (int64_t)(p_q - jb_) * (D / 2) + qoff);
#pragma unroll
                for (int w = 0; w < CPL; ++w) o[w] = __ldg(r + w);
            };
            if (nw > 0) load_qcs(j0 + warp * C, qcs);
            for (int i = 0; i < nw; ++i) {
                const unsigned char* blk = ring_wait(R, qbase + i);
                const int jb = j0 + (warp + kWarps * i) * C;
                const int nch = min(C, j0 + n_sc - jb);
                if (fused && L0 && jb <= nA - 1 && nA - 1 < jb + C)
                    patch_row<T, D, SW>(const_cast<unsigned char*>(blk), nA - 1 - jb, C, knew_row);
                float4 qn[CPL];
                if (i + 1 < nw) load_qcs(jb + kWarps * C, qn);
                if (nch > 0)
                    score_parent<T, D, G, true, SW>(blk, C, jb, qcs, j0, nch, group_first(jb), rc4,
                                                    qsm, tv.scale, s, key, nodes, CH);
#pragma unroll
                for (int w = 0; w < CPL; ++w) qcs[w] = qn[w];
                __syncwarp();
                if (lane == 0 && i + nsw < nk + nw) issue(i + nsw);
            }
        }
        for (int i = threadIdx.x; i < n_sc; i += kThreads) flag[i] = 0;
        __syncthreads();

        if (!L0) {
            const int M = nA - 1;
            if (first) cluster_wait();   // every CTA's zeroed histogram slice is in place
            // 2. exact top-(k-1) over all M keys; this CTA writes S for its entries
            auto mark = [&](int i, int r) {
                if (!in_bounds(r >= 0 && r < K1 && i >= j0 && i < j0 + n_sc &&
                               r / ppc_next < nsplit, wv.status))
                    return;
                const int node = nodes[i - j0];
                sel_ws[r] = node;
                if (sel_usr) sel_usr[r] = node;
                flag[i - j0] = 1;
                cluster.map_shared_rank(par_next, r / ppc_next)[r] = node;
            };
            bool done = true;
            if (K1 > 0) {   // k = 1: only the current node is selected
                uint2* pub = reinterpret_cast<uint2*>(mkey);
                done = cluster_select(key, n_sc, j0, K1, csize, crank, gsw, hist, gs, pub,
                                      pub + kSelCand, misc, mark);
            }
            if (!done) {
                // heavy ties: every CTA's keys in list order (list position = merged
                // index), then the block-wide select (same set)
                for (int r = 0; r < csize; ++r) {
                    const int lo = r * chunk, hi = min(M, lo + chunk);
                    if (hi <= lo) break;
                    const uint32_t* rk = cluster.map_shared_rank(key, r);
#pragma unroll 4
                    for (int i = threadIdx.x; i < hi - lo; i += kThreads) mkey[lo + i] = rk[i];
                }
                __syncthreads();
                select_topk(mkey, M, K1, hist, misc, j0, j0 + n_sc, mark);
            }
            if (crank == 0 && threadIdx.x == 0) {
                const int64_t cur = apow(t, level, C, lgC);
                sel_ws[K1] = (int)cur;
                if (sel_usr) sel_usr[K1] = (int)cur;
                cluster.map_shared_rank(par_next, K1 / ppc_next)[K1] = (int)cur;
            }
            // every remote read of this level is done (the other CTAs' keys, candidates,
            // counts and histogram slices) and every store of S^(level) into the other
            // CTAs has been issued; the slice is zeroed for the level below.  The
            // release publishes both; the level's end waits for every CTA.
            for (int i = threadIdx.x; i < gsw; i += kThreads) gs[i] = 0u;
            __syncthreads();
            cluster_arrive();
            // No L2 prefetch of the kept nodes' children here: bulk prefetches queue in
            // the same TMA unit as the rings' copies, and delayed this level's value
            // blocks and the next level's first blocks by more than they saved.
        }

        // 3. softmax partial over the unselected (level) or all (level 0) entries
        float lsum[G];
        // (scratch: the histogram area; the ring, and so red, still holds V blocks)
        softmax_weights<G>(s, n_sc, L0 ? nullptr : flag, CH, reinterpret_cast<float*>(hist), fm,
                           lsum);
        if constexpr (SW) {
            float acc[D / 16][4];
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
            for (int i = 0; i < nw; ++i) {
                const int q = nk + i;
                const unsigned char* blk = ring_wait(R, qbase + q);
                const int jb = j0 + (warp + kWarps * i) * C;
                const int nrow = min(C, j0 + n_sc - jb);
                if (fused && L0 && jb <= nA - 1 && nA - 1 < jb + C)
                    patch_row<T, D, SW>(const_cast<unsigned char*>(blk), nA - 1 - jb, C, vnew_row);
                if (nrow > 0 && fm[0] > -INFINITY)
                    accum_parent_mma<D, G>(blk, C, jb, j0, nrow, L0 ? nullptr : flag, s, CH, acc);
                __syncwarp();
                if (lane == 0 && q + nsw < nk + nw) issue(q + nsw);
            }
            __syncthreads();   // every block consumed: the ring area becomes the reduction buffer
            finish_partial_mma<D, G>(acc, lsum, fm, red, outp);
        } else {
            float2 acc[G][V2];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < V2; ++e) acc[g][e] = make_float2(0.f, 0.f);
            for (int i = 0; i < nw; ++i) {
                const int q = nk + i;
                const unsigned char* blk = ring_wait(R, qbase + q);
                const int jb = j0 + (warp + kWarps * i) * C;
                const int nrow = min(C, j0 + n_sc - jb);
                if (fused && L0 && jb <= nA - 1 && nA - 1 < jb + C)
                    patch_row<T, D, SW>(const_cast<unsigned char*>(blk), nA - 1 - jb, C, vnew_row);
                if (nrow > 0 && fm[0] > -INFINITY)
                    accum_parent<T, D, G>(blk, jb, j0, nrow, L0 ? nullptr : flag, s, CH, acc);
                __syncwarp();
                if (lane == 0 && q + nsw < nk + nw) issue(q + nsw);
            }
            __syncthreads();   // every block consumed: the ring area becomes the reduction buffer
            finish_partial<T, D, G>(acc, lsum, fm, red, outp);
        }
        qbase += nk + nw;
        // red (the ring) is read: the next level's tensor copies may overwrite it
        __syncthreads();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (!L0) cluster_wait();   // every CTA's arrive after its selection
    }

    if (split == 0 && qv.phase != 2) {
        // the levels above the first scored one: their whole lists are selected
        for (int l = lstar + 1; l <= NL; ++l) {
            if (qv.sel_out)
                for (int i = threadIdx.x; i < k; i += kThreads)
                    qv.sel_out[(((int64_t)gq * tv.Hkv + kvh) * NL + (l - 1)) * k + i] = -1;
            if (threadIdx.x == 0) {
                cnt_ws[l] = 0;
                if (cnt_usr) cnt_usr[l] = 0;
            }
        }
    }
    if (qv.phase == 1) {
        // the peers' parent-list stores into this CTA's shared memory have landed
        // before any CTA of the cluster exits
        pdl_launch_dependents();
        cluster.sync();
        return;
    }
    // every partial of the unit is written: merge them, this CTA taking a slice of
    // the G output heads
    cluster.sync();
    const int per = (G * D + csize - 1) / csize;
    combine_unit<T, D, G>(part, lstar, wv.SPL, wv.NS0, NL, out, red,
                          (int)((SL.total - SL.red) / sizeof(float)),
                          reinterpret_cast<float*>(misc + kMiscFloat + 8), crank * per,
                          min(G * D, (crank + 1) * per));
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
static inline int chunk_cap(int k, int splits, int C) { return ((k + splits - 1) / splits) * C; }

// blocks in flight per warp: two when a parent group is at most 4 KB
static inline int slots_per_warp(int C, int D, int esize) { return C * D * esize <= 4096 ? 2 : 1; }

// Shared memory of the pass kernel (walk CTAs included when `walk`).
template <typename T, int D, int G>
static size_t pass_smem(int C, int k, int splits, int nslot, int n_levels, bool walk) {
    const int CH = chunk_cap(k, splits, C);
    const int nsw = slots_per_warp(C, D, (int)sizeof(T));
    const size_t sm = smem_layout(G, D, CH, k, C, C * k, gs_words(splits), nslot,
                                  kWarps * nsw * C * D * (int)sizeof(T))
                          .total;
    const size_t ws = walk ? ancestor_walk_smem(n_levels, D) : 0;
    return sm > ws ? sm : ws;
}

template <typename T, int D, int G, bool SW, bool FU>
static cudaError_t prepare_one(size_t sm, int SPL) {
    cudaError_t e = cudaFuncSetAttribute(pass_kernel<T, D, G, SW, FU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    if (SPL > 8)
        e = cudaFuncSetAttribute(pass_kernel<T, D, G, SW, FU>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}
template <typename T, int D, int G, bool SW>
static cudaError_t prepare_variant(size_t sm, int SPL) {
    cudaError_t e = prepare_one<T, D, G, SW, false>(sm, SPL);
    return e == cudaSuccess ? prepare_one<T, D, G, SW, true>(sm, SPL) : e;
}

template <typename T, int D, int G>
static cudaError_t prepare_impl(int SPL, int NS0, int C, int k) {
    if (NS0 != SPL) return cudaErrorInvalidValue;   // level 0 runs on the same cluster
    const size_t sm = pass_smem<T, D, G>(C, k, SPL, kMaxLevels * SPL + NS0, kMaxLevels, true);
    if (sm > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = prepare_variant<T, D, G, false>(sm, SPL);
    if constexpr (kSwzCapable<T, D>)
        if (e == cudaSuccess) e = prepare_variant<T, D, G, true>(sm, SPL);
    return e;
}

template <typename T, int D, int G, bool SW>
static cudaError_t select_attend_variant(const TreeView& tv, const WorkView& wv,
                                         const QueryView& qv, cudaStream_t s, const ProfHook* prof,
                                         const KVMaps* maps) {
    PassMaps pm = {};
    if (SW)
        for (int l = 0; l < tv.n_levels && l < kMapLevels; ++l) pm.m[l] = maps[l];
    const int CH = chunk_cap(tv.k, wv.SPL, tv.C);
    const int NA = tv.C * tv.k;
    const int nsw = slots_per_warp(tv.C, D, (int)sizeof(T));
    const unsigned units = (unsigned)(qv.nq * tv.Hkv);
    // with a pending ancestor walk, extra rows of CTAs (one CTA per sequence and KV head)
    const unsigned walk_rows = qv.walk ? (unsigned)((tv.B * tv.Hkv + wv.SPL - 1) / wv.SPL) : 0u;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)wv.SPL, units + walk_rows, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = pass_smem<T, D, G>(tv.C, tv.k, wv.SPL, wv.NSLOT, tv.n_levels, qv.walk != 0);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)wv.SPL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attribute();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    prof_mark(prof, 0, true, s);
    NvtxRange nv(qv.phase == 1 ? "recsa pass (levels >= 1)" : qv.phase == 2 ? "recsa pass (level 0)"
                 : "recsa pass");
    cudaError_t e = qv.knew != nullptr
                        ? cudaLaunchKernelEx(&cfg, pass_kernel<T, D, G, SW, true>, tv, wv, qv, pm, CH, NA, nsw)
                        : cudaLaunchKernelEx(&cfg, pass_kernel<T, D, G, SW, false>, tv, wv, qv, pm, CH, NA, nsw);
    prof_mark(prof, 0, false, s);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// maps: the tensor maps of every level when the tree stages through them (bf16,
// d = 128, C a multiple of 16, at most kMapLevels levels), else null.
template <typename T, int D, int G>
static cudaError_t select_attend_impl(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                      cudaStream_t s, const ProfHook* prof, const KVMaps* maps) {
    if constexpr (kSwzCapable<T, D>) {
        if (maps && tv.C % 16 == 0 && tv.n_levels <= kMapLevels)
            return select_attend_variant<T, D, G, true>(tv, wv, qv, s, prof, maps);
    }
    return select_attend_variant<T, D, G, false>(tv, wv, qv, s, prof, nullptr);
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
                                 int dtype, cudaStream_t s, const ProfHook* prof,
                                 const KVMaps* maps) {
    RECSA_DISPATCH_TDG(dtype, tv.D, tv.G, select_attend_impl, tv, wv, qv, s, prof, maps);
}

}  // namespace recsa

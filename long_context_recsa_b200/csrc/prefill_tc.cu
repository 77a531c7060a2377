// Tensor-core scoring of the first scored level for a chunk of prefill queries
// ("Hierarchical Selection", Eq.3: at that level every query's list is the node
// range [0..a_t], so a chunk of queries shares one candidate set up to its causal
// cut), sm_100a tcgen05.
//
//   logits[q][h][g][j] = scale * < R(a_t) q_g , R(j) K_j >
//
// is candidate-local RoPE ("Key Theoretical Insight"): entry j sits at list index
// j and the query at its own index a_t.  Per KV head this is one dense product
// A . B^T with A = the chunk's query heads rotated by R(a_t) (M = queries x G
// rows), B = the level's nodes rotated by R(j) (N = a_max + 1 rows), and K = d.
//
// Precision: the selection has to agree with an fp64 evaluation up to a 1e-5
// relative band, which a single tf32 or bf16 product cannot do.  Each operand is
// split as hi = tf32(x), lo = tf32(x - hi) (round to nearest), and three MMAs
// accumulate hi.hi + hi.lo + lo.hi in fp32; the dropped lo.lo term and the two
// roundings are about 2^-21 of each product.
//
// Staging: the split kernels write each operand as the exact shared-memory image
// that tcgen05 reads for a K-major operand with 128-byte swizzle (rows of 32 tf32
// = 128 bytes, the 16-byte chunk c of row r stored at chunk c ^ (r mod 8), 8-row
// groups 1024 bytes apart), one image per 32-wide K slice.  A plain bulk copy of
// an image into 1024-byte-aligned shared memory is then a valid operand, so no
// tensor map is involved.  No copy uses cluster multicast.
#include "recsa_internal.cuh"

namespace recsa {

namespace {

constexpr int kTileM = 128;   // query-head rows per tile (TMEM lanes)
constexpr int kTileN = 256;   // nodes per tile (TMEM fp32 columns)
constexpr int kKSlice = 32;   // tf32 elements per 128-byte row
constexpr uint32_t kImgA = kTileM * 128;   // bytes of one A slice image
constexpr uint32_t kImgB = kTileN * 128;   // bytes of one B slice image
constexpr uint32_t kStageBytes = 2 * kImgA + 2 * kImgB;   // hi and lo of A and B
constexpr int kStages = 2;
constexpr int kGemmThreads = 128;

// Byte offset of element e (0..31) of row r in a 128-byte-swizzled slice image.
__device__ __forceinline__ uint32_t sw128_offset(int r, int e) {
    const int chunk = e >> 2;
    return (uint32_t)r * 128u + ((uint32_t)((chunk ^ (r & 7)) << 4) | (uint32_t)((e & 3) << 2));
}

__device__ __forceinline__ uint32_t tf32_rna(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
    return y;
}

// Writes x as (hi, lo) tf32 words at word index idx of the two images.
__device__ __forceinline__ void put_split(uint32_t* hi, uint32_t* lo, size_t idx, float x) {
    const uint32_t h = tf32_rna(x);
    const float rem = x - __uint_as_float(h);   // exact: hi is x rounded to 11 bits
    hi[idx] = h;
    lo[idx] = tf32_rna(rem);
}

// ---------------------------------------------------------------------------
// tcgen05 / TMEM helpers (inline PTX)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B
// apart (stride byte offset), leading byte offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of kind::tf32: fp32 accumulator, tf32 A and B, both
// K-major, N and M as given.
__host__ __device__ constexpr uint32_t tf32_idesc(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                         uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t"
        "}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace

// ---------------------------------------------------------------------------
// operand split kernels: one warp per operand row
// ---------------------------------------------------------------------------

// A rows of KV head hh: row r = (query ql, head g) with r = ql * G + g, rotated by
// R(a_t) where a_t is the query's index in the level-lt list.  Rows past the
// chunk are zero.
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) tc_split_q_kernel(TreeView tv, WorkView wv, QueryView qv,
                                                         TcView tc, int lt) {
    constexpr int H = D / 2, PPL = H / 32, KS = D / kKSlice;
    const int row = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    const int rows_head = tc.MB * kTileM;
    if (row >= tv.Hkv * rows_head) return;
    const int hh = row / rows_head, r = row % rows_head;
    const int ql = r / G, g = r % G;
    float x1[PPL], x2[PPL];
    if (ql < qv.nq) {
        const int gq = qv.q_begin + ql;
        const int b = gq / qv.n_per_b;
        const int64_t t = qv.pos0 + (gq - (int64_t)b * qv.n_per_b);
        const int64_t p = apow(t, lt, tv.C, tv.lgC);
        const T* q = reinterpret_cast<const T*>(qv.q) + ((int64_t)gq * tv.Hq + hh * G + g) * D;
        const float2* cs = wv.rope + p * H;
#pragma unroll
        for (int i = 0; i < PPL; ++i) {
            const int j = lane + 32 * i;
            const float a = (float)q[j], c = (float)q[j + H];
            const float2 w = cs[j];
            x1[i] = a * w.x - c * w.y;
            x2[i] = a * w.y + c * w.x;
        }
    } else {
#pragma unroll
        for (int i = 0; i < PPL; ++i) { x1[i] = 0.f; x2[i] = 0.f; }
    }
    const int mb = r / kTileM, rr = r % kTileM;
    const size_t img0 = ((size_t)(hh * tc.MB + mb) * KS) * (kImgA / 4);
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
        const int j1 = lane + 32 * i, j2 = j1 + H;
        put_split(tc.a_hi, tc.a_lo, img0 + (j1 / kKSlice) * (kImgA / 4) + sw128_offset(rr, j1 % kKSlice) / 4, x1[i]);
        put_split(tc.a_hi, tc.a_lo, img0 + (j2 / kKSlice) * (kImgA / 4) + sw128_offset(rr, j2 % kKSlice) / 4, x2[i]);
    }
}

// B rows of KV head hh: node j of level lt of sequence b rotated by R(j); rows
// j >= n_nodes are zero.
template <typename T, int D>
__global__ void __launch_bounds__(256) tc_split_k_kernel(TreeView tv, WorkView wv, TcView tc, int b,
                                                         int lt, int n_nodes, int nb_used) {
    constexpr int H = D / 2, PPL = H / 32, KS = D / kKSlice;
    const int row = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    const int rows_head = nb_used * kTileN;
    if (row >= tv.Hkv * rows_head) return;
    const int hh = row / rows_head, j = row % rows_head;
    float x1[PPL], x2[PPL];
    if (j < n_nodes) {
        const T* kr = level_k<T>(tv, lt, b, hh) + (int64_t)j * D;
        const float2* cs = wv.rope + (int64_t)j * H;
#pragma unroll
        for (int i = 0; i < PPL; ++i) {
            const int e = lane + 32 * i;
            const float a = (float)kr[e], c = (float)kr[e + H];
            const float2 w = cs[e];
            x1[i] = a * w.x - c * w.y;
            x2[i] = a * w.y + c * w.x;
        }
    } else {
#pragma unroll
        for (int i = 0; i < PPL; ++i) { x1[i] = 0.f; x2[i] = 0.f; }
    }
    const int nb = j / kTileN, rr = j % kTileN;
    const size_t img0 = ((size_t)(hh * tc.NB + nb) * KS) * (kImgB / 4);
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
        const int e1 = lane + 32 * i, e2 = e1 + H;
        put_split(tc.b_hi, tc.b_lo, img0 + (e1 / kKSlice) * (kImgB / 4) + sw128_offset(rr, e1 % kKSlice) / 4, x1[i]);
        put_split(tc.b_hi, tc.b_lo, img0 + (e2 / kKSlice) * (kImgB / 4) + sw128_offset(rr, e2 % kKSlice) / 4, x2[i]);
    }
}

// ---------------------------------------------------------------------------
// the product: one CTA per (N tile, M tile, KV head), 4 warps.
//   warp 0 lane 0: stages the K slices (hi and lo of A and B) through a 2-deep
//                  ring of bulk copies completed on mbarriers;
//   warp 1 lane 0: issues the MMAs (3 per 8-wide K step) into one TMEM
//                  accumulator of 128 lanes x 256 fp32 columns and commits;
//   all 4 warps:   read their 32 TMEM lanes back and store scale * accumulator.
// Every wait is bounded; a timeout records RECSA_E_TIMEOUT, skips the remaining
// MMAs, still drains the copies it issued and frees TMEM before returning.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kGemmThreads, 1) tc_logits_kernel(TcView tc, WorkView wv, int Hkv,
                                                                    int G, int nq, float scale) {
    constexpr int KS = D / kKSlice;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* done = empty + kStages;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
    const int nb = blockIdx.x, mb = blockIdx.y, hh = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTileN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp == 0 && lane == 0) {
        const unsigned char* ah = reinterpret_cast<const unsigned char*>(tc.a_hi) + (size_t)(hh * tc.MB + mb) * KS * kImgA;
        const unsigned char* al = reinterpret_cast<const unsigned char*>(tc.a_lo) + (size_t)(hh * tc.MB + mb) * KS * kImgA;
        const unsigned char* bh = reinterpret_cast<const unsigned char*>(tc.b_hi) + (size_t)(hh * tc.NB + nb) * KS * kImgB;
        const unsigned char* bl = reinterpret_cast<const unsigned char*>(tc.b_lo) + (size_t)(hh * tc.NB + nb) * KS * kImgB;
        for (int c = 0; c < KS; ++c) {
            const int s = c % kStages;
            if (c >= kStages && !mbar_wait_bounded(&empty[s], (uint32_t)((c / kStages - 1) & 1), wv.status))
                break;   // the MMA side gave up; issue nothing more
            unsigned char* st = smem + s * kStageBytes;
            mbar_expect_tx(&full[s], kStageBytes);
            bulk_g2s(st, ah + (size_t)c * kImgA, kImgA, &full[s]);
            bulk_g2s(st + kImgA, al + (size_t)c * kImgA, kImgA, &full[s]);
            bulk_g2s(st + 2 * kImgA, bh + (size_t)c * kImgB, kImgB, &full[s]);
            bulk_g2s(st + 2 * kImgA + kImgB, bl + (size_t)c * kImgB, kImgB, &full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t idesc = tf32_idesc(kTileM, kTileN);
        bool ok = true;
        for (int c = 0; c < KS; ++c) {
            const int s = c % kStages;
            // wait even after a failure, so no copy is still landing when the CTA exits
            const bool got = mbar_wait_bounded(&full[s], (uint32_t)((c / kStages) & 1), wv.status);
            ok = ok && got;
            tc_fence_after();
            if (ok) {
                const uint32_t st = smem_u32(smem + s * kStageBytes);
#pragma unroll
                for (int kk = 0; kk < kKSlice / 8; ++kk) {
                    const uint64_t dah = sw128_desc(st + kk * 32);
                    const uint64_t dal = sw128_desc(st + kImgA + kk * 32);
                    const uint64_t dbh = sw128_desc(st + 2 * kImgA + kk * 32);
                    const uint64_t dbl = sw128_desc(st + 2 * kImgA + kImgB + kk * 32);
                    mma_tf32(tmem, dah, dbh, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                    mma_tf32(tmem, dah, dbl, idesc, 1u);
                    mma_tf32(tmem, dal, dbh, idesc, 1u);
                }
            }
            mma_commit(&empty[s]);   // the slot is free once these MMAs have read it
            if (!got) break;         // a copy never completed: stop here
        }
        mma_commit(done);
    }
    __syncwarp();
    const bool fin = mbar_wait_bounded(done, 0u, wv.status);
    tc_fence_after();

    // epilogue: TMEM lane = tile row, column = node within the tile
    const int rr = warp * 32 + lane;
    const int r = mb * kTileM + rr;
    const int ql = r / G, g = r % G;
    const bool valid = fin && ql < nq;
    float* dst = tc.logits + ((size_t)(ql * Hkv + hh) * G + g) * tc.npad + (size_t)nb * kTileN;
#pragma unroll 1
    for (int c0 = 0; c0 < kTileN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
        if (valid) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + c0 + i) =
                    make_float4(__uint_as_float(v[i]) * scale, __uint_as_float(v[i + 1]) * scale,
                                __uint_as_float(v[i + 2]) * scale, __uint_as_float(v[i + 3]) * scale);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTileN);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static size_t tc_smem_bytes() { return kStages * kStageBytes + 1024 + 64; }

template <int D>
static cudaError_t prepare_tc_impl() {
    return cudaFuncSetAttribute(tc_logits_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)tc_smem_bytes());
}

cudaError_t prepare_tc_kernels(int D) {
    if (D == 128) return prepare_tc_impl<128>();
    if (D == 64) return prepare_tc_impl<64>();
    return cudaErrorInvalidValue;
}

template <typename T, int D, int G>
static cudaError_t prefill_top_impl(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                    const TcView& tc, int lt, int64_t a_max, cudaStream_t s,
                                    const ProfHook* prof) {
    const int n_nodes = (int)(a_max + 1);
    const int nb_used = (n_nodes + kTileN - 1) / kTileN;
    const int mb_used = (qv.nq * G + kTileM - 1) / kTileM;
    if (nb_used > tc.NB || mb_used > tc.MB || qv.nq > tc.nsub) return cudaErrorInvalidValue;
    const int b = qv.q_begin / qv.n_per_b;
    {
        const int64_t threads = (int64_t)tv.Hkv * nb_used * kTileN * 32;
        tc_split_k_kernel<T, D><<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(tv, wv, tc, b, lt,
                                                                                  n_nodes, nb_used);
    }
    {
        const int64_t threads = (int64_t)tv.Hkv * tc.MB * kTileM * 32;
        tc_split_q_kernel<T, D, G><<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(tv, wv, qv, tc, lt);
    }
    // the split kernels lay B out with tc.NB images per head but fill only nb_used
    prof_mark(prof, -2, true, s);
    tc_logits_kernel<D><<<dim3((unsigned)nb_used, (unsigned)mb_used, (unsigned)tv.Hkv), kGemmThreads,
                          tc_smem_bytes(), s>>>(tc, wv, tv.Hkv, G, qv.nq, tv.scale);
    prof_mark(prof, -2, false, s);
    return cudaGetLastError();
}

cudaError_t launch_prefill_top_tc(const TreeView& tv, const WorkView& wv, const QueryView& qv,
                                  const TcView& tc, int lt, int64_t a_max, int dtype, cudaStream_t s,
                                  const ProfHook* prof) {
    NvtxRange nv("recsa prefill top-level product");
#define RECSA_TC_G(T, D)                                                       \
    do {                                                                       \
        if (tv.G == 1) return prefill_top_impl<T, D, 1>(tv, wv, qv, tc, lt, a_max, s, prof); \
        if (tv.G == 2) return prefill_top_impl<T, D, 2>(tv, wv, qv, tc, lt, a_max, s, prof); \
        if (tv.G == 4) return prefill_top_impl<T, D, 4>(tv, wv, qv, tc, lt, a_max, s, prof); \
        if (tv.G == 8) return prefill_top_impl<T, D, 8>(tv, wv, qv, tc, lt, a_max, s, prof); \
    } while (0)
    if (dtype == RECSA_BF16 && tv.D == 128) RECSA_TC_G(__nv_bfloat16, 128);
    if (dtype == RECSA_BF16 && tv.D == 64) RECSA_TC_G(__nv_bfloat16, 64);
    if (dtype == RECSA_F32 && tv.D == 128) RECSA_TC_G(float, 128);
    if (dtype == RECSA_F32 && tv.D == 64) RECSA_TC_G(float, 64);
#undef RECSA_TC_G
    return cudaErrorInvalidValue;
}

}  // namespace recsa

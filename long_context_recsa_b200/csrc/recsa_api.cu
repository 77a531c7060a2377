// Host side of the RecSA C ABI: argument checks, buffer layout, kernel dispatch.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "recsa_internal.cuh"

namespace recsa {

constexpr int kSplits = 8;    // CTAs (one thread-block cluster) per unit, levels >= 1
constexpr int kSplits0 = 8;   // CTAs per unit at level 0
constexpr int kTcMinQueries = 128;   // trees with this many queries get the tensor-core path
constexpr int kTcQueries = 128;      // prefill rows per tensor-core product
constexpr int kTcMinRows = 32;       // smaller groups are scored per row

struct Layout {
    int esize, D, G;
    int n_levels;
    int64_t rows[kMaxLevels];
    int64_t off_k[kMaxLevels], off_v[kMaxLevels];
    size_t level_bytes;
    int NL, SPL, NS0, NSLOT;
    size_t o_status, o_lens, o_done, o_alpha, o_rope, o_sel, o_cnt, o_part, o_ucnt, ws_bytes;
    // tensor-core prefill buffers (tc_nsub == 0: disabled)
    int tc_nsub, tc_npad, tc_MB, tc_NB;
    size_t o_tca_hi, o_tca_lo, o_tcb_hi, o_tcb_lo, o_tclog;
};

static size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

static recsa_status check_config(const recsa_config* c) {
    if (!c) return RECSA_E_INVAL;
    if (c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->n_q_heads % c->n_kv_heads) return RECSA_E_INVAL;
    if (c->C < 2 || c->k < 1) return RECSA_E_INVAL;
    if (c->dtype != RECSA_F32 && c->dtype != RECSA_BF16) return RECSA_E_INVAL;
    if (!(c->rope_base > 1.0) || !isfinite(c->rope_base)) return RECSA_E_INVAL;
    if (!(c->scale >= 0.0f) || !isfinite(c->scale)) return RECSA_E_INVAL;
    if (c->head_dim != 64 && c->head_dim != 128) return RECSA_E_UNSUPPORTED;
    const int G = c->n_q_heads / c->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return RECSA_E_UNSUPPORTED;
    if (c->C > RECSA_MAX_C || c->k > 512 || (int64_t)c->C * c->k > 8192) return RECSA_E_UNSUPPORTED;
    for (int i = 0; i < c->C; ++i)
        if (!isfinite(c->pooler_w[i])) return RECSA_E_INVAL;
    return RECSA_OK;
}

static recsa_status compute_layout(const recsa_config* c, int64_t cap, int B, int Qmax, Layout* L) {
    recsa_status st = check_config(c);
    if (st != RECSA_OK) return st;
    if (cap < 1 || cap > ((int64_t)1 << 40)) return RECSA_E_INVAL;
    if (B < 1 || B > RECSA_MAX_BATCH) return RECSA_E_INVAL;
    if (Qmax < B || Qmax > (1 << 20)) return RECSA_E_INVAL;
    memset(L, 0, sizeof(*L));
    L->esize = c->dtype == RECSA_BF16 ? 2 : 4;
    L->D = c->head_dim;
    L->G = c->n_q_heads / c->n_kv_heads;
    const int Hkv = c->n_kv_heads;
    L->rows[0] = cap;
    int n = 1;
    while (L->rows[n - 1] > 1) {
        if (n >= kMaxLevels - 2) return RECSA_E_UNSUPPORTED;
        L->rows[n] = (L->rows[n - 1] + c->C - 1) / c->C;
        ++n;
    }
    L->n_levels = n;
    size_t o = 0;
    for (int l = 1; l < n; ++l) {
        const size_t bytes = al256((size_t)B * Hkv * L->rows[l] * L->D * L->esize);
        L->off_k[l] = (int64_t)o;
        o += bytes;
        L->off_v[l] = (int64_t)o;
        o += bytes;
    }
    L->level_bytes = o > 0 ? o : 256;
    // highest level any position t < cap can score: floor(t / C^l) >= k
    int NL = 0;
    {
        int64_t p = cap - 1;
        int l = 0;
        while (p > 0) {
            p /= c->C;
            ++l;
            if (p >= c->k) NL = l;
        }
    }
    L->NL = NL;
    L->SPL = kSplits;
    L->NS0 = kSplits0;
    L->NSLOT = NL * L->SPL + L->NS0;
    const int ck = c->C * c->k;
    size_t w = 0;
    L->o_status = w; w = al256(w + 64);
    L->o_lens = w;   w = al256(w + sizeof(int64_t) * B);
    L->o_done = w;   w = al256(w + sizeof(uint32_t) * B);
    L->o_alpha = w;  w = al256(w + sizeof(double) * RECSA_MAX_C * RECSA_MAX_C);
    L->o_rope = w;   w = al256(w + sizeof(float2) * (size_t)ck * (L->D / 2));
    L->o_sel = w;    w = al256(w + sizeof(int32_t) * (size_t)Qmax * Hkv * (NL > 0 ? NL : 1) * c->k);
    L->o_cnt = w;    w = al256(w + sizeof(int32_t) * (size_t)Qmax * Hkv * (NL + 1));
    L->o_part = w;   w = al256(w + sizeof(float) * (size_t)Qmax * Hkv * L->NSLOT * L->G * (L->D + 2));
    L->o_ucnt = w;   w = al256(w + sizeof(uint32_t) * (size_t)Qmax * Hkv);
    // tensor-core prefill: trees meant for chunks of queries (max_queries >= 128)
    L->tc_nsub = 0;
    L->o_tca_hi = L->o_tca_lo = L->o_tcb_hi = L->o_tcb_lo = L->o_tclog = 0;
    if (Qmax >= kTcMinQueries && NL >= 1 && (L->D == 64 || L->D == 128)) {
        const int nsub = kTcQueries < Qmax ? kTcQueries : Qmax;
        L->tc_nsub = nsub;
        L->tc_MB = (nsub * L->G + 127) / 128;
        L->tc_NB = (ck + 255) / 256;
        L->tc_npad = L->tc_NB * 256;
        const size_t a_img = (size_t)Hkv * L->tc_MB * (L->D / 32) * 128 * 128;
        const size_t b_img = (size_t)Hkv * L->tc_NB * (L->D / 32) * 256 * 128;
        w = (w + 1023) & ~size_t(1023);
        L->o_tca_hi = w; w = al256(w + a_img);
        L->o_tca_lo = w; w = al256(w + a_img);
        L->o_tcb_hi = w; w = al256(w + b_img);
        L->o_tcb_lo = w; w = al256(w + b_img);
        L->o_tclog = w;  w = al256(w + sizeof(float) * (size_t)nsub * Hkv * L->G * L->tc_npad);
    }
    L->ws_bytes = w;
    return RECSA_OK;
}

// Tree and workspace views over caller buffers and a scratch base `ws`, without a
// tree handle (used by recsa_decode_noalloc).  Same layout as recsa_tree_init.
// With ws == nullptr only *ws_bytes is computed.
recsa_status views_for(const recsa_config* cfg, int64_t cap, int B, int Qmax, const void* k0,
                       const void* v0, const int64_t strides[3], const void* levels,
                       size_t level_bytes, char* ws, size_t* ws_bytes, TreeView* tv,
                       WorkView* wv) {
    Layout L;
    recsa_status st = compute_layout(cfg, cap, B, Qmax, &L);
    if (st != RECSA_OK) return st;
    *ws_bytes = L.ws_bytes;
    if (ws == nullptr) return RECSA_OK;
    if (!k0 || !v0 || !strides || !levels) return RECSA_E_INVAL;
    if ((((uintptr_t)k0) & 15u) || (((uintptr_t)v0) & 15u) || (((uintptr_t)levels) & 255u))
        return RECSA_E_INVAL;
    const int64_t per16 = 16 / L.esize;
    if (strides[0] < 0 || strides[1] < 0 || strides[2] < L.D) return RECSA_E_INVAL;
    if (strides[0] % per16 || strides[1] % per16 || strides[2] % per16) return RECSA_E_INVAL;
    if (level_bytes < L.level_bytes) return RECSA_E_CAPACITY;
    memset(tv, 0, sizeof(*tv));
    memset(wv, 0, sizeof(*wv));
    tv->k0 = k0; tv->v0 = v0; tv->k0w = nullptr; tv->v0w = nullptr;
    tv->s_b = strides[0]; tv->s_h = strides[1]; tv->s_t = strides[2];
    tv->levels = (char*)levels;
    for (int l = 0; l < kMaxLevels; ++l) {
        tv->off_k[l] = L.off_k[l];
        tv->off_v[l] = L.off_v[l];
        tv->rows[l] = L.rows[l];
    }
    tv->B = B;
    tv->Hkv = cfg->n_kv_heads;
    tv->Hq = cfg->n_q_heads;
    tv->G = L.G;
    tv->D = L.D;
    tv->C = cfg->C;
    tv->k = cfg->k;
    tv->lgC = (cfg->C & (cfg->C - 1)) == 0 ? __builtin_ctz((unsigned)cfg->C) : -1;
    tv->n_levels = L.n_levels;
    tv->cap = cap;
    tv->scale = cfg->scale > 0.0f ? cfg->scale : (float)(1.0 / sqrt((double)L.D));
    tv->rope_base = cfg->rope_base;
    for (int i = 0; i < RECSA_MAX_C; ++i) tv->w[i] = i < cfg->C ? cfg->pooler_w[i] : 0.0f;
    wv->status = (uint32_t*)(ws + L.o_status);
    wv->lens = (int64_t*)(ws + L.o_lens);
    wv->done = (uint32_t*)(ws + L.o_done);
    wv->alpha = (const double*)(ws + L.o_alpha);
    wv->rope = (const float2*)(ws + L.o_rope);
    wv->sel = (int32_t*)(ws + L.o_sel);
    wv->cnt = (int32_t*)(ws + L.o_cnt);
    wv->part = (float*)(ws + L.o_part);
    wv->ucnt = (uint32_t*)(ws + L.o_ucnt);
    wv->nunits = Qmax * cfg->n_kv_heads;
    wv->NL = L.NL;
    wv->SPL = L.SPL;
    wv->NS0 = L.NS0;
    wv->NSLOT = L.NSLOT;
    wv->ck = cfg->C * cfg->k;
    return RECSA_OK;
}

}  // namespace recsa

using namespace recsa;

struct recsa_tree {
    recsa_config cfg;
    Layout L;
    int64_t cap;
    int B, Qmax;
    TreeView tv;
    WorkView wv;
    int64_t host_len[RECSA_MAX_BATCH];
    ProfHook prof;
    TcView tc;                 // tensor-core prefill buffers (tc.nsub == 0: none)
    KVMaps maps[kMaxLevels];   // swizzled TMA maps of every level (bf16, d = 128 trees)
    bool has_maps;
    // a single-token append left the ancestors of the new tokens to re-pool: the next
    // decode does it in its level-0 launch, any other call first
    bool walk_pending;
    // Eq.5 gated key pooler in place of the stand-in (recsa_tree_set_gated_pooler)
    bool gated;
    GatedView gv;
    // level 0 in pinned host memory (tv.l0_host): decode stages each query's level-0
    // list in this device buffer (recsa_tree_set_offload_staging)
    char* stage;
    size_t stage_bytes;
    KVMaps stage_map;
    bool has_stage_map;
};

namespace recsa {
cudaError_t encode_stage_map(const void* base, int64_t rows, int Hkv, int nq, int C, CUtensorMap* m);
}  // namespace recsa

// Where a level-0 buffer lives: 1 pinned host memory (its device address in *dev),
// 0 device memory, -1 memory the GPU cannot read (pageable host memory).
static int level0_residence(const void* p, const void** dev) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    if (a.type == cudaMemoryTypeHost) {
        if (!a.devicePointer) return -1;
        *dev = a.devicePointer;
        return 1;
    }
    if (a.type == cudaMemoryTypeUnregistered) return -1;
    *dev = p;
    return 0;
}

// Runs a pending ancestor re-pooling on `stream` (before a call that needs the
// complete tree).
static recsa_status finish_walk(recsa_tree* t, cudaStream_t stream) {
    if (!t->walk_pending) return RECSA_OK;
    t->walk_pending = false;
    return launch_append_walk(t->tv, t->wv, t->cfg.dtype, stream) == cudaSuccess ? RECSA_OK
                                                                                 : RECSA_E_CUDA;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }


namespace recsa {
// tree_kernels.cu: the bounded-wait self-test kernel
cudaError_t launch_bounded_wait_probe(uint32_t* status, cudaStream_t s);
}  // namespace recsa

extern "C" {

const char* recsa_status_str(recsa_status s) {
    switch (s) {
        case RECSA_OK: return "ok";
        case RECSA_E_INVAL: return "invalid argument";
        case RECSA_E_UNSUPPORTED: return "unsupported configuration";
        case RECSA_E_CAPACITY: return "capacity exceeded or buffer too small";
        case RECSA_E_CUDA: return "CUDA error";
        case RECSA_E_TIMEOUT: return "device wait timed out";
        case RECSA_E_DEVICE: return "device-side check failed";
    }
    return "unknown status";
}

recsa_status recsa_query_sizes(const recsa_config* cfg, int64_t capacity, int32_t batch,
                               int32_t max_queries, size_t* level_bytes, size_t* workspace_bytes,
                               int32_t* n_levels) {
    Layout L;
    recsa_status st = compute_layout(cfg, capacity, batch, max_queries, &L);
    if (st != RECSA_OK) return st;
    if (level_bytes) *level_bytes = L.level_bytes;
    if (workspace_bytes) *workspace_bytes = L.ws_bytes;
    if (n_levels) *n_levels = L.n_levels;
    return RECSA_OK;
}

recsa_status recsa_tree_init(const recsa_config* cfg, int64_t capacity, int32_t batch,
                             int32_t max_queries, void* k0, void* v0, const int64_t kv_strides[3],
                             void* levels, size_t level_bytes, void* workspace,
                             size_t workspace_bytes, void* stream, recsa_tree** out) {
    if (!out) return RECSA_E_INVAL;
    *out = nullptr;
    Layout L;
    recsa_status st = compute_layout(cfg, capacity, batch, max_queries, &L);
    if (st != RECSA_OK) return st;
    if (!k0 || !v0 || !kv_strides || !levels || !workspace) return RECSA_E_INVAL;
    if (!aligned16(k0) || !aligned16(v0)) return RECSA_E_INVAL;
    if (((uintptr_t)levels & 255u) || ((uintptr_t)workspace & 255u)) return RECSA_E_INVAL;
    const int64_t sb = kv_strides[0], sh = kv_strides[1], stt = kv_strides[2];
    const int64_t per16 = 16 / L.esize;
    if (sb < 0 || sh < 0 || stt < L.D) return RECSA_E_INVAL;
    if (sb % per16 || sh % per16 || stt % per16) return RECSA_E_INVAL;
    if (level_bytes < L.level_bytes || workspace_bytes < L.ws_bytes) return RECSA_E_CAPACITY;

    const void *k0d = nullptr, *v0d = nullptr;
    const int rk = level0_residence(k0, &k0d), rv = level0_residence(v0, &v0d);
    if (rk < 0 || rv < 0 || rk != rv) return RECSA_E_INVAL;
    recsa_tree* t = (recsa_tree*)calloc(1, sizeof(recsa_tree));
    if (!t) return RECSA_E_INVAL;
    t->cfg = *cfg;
    t->L = L;
    t->cap = capacity;
    t->B = batch;
    t->Qmax = max_queries;
    TreeView& tv = t->tv;
    tv.k0 = k0d; tv.v0 = v0d; tv.k0w = const_cast<void*>(k0d); tv.v0w = const_cast<void*>(v0d);
    tv.l0_host = rk;
    tv.s_b = sb; tv.s_h = sh; tv.s_t = stt;
    tv.levels = (char*)levels;
    for (int l = 0; l < kMaxLevels; ++l) {
        tv.off_k[l] = L.off_k[l];
        tv.off_v[l] = L.off_v[l];
        tv.rows[l] = L.rows[l];
    }
    tv.B = batch;
    tv.Hkv = cfg->n_kv_heads;
    tv.Hq = cfg->n_q_heads;
    tv.G = L.G;
    tv.D = L.D;
    tv.C = cfg->C;
    tv.k = cfg->k;
    tv.lgC = (cfg->C & (cfg->C - 1)) == 0 ? __builtin_ctz((unsigned)cfg->C) : -1;
    tv.n_levels = L.n_levels;
    tv.cap = capacity;
    tv.scale = cfg->scale > 0.0f ? cfg->scale : (float)(1.0 / sqrt((double)L.D));
    tv.rope_base = cfg->rope_base;
    for (int i = 0; i < RECSA_MAX_C; ++i) tv.w[i] = i < cfg->C ? cfg->pooler_w[i] : 0.0f;
    WorkView& wv = t->wv;
    char* ws = (char*)workspace;
    wv.status = (uint32_t*)(ws + L.o_status);
    wv.lens = (int64_t*)(ws + L.o_lens);
    wv.done = (uint32_t*)(ws + L.o_done);
    wv.alpha = (const double*)(ws + L.o_alpha);
    wv.rope = (const float2*)(ws + L.o_rope);
    wv.sel = (int32_t*)(ws + L.o_sel);
    wv.cnt = (int32_t*)(ws + L.o_cnt);
    wv.part = (float*)(ws + L.o_part);
    wv.ucnt = (uint32_t*)(ws + L.o_ucnt);
    wv.nunits = max_queries * cfg->n_kv_heads;
    wv.NL = L.NL;
    wv.SPL = L.SPL;
    wv.NS0 = L.NS0;
    wv.NSLOT = L.NSLOT;
    wv.ck = cfg->C * cfg->k;
    TcView& tc = t->tc;
    memset(&tc, 0, sizeof(tc));
    if (L.tc_nsub > 0) {
        tc.a_hi = (uint32_t*)(ws + L.o_tca_hi);
        tc.a_lo = (uint32_t*)(ws + L.o_tca_lo);
        tc.b_hi = (uint32_t*)(ws + L.o_tcb_hi);
        tc.b_lo = (uint32_t*)(ws + L.o_tcb_lo);
        tc.logits = (float*)(ws + L.o_tclog);
        tc.nsub = L.tc_nsub;
        tc.npad = L.tc_npad;
        tc.MB = L.tc_MB;
        tc.NB = L.tc_NB;
    }

    cudaError_t e = prepare_kernels(cfg->dtype, L.D, L.G, L.SPL, L.NS0, cfg->C, cfg->k);
    if (e == cudaSuccess) e = prepare_tree_kernels(tv, cfg->dtype);
    if (e == cudaSuccess && L.tc_nsub > 0) e = prepare_tc_kernels(L.D);
    // tables the tensor maps cannot describe (strides off 16 bytes) keep plain copies
    t->has_maps = e == cudaSuccess && uses_kv_maps(cfg->dtype, L.D, cfg->C) &&
                  encode_kv_maps(tv, t->maps) == cudaSuccess;
    if (e == cudaSuccess) e = launch_init_workspace(tv, wv, cfg->rope_base, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        free(t);
        return RECSA_E_CUDA;
    }
    *out = t;
    return RECSA_OK;
}

recsa_status recsa_build(recsa_tree* t, const int64_t* lengths, void* stream) {
    if (!t || !lengths) return RECSA_E_INVAL;
    for (int b = 0; b < t->B; ++b)
        if (lengths[b] < 0 || lengths[b] > t->cap) return RECSA_E_CAPACITY;
    t->walk_pending = false;   // the build pools every node anew
    cudaError_t e;
    if (t->gated) {
        e = launch_set_lengths(t->wv, lengths, t->B, (cudaStream_t)stream);
        if (e == cudaSuccess)
            e = launch_gated_levels(t->tv, t->wv, t->gv, 0, t->cfg.dtype, (cudaStream_t)stream);
    } else {
        e = launch_build(t->tv, t->wv, lengths, t->cfg.dtype, (cudaStream_t)stream);
    }
    if (e != cudaSuccess) return RECSA_E_CUDA;
    for (int b = 0; b < t->B; ++b) t->host_len[b] = lengths[b];
    return RECSA_OK;
}

recsa_status recsa_append(recsa_tree* t, const void* k_new, const void* v_new, int32_t n,
                          void* stream) {
    if (!t || !k_new || !v_new || n < 1) return RECSA_E_INVAL;
    if (!aligned16(k_new) || !aligned16(v_new)) return RECSA_E_INVAL;
    for (int b = 0; b < t->B; ++b)
        if (t->host_len[b] + n > t->cap) return RECSA_E_CAPACITY;
    const cudaStream_t s = (cudaStream_t)stream;
    if (finish_walk(t, s) != RECSA_OK) return RECSA_E_CUDA;
    cudaError_t e;
    if (t->gated) {
        // rows at the old lengths, every level's nodes over them, then the lengths
        e = launch_append_rows(t->tv, t->wv, k_new, v_new, n, t->cfg.dtype, s);
        if (e == cudaSuccess) e = launch_gated_levels(t->tv, t->wv, t->gv, n, t->cfg.dtype, s);
        if (e == cudaSuccess) e = launch_commit_lengths(t->wv, t->B, n, t->cap, s);
    } else if (n == 1) {
        e = launch_append_token(t->tv, t->wv, k_new, v_new, t->cfg.dtype, s, &t->prof);
        if (e == cudaSuccess) t->walk_pending = true;
    } else {
        e = launch_append(t->tv, t->wv, k_new, v_new, n, t->cfg.dtype, s, &t->prof);
    }
    if (e != cudaSuccess) return RECSA_E_CUDA;
    for (int b = 0; b < t->B; ++b) t->host_len[b] += n;
    return RECSA_OK;
}

recsa_status recsa_decode(recsa_tree* t, const void* q, void* out, int32_t* sel_out,
                          int32_t* counts_out, void* stream) {
    if (!t || !q || !out) return RECSA_E_INVAL;
    if (!aligned16(q) || !aligned16(out)) return RECSA_E_INVAL;
    QueryView qv = {};
    qv.q = q;
    qv.out = out;
    qv.sel_out = sel_out;
    qv.cnt_out = counts_out;
    qv.mode = 0;
    qv.n_per_b = 1;
    qv.pos0 = 0;
    qv.q_begin = 0;
    qv.nq = t->B;
    qv.walk = t->walk_pending ? 1 : 0;
    const cudaStream_t s = (cudaStream_t)stream;
    if (t->tv.l0_host) {
        // level 0 in host memory: levels >= 1, the gather of each query's level-0 list
        // into the staging buffer, then level 0 from there and the merge
        if (!t->stage) return RECSA_E_UNSUPPORTED;
        const size_t half = t->stage_bytes / 2;
        qv.phase = 1;
        cudaError_t e = launch_select_attend(t->tv, t->wv, qv, t->cfg.dtype, s, &t->prof,
                                             t->has_maps ? t->maps : nullptr);
        if (e == cudaSuccess)
            e = launch_gather_level0(t->tv, t->wv, qv, t->stage, t->stage + half, t->cfg.dtype, s);
        if (e != cudaSuccess) return RECSA_E_CUDA;
        t->walk_pending = false;
        qv.phase = 2;
        qv.walk = 0;
        qv.l0k = t->stage;
        qv.l0v = t->stage + half;
        KVMaps m2[kMaxLevels];
        const bool sw = t->has_maps && t->has_stage_map;
        if (sw) {
            memcpy(m2, t->maps, sizeof(m2));
            m2[0] = t->stage_map;
        }
        e = launch_select_attend(t->tv, t->wv, qv, t->cfg.dtype, s, &t->prof, sw ? m2 : nullptr);
        return e == cudaSuccess ? RECSA_OK : RECSA_E_CUDA;
    }
    cudaError_t e =
        launch_select_attend(t->tv, t->wv, qv, t->cfg.dtype, s, &t->prof,
                             t->has_maps ? t->maps : nullptr);
    if (e != cudaSuccess) return RECSA_E_CUDA;
    t->walk_pending = false;
    return RECSA_OK;
}

recsa_status recsa_append_decode(recsa_tree* t, const void* k_new, const void* v_new,
                                 const void* q, void* out, int32_t* sel_out, int32_t* counts_out,
                                 void* stream) {
    if (!t || !k_new || !v_new || !q || !out) return RECSA_E_INVAL;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(q) || !aligned16(out))
        return RECSA_E_INVAL;
    // the separate calls serve the gated pooler and level 0 in host memory
    if (t->gated || t->tv.l0_host) return RECSA_E_UNSUPPORTED;
    for (int b = 0; b < t->B; ++b)
        if (t->host_len[b] + 1 > t->cap) return RECSA_E_CAPACITY;
    const cudaStream_t s = (cudaStream_t)stream;
    if (finish_walk(t, s) != RECSA_OK) return RECSA_E_CUDA;   // an earlier append's walk
    QueryView qv = {};
    qv.q = q;
    qv.out = out;
    qv.sel_out = sel_out;
    qv.cnt_out = counts_out;
    qv.mode = 0;
    qv.n_per_b = 1;
    qv.nq = t->B;
    qv.walk = 1;   // the walk CTAs write the token's rows and re-pool its ancestors
    qv.knew = k_new;
    qv.vnew = v_new;
    cudaError_t e = launch_select_attend(t->tv, t->wv, qv, t->cfg.dtype, s, &t->prof,
                                         t->has_maps ? t->maps : nullptr);
    if (e != cudaSuccess) return RECSA_E_CUDA;
    for (int b = 0; b < t->B; ++b) t->host_len[b] += 1;
    return RECSA_OK;
}

// t / C^l and the first scored level of position t (host side of Eq.3's sizes).
static int64_t host_apow(int64_t t, int l, int C) {
    for (int i = 0; i < l; ++i) t /= C;
    return t;
}
static int host_first_scored_level(int64_t t, int C, int k) {
    int lstar = 0, l = 0;
    for (int64_t p = t; p > 0 && l + 1 < kMaxLevels;) {
        p /= C;
        ++l;
        if (p >= k) lstar = l;
    }
    return lstar;
}

recsa_status recsa_prefill_chunk(recsa_tree* t, const void* Q, int64_t pos0, int32_t n, void* O,
                                 int32_t* sel_out, int32_t* counts_out, void* stream) {
    if (!t || !Q || !O || n < 1 || pos0 < 0) return RECSA_E_INVAL;
    if (!aligned16(Q) || !aligned16(O)) return RECSA_E_INVAL;
    if (t->tv.l0_host) return RECSA_E_UNSUPPORTED;   // offloaded level 0: decode only
    for (int b = 0; b < t->B; ++b)
        if (pos0 + n > t->host_len[b]) return RECSA_E_CAPACITY;
    const cudaStream_t s = (cudaStream_t)stream;
    if (finish_walk(t, s) != RECSA_OK) return RECSA_E_CUDA;
    auto base_view = [&]() {
        QueryView qv = {};
        qv.q = Q;
        qv.out = O;
        qv.sel_out = sel_out;
        qv.cnt_out = counts_out;
        qv.mode = 1;
        qv.n_per_b = n;
        qv.pos0 = pos0;
        return qv;
    };
    if (t->tc.nsub > 0 && n >= kTcMinRows) {
        // per sequence, groups of up to tc.nsub rows: the group's first scored level
        // comes from one tensor-core product, the levels below from the row kernels
        for (int b = 0; b < t->B; ++b) {
            for (int i0 = 0; i0 < n; i0 += t->tc.nsub) {
                const int cnt = n - i0 < t->tc.nsub ? n - i0 : t->tc.nsub;
                QueryView qv = base_view();
                qv.q_begin = b * n + i0;
                qv.nq = cnt;
                const int64_t t_last = pos0 + i0 + cnt - 1;
                const int lt = host_first_scored_level(t_last, t->cfg.C, t->cfg.k);
                if (lt >= 1 && cnt >= kTcMinRows) {
                    cudaError_t e = launch_prefill_top_tc(t->tv, t->wv, qv, t->tc, lt,
                                                          host_apow(t_last, lt, t->cfg.C),
                                                          t->cfg.dtype, s, &t->prof);
                    if (e != cudaSuccess) return RECSA_E_CUDA;
                    qv.pre = t->tc.logits;
                    qv.pre_level = lt;
                    qv.pre_stride = t->tc.npad;
                }
                cudaError_t e = launch_select_attend(t->tv, t->wv, qv, t->cfg.dtype, s, &t->prof,
                                                     t->has_maps ? t->maps : nullptr);
                if (e != cudaSuccess) return RECSA_E_CUDA;
            }
        }
        return RECSA_OK;
    }
    const int total = t->B * n;
    for (int q0 = 0; q0 < total; q0 += t->Qmax) {
        QueryView qv = base_view();
        qv.q_begin = q0;
        qv.nq = total - q0 < t->Qmax ? total - q0 : t->Qmax;
        cudaError_t e = launch_select_attend(t->tv, t->wv, qv, t->cfg.dtype, s, &t->prof,
                                                     t->has_maps ? t->maps : nullptr);
        if (e != cudaSuccess) return RECSA_E_CUDA;
    }
    return RECSA_OK;
}

recsa_status recsa_offload_staging_bytes(const recsa_config* cfg, int32_t batch, size_t* bytes) {
    recsa_status st = check_config(cfg);
    if (st != RECSA_OK) return st;
    if (!bytes || batch < 1 || batch > RECSA_MAX_BATCH) return RECSA_E_INVAL;
    const size_t es = cfg->dtype == RECSA_BF16 ? 2 : 4;
    *bytes = 2 * (size_t)batch * cfg->n_kv_heads * (size_t)cfg->C * cfg->k * cfg->head_dim * es;
    return RECSA_OK;
}

recsa_status recsa_tree_set_offload_staging(recsa_tree* t, void* staging, size_t bytes) {
    if (!t) return RECSA_E_INVAL;
    if (!t->tv.l0_host) return RECSA_E_UNSUPPORTED;   // level 0 is already in device memory
    size_t need = 0;
    recsa_status st = recsa_offload_staging_bytes(&t->cfg, t->B, &need);
    if (st != RECSA_OK) return st;
    if (!staging || ((uintptr_t)staging & 255u)) return RECSA_E_INVAL;
    if (bytes < need) return RECSA_E_CAPACITY;
    const void* d = nullptr;
    if (level0_residence(staging, &d) != 0) return RECSA_E_INVAL;   // must be device memory
    t->stage = (char*)staging;
    t->stage_bytes = need;
    t->has_stage_map = false;
    if (t->has_maps) {
        const size_t half = need / 2;
        t->has_stage_map =
            encode_stage_map(t->stage, t->wv.ck, t->tv.Hkv, t->B, t->tv.C, &t->stage_map.k) ==
                cudaSuccess &&
            encode_stage_map(t->stage + half, t->wv.ck, t->tv.Hkv, t->B, t->tv.C,
                             &t->stage_map.v) == cudaSuccess;
        if (!t->has_stage_map) return RECSA_E_CUDA;
    }
    return RECSA_OK;
}

recsa_status recsa_tree_set_gated_pooler(recsa_tree* t, const recsa_gated_pooler* p) {
    if (!t) return RECSA_E_INVAL;
    if (p == nullptr) {
        t->gated = false;
        return RECSA_OK;
    }
    if (!p->w || !p->W1t || !p->b1 || !p->W2t) return RECSA_E_INVAL;
    if ((((uintptr_t)p->w) | ((uintptr_t)p->W1t) | ((uintptr_t)p->b1) | ((uintptr_t)p->W2t)) & 7u)
        return RECSA_E_INVAL;
    if (p->hidden < 1) return RECSA_E_INVAL;
    if (p->hidden > kGatedMaxHidden) return RECSA_E_UNSUPPORTED;
    if (!isfinite(p->tau) || !isfinite(p->g) || !isfinite(p->rho) || p->rho == 0.0)
        return RECSA_E_INVAL;
    t->walk_pending = false;   // (a pending stand-in walk is dropped: rebuild after switching)
    t->gv.h = p->hidden;
    t->gv.tau = p->tau;
    t->gv.g = p->g;
    t->gv.rho = p->rho;
    t->gv.w = p->w;
    t->gv.W1t = p->W1t;
    t->gv.b1 = p->b1;
    t->gv.W2t = p->W2t;
    t->gated = true;
    return RECSA_OK;
}

recsa_status recsa_get_status(recsa_tree* t, void* stream) {
    if (!t) return RECSA_E_INVAL;
    const cudaStream_t s = (cudaStream_t)stream;
    if (finish_walk(t, s) != RECSA_OK) return RECSA_E_CUDA;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, t->wv.status, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return RECSA_E_CUDA;
    if (v != 0 && (cudaMemsetAsync(t->wv.status, 0, sizeof(v), s) != cudaSuccess ||
                   cudaStreamSynchronize(s) != cudaSuccess))
        return RECSA_E_CUDA;
    switch (v) {
        case kStatusOk: return RECSA_OK;
        case kStatusCapacity: return RECSA_E_CAPACITY;
        case kStatusTimeout: return RECSA_E_TIMEOUT;
        default: return RECSA_E_DEVICE;
    }
}

recsa_status recsa_probe_bounded_wait(uint32_t* status_dev, void* stream) {
    if (!status_dev) return RECSA_E_INVAL;
    const cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(status_dev, 0, sizeof(uint32_t), s) != cudaSuccess) return RECSA_E_CUDA;
    if (launch_bounded_wait_probe(status_dev, s) != cudaSuccess) return RECSA_E_CUDA;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, status_dev, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return RECSA_E_CUDA;
    return v == kStatusTimeout ? RECSA_E_TIMEOUT : RECSA_OK;
}

recsa_status recsa_tree_info(const recsa_tree* t, recsa_tree_info_t* info) {
    if (!t || !info) return RECSA_E_INVAL;
    info->n_levels = t->L.n_levels;
    info->n_sel_levels = t->L.NL;
    info->splits = t->L.SPL;
    info->splits0 = t->L.NS0;
    info->capacity = t->cap;
    info->batch = t->B;
    info->max_queries = t->Qmax;
    info->tc_queries = t->tc.nsub;
    info->tc_row_stride = t->tc.npad;
    info->tc_logits_offset = t->tc.nsub ? (int64_t)t->L.o_tclog : 0;
    return RECSA_OK;
}

recsa_status recsa_level_info(const recsa_tree* t, int32_t level, int64_t* k_offset,
                              int64_t* v_offset, int64_t* rows) {
    if (!t || level < 1 || level >= t->L.n_levels) return RECSA_E_INVAL;
    if (k_offset) *k_offset = t->L.off_k[level];
    if (v_offset) *v_offset = t->L.off_v[level];
    if (rows) *rows = t->L.rows[level];
    return RECSA_OK;
}

recsa_status recsa_host_lengths(const recsa_tree* t, int64_t* lengths) {
    if (!t || !lengths) return RECSA_E_INVAL;
    for (int b = 0; b < t->B; ++b) lengths[b] = t->host_len[b];
    return RECSA_OK;
}

recsa_status recsa_set_profile_events(recsa_tree* t, int32_t which, void* start, void* stop) {
    if (!t || ((start == nullptr) != (stop == nullptr))) return RECSA_E_INVAL;
    if (start != nullptr && (which < -2 || which > t->L.NL)) return RECSA_E_INVAL;
    t->prof.which = start ? which : -100;
    t->prof.start = (cudaEvent_t)start;
    t->prof.stop = (cudaEvent_t)stop;
    return RECSA_OK;
}

recsa_status recsa_tree_free(recsa_tree* t) {
    if (!t) return RECSA_E_INVAL;
    free(t);
    return RECSA_OK;
}

}  // extern "C"

// ----------------------------------------------------------------------------
// TMA tensor maps of the level tables (see KVMaps)
// ----------------------------------------------------------------------------
namespace recsa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// One table: rows of 128 bf16 at row pitch `row_b` bytes, heads `head_b`, sequences
// `seq_b` apart; boxes of 64 dims x C rows.
static cudaError_t encode_table(CUtensorMap* m, const void* base, int64_t rows, int Hkv, int B,
                                int64_t row_b, int64_t head_b, int64_t seq_b, int C) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (rows >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;   // row coordinates are int32
    const cuuint64_t dims[4] = {128, (cuuint64_t)rows, (cuuint64_t)Hkv, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)row_b, (cuuint64_t)head_b, (cuuint64_t)seq_b};
    const cuuint32_t box[4] = {64, (cuuint32_t)C, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_stage_map(const void* base, int64_t rows, int Hkv, int nq, int C, CUtensorMap* m) {
    return encode_table(m, base, rows, Hkv, nq, 256, rows * 256, rows * 256 * Hkv, C);
}

cudaError_t encode_kv_maps(const TreeView& tv, KVMaps* maps) {
    for (int l = 0; l < tv.n_levels && l < kMaxLevels; ++l) {
        cudaError_t e;
        if (l == 0 && tv.l0_host) {
            // a host-resident level 0 is never staged by TMA (decode stages it through
            // the gather into a device buffer with its own map)
            memset(&maps[0], 0, sizeof(maps[0]));
            continue;
        }
        if (l == 0) {
            const int64_t es = 2;
            e = encode_table(&maps[0].k, tv.k0, tv.cap, tv.Hkv, tv.B, tv.s_t * es, tv.s_h * es,
                             tv.s_b * es, tv.C);
            if (e == cudaSuccess)
                e = encode_table(&maps[0].v, tv.v0, tv.cap, tv.Hkv, tv.B, tv.s_t * es,
                                 tv.s_h * es, tv.s_b * es, tv.C);
        } else {
            const int64_t rows = tv.rows[l], row_b = 256;
            e = encode_table(&maps[l].k, tv.levels + tv.off_k[l], rows, tv.Hkv, tv.B, row_b,
                             rows * row_b, rows * row_b * tv.Hkv, tv.C);
            if (e == cudaSuccess)
                e = encode_table(&maps[l].v, tv.levels + tv.off_v[l], rows, tv.Hkv, tv.B, row_b,
                                 rows * row_b, rows * row_b * tv.Hkv, tv.C);
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace recsa

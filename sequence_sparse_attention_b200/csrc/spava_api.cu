// spava_api.cu -- the C ABI (include/spava.h): argument checks, the plan of work
// items, TMA descriptors, workspace layout and kernel launches.  Every step of
// the computation runs in the kernels; this file only prepares and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/spava.h"
#include "attn_kernel.cuh"
#include "plan.cuh"
#include "score_kernel.cuh"
#include "select_kernels.cuh"
#include "shard_kernels.cuh"

using namespace spava;

namespace {

thread_local int32_t g_last_cuda_error = 0;

spava_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = static_cast<int32_t>(e);
    return SPAVA_ERR_CUDA;
}

spava_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? SPAVA_OK : cuda_fail(e); }

#define SPAVA_CUDA(...)                                    \
    do {                                                   \
        cudaError_t e_ = (__VA_ARGS__);                           \
        if (e_ != cudaSuccess) return cuda_fail(e_);       \
    } while (0)

#define SPAVA_TRY(...)                                     \
    do {                                                   \
        spava_status s_ = (__VA_ARGS__);                          \
        if (s_ != SPAVA_OK) return s_;                     \
    } while (0)

// ---------------------------------------------------------------- config
spava_status make_layer(const spava_config *c, Layer *L) {
    if (!c || !L || !c->chunk_offsets) return SPAVA_ERR_INVALID_ARG;
    if (c->H < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 || c->head_dim < 1)
        return SPAVA_ERR_INVALID_ARG;
    if (c->n_q_heads % c->n_kv_heads) return SPAVA_ERR_INVALID_ARG;
    if (c->anchor_len < 0 || c->query_len < 1 || c->top_l < 0 || c->n_tokens < 1)
        return SPAVA_ERR_INVALID_ARG;
    if (c->local_pair_full != 0 && c->local_pair_full != 1) return SPAVA_ERR_INVALID_ARG;
    if (c->score_norm != 0 && c->score_norm != 1) return SPAVA_ERR_INVALID_ARG;
    if (c->score_pool < 0 || (c->score_pool > 1 && c->score_pool % 2 == 0)) return SPAVA_ERR_INVALID_ARG;
    if (c->score_pool > kMaxPool) return SPAVA_ERR_UNSUPPORTED;
    if (c->H > kMaxChunks / 2) return SPAVA_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return SPAVA_ERR_UNSUPPORTED;
    if (c->n_tokens >= (1LL << 31)) return SPAVA_ERR_UNSUPPORTED;
    const int nc = 2 * c->H;
    const int64_t *off = c->chunk_offsets;
    if (off[0] != c->anchor_len || off[nc] != c->n_tokens - c->query_len) return SPAVA_ERR_INVALID_ARG;
    for (int v = 0; v < nc; ++v)
        if (off[v + 1] <= off[v]) return SPAVA_ERR_INVALID_ARG;
    std::memset(L, 0, sizeof(*L));
    L->H = c->H;
    L->Hq = c->n_q_heads;
    L->Hkv = c->n_kv_heads;
    L->d = c->head_dim;
    L->G = c->n_q_heads / c->n_kv_heads;
    L->lpf = c->local_pair_full;
    L->norm = c->score_norm;
    L->pool = c->score_pool > 1 ? c->score_pool : 1;
    L->l = c->top_l;
    L->n_chunks = nc;
    L->N = static_cast<int32_t>(c->n_tokens);
    L->a = static_cast<int32_t>(c->anchor_len);
    L->q = static_cast<int32_t>(c->query_len);
    L->C = L->N - L->a - L->q;
    for (int v = 0; v <= nc; ++v) L->off[v] = static_cast<int32_t>(off[v]);
    L->pcum[0] = L->a;
    for (int u = 0; u < nc - 1; ++u) {
        const int n_u = L->off[u + 1] - L->off[u];
        L->pcum[u + 1] = L->pcum[u] + std::min(L->l, n_u);
    }
    L->L = L->pcum[nc - 1];
    // One GPU: every region held at its global position.
    L->Nl = L->N;
    L->own = nc >= 64 ? ~0ULL : ((1ULL << nc) - 1);
    for (int r = 0; r < nc + 2; ++r) L->loc[r] = region_first(*L, r);
    const double scale = c->scale > 0.f ? static_cast<double>(c->scale) : 1.0 / std::sqrt(double(c->head_dim));
    L->scale_log2 = static_cast<float>(scale * 1.4426950408889634);
    return SPAVA_OK;
}

// ---------------------------------------------------------------- plan
int item_tiles(const Layer &L, const Item &it) {
    Seg s[kMaxSegs];
    const int n = build_segments(L, it, s);
    return count_tiles(s, n);
}

// Rows of the region a group covers.
void region_rows(const Layer &L, int kind, int sub, int &lo, int &hi) {
    Item it{kind, sub, 0, 0};
    int r0, re;
    item_rows(L, it, r0, re);
    lo = r0;
    hi = kind == kCtx ? L.off[sub + 1] : kind == kAnchor ? L.a : L.N;
}

// Groups of the attention launch, most expensive first: the persistent
// attention grid claims work items from a queue in index order (and the
// hardware block scheduler hands out the statistics pass's CTAs in index
// order), so a cost-descending order is a longest-processing-time-first
// schedule over the SMs.  Inside a group, items run KV head by KV head, row
// tile descending, with the query heads of a KV head adjacent (shared K/V tiles
// in L2; see decode_pair_item).  Only regions lying inside
// rows [row_lo, row_hi) are planned (the whole layer by default).
constexpr unsigned kAllKinds = (1u << kCtx) | (1u << kAnchor) | (1u << kQueryPart);
int plan_attention(const Layer &L, bool stats, Group *out, int row_lo = 0, int row_hi = INT32_MAX,
                   unsigned kinds = kAllKinds) {
    struct G { Group g; int cost; };
    std::vector<G> gs;
    auto push = [&](int kind, int sub, int n_rt) {
        if (n_rt <= 0) return;
        if (!stats && !((kinds >> kind) & 1u)) return;
        int lo, hi;
        region_rows(L, kind, sub, lo, hi);
        if (lo < row_lo || hi > row_hi) return;
        Item it{kind, sub, n_rt - 1, 0};
        gs.push_back({Group{kind, sub, n_rt, 0}, item_tiles(L, it)});
    };
    // A query-row segment is computed where its keys are held: the anchor and
    // the query block everywhere, chunk v where v is held.
    auto seg_held = [&](int s) { return s == 0 || s > L.n_chunks || owns(L, s - 1); };
    const int n_qrt = cdiv(L.q, kRowTile);
    if (stats && L.norm == 0) {
        for (int u = 0; u < L.n_chunks - 1; ++u)
            if (owns(L, u)) push(kStats, u, n_qrt);
    } else if (stats) {
        // Row-normalised scores: the query rows' statistics over every segment
        // they attend (anchor, each chunk, the query block up to the row), the
        // same segments as the query-row partials of the attention.
        for (int s = (L.a > 0 ? 0 : 1); s < L.n_chunks + 2; ++s) push(kQueryPart, s, n_qrt);
    } else {
        for (int v = 0; v < L.n_chunks; ++v)
            if (owns(L, v)) push(kCtx, v, cdiv(L.off[v + 1] - L.off[v], kRowTile));
        if (L.a > 0) push(kAnchor, 0, cdiv(L.a, kRowTile));
        for (int s = (L.a > 0 ? 0 : 1); s < L.n_chunks + 2; ++s)
            if (seg_held(s)) push(kQueryPart, s, n_qrt);
    }
    std::stable_sort(gs.begin(), gs.end(), [](const G &x, const G &y) { return x.cost > y.cost; });
    // Work items of two 128-row tiles each (statistics pass and attention alike).
    int begin = 0, n = 0;
    for (auto &g : gs) {
        g.g.item_begin = begin;
        begin += pair_items(g.g.n_rt, L.G) * L.Hkv;
        out[n++] = g.g;
    }
    return n;
}

int64_t plan_items(const Group *g, int n, const Layer &L) {
    if (!n) return 0;
    return static_cast<int64_t>(g[n - 1].item_begin) + pair_items(g[n - 1].n_rt, L.G) * L.Hkv;
}

// ---------------------------------------------------------------- workspace
struct WsLayout {
    size_t status, stats, scores, idx, pk, pv, part_o, part_lse, counters, total;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(const Layer &L) {
    WsLayout w{};
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
    w.status = take(256);
    w.stats = take(sizeof(float) * size_t(L.n_chunks - 1) * L.Hq * L.q);
    w.scores = take(sizeof(float) * size_t(L.Hkv) * L.C);
    w.idx = take(sizeof(int32_t) * size_t(L.n_chunks - 1) * L.Hkv * L.l);
    w.pk = take(2 * size_t(L.Hkv) * L.L * L.d);
    w.pv = take(2 * size_t(L.Hkv) * L.L * L.d);
    w.part_o = take(sizeof(float) * size_t(L.n_chunks + 2) * L.Hq * L.q * L.d);
    w.part_lse = take(sizeof(float) * size_t(L.n_chunks + 2) * L.Hq * L.q);
    w.counters = take(sizeof(int32_t) * size_t(L.n_chunks - 1) * L.Hkv);
    w.total = o;
    return w;
}

spava_status check_ws(const Layer &L, void *ws, size_t ws_bytes) {
    if (!ws) return SPAVA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return SPAVA_ERR_MISALIGNED;
    if (ws_bytes < ws_layout(L).total) return SPAVA_ERR_WORKSPACE;
    return SPAVA_OK;
}

// Work-queue counters of the persistent attention launches, inside the
// workspace's first 256 bytes (the status block: status word at 0): slot 0
// serves every launch on the caller's stream and the statistics pass; launches
// that may run at the same time as another attention launch take slots 1 and 2.
int *queue_slot(char *ws, int slot) { return reinterpret_cast<int *>(ws + 128 + 32 * slot); }

spava_status check_ptr(const void *p, bool required = true) {
    if (!p) return required ? SPAVA_ERR_INVALID_ARG : SPAVA_OK;
    return (reinterpret_cast<uintptr_t>(p) & 15) ? SPAVA_ERR_MISALIGNED : SPAVA_OK;
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

spava_status get_encoder(EncodeTiledFn *fn) {
    std::call_once(g_encode_once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(p);
        else if (g_encode_err == cudaSuccess)
            g_encode_err = cudaErrorSymbolNotFound;
    });
    if (!g_encode) return cuda_fail(g_encode_err);
    *fn = g_encode;
    return SPAVA_OK;
}

// bf16 3-D map {d0 inner, d1, d2}, 128-byte swizzle, zero fill out of bounds.
spava_status encode_3d(CUtensorMap *tm, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint32_t b0, uint32_t b1, uint32_t b2) {
    EncodeTiledFn fn;
    SPAVA_TRY(get_encoder(&fn));
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = static_cast<int32_t>(r);
        return SPAVA_ERR_CUDA;
    }
    return SPAVA_OK;
}

// Token-major [Nl, H, D] tensor (the rows held here), boxes of 64 columns x 1
// head x 128 tokens.
spava_status map_tokens(CUtensorMap *tm, const void *p, const Layer &L, int heads) {
    return encode_3d(tm, p, L.d, heads, L.Nl, 64, 1, 128);
}
// Packed [Hkv, rows, D] tensor, boxes of 64 columns x 128 rows x 1 head.
spava_status map_packed(CUtensorMap *tm, const void *p, const Layer &L) {
    return encode_3d(tm, p, L.d, std::max(L.L, 1), L.Hkv, 64, 128, 1);
}

template <typename K>
spava_status set_smem(K kernel, int bytes) {
    SPAVA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    return SPAVA_OK;
}

spava_status launched() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SPAVA_OK : cuda_fail(e);
}

// ---------------------------------------------------------------- launches
template <int D, bool STATS>
spava_status launch_attn(AttnParams &p, cudaStream_t st) {
    const int64_t items = plan_items(p.groups, p.n_groups, p.L);
    if (items == 0) return SPAVA_OK;
    if (items >= (1LL << 31)) return SPAVA_ERR_UNSUPPORTED;
    using SM = AttnSmem<D>;
    // Persistent grid: one CTA per SM (the shared memory allows no more), each
    // claiming items from the queue counter p.queue.
    int dev = 0, n_sm = 148;
    SPAVA_CUDA(cudaGetDevice(&dev));
    SPAVA_CUDA(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
    p.n_items = static_cast<int32_t>(items);
    SPAVA_CUDA(cudaMemsetAsync(p.queue, 0, sizeof(int), st));
    // The kernel's register split draws on the pool its launch allocates;
    // refuse to launch a build whose per-thread count would leave it short.
    cudaFuncAttributes fa;
    SPAVA_CUDA(cudaFuncGetAttributes(&fa, attn_kernel<D, STATS>));
    if (fa.numRegs < kLaunchRegs) return SPAVA_ERR_UNSUPPORTED;
    SPAVA_TRY(set_smem(attn_kernel<D, STATS>, SM::kAlloc));
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(items, n_sm));
    attn_kernel<D, STATS><<<grid, kAttnThreads, SM::kAlloc, st>>>(p);
    return launched();
}

// The normaliser of the scores: per (chunk u, query head, query row) the base-2
// log-sum-exp of the row's logits over chunk u (score_norm 0), or over every
// key the row attends, the same value for every u (score_norm 1: the segment
// statistics go to the query-partial lse array, free until the attention, and
// are combined there).
spava_status run_stats(const Layer &L, const void *q, const void *k, char *ws, cudaStream_t st) {
    const WsLayout w = ws_layout(L);
    AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.L = L;
    SPAVA_TRY(map_tokens(&p.tmQ, q, L, L.Hq));
    SPAVA_TRY(map_tokens(&p.tmK, k, L, L.Hkv));
    p.n_groups = plan_attention(L, true, p.groups);
    float *stats = reinterpret_cast<float *>(ws + w.stats);
    p.stats = L.norm ? reinterpret_cast<float *>(ws + w.part_lse) : stats;
    p.status = reinterpret_cast<int *>(ws + w.status);
    p.queue = queue_slot(ws, 0);
    SPAVA_TRY(L.d == 128 ? launch_attn<128, true>(p, st) : launch_attn<64, true>(p, st));
    if (!L.norm) return SPAVA_OK;
    const int rows = L.Hq * L.q;
    row_lse_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, st>>>(L, p.stats, stats);
    return launched();
}

// Producing chunks (u < 2H-1) held here.
int owned_producers(const Layer &L) {
    int n = 0;
    for (int u = 0; u < L.n_chunks - 1; ++u) n += owns(L, u);
    return n;
}

// Shared memory for the rank keys of the longest producing chunk held here
// (0 if it does not fit: the selection passes then recompute them).
int select_key_cap(const Layer &L) {
    int n = 0;
    for (int u = 0; u < L.n_chunks - 1; ++u)
        if (owns(L, u)) n = std::max(n, L.off[u + 1] - L.off[u]);
    return n * 4 <= kMaxDynSmem - 4096 ? n : 0;
}

// What the fused scoring launch also needs: where the selection and the gather
// go, and the finished-unit counters.
struct FusedSelect {
    int32_t *idx;
    const void *v;
    void *pk, *pv;
    int *counters;
    bool anchor;  // also copy the anchor rows into the packed buffers
};

// Query-to-context scores of the producing chunks held here, normalised by
// `stats` ([2H-1, Hq, q] base-2 log-sum-exps); `status`: the status word of the
// bounded waits.  With `fused`, the same launch also selects every (chunk, KV
// head)'s passing block into fused->idx and gathers it, and the anchor rows,
// into the packed buffers.
spava_status run_scores(const Layer &L, const void *q, const void *k, const float *stats, float *scores,
                        int *status, cudaStream_t st, const FusedSelect *fused = nullptr) {
    ScoreParams p;
    std::memset(&p, 0, sizeof(p));
    p.L = L;
    SPAVA_TRY(map_tokens(&p.tmQ, q, L, L.Hq));
    SPAVA_TRY(map_tokens(&p.tmK, k, L, L.Hkv));
    p.stats = stats;
    p.scores = scores;
    p.status = status;
    int units = 0;  // score units: pairs of 128-key tiles of one chunk
    for (int u = 0; u < L.n_chunks - 1; ++u) {
        p.unit_begin[u] = units;
        if (owns(L, u)) units += cdiv(cdiv(L.off[u + 1] - L.off[u], 128), kScoreTiles);
    }
    p.unit_begin[L.n_chunks - 1] = units;
    const int64_t score_ctas = static_cast<int64_t>(units) * L.Hkv;
    int64_t blocks = score_ctas;
    if (fused) {
        p.counters = fused->counters;
        p.idx = fused->idx;
        p.K = static_cast<const __nv_bfloat16 *>(k);
        p.V = static_cast<const __nv_bfloat16 *>(fused->v);
        p.PK = static_cast<__nv_bfloat16 *>(fused->pk);
        p.PV = static_cast<__nv_bfloat16 *>(fused->pv);
        p.n_score_ctas = static_cast<int32_t>(score_ctas);
        if (fused->anchor && L.a > 0) blocks += static_cast<int64_t>(L.Hkv) * cdiv(L.a, kAnchorRowsPerCta);
        SPAVA_CUDA(cudaMemsetAsync(p.counters, 0, sizeof(int32_t) * size_t(L.n_chunks - 1) * L.Hkv, st));
    }
    if (blocks == 0) return SPAVA_OK;
    if (blocks >= (1LL << 31)) return SPAVA_ERR_UNSUPPORTED;
    auto go = [&](auto kernel, int smem) -> spava_status {
        SPAVA_TRY(set_smem(kernel, smem));
        kernel<<<static_cast<unsigned>(blocks), kScoreBlockThreads, smem, st>>>(p);
        return launched();
    };
    if (L.d == 128)
        return fused ? go(score_kernel<128, true>, ScoreSmem<128>::kAlloc)
                     : go(score_kernel<128, false>, ScoreSmem<128>::kAlloc);
    return fused ? go(score_kernel<64, true>, ScoreSmem<64>::kAlloc)
                 : go(score_kernel<64, false>, ScoreSmem<64>::kAlloc);
}

// The same, with the workspace's status word and counters.
spava_status run_scores_ws(const Layer &L, const void *q, const void *k, const float *stats, float *scores,
                           char *ws, cudaStream_t st, bool fused = false, int32_t *idx = nullptr,
                           const void *v = nullptr, void *pk = nullptr, void *pv = nullptr,
                           bool anchor = true) {
    const WsLayout w = ws_layout(L);
    int *status = reinterpret_cast<int *>(ws + w.status);
    if (!fused) return run_scores(L, q, k, stats, scores, status, st);
    const FusedSelect f{idx, v, pk, pv, reinterpret_cast<int *>(ws + w.counters), anchor};
    return run_scores(L, q, k, stats, scores, status, st, &f);
}

spava_status run_topk(const Layer &L, const float *scores, int32_t *idx, cudaStream_t st) {
    const int blocks = owned_producers(L) * L.Hkv;
    if (blocks == 0 || L.l == 0) return SPAVA_OK;
    const int cap = select_key_cap(L);
    SPAVA_TRY(set_smem(topk_kernel, cap * 4));
    topk_kernel<<<blocks, kSelectThreads, cap * 4, st>>>(L, scores, idx, cap);  // pools on the fly (L.pool)
    return launched();
}

spava_status run_pack(const Layer &L, const void *k, const void *v, const int32_t *idx, void *pk,
                      void *pv, cudaStream_t st) {
    const int64_t rows = static_cast<int64_t>(L.Hkv) * L.L;
    if (rows == 0) return SPAVA_OK;
    // Persistent grid: a few blocks per SM, each warp walking 32-row groups.
    int dev = 0, n_sm = 148;
    SPAVA_CUDA(cudaGetDevice(&dev));
    SPAVA_CUDA(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
    const int64_t groups = (rows + 31) / 32;
    const int64_t want = (groups + kPackThreads / 32 - 1) / (kPackThreads / 32);
    const int64_t blocks = std::min<int64_t>(want, static_cast<int64_t>(n_sm) * 8);
    auto K = static_cast<const __nv_bfloat16 *>(k);
    auto V = static_cast<const __nv_bfloat16 *>(v);
    auto PK = static_cast<__nv_bfloat16 *>(pk);
    auto PV = static_cast<__nv_bfloat16 *>(pv);
    if (L.d == 128)
        pack_kernel<128><<<static_cast<unsigned>(blocks), kPackThreads, 0, st>>>(L, K, V, idx, PK, PV);
    else
        pack_kernel<64><<<static_cast<unsigned>(blocks), kPackThreads, 0, st>>>(L, K, V, idx, PK, PV);
    return launched();
}

// Selection and gather in one launch (select_pack_kernel): one CTA per
// (producing chunk, KV head), then the anchor rows.
spava_status run_select_pack(const Layer &L, const float *scores, int32_t *idx, const void *k,
                             const void *v, void *pk, void *pv, cudaStream_t st) {
    const int64_t n_sel = static_cast<int64_t>(owned_producers(L)) * L.Hkv;
    const int64_t n_anchor = L.a > 0 ? static_cast<int64_t>(L.Hkv) * cdiv(L.a, kAnchorRowsPerCta) : 0;
    const unsigned blocks = static_cast<unsigned>(n_sel + n_anchor);
    if (blocks == 0) return SPAVA_OK;
    auto K = static_cast<const __nv_bfloat16 *>(k);
    auto V = static_cast<const __nv_bfloat16 *>(v);
    auto PK = static_cast<__nv_bfloat16 *>(pk);
    auto PV = static_cast<__nv_bfloat16 *>(pv);
    const int cap = select_key_cap(L);
    if (L.d == 128) {
        SPAVA_TRY(set_smem(select_pack_kernel<128>, cap * 4));
        select_pack_kernel<128><<<blocks, kSelectThreads, cap * 4, st>>>(L, scores, idx, K, V, PK, PV,
                                                                         static_cast<int>(n_sel), cap);
    } else {
        SPAVA_TRY(set_smem(select_pack_kernel<64>, cap * 4));
        select_pack_kernel<64><<<blocks, kSelectThreads, cap * 4, st>>>(L, scores, idx, K, V, PK, PV,
                                                                        static_cast<int>(n_sel), cap);
    }
    return launched();
}

// The query rows: the per-segment partials merged by log-sum-exp.
spava_status run_merge(const Layer &L, void *o, float *lse, char *ws, cudaStream_t st) {
    const WsLayout w = ws_layout(L);
    const float *part_O = reinterpret_cast<const float *>(ws + w.part_o);
    const float *part_lse = reinterpret_cast<const float *>(ws + w.part_lse);
    const int64_t warps = static_cast<int64_t>(L.Hq) * L.q;
    const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
    auto O = static_cast<__nv_bfloat16 *>(o);
    if (L.d == 128)
        merge_kernel<128><<<blocks, 256, 0, st>>>(L, part_O, part_lse, O, lse);
    else
        merge_kernel<64><<<blocks, 256, 0, st>>>(L, part_O, part_lse, O, lse);
    return launched();
}

spava_status run_attn(const Layer &L, const void *q, const void *k, const void *v, const void *pk,
                      const void *pv, void *o, float *lse, char *ws, cudaStream_t st,
                      int row_lo = 0, int row_hi = INT32_MAX, unsigned kinds = kAllKinds,
                      bool merge = true, int slot = 0) {
    const WsLayout w = ws_layout(L);
    AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.L = L;
    SPAVA_TRY(map_tokens(&p.tmQ, q, L, L.Hq));
    SPAVA_TRY(map_tokens(&p.tmK, k, L, L.Hkv));
    SPAVA_TRY(map_tokens(&p.tmV, v, L, L.Hkv));
    // With no packed rows (a = 0, l = 0) no segment reads the packed maps.
    SPAVA_TRY(L.L > 0 ? map_packed(&p.tmPK, pk, L) : map_tokens(&p.tmPK, k, L, L.Hkv));
    SPAVA_TRY(L.L > 0 ? map_packed(&p.tmPV, pv, L) : map_tokens(&p.tmPV, v, L, L.Hkv));
    p.n_groups = plan_attention(L, false, p.groups, row_lo, row_hi, kinds);
    p.O = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.part_O = reinterpret_cast<float *>(ws + w.part_o);
    p.part_lse = reinterpret_cast<float *>(ws + w.part_lse);
    p.status = reinterpret_cast<int *>(ws + w.status);
    p.queue = queue_slot(ws, slot);
    SPAVA_TRY(L.d == 128 ? launch_attn<128, false>(p, st) : launch_attn<64, false>(p, st));
    if (!merge || L.N - L.q < row_lo || L.N > row_hi) return SPAVA_OK;  // query block not in this range
    return run_merge(L, o, lse, ws, st);
}

// Scoring, selection and gather: everything of the layer before the attention,
// from the statistics pass.  Scoring reads only K and the query block's Q rows;
// with `v_ready` (the host entry point's copy pipeline) the selection and the
// gather -- the first step that reads V -- run as their own launch after it,
// otherwise in the scoring launch.
spava_status run_front(const Layer &L, const void *q, const void *k, const void *v,
                       int32_t *idx_out, char *w, cudaStream_t st, cudaEvent_t v_ready = nullptr) {
    const WsLayout lay = ws_layout(L);
    float *scores = reinterpret_cast<float *>(w + lay.scores);
    const float *stats = reinterpret_cast<const float *>(w + lay.stats);
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(w + lay.idx);
    if (L.n_chunks > 1 && L.l > 0) {
        SPAVA_TRY(run_stats(L, q, k, w, st));
        if (!v_ready)
            return run_scores_ws(L, q, k, stats, scores, w, st, true, idx, v, w + lay.pk, w + lay.pv);
        SPAVA_TRY(run_scores_ws(L, q, k, stats, scores, w, st));
        SPAVA_CUDA(cudaStreamWaitEvent(st, v_ready, 0));
        return run_select_pack(L, scores, idx, k, v, w + lay.pk, w + lay.pv, st);
    }
    if (v_ready) SPAVA_CUDA(cudaStreamWaitEvent(st, v_ready, 0));
    return run_pack(L, k, v, idx, w + lay.pk, w + lay.pv, st);  // anchor rows only
}

// The whole layer on device buffers, in the order of the pages' fused forward
// ("Forward Fuso di Contesto e Query"): first the work that needs no passing
// block -- the anchor rows and the query rows' partials over every segment,
// whose per-chunk log-sum-exps ARE the scoring's normaliser (the statistics
// pass computes the same values bit for bit) -- then scoring fused with the
// selection and the gather, then the context rows and the query-row merge.
spava_status run_layer(const Layer &L, const void *q, const void *k, const void *v, void *o,
                       float *lse, int32_t *idx_out, char *w, cudaStream_t st) {
    const WsLayout lay = ws_layout(L);
    if (!(L.n_chunks > 1 && L.l > 0)) {
        SPAVA_TRY(run_front(L, q, k, v, idx_out, w, st));
        return run_attn(L, q, k, v, w + lay.pk, w + lay.pv, o, lse, w, st);
    }
    SPAVA_TRY(run_attn(L, q, k, v, w + lay.pk, w + lay.pv, o, lse, w, st, 0, INT32_MAX,
                       (1u << kAnchor) | (1u << kQueryPart), false));
    float *part_lse = reinterpret_cast<float *>(w + lay.part_lse);
    const float *stats = part_lse + size_t(L.Hq) * L.q;  // segment 1 + u = chunk u
    if (L.norm) {  // each row's log-sum-exp over all its segments
        float *row = reinterpret_cast<float *>(w + lay.stats);
        const int rows = L.Hq * L.q;
        row_lse_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, st>>>(L, part_lse, row);
        SPAVA_TRY(launched());
        stats = row;
    }
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(w + lay.idx);
    SPAVA_TRY(run_scores_ws(L, q, k, stats, reinterpret_cast<float *>(w + lay.scores), w, st, true, idx, v,
                            w + lay.pk, w + lay.pv));
    return run_attn(L, q, k, v, w + lay.pk, w + lay.pv, o, lse, w, st, 0, INT32_MAX, 1u << kCtx, true);
}

// Row groups of the copy/compute pipeline of the host entry point, in the
// order they run: the query block first (its Q rows go up with K, ahead of
// everything else), then the chunks and the anchor in DESCENDING token order.
// Later chunks attend more keys, so the first context groups bring the most
// work per uploaded row and the copies run ahead of the kernels; the last
// group, whose download no kernel hides, is the first region alone (the
// cheapest).  The last chunk is alone too; the regions between are cut into
// runs of about equal rows.  Group g covers rows [lo[g], hi[g]); returns the
// count (at most kCopyGroups).
constexpr int kCopyGroups = 8;
int copy_groups(const Layer &L, int *lo, int *hi) {
    std::vector<int> starts;  // starts of the anchor and chunk regions, in token order
    if (L.a > 0) starts.push_back(0);
    for (int v = 0; v < L.n_chunks; ++v) starts.push_back(L.off[v]);
    const int ctx_end = L.N - L.q;
    int n = 0;
    lo[n] = ctx_end, hi[n++] = L.N;
    const int m = static_cast<int>(starts.size());
    lo[n] = starts[m - 1], hi[n++] = ctx_end;  // the last chunk
    if (m == 1) return n;
    // regions m-2 .. 1 (descending), then region 0 alone
    const int mid_hi = starts[m - 1], mid_lo = starts[1];
    const int mid_groups = kCopyGroups - 3;
    int end = mid_hi;
    for (int i = m - 2; i >= 1; --i) {
        const int64_t k = n - 1;  // middle groups cut so far + 1
        const int64_t target = mid_hi - static_cast<int64_t>(mid_hi - mid_lo) * k / mid_groups;
        if (starts[i] <= target || i == 1) {
            lo[n] = starts[i], hi[n++] = end;
            end = starts[i];
        }
    }
    lo[n] = 0, hi[n++] = starts[1];
    return n;
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

spava_status spava_workspace_size(const spava_config *cfg, size_t *bytes) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    if (!bytes) return SPAVA_ERR_INVALID_ARG;
    *bytes = ws_layout(L).total;
    return SPAVA_OK;
}

spava_status spava_packed_len(const spava_config *cfg, int64_t *rows) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    if (!rows) return SPAVA_ERR_INVALID_ARG;
    *rows = L.L;
    return SPAVA_OK;
}

spava_status spava_score(const spava_config *cfg, const void *q, const void *k, float *scores,
                         void *ws, size_t ws_bytes, void *stream) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(scores));
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(ws);
    SPAVA_TRY(run_stats(L, q, k, w, st));
    return run_scores_ws(L, q, k, reinterpret_cast<const float *>(w + ws_layout(L).stats), scores, w, st);
}

spava_status spava_topk_select(const spava_config *cfg, const float *scores, int32_t *idx,
                               void *stream) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    SPAVA_TRY(check_ptr(scores));
    if (L.l > 0) SPAVA_TRY(check_ptr(idx));
    return run_topk(L, scores, idx, static_cast<cudaStream_t>(stream));
}

spava_status spava_pack_passing(const spava_config *cfg, const void *k, const void *v,
                                const int32_t *idx, void *pk, void *pv, void *stream) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(v));
    if (L.l > 0) SPAVA_TRY(check_ptr(idx));
    if (L.L > 0) {
        SPAVA_TRY(check_ptr(pk));
        SPAVA_TRY(check_ptr(pv));
    }
    return run_pack(L, k, v, idx, pk, pv, static_cast<cudaStream_t>(stream));
}

spava_status spava_attn(const spava_config *cfg, const void *q, const void *k, const void *v,
                        const void *pk, const void *pv, void *o, float *lse, void *ws,
                        size_t ws_bytes, void *stream) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(v));
    SPAVA_TRY(check_ptr(o));
    SPAVA_TRY(check_ptr(lse, false));
    if (L.L > 0) {
        SPAVA_TRY(check_ptr(pk));
        SPAVA_TRY(check_ptr(pv));
    }
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    return run_attn(L, q, k, v, pk, pv, o, lse, static_cast<char *>(ws),
                    static_cast<cudaStream_t>(stream));
}

spava_status spava_prefill_attention(const spava_config *cfg, const void *q, const void *k,
                                     const void *v, void *o, float *lse, int32_t *idx_out,
                                     void *ws, size_t ws_bytes, void *stream) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(v));
    SPAVA_TRY(check_ptr(o));
    SPAVA_TRY(check_ptr(lse, false));
    SPAVA_TRY(check_ptr(idx_out, false));
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    return run_layer(L, q, k, v, o, lse, idx_out, static_cast<char *>(ws), static_cast<cudaStream_t>(stream));
}

spava_status spava_prefill_attention_host(const spava_config *cfg, const void *q_host,
                                          const void *k_host, const void *v_host, void *o_host,
                                          float *lse_host, void *q, void *k, void *v, void *o,
                                          float *lse, void *ws, size_t ws_bytes, void *stream,
                                          void *copy_stream) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    if (!q_host || !k_host || !v_host || !o_host) return SPAVA_ERR_INVALID_ARG;
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(v));
    SPAVA_TRY(check_ptr(o));
    SPAVA_TRY(check_ptr(lse, false));
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t row_q = size_t(L.Hq) * L.d * 2, row_k = size_t(L.Hkv) * L.d * 2;
    const bool want_lse = lse && lse_host;
    auto cq = static_cast<const char *>(q_host);
    auto oh = static_cast<char *>(o_host);
    char *qd = static_cast<char *>(q), *od = static_cast<char *>(o);
    auto d2h_rows = [&](int r0, int r1, cudaStream_t s) -> spava_status {
        SPAVA_CUDA(cudaMemcpyAsync(oh + r0 * row_q, od + r0 * row_q, (r1 - r0) * row_q,
                                   cudaMemcpyDeviceToHost, s));
        if (want_lse)  // lse is [Hq, N]: the rows of every head, one strided copy
            SPAVA_CUDA(cudaMemcpy2DAsync(lse_host + r0, sizeof(float) * L.N, lse + r0,
                                         sizeof(float) * L.N, sizeof(float) * (r1 - r0), L.Hq,
                                         cudaMemcpyDeviceToHost, s));
        return SPAVA_OK;
    };
    if (!copy_stream || copy_stream == stream) {
        SPAVA_CUDA(cudaMemcpyAsync(q, q_host, L.N * row_q, cudaMemcpyHostToDevice, st));
        SPAVA_CUDA(cudaMemcpyAsync(k, k_host, L.N * row_k, cudaMemcpyHostToDevice, st));
        SPAVA_CUDA(cudaMemcpyAsync(v, v_host, L.N * row_k, cudaMemcpyHostToDevice, st));
        SPAVA_TRY(spava_prefill_attention(cfg, q, k, v, o, want_lse ? lse : nullptr, nullptr, ws,
                                          ws_bytes, stream));
        return d2h_rows(0, L.N, st);
    }
    cudaStream_t cs = static_cast<cudaStream_t>(copy_stream);
    char *w = static_cast<char *>(ws);
    const WsLayout lay = ws_layout(L);
    auto cv = static_cast<const char *>(v_host), ck = static_cast<const char *>(k_host);
    char *kd = static_cast<char *>(k), *vd = static_cast<char *>(v);
    auto h2d_rows = [&](int r0, int r1, bool qkv) -> spava_status {  // Q rows, and K/V rows if qkv
        if (r1 <= r0) return SPAVA_OK;
        SPAVA_CUDA(cudaMemcpyAsync(qd + r0 * row_q, cq + r0 * row_q, (r1 - r0) * row_q,
                                   cudaMemcpyHostToDevice, cs));
        if (qkv) {
            SPAVA_CUDA(cudaMemcpyAsync(kd + r0 * row_k, ck + r0 * row_k, (r1 - r0) * row_k,
                                       cudaMemcpyHostToDevice, cs));
            SPAVA_CUDA(cudaMemcpyAsync(vd + r0 * row_k, cv + r0 * row_k, (r1 - r0) * row_k,
                                       cudaMemcpyHostToDevice, cs));
        }
        return SPAVA_OK;
    };
    std::vector<cudaEvent_t> ev;
    spava_status rc = SPAVA_OK;
    auto new_event = [&]() -> cudaEvent_t {
        cudaEvent_t e = nullptr;
        if (rc == SPAVA_OK && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
            rc = cuda_fail(cudaGetLastError());
        ev.push_back(e);
        return e;
    };
    const bool chunkwise = L.norm == 0;
    // The chunk pipeline's own streams: scoring (at the device's highest
    // priority, so that its CTAs take the first SMs an attention launch frees)
    // and two for the attention launches.  Destroying a stream with work still
    // queued is safe: it is released once that work completes.
    cudaStream_t side[3] = {nullptr, nullptr, nullptr};
    if (chunkwise) {
        int prio_least = 0, prio_greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&prio_least, &prio_greatest) != cudaSuccess)
            return cuda_fail(cudaGetLastError());
        for (int i = 0; i < 3; ++i)
            if (cudaStreamCreateWithPriority(&side[i], cudaStreamNonBlocking,
                                             i == 0 ? prio_greatest : prio_least) != cudaSuccess) {
                const cudaError_t e = cudaGetLastError();
                for (int j = 0; j < i; ++j) cudaStreamDestroy(side[j]);
                return cuda_fail(e);
            }
    }
    auto body = [&]() -> spava_status {
        cudaEvent_t e_start = new_event();
        if (rc != SPAVA_OK) return rc;
        // The copies start only once everything already on `stream` is done (an
        // earlier call's kernels may still be reading the buffers they overwrite).
        SPAVA_CUDA(cudaEventRecord(e_start, st));
        SPAVA_CUDA(cudaStreamWaitEvent(cs, e_start, 0));
        std::vector<std::pair<int, int>> rows;      // row groups, in the order they compute
        std::vector<cudaEvent_t> computed;          // one per row group
        if (chunkwise) {
            // Chunk by chunk, in token order: chunk v's rows need the anchor, the
            // passing blocks of the chunks before it, its partner chunk (an
            // earlier one) and itself -- all on the device by the time chunk v
            // has arrived -- so each chunk is scored, selected and gathered, and
            // its rows computed, as soon as its Q/K/V rows land, while the next
            // chunk is still on its way.  The query block's Q rows (the scorer)
            // go up first, its K/V last; its rows compute last.
            const int q0 = L.N - L.q;
            SPAVA_TRY(h2d_rows(q0, L.N, false));
            SPAVA_TRY(h2d_rows(0, L.a, true));
            cudaEvent_t e_anchor = new_event();
            std::vector<cudaEvent_t> e_chunk(L.n_chunks);
            for (auto &e : e_chunk) e = new_event();
            cudaEvent_t e_query = new_event();
            if (rc != SPAVA_OK) return rc;
            SPAVA_CUDA(cudaEventRecord(e_anchor, cs));
            for (int c = 0; c < L.n_chunks; ++c) {
                SPAVA_TRY(h2d_rows(L.off[c], L.off[c + 1], true));
                SPAVA_CUDA(cudaEventRecord(e_chunk[c], cs));
            }
            SPAVA_CUDA(cudaMemcpyAsync(kd + q0 * row_k, ck + q0 * row_k, L.q * row_k, cudaMemcpyHostToDevice, cs));
            SPAVA_CUDA(cudaMemcpyAsync(vd + q0 * row_k, cv + q0 * row_k, L.q * row_k, cudaMemcpyHostToDevice, cs));
            SPAVA_CUDA(cudaEventRecord(e_query, cs));
            // A region's last 128-row tile reads up to 127 rows past the region's
            // end: their keys are masked, but their V rows meet a zero weight in
            // the PV product, and 0 x (a NaN or Inf not yet overwritten) is NaN.
            // So a region's attention waits until every row its tiles touch has
            // arrived.
            auto wait_rows = [&](cudaStream_t s, int end) -> spava_status {  // rows [0, end) on the device
                if (end > L.off[L.n_chunks]) return cuda_ok(cudaStreamWaitEvent(s, e_query, 0));
                int c = 0;
                while (L.off[c + 1] < end) ++c;
                return cuda_ok(cudaStreamWaitEvent(s, e_chunk[c], 0));
            };
            auto tiles_end = [&](int r0, int r1) { return std::min(L.N, r0 + kRowTile * cdiv(r1 - r0, kRowTile)); };
            const bool select = L.n_chunks > 1 && L.l > 0;
            float *scores = reinterpret_cast<float *>(w + lay.scores);
            const float *stats = reinterpret_cast<const float *>(w + lay.stats);
            int32_t *idx = reinterpret_cast<int32_t *>(w + lay.idx);
            // Scoring runs on its own stream, ahead of the attention; the
            // attention launches alternate between two streams, each waiting only
            // for its rows and the passing blocks before them, so that a launch's
            // persistent CTAs take over the SMs its predecessor's tail frees.
            cudaStream_t ss = side[0];
            for (int i = 0; i < 3; ++i) SPAVA_CUDA(cudaStreamWaitEvent(side[i], e_start, 0));
            // The packed passing blocks fill up chunk by chunk, and a packed
            // segment's last tile reads past its end into blocks not yet written:
            // those rows start as zeros, not as whatever the workspace held.
            if (select) {
                const size_t packed = 2 * size_t(L.Hkv) * L.L * L.d;
                SPAVA_CUDA(cudaMemsetAsync(w + lay.pk, 0, packed, ss));
                SPAVA_CUDA(cudaMemsetAsync(w + lay.pv, 0, packed, ss));
            }
            SPAVA_CUDA(cudaStreamWaitEvent(ss, e_anchor, 0));
            if (!select) SPAVA_TRY(run_pack(L, k, v, idx, w + lay.pk, w + lay.pv, ss));  // anchor rows
            cudaEvent_t e_init = new_event();
            if (rc != SPAVA_OK) return rc;
            SPAVA_CUDA(cudaEventRecord(e_init, ss));
            int turn = 0;
            auto attend = [&](int r0, int r1, cudaEvent_t after) -> spava_status {
                if (r1 <= r0) return SPAVA_OK;
                cudaStream_t sa = side[1 + turn];
                const int slot = 1 + turn;
                turn ^= 1;
                SPAVA_TRY(wait_rows(sa, tiles_end(r0, r1)));
                SPAVA_CUDA(cudaStreamWaitEvent(sa, after, 0));
                SPAVA_TRY(run_attn(L, q, k, v, w + lay.pk, w + lay.pv, o, want_lse ? lse : nullptr, w, sa,
                                   r0, r1, kAllKinds, true, slot));
                cudaEvent_t e = new_event();
                if (rc != SPAVA_OK) return rc;
                SPAVA_CUDA(cudaEventRecord(e, sa));
                rows.emplace_back(r0, r1);
                computed.push_back(e);
                return SPAVA_OK;
            };
            if (L.a > 0) SPAVA_TRY(attend(0, L.a, e_init));
            cudaEvent_t sel_before = e_init;  // the passing blocks of every chunk before c
            for (int c = 0; c < L.n_chunks; ++c) {
                cudaEvent_t sel_c = sel_before;
                if (select && c < L.n_chunks - 1) {
                    // this chunk's passing block: the same kernels as the whole
                    // layer's front, restricted to chunk c
                    Layer Lc = L;
                    Lc.own = 1ULL << c;
                    SPAVA_CUDA(cudaStreamWaitEvent(ss, e_chunk[c], 0));
                    SPAVA_TRY(run_stats(Lc, q, k, w, ss));
                    SPAVA_TRY(run_scores_ws(Lc, q, k, stats, scores, w, ss, true, idx, v, w + lay.pk,
                                            w + lay.pv, c == 0));
                    sel_c = new_event();
                    if (rc != SPAVA_OK) return rc;
                    SPAVA_CUDA(cudaEventRecord(sel_c, ss));
                }
                // chunk 0's scoring launch also copies the anchor rows
                SPAVA_TRY(attend(L.off[c], L.off[c + 1], c == 0 ? sel_c : sel_before));
                sel_before = sel_c;
            }
            SPAVA_TRY(attend(q0, L.N, sel_before));
        } else {
            // Row-normalised scores need every segment's statistics first: K and
            // the query block's Q rows go up first, then V, then the Q rows of
            // each context group; the attention runs group by group as its Q rows
            // arrive.
            int lo[kCopyGroups], hi[kCopyGroups];
            const int ng = copy_groups(L, lo, hi);
            cudaEvent_t e_front = new_event(), e_v = new_event();
            std::vector<cudaEvent_t> e_q(ng);
            for (auto &e : e_q) e = new_event();
            if (rc != SPAVA_OK) return rc;
            SPAVA_CUDA(cudaMemcpyAsync(k, k_host, L.N * row_k, cudaMemcpyHostToDevice, cs));
            SPAVA_TRY(h2d_rows(lo[0], hi[0], false));
            SPAVA_CUDA(cudaEventRecord(e_front, cs));
            SPAVA_CUDA(cudaMemcpyAsync(v, v_host, L.N * row_k, cudaMemcpyHostToDevice, cs));
            SPAVA_CUDA(cudaEventRecord(e_v, cs));
            for (int g = 1; g < ng; ++g) {
                SPAVA_TRY(h2d_rows(lo[g], hi[g], false));
                SPAVA_CUDA(cudaEventRecord(e_q[g], cs));
            }
            SPAVA_CUDA(cudaStreamWaitEvent(st, e_front, 0));
            SPAVA_TRY(run_front(L, q, k, v, nullptr, w, st, e_v));
            for (int g = 0; g < ng; ++g) {
                if (g > 0) SPAVA_CUDA(cudaStreamWaitEvent(st, e_q[g], 0));
                SPAVA_TRY(run_attn(L, q, k, v, w + lay.pk, w + lay.pv, o, want_lse ? lse : nullptr, w,
                                   st, lo[g], hi[g]));
                cudaEvent_t e = new_event();
                if (rc != SPAVA_OK) return rc;
                SPAVA_CUDA(cudaEventRecord(e, st));
                rows.emplace_back(lo[g], hi[g]);
                computed.push_back(e);
            }
        }
        // Each row group's O (and lse) goes down once it is computed.
        for (size_t g = 0; g < rows.size(); ++g) {
            SPAVA_CUDA(cudaStreamWaitEvent(cs, computed[g], 0));
            SPAVA_TRY(d2h_rows(rows[g].first, rows[g].second, cs));
        }
        // The call's work ends on `stream`, after the last copy.
        cudaEvent_t e_done = new_event();
        if (rc != SPAVA_OK) return rc;
        SPAVA_CUDA(cudaEventRecord(e_done, cs));
        SPAVA_CUDA(cudaStreamWaitEvent(st, e_done, 0));
        return SPAVA_OK;
    };
    const spava_status rb = body();
    if (rc == SPAVA_OK) rc = rb;
    // Destroying a recorded event is safe: its resources go once it completes.
    for (auto e : ev)
        if (e) cudaEventDestroy(e);
    for (auto s : side)
        if (s) cudaStreamDestroy(s);
    return rc;
}

spava_status spava_device_status(void *ws, size_t ws_bytes, void *stream, int32_t *flags) {
    if (!ws || ws_bytes < 256 || !flags) return SPAVA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    SPAVA_CUDA(cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st));
    SPAVA_CUDA(cudaStreamSynchronize(st));
    if (h) {
        SPAVA_CUDA(cudaMemsetAsync(ws, 0, sizeof(h), st));
        SPAVA_CUDA(cudaStreamSynchronize(st));
    }
    *flags = h;
    return (h & kStatusTimeout) ? SPAVA_ERR_TIMEOUT : SPAVA_OK;
}

spava_status spava_selftest_wait_timeout(void *ws, size_t ws_bytes, void *stream) {
    if (!ws || ws_bytes < 256) return SPAVA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return SPAVA_ERR_MISALIGNED;
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int *>(ws));
    return launched();
}

spava_status spava_plan_chunks(int32_t H, const int64_t *frame_tokens, int64_t n_frames,
                               int64_t anchor_len, int64_t *chunk_offsets) {
    if (!frame_tokens || !chunk_offsets || H < 1 || H > kMaxChunks / 2 || anchor_len < 0)
        return SPAVA_ERR_INVALID_ARG;
    const int nc = 2 * H;
    if (n_frames < nc) return SPAVA_ERR_INVALID_ARG;
    const int64_t per = n_frames / nc, extra = n_frames % nc;
    int64_t f = 0, tok = anchor_len;
    chunk_offsets[0] = anchor_len;
    for (int v = 0; v < nc; ++v) {
        const int64_t take = per + (v < extra ? 1 : 0);
        for (int64_t i = 0; i < take; ++i, ++f) {
            if (frame_tokens[f] < 1) return SPAVA_ERR_INVALID_ARG;
            tok += frame_tokens[f];
            if (tok >= (1LL << 31)) return SPAVA_ERR_INVALID_ARG;
        }
        chunk_offsets[v + 1] = tok;
    }
    return SPAVA_OK;
}

spava_status spava_attended_pairs(const spava_config *cfg, int64_t pairs[3], int64_t *per_host) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    if (!pairs) return SPAVA_ERR_INVALID_ARG;
    pairs[0] = pairs[1] = pairs[2] = 0;
    if (per_host)
        for (int p = 0; p < L.H; ++p) per_host[p] = 0;
    Group groups[sizeof(AttnParams::groups) / sizeof(Group)];
    const int ng = plan_attention(L, false, groups);
    for (int k = 0; k < ng; ++k) {
        for (int rt = 0; rt < groups[k].n_rt; ++rt) {
            Item it{groups[k].kind, groups[k].sub, rt, 0};
            Seg s[kMaxSegs];
            const int n = build_segments(L, it, s);
            int row0, row_end;
            item_rows(L, it, row0, row_end);
            int64_t cnt = 0;
            for (int t = row0; t < row_end; ++t)
                for (int i = 0; i < n; ++i) {
                    const int e = s[i].causal ? std::min(s[i].end, t + 1) : s[i].end;
                    cnt += std::max(0, e - s[i].begin);
                }
            const int cls = it.kind == kAnchor ? 0 : it.kind == kCtx ? 1 : 2;
            pairs[cls] += cnt;
            if (per_host && it.kind == kCtx) per_host[pair_of(L.H, it.sub)] += cnt;
        }
    }
    return SPAVA_OK;
}

const char *spava_status_string(spava_status s) {
    switch (s) {
        case SPAVA_OK: return "ok";
        case SPAVA_ERR_INVALID_ARG: return "invalid argument";
        case SPAVA_ERR_UNSUPPORTED: return "unsupported configuration";
        case SPAVA_ERR_MISALIGNED: return "misaligned pointer";
        case SPAVA_ERR_WORKSPACE: return "workspace missing or too small";
        case SPAVA_ERR_CUDA: return "CUDA error";
        case SPAVA_ERR_TIMEOUT: return "kernel wait timed out";
    }
    return "unknown status";
}

int32_t spava_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"

// ==================================================================== shards
// Multi-GPU ZigZag sequence parallelism ("Disposizione ZigZag", "Comunicazione
// Sovrapposta"): `world` GPUs, rank r holding the physical hosts
// p in [r*m, (r+1)*m), m = H / world, i.e. the chunks v with pair(v) / m == r,
// in local buffers laid out [anchor | its chunks in increasing v | query].
namespace {

// The layer as rank `rank` of `world` sees it.
spava_status make_shard_layer(const spava_config *c, int32_t rank, int32_t world, Layer *L) {
    SPAVA_TRY(make_layer(c, L));
    if (world < 1 || rank < 0 || rank >= world) return SPAVA_ERR_INVALID_ARG;
    if (L->H % world) return SPAVA_ERR_UNSUPPORTED;
    // Row-normalised scores need every chunk's statistics of the query rows
    // before scoring, an exchange this path does not make.
    if (L->norm) return SPAVA_ERR_UNSUPPORTED;
    const int m = L->H / world, nc = L->n_chunks;
    L->own = 0;
    for (int v = 0; v < nc; ++v)
        if (pair_of(L->H, v) / m == rank) L->own |= 1ULL << v;
    for (int r = 0; r < nc + 2; ++r) L->loc[r] = -1;
    int row = 0;
    L->loc[0] = row;
    row += L->a;
    for (int v = 0; v < nc; ++v)
        if (owns(*L, v)) {
            L->loc[1 + v] = row;
            row += L->off[v + 1] - L->off[v];
        }
    L->loc[nc + 1] = row;
    L->Nl = row + L->q;
    return SPAVA_OK;
}

// Chunks of rank r (ascending): the slots of its exchange messages.
int shard_chunks(const Layer &L, int world, int r, int *out) {
    const int m = L.H / world;
    int n = 0;
    for (int v = 0; v < L.n_chunks; ++v)
        if (pair_of(L.H, v) / m == r) out[n++] = v;
    return n;
}

// Passing-block message of one rank: per slot (one of its 2m chunks) the
// indices [Hkv, l] int32, then K rows [Hkv, l, d] and V rows [Hkv, l, d] bf16;
// the slot of the last chunk (no successor) stays unused.
struct PassMsg { size_t idx, k, v, total; };
PassMsg pass_msg(const Layer &L, int world) {
    const size_t slots = 2 * (L.H / world);
    PassMsg g{};
    size_t o = 0;
    auto take = [&](size_t b) { size_t at = o; o = align256(o + b); return at; };
    g.idx = take(slots * L.Hkv * L.l * 4);
    g.k = take(slots * L.Hkv * L.l * L.d * 2);
    g.v = take(slots * L.Hkv * L.l * L.d * 2);
    g.total = std::max<size_t>(o, 256);
    return g;
}

// Query-partial message of one rank: per slot the normalised partial O
// [Hq, q, d] and the base-2 lse [Hq, q] of the query rows over that chunk.
struct PartMsg { size_t o, lse, total; };
PartMsg part_msg(const Layer &L, int world) {
    const size_t slots = 2 * (L.H / world);
    PartMsg g{};
    size_t o = 0;
    auto take = [&](size_t b) { size_t at = o; o = align256(o + b); return at; };
    g.o = take(slots * L.Hq * L.q * L.d * 4);
    g.lse = take(slots * L.Hq * L.q * 4);
    g.total = o;
    return g;
}

// Collects 2-D copies and launches them, kMaxCopyJobs per launch.  The jobs
// of one launch run concurrently: none may read what another writes (flush
// between dependent copies).
struct Copier {
    CopyBatch b{};
    int64_t most = 0;  // units of the largest job of the batch
    cudaStream_t st;
    explicit Copier(cudaStream_t s) : st(s) {}
    spava_status add(const void *src, int64_t src_pitch, void *dst, int64_t dst_pitch, int64_t width,
                     int64_t height) {
        if (width <= 0 || height <= 0) return SPAVA_OK;
        const auto a = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                       static_cast<uintptr_t>(src_pitch) | static_cast<uintptr_t>(dst_pitch) |
                       static_cast<uintptr_t>(width);
        const int unit = (a & 15) == 0 ? 16 : 4;
        if (a & 3) return SPAVA_ERR_MISALIGNED;
        if (width >= (1LL << 31) || height >= (1LL << 31)) return SPAVA_ERR_UNSUPPORTED;
        if (b.n == kMaxCopyJobs) SPAVA_TRY(flush());
        b.job[b.n++] = CopyJob{static_cast<const char *>(src), static_cast<char *>(dst), src_pitch,
                               dst_pitch, static_cast<int32_t>(width), static_cast<int32_t>(height),
                               unit, 0};
        most = std::max(most, width / unit * height);
        return SPAVA_OK;
    }
    spava_status flush() {
        if (b.n == 0) return SPAVA_OK;
        const int64_t blocks = std::min<int64_t>((most + 255) / 256, 1024);
        batched_copy_kernel<<<dim3(static_cast<unsigned>(blocks), static_cast<unsigned>(b.n)), 256, 0, st>>>(b);
        b.n = 0;
        most = 0;
        return launched();
    }
};

// Copies between the workspace's passing blocks (idx [2H-1, Hkv, l], packed
// K/V [Hkv, L, d]) and slot k of a pass message: to_msg = export.
spava_status pass_slot_copy(Copier &cp, const Layer &L, char *ws, char *msg, const PassMsg &g, int k,
                            int u, bool to_msg) {
    if (u >= L.n_chunks - 1 || L.l == 0) return SPAVA_OK;  // no passing block
    const WsLayout w = ws_layout(L);
    const int64_t l_eff = std::min(L.l, L.off[u + 1] - L.off[u]);
    const int64_t row = int64_t(L.d) * 2;
    char *idx_ws = ws + w.idx + size_t(u) * L.Hkv * L.l * 4;
    char *idx_m = msg + g.idx + size_t(k) * L.Hkv * L.l * 4;
    const int64_t idx_bytes = int64_t(L.Hkv) * L.l * 4;
    if (to_msg) SPAVA_TRY(cp.add(idx_ws, idx_bytes, idx_m, idx_bytes, idx_bytes, 1));
    else SPAVA_TRY(cp.add(idx_m, idx_bytes, idx_ws, idx_bytes, idx_bytes, 1));
    for (int kv = 0; kv < 2; ++kv) {
        char *packed = ws + (kv ? w.pv : w.pk) + size_t(L.pcum[u]) * row;     // KV head 0
        char *slot = msg + (kv ? g.v : g.k) + size_t(k) * L.Hkv * L.l * row;  // KV head 0
        const int64_t packed_pitch = int64_t(L.L) * row, slot_pitch = int64_t(L.l) * row;
        if (to_msg) SPAVA_TRY(cp.add(packed, packed_pitch, slot, slot_pitch, l_eff * row, L.Hkv));
        else SPAVA_TRY(cp.add(slot, slot_pitch, packed, packed_pitch, l_eff * row, L.Hkv));
    }
    return SPAVA_OK;
}

// Copies between the workspace's query partials of segment 1+v and slot k of
// a partial message.
spava_status part_slot_copy(Copier &cp, const Layer &L, char *ws, char *msg, const PartMsg &g, int k,
                            int v, bool to_msg) {
    const WsLayout w = ws_layout(L);
    const int64_t o_bytes = int64_t(L.Hq) * L.q * L.d * 4, l_bytes = int64_t(L.Hq) * L.q * 4;
    char *o_ws = ws + w.part_o + size_t(1 + v) * o_bytes, *o_m = msg + g.o + size_t(k) * o_bytes;
    char *l_ws = ws + w.part_lse + size_t(1 + v) * l_bytes, *l_m = msg + g.lse + size_t(k) * l_bytes;
    // Rows of d floats (o) and one row of Hq*q floats (lse).
    const int64_t o_row = int64_t(L.d) * 4, o_rows = int64_t(L.Hq) * L.q;
    if (to_msg) {
        SPAVA_TRY(cp.add(o_ws, o_row, o_m, o_row, o_row, o_rows));
        SPAVA_TRY(cp.add(l_ws, l_bytes, l_m, l_bytes, l_bytes, 1));
    } else {
        SPAVA_TRY(cp.add(o_m, o_row, o_ws, o_row, o_row, o_rows));
        SPAVA_TRY(cp.add(l_m, l_bytes, l_ws, l_bytes, l_bytes, 1));
    }
    return SPAVA_OK;
}


}  // namespace

extern "C" {

spava_status spava_shard_layout(const spava_config *cfg, int32_t rank, int32_t world,
                                int64_t *local_first, int64_t *n_local, int32_t *slot_chunk) {
    Layer L;
    SPAVA_TRY(make_shard_layer(cfg, rank, world, &L));
    if (local_first)
        for (int r = 0; r < L.n_chunks + 2; ++r) local_first[r] = L.loc[r];
    if (n_local) *n_local = L.Nl;
    if (slot_chunk) {
        int ch[kMaxChunks];
        const int n = shard_chunks(L, world, rank, ch);
        for (int k = 0; k < n; ++k) slot_chunk[k] = ch[k];
    }
    return SPAVA_OK;
}

spava_status spava_shard_sizes(const spava_config *cfg, int32_t world, size_t *ws_bytes,
                               size_t *pass_msg_bytes, size_t *part_msg_bytes) {
    Layer L;
    SPAVA_TRY(make_shard_layer(cfg, 0, world, &L));
    if (ws_bytes) *ws_bytes = ws_layout(L).total;
    if (pass_msg_bytes) *pass_msg_bytes = pass_msg(L, world).total;
    if (part_msg_bytes) *part_msg_bytes = part_msg(L, world).total;
    return SPAVA_OK;
}

spava_status spava_shard_front(const spava_config *cfg, int32_t rank, int32_t world, const void *q,
                               const void *k, const void *v, void *pass_send, void *ws,
                               size_t ws_bytes, void *stream) {
    Layer L;
    SPAVA_TRY(make_shard_layer(cfg, rank, world, &L));
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(v));
    SPAVA_TRY(check_ptr(pass_send));
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(ws);
    SPAVA_TRY(run_front(L, q, k, v, nullptr, w, st));
    const PassMsg g = pass_msg(L, world);
    int ch[kMaxChunks];
    const int n = shard_chunks(L, world, rank, ch);
    Copier cp(st);
    for (int s = 0; s < n; ++s)
        SPAVA_TRY(pass_slot_copy(cp, L, w, static_cast<char *>(pass_send), g, s, ch[s], true));
    return cp.flush();
}

spava_status spava_shard_local_attn(const spava_config *cfg, int32_t rank, int32_t world,
                                    const void *q, const void *k, const void *v, void *o, float *lse,
                                    void *part_send, void *ws, size_t ws_bytes, void *stream) {
    Layer L;
    SPAVA_TRY(make_shard_layer(cfg, rank, world, &L));
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(v));
    SPAVA_TRY(check_ptr(o));
    SPAVA_TRY(check_ptr(lse, false));
    SPAVA_TRY(check_ptr(part_send));
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(ws);
    const WsLayout lay = ws_layout(L);
    // Anchor rows and the query rows' partials over the anchor, this rank's
    // chunks and the query block: nothing from another rank is needed.
    SPAVA_TRY(run_attn(L, q, k, v, w + lay.pk, w + lay.pv, o, lse, w, st, 0, INT32_MAX,
                       (1u << kAnchor) | (1u << kQueryPart), false));
    const PartMsg g = part_msg(L, world);
    int ch[kMaxChunks];
    const int n = shard_chunks(L, world, rank, ch);
    Copier cp(st);
    for (int s = 0; s < n; ++s)
        SPAVA_TRY(part_slot_copy(cp, L, w, static_cast<char *>(part_send), g, s, ch[s], true));
    return cp.flush();
}

spava_status spava_shard_context_attn(const spava_config *cfg, int32_t rank, int32_t world,
                                      const void *q, const void *k, const void *v,
                                      const void *pass_all, void *o, float *lse, int32_t *idx_out,
                                      void *ws, size_t ws_bytes, void *stream) {
    Layer L;
    SPAVA_TRY(make_shard_layer(cfg, rank, world, &L));
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(v));
    SPAVA_TRY(check_ptr(o));
    SPAVA_TRY(check_ptr(lse, false));
    SPAVA_TRY(check_ptr(pass_all));
    SPAVA_TRY(check_ptr(idx_out, false));
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(ws);
    const WsLayout lay = ws_layout(L);
    const PassMsg g = pass_msg(L, world);
    // Every other rank's passing blocks into the packed buffer.
    Copier cp(st);
    for (int r = 0; r < world; ++r) {
        if (r == rank) continue;
        int ch[kMaxChunks];
        const int n = shard_chunks(L, world, r, ch);
        char *msg = const_cast<char *>(static_cast<const char *>(pass_all)) + size_t(r) * g.total;
        for (int s = 0; s < n; ++s) SPAVA_TRY(pass_slot_copy(cp, L, w, msg, g, s, ch[s], false));
    }
    SPAVA_TRY(cp.flush());
    if (idx_out && L.l > 0) {  // after the imports that complete the indices
        const int64_t b = int64_t(L.n_chunks - 1) * L.Hkv * L.l * 4;
        SPAVA_TRY(cp.add(w + lay.idx, b, idx_out, b, b, 1));
        SPAVA_TRY(cp.flush());
    }
    return run_attn(L, q, k, v, w + lay.pk, w + lay.pv, o, lse, w, st, 0, INT32_MAX, 1u << kCtx, false);
}

spava_status spava_shard_merge(const spava_config *cfg, int32_t rank, int32_t world,
                               const void *part_all, void *o, float *lse, void *ws, size_t ws_bytes,
                               void *stream) {
    Layer L;
    SPAVA_TRY(make_shard_layer(cfg, rank, world, &L));
    SPAVA_TRY(check_ptr(o));
    SPAVA_TRY(check_ptr(lse, false));
    SPAVA_TRY(check_ptr(part_all));
    SPAVA_TRY(check_ws(L, ws, ws_bytes));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(ws);
    const PartMsg g = part_msg(L, world);
    Copier cp(st);
    for (int r = 0; r < world; ++r) {
        if (r == rank) continue;
        int ch[kMaxChunks];
        const int n = shard_chunks(L, world, r, ch);
        char *msg = const_cast<char *>(static_cast<const char *>(part_all)) + size_t(r) * g.total;
        for (int s = 0; s < n; ++s) SPAVA_TRY(part_slot_copy(cp, L, w, msg, g, s, ch[s], false));
    }
    SPAVA_TRY(cp.flush());
    return run_merge(L, o, lse, w, st);
}

}  // extern "C"

// ==================================================================== scores
// without caller-provided scratch
//
// spava_score needs scratch memory for the per-chunk softmax statistics of the
// query block, which normally lives in the caller's workspace.  Some callers
// cannot provide one: a plug-in inside a host engine that owns all device
// memory and hands a kernel only its input and output buffers, or code that
// must not allocate after start-up (real-time or certified deployments, and
// latency-critical paths where cudaMalloc would synchronise the device).  For
// them the scratch lives in the fixed array below, compiled into the library:
// every GPU that loads the library holds these bytes until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr size_t kNoAllocStatusBytes = 256;  // status word (byte 0), work-item counter (byte 128)

static __device__ __align__(256) unsigned char g_score_scratch[kNoAllocScratchBytes];

// Device address of g_score_scratch on the current device.  The name is only
// a host-side stand-in for the array, so the address is looked up with the
// device current, on every call: the lookup is cheap once the module is
// loaded, and no address can outlive a reset of the device's context.
spava_status scratch_address(void **out) {
    void *p = nullptr;
    SPAVA_CUDA(cudaGetSymbolAddress(&p, g_score_scratch));
    *out = p;
    return SPAVA_OK;
}

}  // namespace

extern "C" spava_status spava_score_noalloc(const spava_config *cfg, const void *q, const void *k,
                                            float *scores, void *stream) {
    Layer L;
    SPAVA_TRY(make_layer(cfg, &L));
    SPAVA_TRY(check_ptr(q));
    SPAVA_TRY(check_ptr(k));
    SPAVA_TRY(check_ptr(scores));
    // The fixed scratch holds the per-chunk statistics only: the row-normalised
    // variant (statistics of every segment first) is not offered here.
    if (L.norm) return SPAVA_ERR_UNSUPPORTED;
    const size_t stats_bytes = sizeof(float) * size_t(L.n_chunks - 1) * L.Hq * L.q;
    if (kNoAllocStatusBytes + stats_bytes > kNoAllocScratchBytes) return SPAVA_ERR_WORKSPACE;
    void *scratch = nullptr;
    SPAVA_TRY(scratch_address(&scratch));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *base = static_cast<char *>(scratch);
    int *status = reinterpret_cast<int *>(base);
    float *stats = reinterpret_cast<float *>(base + kNoAllocStatusBytes);
    // The array keeps the previous call's contents: the status word must start
    // at zero; every statistic is written before it is read.
    SPAVA_CUDA(cudaMemsetAsync(status, 0, sizeof(int), st));

    AttnParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.L = L;
    SPAVA_TRY(map_tokens(&sp.tmQ, q, L, L.Hq));
    SPAVA_TRY(map_tokens(&sp.tmK, k, L, L.Hkv));
    sp.n_groups = plan_attention(L, true, sp.groups);
    sp.stats = stats;
    sp.status = status;
    sp.queue = reinterpret_cast<int *>(base + 128);  // work-item counter, inside the status block
    SPAVA_TRY(L.d == 128 ? launch_attn<128, true>(sp, st) : launch_attn<64, true>(sp, st));

    return run_scores(L, q, k, stats, scores, status, st);
}

extern "C" spava_status spava_score_noalloc_status(void *stream, int32_t *flags) {
    if (!flags) return SPAVA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    SPAVA_TRY(scratch_address(&scratch));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    SPAVA_CUDA(cudaMemcpyAsync(&h, scratch, sizeof(h), cudaMemcpyDeviceToHost, st));
    SPAVA_CUDA(cudaStreamSynchronize(st));
    if (h) {
        SPAVA_CUDA(cudaMemsetAsync(scratch, 0, sizeof(h), st));
        SPAVA_CUDA(cudaStreamSynchronize(st));
    }
    *flags = h;
    return (h & kStatusTimeout) ? SPAVA_ERR_TIMEOUT : SPAVA_OK;
}

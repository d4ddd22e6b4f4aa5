// plan.cuh -- work items and key segments of the approximate attention, shared
// by the host planner and the kernels (__host__ __device__, integer only).
//
// Sequence split ("Riepilogo Tecnico: APB-V", Metodologia, "Suddivisione del
// Contesto e Disposizione ZigZag"): [anchor | chunk 0 .. chunk 2H-1 | query].
// Physical host p holds virtual hosts p and 2H-1-p.
//
// Key set of a row ("Meccanismo di Attenzione Approssimata", "Computazione"),
// expressed as at most four contiguous segments of either the original K/V
// (src 0, token positions) or the packed passing K/V (src 1, packed rows
// [anchor | P_0 | P_1 | ...]):
//   context row t of chunk v:
//     local_pair_full and v >= H (partner p = 2H-1-v, an earlier chunk):
//        packed [0, pcum[p])            anchor + P_0..P_{p-1}
//        packed [pcum[p+1], pcum[v])    P_{p+1}..P_{v-1}
//        K      [off[p], off[p+1])      the partner chunk in full
//     otherwise:
//        packed [0, pcum[v])            anchor + P_0..P_{v-1}
//     and   K   [off[v], t]             own chunk, causal
//   anchor row t:  K [0, t]
//   query rows ("Forward Fuso di Contesto e Query"): one partial per segment
//     s = 0 anchor [0,a), s = 1+v chunk v, s = 2H+1 query block [N-q, t];
//     the partials are merged by log-sum-exp afterwards.
//   score statistics of chunk u: K [off[u], off[u+1]) for the query rows.
//
// Positions are global token positions throughout.  The token-major buffers
// (Q, K, V, O, lse) may hold only some regions of the sequence -- a shard of
// the ZigZag sequence parallelism holds the anchor, its own chunks and the
// query block ("Comunicazione Sovrapposta": one physical host per GPU) -- laid
// out region after region; Layer::loc gives each region's first local row,
// and every load or store of a token row subtracts its region's shift.  On one
// GPU every region is held at its global position (all shifts 0).
#pragma once

#include <stdint.h>

namespace spava {

constexpr int kMaxChunks = 64;   // 2H <= 64
constexpr int kMaxGroups = 2 * kMaxChunks + 8 + 2 * kMaxChunks;
constexpr int kRowTile = 128;    // query rows per work item
constexpr int kKeyTile = 128;    // keys per pipeline step
constexpr int kMaxSegs = 4;      // key segments of one work item
constexpr int kMaxPool = 255;    // widest score-pooling window

enum ItemKind : int32_t { kCtx = 0, kAnchor = 1, kQueryPart = 2, kStats = 3 };

// Regions of the sequence: 0 the anchor, 1 + v chunk v, 2H + 1 the query block.
constexpr int kMaxRegions = kMaxChunks + 2;

struct Layer {
    int32_t H, Hq, Hkv, d, G, lpf, l, n_chunks;
    int32_t norm, pool;                // selection variants: row-normalised scores, window width
    int32_t N, a, q, C, L;             // tokens, anchor, query, context, packed rows
    int32_t Nl;                        // rows of the (local) token-major buffers
    float scale_log2;                  // softmax scale * log2(e)
    uint64_t own;                      // bit v: chunk v is held (and computed) here
    int32_t off[kMaxChunks + 1];       // chunk offsets
    int32_t pcum[kMaxChunks + 1];      // packed row where P_u starts; pcum[0] = a
    int32_t loc[kMaxRegions];          // first local row of each region, -1 if not held
};

__host__ __device__ inline int region_first(const Layer &L, int r) {
    return r == 0 ? 0 : (r <= L.n_chunks ? L.off[r - 1] : L.N - L.q);
}
// Global position minus local row, for the rows of region r.
__host__ __device__ inline int region_shift(const Layer &L, int r) { return region_first(L, r) - L.loc[r]; }
__host__ __device__ inline int query_region(const Layer &L) { return L.n_chunks + 1; }
__host__ __device__ inline bool owns(const Layer &L, int v) { return (L.own >> v) & 1u; }

// A run of work items of one kind and one chunk/segment.  Items inside a group
// run KV head by KV head, the costlier row tiles first (decode_pair_item): the
// CTAs resident at any moment then work on one KV head's packed passing K/V and
// chunks, which fit in L2.
struct Group {
    int32_t kind, sub, n_rt, item_begin;
};

struct Item {
    int32_t kind, sub, rt, h;
};

struct Seg {
    int32_t src, begin, end, causal;
    int32_t shift;  // src 0: global position minus local row of this segment's keys
};

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ inline int pair_of(int H, int v) { return v < H ? v : 2 * H - 1 - v; }

// Rows [row0, row_end) of the item.
__host__ __device__ inline void item_rows(const Layer &L, const Item &it, int &row0, int &row_end) {
    int lo, hi;
    if (it.kind == kCtx) {
        lo = L.off[it.sub];
        hi = L.off[it.sub + 1];
    } else if (it.kind == kAnchor) {
        lo = 0;
        hi = L.a;
    } else {
        lo = L.N - L.q;
        hi = L.N;
    }
    row0 = lo + it.rt * kRowTile;
    row_end = row0 + kRowTile < hi ? row0 + kRowTile : hi;
}

// Segment [b, e) of the packed passing K/V (src 1), or of region r's token
// rows (src 0).
__host__ __device__ inline void add_seg(const Layer &L, Seg *s, int &n, int src, int b, int e,
                                        int causal, int region = 0) {
    if (e > b) {
        s[n].src = src;
        s[n].begin = b;
        s[n].end = e;
        s[n].causal = causal;
        s[n].shift = src == 0 ? region_shift(L, region) : 0;
        ++n;
    }
}

// Region whose rows an item computes.
__host__ __device__ inline int item_region(const Layer &L, const Item &it) {
    return it.kind == kCtx ? 1 + it.sub : (it.kind == kAnchor ? 0 : query_region(L));
}

// Segments of the item's key sequence (at most kMaxSegs).  Returns their count.
__host__ __device__ inline int build_segments(const Layer &L, const Item &it, Seg *s) {
    int n = 0, row0, row_end;
    item_rows(L, it, row0, row_end);
    switch (it.kind) {
        case kCtx: {
            const int v = it.sub;
            if (L.lpf && v >= L.H) {
                const int p = 2 * L.H - 1 - v;
                add_seg(L, s, n, 1, 0, L.pcum[p], 0);
                add_seg(L, s, n, 1, L.pcum[p + 1], L.pcum[v], 0);
                add_seg(L, s, n, 0, L.off[p], L.off[p + 1], 0, 1 + p);
            } else {
                add_seg(L, s, n, 1, 0, L.pcum[v], 0);
            }
            add_seg(L, s, n, 0, L.off[v], row_end, 1, 1 + v);
            break;
        }
        case kAnchor:
            add_seg(L, s, n, 0, 0, row_end, 1, 0);
            break;
        case kQueryPart: {
            const int sg = it.sub;
            if (sg == 0)
                add_seg(L, s, n, 0, 0, L.a, 0, 0);
            else if (sg <= L.n_chunks)
                add_seg(L, s, n, 0, L.off[sg - 1], L.off[sg], 0, sg);
            else
                add_seg(L, s, n, 0, L.N - L.q, row_end, 1, query_region(L));
            break;
        }
        default:  // kStats
            add_seg(L, s, n, 0, L.off[it.sub], L.off[it.sub + 1], 0, 1 + it.sub);
            break;
    }
    return n;
}

// Position in an item's key sequence: segment index and 128-key tile inside it.
struct TileCursor {
    int seg = 0, tile = 0;
    __host__ __device__ void advance(const Seg *s) {
        if (s[seg].begin + (tile + 1) * kKeyTile >= s[seg].end) {
            ++seg;
            tile = 0;
        } else {
            ++tile;
        }
    }
};

__host__ __device__ inline int count_tiles(const Seg *s, int n) {
    int t = 0;
    for (int i = 0; i < n; ++i) t += cdiv(s[i].end - s[i].begin, kKeyTile);
    return t;
}

}  // namespace spava

// select_kernels.cuh -- passing-block selection, aggregation, and the merge of
// the query-row partials.
//
// "Riepilogo Tecnico: APB-V", Metodologia, "Blocchi di Passaggio": per host,
// the most essential KV (top-l per KV head by query-to-context score) are
// aggregated into passing blocks; on one GPU the cross-host transfer of those
// blocks ("Comunicazione Sovrapposta") becomes the gather in pack_kernel.
// "Forward Fuso di Contesto e Query": the query rows' per-segment partial
// results are merged through their log-sum-exp (merge_kernel).
#pragma once

#include "plan.cuh"
#include "sm100.cuh"

namespace spava {

// fp32 -> uint32 key whose unsigned order equals the float order.
__device__ __forceinline__ uint32_t ordered_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the block (blockDim.x multiple of 32, <= 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < nw) warp_sums[lane] = s;  // inclusive over warps
        if (lane == nw - 1) *total = s;
    }
    __syncthreads();
    const int before = (w > 0 ? warp_sums[w - 1] : 0) + x - v;
    __syncthreads();
    return before;
}

// One CTA per (chunk u < 2H-1, KV head g): the min(l, n_u) largest scores (or
// pooled window sums, rank_value) of
// the chunk, ties to the lower token index, written ascending as absolute
// positions; padding -1.  Radix select on the ordered 32-bit key (4 passes of
// 8 bits) finds the exact threshold key T and how many keys equal to T are
// kept; a final pass in index order emits the set, so the output is sorted and
// the lower-index rule holds for the keys equal to T.
constexpr int kSelectThreads = 1024;

// The value a key is ranked by: its score, or with pooling (L.pool = w >= 3)
// the sum of the scores of the w keys centred on it inside the chunk, added in
// ascending order with plain fp32 adds (the window mean with zero padding up to
// the factor 1/w, which does not change the ranking).  Scores are read through
// L2 (another CTA of the same launch may have written them).
__device__ __forceinline__ float rank_value(const float *S, int n, int j, int pool) {
    if (pool <= 1) return __ldcg(S + j);
    const int h = pool >> 1;
    const int k0 = j - h < 0 ? 0 : j - h, k1 = j + h < n ? j + h : n - 1;
    float s = 0.f;
    for (int k = k0; k <= k1; ++k) s = __fadd_rn(s, __ldcg(S + k));
    return s;
}

// The selection of one (chunk u, KV head g) by the whole CTA; returns l_eff.
// `keys` (shared memory, room for `cap` entries, or null): when the chunk
// fits, each key's ordered rank value is computed once into it and the five
// passes read it from there.
__device__ __forceinline__ int select_chunk(const Layer &L, const float *scores, int32_t *idx, int u,
                                            int g, uint32_t *keys = nullptr, int cap = 0) {
    __shared__ int hist[256];
    __shared__ int warp_sums[32];
    __shared__ int s_digit, s_need, s_total;
    const int base = L.off[u];
    const int n = L.off[u + 1] - base;
    const int l_eff = min(L.l, n);
    const float *S = scores + static_cast<size_t>(g) * L.C + (base - L.a);
    int32_t *out = idx + (static_cast<size_t>(u) * L.Hkv + g) * L.l;
    const int tid = threadIdx.x;

    for (int r = l_eff + tid; r < L.l; r += blockDim.x) out[r] = -1;
    if (l_eff == 0) return 0;
    if (l_eff == n) {
        for (int r = tid; r < n; r += blockDim.x) out[r] = base + r;
        return l_eff;
    }
    const bool cached = keys != nullptr && n <= cap;
    if (cached) {
        for (int j = tid; j < n; j += blockDim.x) keys[j] = ordered_key(rank_value(S, n, j, L.pool));
        __syncthreads();
    }
    auto key_of = [&](int j) -> uint32_t {
        return cached ? keys[j] : ordered_key(rank_value(S, n, j, L.pool));
    };

    uint32_t prefix = 0, mask = 0;
    int need = l_eff;
    for (int shift = 24; shift >= 0; shift -= 8) {
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int j = tid; j < n; j += blockDim.x) {
            const uint32_t k = key_of(j);
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
        }
        __syncthreads();
        if (tid == 0) {
            int cum = 0, d = 0;
            for (int b = 255; b >= 0; --b) {
                if (cum + hist[b] >= need) {
                    d = b;
                    break;
                }
                cum += hist[b];
            }
            s_digit = d;
            s_need = need - cum;
        }
        __syncthreads();
        prefix |= static_cast<uint32_t>(s_digit) << shift;
        mask |= 255u << shift;
        need = s_need;
        __syncthreads();
    }
    const uint32_t T = prefix;  // key of the l_eff-th largest score
    const int need_eq = need;   // how many keys equal to T are kept

    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int j0 = min(n, tid * per), j1 = min(n, j0 + per);
    int gt = 0, eq = 0;
    for (int j = j0; j < j1; ++j) {
        const uint32_t k = key_of(j);
        gt += k > T;
        eq += k == T;
    }
    const int eq_before = block_exclusive_scan(eq, warp_sums, &s_total);
    const int take_eq = max(0, min(eq, need_eq - eq_before));
    int pos = block_exclusive_scan(gt + take_eq, warp_sums, &s_total);
    int taken = 0;
    for (int j = j0; j < j1; ++j) {
        const uint32_t k = key_of(j);
        if (k > T || (k == T && taken < take_eq)) {
            out[pos++] = base + j;
            taken += (k == T);
        }
    }
    return l_eff;
}

// The k-th producing chunk (u < 2H-1) held here, in increasing u; -1 if there
// is none (the host sizes the grids so that there always is).
__device__ __forceinline__ int nth_owned_producer(const Layer &L, int k) {
    for (int u = 0; u < L.n_chunks - 1; ++u)
        if (owns(L, u) && k-- == 0) return u;
    return -1;
}

// Dynamic shared memory of the selection kernels: room for the rank keys of
// the longest chunk (0 if it does not fit; the passes then recompute them).
__global__ void __launch_bounds__(kSelectThreads) topk_kernel(const Layer L, const float *scores,
                                                              int32_t *idx, int key_cap) {
    extern __shared__ uint32_t sel_keys[];
    const int u = nth_owned_producer(L, blockIdx.x / L.Hkv);
    if (u >= 0) select_chunk(L, scores, idx, u, blockIdx.x % L.Hkv, sel_keys, key_cap);
}

// Copies packed rows [r0, r1) of KV head g from the local token rows src(r): one warp
// per row, lanes 0-15 the K row and lanes 16-31 the V row in 16-byte pieces,
// 8 rows in flight per warp.
template <int D, typename Src>
__device__ __forceinline__ void copy_rows(const Layer &L, const __nv_bfloat16 *K,
                                          const __nv_bfloat16 *V, __nv_bfloat16 *PK,
                                          __nv_bfloat16 *PV, int g, int r0, int r1, int warp0,
                                          int n_warps, Src src) {
    constexpr int kPieces = D * 2 / 16;
    const int lane = threadIdx.x & 31, half = lane >> 4, c = lane & 15;
    const __nv_bfloat16 *from = half ? V : K;
    __nv_bfloat16 *to = half ? PV : PK;
    for (int b = r0 + warp0 * 8; b < r1; b += n_warps * 8) {
        uint4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            v[k] = make_uint4(0, 0, 0, 0);
            if (b + k < r1 && c < kPieces) {
                const int t = src(b + k);
                v[k] = __ldg(reinterpret_cast<const uint4 *>(from + (static_cast<size_t>(t) * L.Hkv + g) * D) + c);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (b + k < r1 && c < kPieces)
                reinterpret_cast<uint4 *>(to + (static_cast<size_t>(g) * L.L + b + k) * D)[c] = v[k];
    }
}

// Selection and gather in one launch (the layer entry points): CTA (u, g) for
// each producing chunk u < 2H-1 held here selects the passing block of chunk u
// for KV head g exactly as topk_kernel, then copies those K/V rows to the
// packed rows pcum[u] + r; the CTAs after them copy the anchor rows.  The
// selected indices are read back from idx by the CTA that wrote them (visible
// after __syncthreads).
constexpr int kAnchorRowsPerCta = 256;
template <int D>
__global__ void __launch_bounds__(kSelectThreads) select_pack_kernel(
    const Layer L, const float *scores, int32_t *idx, const __nv_bfloat16 *K,
    const __nv_bfloat16 *V, __nv_bfloat16 *PK, __nv_bfloat16 *PV, int n_sel_ctas, int key_cap) {
    extern __shared__ uint32_t sel_keys[];
    const int n_sel = n_sel_ctas;
    const int warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
    if (static_cast<int>(blockIdx.x) < n_sel) {
        const int u = nth_owned_producer(L, blockIdx.x / L.Hkv), g = blockIdx.x % L.Hkv;
        if (u < 0) return;
        const int l_eff = select_chunk(L, scores, idx, u, g, sel_keys, key_cap);
        __syncthreads();
        const int32_t *sel = idx + (static_cast<size_t>(u) * L.Hkv + g) * L.l;
        const int p0 = L.pcum[u], sh = region_shift(L, 1 + u);
        copy_rows<D>(L, K, V, PK, PV, g, p0, p0 + l_eff, warp, n_warps,
                     [&](int r) { return sel[r - p0] - sh; });
    } else {
        const int b = blockIdx.x - n_sel;
        const int per_g = (L.a + kAnchorRowsPerCta - 1) / kAnchorRowsPerCta;
        const int g = b / per_g, r0 = (b % per_g) * kAnchorRowsPerCta;
        const int r1 = min(L.a, r0 + kAnchorRowsPerCta);
        const int sh = region_shift(L, 0);
        copy_rows<D>(L, K, V, PK, PV, g, r0, r1, warp, n_warps, [&](int r) { return r - sh; });
    }
}

// Packed passing K/V: packed row `row` = g*L + r of KV head g is the anchor row r
// (r < a) or the s-th kept key of chunk u (r = pcum[u] + s); the rows of chunks
// not held here are left alone.  HBM-bound gather:
// persistent warps walk groups of 32 packed rows; lane i resolves the source of
// row i with one coalesced index load, the sources are shuffled out, and rows are
// copied 8 at a time (first half-warp K, second half V, 16 bytes per lane) with
// all 8 loads of a lane issued before its stores.
constexpr int kPackThreads = 256;
constexpr int kPackBatch = 8;

// Local token row of packed row r of KV head g; -1: a row to zero (an index
// that is not a position of chunk u); -2: a row of a chunk not held here.
__device__ __forceinline__ int packed_source(const Layer &L, const int32_t *idx, int g, int r) {
    if (r < L.a) return r - region_shift(L, 0);
    int u = 0;
    while (u + 1 < L.n_chunks - 1 && r >= L.pcum[u + 1]) ++u;
    if (!owns(L, u)) return -2;
    const int t = idx[(static_cast<size_t>(u) * L.Hkv + g) * L.l + (r - L.pcum[u])];
    return (t >= L.off[u] && t < L.off[u + 1]) ? t - region_shift(L, 1 + u) : -1;
}

template <int D>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(const Layer L, const __nv_bfloat16 *K,
                                                            const __nv_bfloat16 *V, const int32_t *idx,
                                                            __nv_bfloat16 *PK, __nv_bfloat16 *PV) {
    constexpr int kChunks = D * 2 / 16;  // 16-byte pieces per row
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4, c = lane & 15;
    const long long total = static_cast<long long>(L.Hkv) * L.L;
    const long long n_groups = (total + 31) / 32;
    const long long stride = static_cast<long long>(gridDim.x) * (kPackThreads / 32);
    const __nv_bfloat16 *src_base = half ? V : K;
    __nv_bfloat16 *dst_base = half ? PV : PK;
    for (long long grp = static_cast<long long>(blockIdx.x) * (kPackThreads / 32) + (threadIdx.x >> 5);
         grp < n_groups; grp += stride) {
        // Source element offset of this lane's row, or -1 (past the end, or an
        // index that is not a token position: written as a zero row).
        const long long row_l = grp * 32 + lane;
        long long src_l = -1;
        int src = -2;
        if (row_l < total) {
            const int g = static_cast<int>(row_l / L.L);
            src = packed_source(L, idx, g, static_cast<int>(row_l % L.L));
            if (src >= 0) src_l = (static_cast<long long>(src) * L.Hkv + g) * D;
        }
        // rows to leave alone: past the end, or of a chunk not held here
        const uint32_t keep = __ballot_sync(0xffffffffu, src != -2);
#pragma unroll 1
        for (int b = 0; b < 32; b += kPackBatch) {
            uint4 v[kPackBatch];
#pragma unroll
            for (int k = 0; k < kPackBatch; ++k) {
                const long long so = __shfl_sync(0xffffffffu, src_l, b + k);
                v[k] = make_uint4(0, 0, 0, 0);
                if (so >= 0 && c < kChunks) v[k] = __ldg(reinterpret_cast<const uint4 *>(src_base + so) + c);
            }
#pragma unroll
            for (int k = 0; k < kPackBatch; ++k) {
                const long long row = grp * 32 + b + k;
                if (((keep >> (b + k)) & 1u) && c < kChunks)
                    reinterpret_cast<uint4 *>(dst_base + row * D)[c] = v[k];
            }
        }
    }
}

// Query rows: O = sum_s w_s O_s / sum_s w_s, w_s = 2^(lse2_s - max), over the
// segments s present (anchor if a > 0, every chunk, the query block itself).
// One warp per (head, query row); D/4 lanes hold 4 columns each.
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const Layer L, const float *part_O,
                                                    const float *part_lse, __nv_bfloat16 *O,
                                                    float *lse) {
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= L.Hq * L.q) return;
    const int h = w / L.q, i = w % L.q;
    const int n_seg = L.n_chunks + 2;
    const int s_first = L.a > 0 ? 0 : 1;
    float m = -INFINITY;
    for (int s = s_first; s < n_seg; ++s)
        m = fmaxf(m, part_lse[(static_cast<size_t>(s) * L.Hq + h) * L.q + i]);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float wsum = 0.f;
    for (int s = s_first; s < n_seg; ++s) {
        const size_t row = (static_cast<size_t>(s) * L.Hq + h) * L.q + i;
        const float ws = ex2(part_lse[row] - m);
        wsum += ws;
        if (lane < D / 4) {
            const float4 o = __ldg(reinterpret_cast<const float4 *>(part_O + row * D) + lane);
            acc[0] += ws * o.x;
            acc[1] += ws * o.y;
            acc[2] += ws * o.z;
            acc[3] += ws * o.w;
        }
    }
    const float inv = 1.f / wsum;
    const int t = L.N - L.q + i - region_shift(L, query_region(L));  // local row
    if (lane < D / 4) {
        uint2 v;
        v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        reinterpret_cast<uint2 *>(O + (static_cast<size_t>(t) * L.Hq + h) * D)[lane] = v;
    }
    if (lane == 0 && lse) lse[static_cast<size_t>(h) * L.Nl + t] = (m + __log2f(wsum)) * 0.69314718055994531f;
}

// Failure-path self-test: one thread waits on an mbarrier that nothing ever
// arrives on.  The bounded wait gives up after kWaitLimitCycles, flags the
// workspace status word and the kernel returns normally -- the same path every
// pipeline wait takes when a partner stops making progress.
__global__ void selftest_wait_kernel(int *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const AbortState ab{&abort_flag, status};
        mbar_wait(&bar, 0, ab);  // never completes: returns false after the limit
    }
}

}  // namespace spava

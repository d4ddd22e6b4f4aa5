// score_kernel.cuh -- query-to-context scores of the passing-block selection.
//
// "Riepilogo Tecnico: APB-V", Metodologia, "Blocchi di Passaggio": the most
// essential KV of each host are identified by query-to-context attention
// scores.  Score of key j of chunk u for KV head g:
//     S[g, j] = sum_{h in g} sum_{i in query block} exp2(x_{h,i,j} - lse2_{u,h,i}),
//     x = scale*log2(e) * q_{h,i} . k_{g,j},
// where lse2_{u,h,i} is the base-2 log-sum-exp of row (h, i) over chunk u:
// from the attention kernel's statistics mode, or -- the same values -- from
// the query-row partial of chunk u ("Forward Fuso di Contesto e Query").
// Equivalently: softmax over the chunk, summed over query rows and group heads.
//
// One CTA = a score unit: two 128-key tiles (the last unit of a chunk may have
// one) of one chunk and one KV head.  The product is formed transposed,
// S^T = K Q^T (M = 128 keys, N = 128 query rows of one head per block, K = d),
// so that TMEM lane j holds key j and each thread sums its own keys'
// probabilities without any cross-thread reduction; both tiles of a unit take
// the same query block from shared memory and the same log-sum-exp loads.  The
// summation order is fixed, so the result is deterministic.
//
// The exponentials are MUFU-bound (one per 2*d tensor FLOPs, against a MUFU
// rate of 16 per SM per clock), with the FMA pipe idle: a quarter of them run
// on the FMA pipe instead, as 2^a = 2^n * p(f) with n = round(a), f = a - n in
// [-1/2, 1/2] (Cody-Waite style reduction; n is read off the low mantissa bits
// of a + 1.5*2^23) and p a degree-4 polynomial fitted to 2^f in relative error
// by Lawson's iteratively reweighted least squares (fit_exp2_poly.py in this
// directory; max relative error 2.7e-6 in fp32 Horner form).
//
// FUSED = true also selects and gathers (the layer entry points): the CTA that
// writes the last 128-key tile of a (chunk, KV head) -- counted with an atomic
// per (chunk, KV head) -- selects that chunk's passing block for the KV head
// (select_chunk) and copies its K/V rows into the packed buffer; the CTAs after
// the scoring ones copy the anchor rows.  Selections of finished chunks thus
// run while later chunks are still being scored.
#pragma once

#include "plan.cuh"
#include "select_kernels.cuh"
#include "sm100.cuh"

namespace spava {

struct ScoreParams {
    CUtensorMap tmQ, tmK;
    Layer L;
    const float *stats;  // [2H-1, Hq, q] log2 domain
    float *scores;       // [Hkv, C]
    int *status;
    int32_t unit_begin[kMaxChunks + 1];  // prefix of score units over chunks u < 2H-1
    // FUSED only
    int *counters;       // [2H-1, Hkv] finished units, zero at launch
    int32_t *idx;        // [2H-1, Hkv, l]
    const __nv_bfloat16 *K, *V;
    __nv_bfloat16 *PK, *PV;  // [Hkv, L, D]
    int32_t n_score_ctas;
};

constexpr int kScoreTiles = 2;                  // 128-key tiles per score unit
constexpr int kScoreWarps = 16;                 // 4 per TMEM lane quarter
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kScoreProducer = kScoreWarps;
constexpr int kScoreMma = kScoreWarps + 1;
constexpr int kScoreBlockThreads = (kScoreWarps + 2) * 32;
constexpr int kPolyEvery = 4;                   // every 4th exponential pair on the FMA pipe

// Coefficients of p(f) ~ 2^f on [-1/2, 1/2] (fit_exp2_poly.py).
constexpr float kExp2C0 = 0.9999992847442627f;
constexpr float kExp2C1 = 0.6931217908859253f;
constexpr float kExp2C2 = 0.240247443318367f;
constexpr float kExp2C3 = 0.05591782182455063f;
constexpr float kExp2C4 = 0.009570080786943436f;

// 2^a for a pair of arguments on the FMA pipe.  Arguments below -126 are taken
// as -126 (2^-126 and below contribute nothing to a score).
__device__ __forceinline__ float2 exp2_fma2(float2 a) {
    a = make_float2(fmaxf(a.x, -126.f), fmaxf(a.y, -126.f));
    const float2 shifter = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
    const float2 t = fadd2(a, shifter);                            // n in the low mantissa bits
    const float2 n = fadd2(t, make_float2(-12582912.f, -12582912.f));
    const float2 f = ffma2(n, make_float2(-1.f, -1.f), a);        // a - n, exact
    float2 p = ffma2(make_float2(kExp2C4, kExp2C4), f, make_float2(kExp2C3, kExp2C3));
    p = ffma2(p, f, make_float2(kExp2C2, kExp2C2));
    p = ffma2(p, f, make_float2(kExp2C1, kExp2C1));
    p = ffma2(p, f, make_float2(kExp2C0, kExp2C0));
    // times 2^n: n added to the exponent field (t's low bits shifted into place)
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

template <int D>
struct ScoreSmem {
    static constexpr int kPanels = D / 64;
    static constexpr int kTile = 128 * D * 2;
    static constexpr int QS = 4;
    static constexpr int kOffK = 0;                        // the unit's key tiles
    static constexpr int kOffQ = kScoreTiles * kTile;      // query-block ring
    static constexpr int kOffBar = kOffQ + QS * kTile;
    static constexpr int kNumBar = 1 + 2 * QS + 2 * 2 + 1;
    static constexpr int kOffRed = kOffBar + kNumBar * 8;  // [4 parts][256 keys] partial sums
    static constexpr int kOffMisc = kOffRed + 4 * kScoreTiles * 128 * 4;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

static_assert(ScoreSmem<128>::kAlloc + 2048 <= 232448, "scoring smem over budget");

template <int D, bool FUSED = false>
__global__ void __launch_bounds__(kScoreBlockThreads, 1) score_kernel(const __grid_constant__ ScoreParams P) {
    using SM = ScoreSmem<D>;
    constexpr int QS = SM::QS;
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, 0, 0);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    if (FUSED && static_cast<int>(blockIdx.x) >= P.n_score_ctas) {
        // anchor rows into the packed buffer
        const Layer &L = P.L;
        const int b = blockIdx.x - P.n_score_ctas;
        const int per_g = (L.a + kAnchorRowsPerCta - 1) / kAnchorRowsPerCta;
        const int g = b / per_g, r0 = (b % per_g) * kAnchorRowsPerCta;
        const int r1 = min(L.a, r0 + kAnchorRowsPerCta);
        const int sh = region_shift(L, 0);
        copy_rows<D>(L, P.K, P.V, P.PK, P.PV, g, r0, r1, threadIdx.x >> 5, blockDim.x >> 5,
                     [&](int r) { return r - sh; });
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffBar);
    uint64_t *a_full = bars;
    uint64_t *q_full = a_full + 1;
    uint64_t *q_empty = q_full + QS;
    uint64_t *s_full = q_empty + QS;  // [2]: S of both tiles of block b in buffer b & 1
    uint64_t *s_free = s_full + 2;
    uint64_t *mma_drain = s_free + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::kOffMisc + 4);

    const Layer &L = P.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blockIdx.x = unit * Hkv + g, units enumerated over the chunks u < 2H-1
    const int g = blockIdx.x % L.Hkv;
    const int unit = blockIdx.x / L.Hkv;
    int u = 0;
    while (u + 1 < L.n_chunks - 1 && unit >= P.unit_begin[u + 1]) ++u;
    const int key0 = L.off[u] + (unit - P.unit_begin[u]) * kScoreTiles * 128;
    const int n_keys = min(kScoreTiles * 128, L.off[u + 1] - key0);  // 1 .. 256
    const int nt = cdiv(n_keys, 128);                                // key tiles: 1 or 2
    const int n_rb = cdiv(L.q, 128);
    const int NBLK = L.G * n_rb;  // column blocks: (head in group, 128 query rows)

    if (threadIdx.x == 0) {
        mbar_init(a_full, 1);
        for (int i = 0; i < QS; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kScoreThreads);
        }
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kScoreProducer && lane == 0) {
        tma_prefetch(&P.tmQ);
        tma_prefetch(&P.tmK);
    }
    if (warp == kScoreMma) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState ab{abort_flag, P.status};

    if (warp == kScoreProducer) {
        if (lane == 0) {
            mbar_expect_tx(a_full, nt * SM::kTile);
            const int krow = key0 - region_shift(L, 1 + u);  // local row of the unit's first key
            for (int t = 0; t < nt; ++t)
                for (int p = 0; p < SM::kPanels; ++p)
                    tma_load_3d(smem + SM::kOffK + t * SM::kTile + p * 16384, &P.tmK, p * 64, g,
                                krow + t * 128, a_full);
            int q_last[QS];
            for (int i = 0; i < QS; ++i) q_last[i] = -1;
            for (int b = 0; b < NBLK; ++b) {
                const int qs = b % QS;
                if (b >= QS && !mbar_wait(&q_empty[qs], ((b / QS) - 1) & 1, ab)) break;
                const int h = g * L.G + b / n_rb;
                const int r0 = L.N - L.q + (b % n_rb) * 128 - region_shift(L, query_region(L));
                mbar_expect_tx(&q_full[qs], SM::kTile);
                for (int p = 0; p < SM::kPanels; ++p)
                    tma_load_3d(smem + SM::kOffQ + qs * SM::kTile + p * 16384, &P.tmQ, p * 64, h, r0,
                                &q_full[qs]);
                q_last[qs] = b;
            }
            mbar_wait_drain(a_full, 0);
            for (int i = 0; i < QS; ++i)
                if (q_last[i] >= 0) mbar_wait_drain(&q_full[i], (q_last[i] / QS) & 1);
        }
    } else if (warp == kScoreMma) {
        if (lane == 0) {
            const uint32_t k_base = smem_u32(smem + SM::kOffK);
            const uint32_t q_base = smem_u32(smem + SM::kOffQ);
            bool ok = mbar_wait(a_full, 0, ab);
            tc_fence_after();
            for (int b = 0; ok && b < NBLK; ++b) {
                const int qs = b % QS, pb = b & 1;
                if (!mbar_wait(&q_full[qs], (b / QS) & 1, ab)) break;
                if (b >= 2 && !mbar_wait(&s_free[pb], ((b >> 1) - 1) & 1, ab)) break;
                tc_fence_after();
                const uint32_t qb = q_base + qs * SM::kTile;
                for (int t = 0; t < nt; ++t) {
                    const uint32_t kb = k_base + t * SM::kTile;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_ss(tmem + pb * 256 + t * 128, sdesc_sw128(kb + off, 16, 1024),
                               sdesc_sw128(qb + off, 16, 1024), kIdesc, kk > 0);
                    }
                }
                tc_commit(&q_empty[qs]);
                tc_commit(&s_full[pb]);
            }
            tc_commit(mma_drain);
            mbar_wait_drain(mma_drain, 0);
        }
        __syncwarp();
    } else {
        // Warp w: keys 32*(w%4) .. +31 of each tile (its TMEM lane quarter),
        // query-row columns 32*(w/4) .. +31 of every 128-column block; the four
        // column parts of a key are added at the end.
        const int quarter = warp & 3, part = warp >> 2;
        const int j = quarter * 32 + lane;  // key within a tile == TMEM lane
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const float2 sl2v = make_float2(L.scale_log2, L.scale_log2);
        float2 acc[kScoreTiles][4];  // per tile 8 independent partial sums, in packed pairs
#pragma unroll
        for (int t = 0; t < kScoreTiles; ++t)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[t][k] = make_float2(0.f, 0.f);
        const bool two = nt > 1;  // CTA-uniform
        // Exponentials of one pair of logits: pair k of the block (0..31 over
        // both tiles) goes to the FMA pipe when k % kPolyEvery is the last slot.
        auto add_pair = [&](int t, int c, float2 arg) {
            const int k = t * 16 + (c >> 1);
            const float2 p = (k % kPolyEvery == kPolyEvery - 1) ? exp2_fma2(arg)
                                                                 : make_float2(ex2(arg.x), ex2(arg.y));
            acc[t][(c >> 1) & 3] = fadd2(acc[t][(c >> 1) & 3], p);
        };
        bool ok = true;
        for (int b = 0; b < NBLK; ++b) {
            const int pb = b & 1;
            const int h = g * L.G + b / n_rb;
            const int i0 = (b % n_rb) * 128 + part * 32;
            const float *lse2 = P.stats + (static_cast<size_t>(u) * L.Hq + h) * L.q + i0;
            const int n_rows = min(32, L.q - i0);  // may be <= 0 for the ragged last block
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[pb], (b >> 1) & 1, ab));
            if (!ok) break;
            tc_fence_after();
            // The two tiles' logits one after the other (32 registers each:
            // 18 warps share each sub-partition's 16K registers).
            const bool vec = n_rows == 32 && ((reinterpret_cast<uintptr_t>(lse2) & 15) == 0);
#pragma unroll
            for (int t = 0; t < kScoreTiles; ++t) {
                if (t > 0 && !two) break;
                uint32_t r[32];
                tmem_ld32(lane_addr + pb * 256 + t * 128 + part * 32, r);
                tmem_wait_ld();
                if (t + 1 == nt) {  // S buffer pb read completely
                    tc_fence_before();
                    mbar_arrive(&s_free[pb]);
                }
                if (vec) {
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        const float4 l4 = __ldg(reinterpret_cast<const float4 *>(lse2 + c));
                        add_pair(t, c, ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v,
                                             make_float2(-l4.x, -l4.y)));
                        add_pair(t, c + 2, ffma2(make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])),
                                                 sl2v, make_float2(-l4.z, -l4.w)));
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float2 nl = make_float2(c < n_rows ? -__ldg(lse2 + c) : -INFINITY,
                                                      c + 1 < n_rows ? -__ldg(lse2 + c + 1) : -INFINITY);
                        add_pair(t, c, ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v, nl));
                    }
                }
            }
        }
        float *red = reinterpret_cast<float *>(smem + SM::kOffRed);  // [4 parts][256 keys]
#pragma unroll
        for (int t = 0; t < kScoreTiles; ++t)
            red[part * 256 + t * 128 + j] = ((acc[t][0].x + acc[t][0].y) + (acc[t][1].x + acc[t][1].y)) +
                                            ((acc[t][2].x + acc[t][2].y) + (acc[t][3].x + acc[t][3].y));
        // All score warps leave the loop together (the abort flag is CTA-wide and
        // every wait is bounded), so this barrier is always reached by all 512.
        bar_sync(1, kScoreThreads);
        if (part == 0 && ok) {
#pragma unroll
            for (int t = 0; t < kScoreTiles; ++t) {
                const int key = t * 128 + j;
                if (key < n_keys)
                    P.scores[static_cast<size_t>(g) * L.C + (key0 - L.a) + key] =
                        (red[key] + red[256 + key]) + (red[512 + key] + red[768 + key]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kScoreMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if constexpr (FUSED) {
        // The last CTA of (chunk u, KV head g) to finish selects and gathers.
        __shared__ int s_last;
        __threadfence();  // this CTA's scores, before its count
        __syncthreads();
        if (threadIdx.x == 0) {
            const int n_units = P.unit_begin[u + 1] - P.unit_begin[u];
            s_last = atomicAdd(&P.counters[u * L.Hkv + g], 1) == n_units - 1;
        }
        __syncthreads();
        if (s_last) {
            __threadfence();  // every other CTA's scores of (u, g), after their counts
            // The tiles' shared memory is free: the rank keys go there.
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            const int l_eff = select_chunk(L, P.scores, P.idx, u, g, reinterpret_cast<uint32_t *>(smem),
                                           SM::kOffBar / 4);
            __syncthreads();
            const int32_t *sel = P.idx + (static_cast<size_t>(u) * L.Hkv + g) * L.l;
            const int p0 = L.pcum[u], sh = region_shift(L, 1 + u);
            copy_rows<D>(L, P.K, P.V, P.PK, P.PV, g, p0, p0 + l_eff, warp, blockDim.x >> 5,
                         [&](int r) { return sel[r - p0] - sh; });
            if (threadIdx.x == 0) P.counters[u * L.Hkv + g] = 0;  // ready for the next launch
        }
    }
}

// Row-normalised scores: the base-2 log-sum-exp of every query row over all the
// segments it attends, seg[s][h][i] combined over s (anchor s = 0 only if
// a > 0, chunks s = 1..2H, query block s = 2H+1), written for every producing
// chunk u so that the scoring pass reads it like a per-chunk statistic.
__global__ void row_lse_kernel(const Layer L, const float *seg, float *stats) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;  // h * q + i
    const int rows = L.Hq * L.q;
    if (r >= rows) return;
    const int s0 = L.a > 0 ? 0 : 1, s1 = L.n_chunks + 1;
    float m = -INFINITY;
    for (int s = s0; s <= s1; ++s) m = fmaxf(m, seg[static_cast<size_t>(s) * rows + r]);
    float sum = 0.f;
    if (m != -INFINITY)
        for (int s = s0; s <= s1; ++s) sum += exp2f(seg[static_cast<size_t>(s) * rows + r] - m);
    const float lse = (m == -INFINITY) ? -INFINITY : m + log2f(sum);
    for (int u = 0; u < L.n_chunks - 1; ++u) stats[static_cast<size_t>(u) * rows + r] = lse;
}

}  // namespace spava

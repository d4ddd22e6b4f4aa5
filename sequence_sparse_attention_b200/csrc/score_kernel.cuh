// score_kernel.cuh -- query-to-context scores of the passing-block selection.
//
// "Riepilogo Tecnico: APB-V", Metodologia, "Blocchi di Passaggio": the most
// essential KV of each host are identified by query-to-context attention
// scores.  Score of key j of chunk u for KV head g:
//     S[g, j] = sum_{h in g} sum_{i in query block} exp2(x_{h,i,j} - lse2_{u,h,i}),
//     x = scale*log2(e) * q_{h,i} . k_{g,j},
// where lse2_{u,h,i} is the base-2 log-sum-exp of row (h, i) over chunk u (the
// statistics pass, stats_kernel.cuh).  Equivalently: softmax over the
// chunk, summed over query rows and group heads.
//
// One CTA = 128 keys of one chunk and one KV head.  The product is formed
// transposed, S^T = K Q^T (M = 128 keys, N = 128 query rows of one head per
// block, K = d), so that TMEM lane j holds key j and each thread sums its own
// key's probabilities without any cross-thread reduction; the summation order
// is fixed, so the result is deterministic.
#pragma once

#include "plan.cuh"
#include "sm100.cuh"

namespace spava {

struct ScoreParams {
    CUtensorMap tmQ, tmK;
    Layer L;
    const float *stats;  // [2H-1, Hq, q] log2 domain
    float *scores;       // [Hkv, C]
    int *status;
    int32_t tile_begin[kMaxChunks + 1];  // prefix of 128-key tiles over chunks u < 2H-1
};

constexpr int kScoreWarps = 16;                 // 4 per TMEM lane quarter
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kScoreProducer = kScoreWarps;
constexpr int kScoreMma = kScoreWarps + 1;
constexpr int kScoreBlockThreads = (kScoreWarps + 2) * 32;

template <int D>
struct ScoreSmem {
    static constexpr int kPanels = D / 64;
    static constexpr int kTile = 128 * D * 2;
    static constexpr int QS = 4;
    static constexpr int NB = 4;  // TMEM S buffers
    static constexpr int kOffK = 0;
    static constexpr int kOffQ = kTile;
    static constexpr int kOffBar = kOffQ + QS * kTile;
    static constexpr int kNumBar = 1 + 2 * QS + 2 * NB + 1;
    static constexpr int kOffRed = kOffBar + kNumBar * 8;   // [4 parts][128 keys] partial sums
    static constexpr int kOffMisc = kOffRed + 4 * 128 * 4;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

static_assert(ScoreSmem<128>::kAlloc <= 232448, "scoring smem over budget");

template <int D>
__global__ void __launch_bounds__(kScoreBlockThreads, 1) score_kernel(const __grid_constant__ ScoreParams P) {
    using SM = ScoreSmem<D>;
    constexpr int QS = SM::QS, NB = SM::NB;
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, 0, 0);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffBar);
    uint64_t *a_full = bars;
    uint64_t *q_full = a_full + 1;
    uint64_t *q_empty = q_full + QS;
    uint64_t *s_full = q_empty + QS;
    uint64_t *s_free = s_full + NB;
    uint64_t *mma_drain = s_free + NB;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::kOffMisc + 4);

    const Layer &L = P.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blockIdx.x = tile * Hkv + g, tiles enumerated over chunks u < 2H-1
    const int g = blockIdx.x % L.Hkv;
    const int tile = blockIdx.x / L.Hkv;
    int u = 0;
    while (u + 1 < L.n_chunks - 1 && tile >= P.tile_begin[u + 1]) ++u;
    const int kt = tile - P.tile_begin[u];
    const int key0 = L.off[u] + kt * 128;
    const int n_valid = min(128, L.off[u + 1] - key0);
    const int n_rb = cdiv(L.q, 128);
    const int NBLK = L.G * n_rb;  // column blocks: (head in group, 128 query rows)

    if (threadIdx.x == 0) {
        mbar_init(a_full, 1);
        for (int i = 0; i < QS; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < NB; ++i) {
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
            mbar_expect_tx(a_full, SM::kTile);
            for (int p = 0; p < SM::kPanels; ++p)
                tma_load_3d(smem + SM::kOffK + p * 16384, &P.tmK, p * 64, g, key0 - region_shift(L, 1 + u),
                            a_full);
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
            const uint32_t a_base = smem_u32(smem + SM::kOffK);
            const uint32_t q_base = smem_u32(smem + SM::kOffQ);
            bool ok = mbar_wait(a_full, 0, ab);
            tc_fence_after();
            for (int b = 0; ok && b < NBLK; ++b) {
                const int qs = b % QS, sb = b % NB;
                if (!mbar_wait(&q_full[qs], (b / QS) & 1, ab)) break;
                if (b >= NB && !mbar_wait(&s_free[sb], ((b / NB) - 1) & 1, ab)) break;
                tc_fence_after();
                const uint32_t qb = q_base + qs * SM::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tmem + sb * 128, sdesc_sw128(a_base + off, 16, 1024),
                           sdesc_sw128(qb + off, 16, 1024), kIdesc, kk > 0);
                }
                tc_commit(&q_empty[qs]);
                tc_commit(&s_full[sb]);
            }
            tc_commit(mma_drain);
            mbar_wait_drain(mma_drain, 0);
        }
        __syncwarp();
    } else {
        // Warp w: keys 32*(w%4) .. +31 (its TMEM lane quarter), query-row columns
        // 32*(w/4) .. +31 of every 128-column block; the four column parts of a
        // key are added at the end.
        const int quarter = warp & 3, part = warp >> 2;
        const int j = quarter * 32 + lane;  // key within the tile == TMEM lane
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const float2 sl2v = make_float2(L.scale_log2, L.scale_log2);
        float2 acc[4];  // 8 independent partial sums, in packed pairs
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
        bool ok = true;
        for (int b = 0; b < NBLK; ++b) {
            const int sb = b % NB;
            const int h = g * L.G + b / n_rb;
            const int i0 = (b % n_rb) * 128 + part * 32;
            const float *lse2 = P.stats + (static_cast<size_t>(u) * L.Hq + h) * L.q + i0;
            const int n_rows = min(32, L.q - i0);  // may be <= 0 for the ragged last block
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (b / NB) & 1, ab));
            if (!ok) break;
            tc_fence_after();
            uint32_t r[32];
            tmem_ld32(lane_addr + sb * 128 + part * 32, r);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&s_free[sb]);
            if (n_rows == 32) {
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 nl = make_float2(-__ldg(lse2 + c), -__ldg(lse2 + c + 1));
                    const float2 arg = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v, nl);
                    acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], make_float2(ex2(arg.x), ex2(arg.y)));
                }
            } else {
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 nl = make_float2(c < n_rows ? -__ldg(lse2 + c) : -INFINITY,
                                                  c + 1 < n_rows ? -__ldg(lse2 + c + 1) : -INFINITY);
                    const float2 arg = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v, nl);
                    acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], make_float2(ex2(arg.x), ex2(arg.y)));
                }
            }
        }
        float *red = reinterpret_cast<float *>(smem + SM::kOffRed);
        red[part * 128 + j] = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                              ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
        // All score warps leave the loop together (the abort flag is CTA-wide and
        // every wait is bounded), so this barrier is always reached by all 512.
        bar_sync(1, kScoreThreads);
        if (part == 0 && ok && j < n_valid)
            P.scores[static_cast<size_t>(g) * L.C + (key0 - L.a) + j] =
                (red[j] + red[128 + j]) + (red[256 + j] + red[384 + j]);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kScoreMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace spava

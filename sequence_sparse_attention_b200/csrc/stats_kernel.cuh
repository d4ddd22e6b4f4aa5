// stats_kernel.cuh -- per-chunk softmax statistics of the query block, the
// normaliser of the scoring pass, on tcgen05/TMEM.
//
// "Riepilogo Tecnico: APB-V", Metodologia, "Meccanismo di Attenzione
// Approssimata": each chunk's keys are scored by the query block's attention
// over that chunk alone, so every query row needs the log-sum-exp of its
// logits against each chunk u:  stats[u, h, i] = log2 sum_{j in B_u} 2^(x_ij),
// x = scale * log2(e) * q_i . k_j  (score_kernel.cuh divides by it).
//
// With row-normalised scores the same kernel runs over every segment a query
// row attends (anchor, chunks, the query block causally), writing one
// statistic per segment; row_lse_kernel combines them.
//
// One CTA = 128 query rows of one head against one segment.  Warp roles:
//   warps 0-7  two warps per TMEM lane quarter, each taking one half of the 128
//              keys of a tile; running max with conditional rescaling of the
//              running sum (the max only moves when it grows by more than 2^8)
//   warp  8    TMA producer: the Q tile once, then K tiles through a ring
//   warp  9    MMA issuer: S = Q K^T (SS, K-major/K-major) into one of two S
//              buffers in TMEM; S_{j+2} is issued once the softmax has loaded S_j
#pragma once

#include "attn_kernel.cuh"

namespace spava {

template <int D>
struct StatsSmem {
    static constexpr int kPanels = D / 64;
    static constexpr int kTile = kRowTile * D * 2;  // one 128-row bf16 tile
    static constexpr int KS = 4;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kTile;
    static constexpr int kOffBar = kOffK + KS * kTile;
    static constexpr int kNumBar = 1 + 2 * KS + 4 + 1;
    static constexpr int kOffRed = kOffBar + kNumBar * 8;  // row-max / row-sum exchange
    static constexpr int kOffMisc = kOffRed + 6 * kRowTile * 4;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(StatsSmem<128>::kAlloc <= kMaxDynSmem, "statistics smem over budget");

constexpr int kStatsSoftWarps = 8;
constexpr int kStatsSoftThreads = kStatsSoftWarps * 32;
constexpr int kStatsProducer = kStatsSoftWarps;
constexpr int kStatsMma = kStatsSoftWarps + 1;
constexpr int kStatsThreads = (kStatsSoftWarps + 2) * 32;
constexpr int kHalf = kKeyTile / 2;  // keys of a tile handled by one warp
constexpr uint32_t kStatsTmemCols = 256;

template <int D>
__global__ void __launch_bounds__(kStatsThreads, 1) stats_kernel(const __grid_constant__ AttnParams P) {
    using SM = StatsSmem<D>;
    constexpr int KS = SM::KS;
    constexpr uint32_t kIdescS = idesc_bf16_f32(128, kKeyTile, 0, 0);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffBar);
    uint64_t *q_full = bars;
    uint64_t *k_full = q_full + 1;
    uint64_t *k_empty = k_full + KS;
    uint64_t *s_full = k_empty + KS;
    uint64_t *s_free = s_full + 2;
    uint64_t *mma_drain = s_free + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layer &L = P.L;
    const Item it = decode_item(P.groups, P.n_groups, blockIdx.x, L.Hq, L.G);
    Seg segs[kMaxSegs];
    const int ns = build_segments(L, it, segs);
    const int T = count_tiles(segs, ns);
    int row0, row_end;
    item_rows(L, it, row0, row_end);
    const int g = it.h / L.G;
    const int rs = region_shift(L, item_region(L, it));  // global minus local row of the Q rows

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < KS; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kStatsSoftThreads);
        }
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kStatsProducer && lane == 0) {
        tma_prefetch(&P.tmQ);
        tma_prefetch(&P.tmK);
    }
    if (warp == kStatsMma) tmem_alloc(tmem_slot, kStatsTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState ab{abort_flag, P.status};

    if (warp == kStatsProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(q_full, SM::kTile);
            for (int p = 0; p < SM::kPanels; ++p)
                tma_load_3d(smem + SM::kOffQ + p * 16384, &P.tmQ, p * 64, it.h, row0 - rs, q_full);
            int k_last[KS];
            for (int i = 0; i < KS; ++i) k_last[i] = -1;
            TileCursor kc;
            for (int j = 0; j < T; ++j) {
                const int ks = j % KS;
                if (j >= KS && !mbar_wait(&k_empty[ks], ((j / KS) - 1) & 1, ab)) break;
                mbar_expect_tx(&k_full[ks], SM::kTile);
                uint8_t *kd = smem + SM::kOffK + ks * SM::kTile;
                const Seg &s = segs[kc.seg];
                const int key0 = s.begin + kc.tile * kKeyTile;
                for (int p = 0; p < SM::kPanels; ++p)
                    tma_load_3d(kd + p * 16384, &P.tmK, p * 64, g, key0 - s.shift, &k_full[ks]);
                k_last[ks] = j;
                kc.advance(segs);
            }
            // Every load this thread issued has landed before the CTA may exit.
            mbar_wait_drain(q_full, 0);
            for (int i = 0; i < KS; ++i)
                if (k_last[i] >= 0) mbar_wait_drain(&k_full[i], (k_last[i] / KS) & 1);
        }
    } else if (warp == kStatsMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr int NK = D / 16;  // K-steps of S = Q K^T
            uint64_t qd[NK];
            const uint64_t q_desc = sdesc_sw128(smem_u32(smem + SM::kOffQ), 16, 1024);
            const uint64_t k_desc = sdesc_sw128(smem_u32(smem + SM::kOffK), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < NK; ++kk) qd[kk] = q_desc + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            bool ok = mbar_wait(q_full, 0, ab);
            tc_fence_after();
            auto issue_s = [&](int j) -> bool {
                const int ks = j % KS;
                if (!mbar_wait(&k_full[ks], (j / KS) & 1, ab)) return false;
                tc_fence_after();
                const uint32_t d_s = tmem + (j & 1) * kKeyTile;
                const uint64_t kd = k_desc + static_cast<uint64_t>((ks * SM::kTile) >> 4);
#pragma unroll
                for (int g4 = 0; g4 < NK / 4; ++g4) {
                    const uint64_t kb = kd + static_cast<uint64_t>(g4 * (16384 >> 4));
                    mma_ss_x4(d_s, qd[4 * g4], qd[4 * g4 + 1], qd[4 * g4 + 2], qd[4 * g4 + 3], kb,
                              kb + 2, kb + 4, kb + 6, kIdescS, g4 > 0);
                }
                tc_commit(&k_empty[ks]);
                tc_commit(&s_full[j & 1]);
                return true;
            };
            if (ok && T > 0) ok = issue_s(0);
            if (ok && T > 1) ok = issue_s(1);
            for (int j = 0; ok && j + 2 < T; ++j) {
                // S buffer (j&1) is reused by S_{j+2} once the softmax has loaded S_j.
                if (!mbar_wait(&s_free[j & 1], (j >> 1) & 1, ab)) break;
                tc_fence_after();
                ok = issue_s(j + 2);
            }
            // No MMA may still be running when TMEM is released.
            tc_commit(mma_drain);
            mbar_wait_drain(mma_drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        // Warp w owns rows 32*(w%4) .. +31 (its TMEM lane quarter) and the key
        // half kh = w/4 of every tile (keys 64*kh .. +63).  The two warps of a
        // quarter exchange their partial row maxima through shared memory; every
        // abort decision is taken jointly with bar.red.and so that both always
        // reach the same named barriers.
        const int quarter = warp & 3, kh = warp >> 2;
        const int r = quarter * 32 + lane;  // row within the tile == TMEM lane
        const int t = row0 + r;
        const int pair_bar = 1 + quarter;   // named barrier of the two warps of a quarter
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        float *red = reinterpret_cast<float *>(smem + SM::kOffRed);  // [2][2][128]
        const float sl2 = L.scale_log2;
        const float2 sl2v = make_float2(sl2, sl2);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        TileCursor cur;
        for (int j = 0; j < T; ++j) {
            const Seg &s = segs[cur.seg];
            int lim_end = s.end;
            if (s.causal && t + 1 < lim_end) lim_end = t + 1;  // the query block up to the row
            const int lim = lim_end - (s.begin + cur.tile * kKeyTile + kh * kHalf);  // valid keys
            cur.advance(segs);

            const bool got = __all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1, ab));
            tc_fence_after();
            float x[kHalf];
            {
                uint32_t u[2][32];
#pragma unroll
                for (int c = 0; c < 2; ++c) tmem_ld32(lane_addr + (j & 1) * kKeyTile + kh * kHalf + c * 32, u[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    reg_fence(u[c]);
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(u[c][e]);
                }
            }
            tc_fence_before();
            mbar_arrive(&s_free[j & 1]);
            if (lim < kHalf) {
#pragma unroll
                for (int c = 0; c < kHalf; ++c)
                    if (c >= lim) x[c] = -INFINITY;
            }
            // Partial row max (3-input max, 4 chains), then the pair's exchange.
            const float mx_mine = max64(x);
            red[((j & 1) * 2 + kh) * kRowTile + r] = mx_mine;
            ok = bar_red_and(pair_bar, 64, got);
            if (!ok) break;
            const float mx = fmaxf(mx_mine, red[((j & 1) * 2 + (kh ^ 1)) * kRowTile + r]) * sl2;
            const float m_new = fmaxf(m_run, mx);
            if (m_new > m_run + 8.0f) {
                l_run *= ex2(m_run - m_new);
                m_run = m_new;
            }
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            const float2 nmu = make_float2(-mu, -mu);
            float2 ps[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) ps[k] = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float2 arg = ffma2(make_float2(x[2 * e], x[2 * e + 1]), sl2v, nmu);
                ps[e & 3] = fadd2(ps[e & 3], make_float2(ex2(arg.x), ex2(arg.y)));
            }
            const float2 pss = fadd2(fadd2(ps[0], ps[1]), fadd2(ps[2], ps[3]));
            l_run += pss.x + pss.y;
        }

        // ------------------------------------------------------------ epilogue
        // Row sum = the two halves' partial sums (same running max in both).
        float *lred = red + 4 * kRowTile;  // [2][128]
        lred[kh * kRowTile + r] = l_run;
        bar_sync(pair_bar, 64);
        const float l_tot = l_run + lred[(kh ^ 1) * kRowTile + r];
        if (ok && t < row_end && kh == 0) {
            const int i = t - (L.N - L.q);
            P.stats[(static_cast<size_t>(it.sub) * L.Hq + it.h) * L.q + i] =
                (l_tot > 0.f) ? m_run + __log2f(l_tot) : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kStatsMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kStatsTmemCols);
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

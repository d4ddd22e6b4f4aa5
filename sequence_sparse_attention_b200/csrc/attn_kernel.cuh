// attn_kernel.cuh -- approximate attention with online softmax on tcgen05/TMEM.
//
// "Riepilogo Tecnico: APB-V", Metodologia, "Meccanismo di Attenzione
// Approssimata" / "Computazione": every row attends its key segments (anchor,
// passing blocks, partner chunk, own chunk; plan.cuh); "Forward Fuso di
// Contesto e Query": query rows are computed as per-segment partials carrying
// their log-sum-exp, merged later.  The same kernel in STATS mode computes the
// per-chunk softmax statistics of the query block that the scoring pass needs.
//
// One CTA = one work item = 128 query rows of one head.  Warp roles:
//   warps 0-7  softmax: two warps per TMEM lane quarter, each taking one half
//              of the 128 keys of a tile; online softmax with conditional
//              rescaling (the running max only moves when it grows by more than
//              2^8), P written back into TMEM as bf16
//   warp  8    TMA producer: Q tile once, then K (and V) tiles through rings
//   warp  9    MMA issuer: S = Q K^T (SS, K-major/K-major) into one of two S
//              buffers in TMEM; O += P V (P from TMEM, V MN-major in smem)
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D), P0 [384,448),
// P1 [448,512) (bf16 pairs).  P has its own columns, so S_{j+2} is issued right
// behind PV_j without waiting for PV_j to finish; the softmax writes P_{j+2} over
// P_j only after S_{j+2} has completed, and that completion (tcgen05.commit
// tracks every earlier MMA of the issuing thread) implies PV_j has completed.
// MMAs with different accumulators are not ordered by the hardware, so every
// hand-off goes through an mbarrier.
#pragma once

#include "plan.cuh"
#include "sm100.cuh"

namespace spava {

struct AttnParams {
    CUtensorMap tmQ, tmK, tmV, tmPK, tmPV;
    Layer L;
    Group groups[4 * (kMaxChunks / 2) + 8];
    int32_t n_groups;
    __nv_bfloat16 *O;   // [N, Hq, D]
    float *lse;         // [Hq, N] natural log, or null
    float *part_O;      // [2H+2, Hq, q, D] normalised partials of the query rows
    float *part_lse;    // [2H+2, Hq, q] log2 domain
    float *stats;       // [2H-1, Hq, q] log2-domain lse of the query rows per chunk
    int *status;        // workspace status word
};

template <int D, bool STATS>
struct AttnSmem {
    static constexpr int kPanels = D / 64;
    static constexpr int kTile = kRowTile * D * 2;  // one 128-row bf16 tile
    static constexpr int KS = STATS ? 4 : 3;
    static constexpr int VS = STATS ? 1 : (D == 128 ? 2 : 3);  // STATS mode leaves V unused
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kTile;
    static constexpr int kOffV = kOffK + KS * kTile;
    static constexpr int kOffBar = kOffV + (STATS ? 0 : VS) * kTile;
    static constexpr int kNumBar = 1 + 2 * KS + 2 * VS + 8 + 1;
    static constexpr int kOffRed = kOffBar + kNumBar * 8;        // row-max / row-sum exchange
    static constexpr int kOffMisc = kOffRed + 6 * kRowTile * 4;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

// sm_100 allows at most 227 KiB of dynamic shared memory per CTA.
constexpr int kMaxDynSmem = 232448;
static_assert(AttnSmem<128, false>::kAlloc <= kMaxDynSmem, "attention smem over budget");
static_assert(AttnSmem<128, true>::kAlloc <= kMaxDynSmem, "statistics smem over budget");
static_assert(AttnSmem<64, false>::kAlloc <= kMaxDynSmem, "attention smem over budget");

constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kAttnThreads = (kSoftmaxWarps + 2) * 32;
constexpr int kHalf = kKeyTile / 2;  // keys of a tile handled by one softmax warp
constexpr uint32_t kTmemCols = 512;
constexpr int kColO = 256;
constexpr int kColP = 384;

template <int D, bool STATS>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_kernel(const __grid_constant__ AttnParams P) {
    using SM = AttnSmem<D, STATS>;
    constexpr int KS = SM::KS, VS = SM::VS;
    constexpr uint32_t kIdescS = idesc_bf16_f32(128, kKeyTile, 0, 0);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffBar);
    uint64_t *q_full = bars;
    uint64_t *k_full = q_full + 1;
    uint64_t *k_empty = k_full + KS;
    uint64_t *v_full = k_empty + KS;
    uint64_t *v_empty = v_full + VS;
    uint64_t *s_full = v_empty + VS;
    uint64_t *s_free = s_full + 2;
    uint64_t *p_full = s_free + 2;
    uint64_t *pv_done = p_full + 2;
    uint64_t *mma_drain = pv_done + 2;
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

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < KS; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < VS; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kSoftmaxThreads);
            mbar_init(&p_full[i], kSoftmaxThreads);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch(&P.tmQ);
        tma_prefetch(&P.tmK);
        if (!STATS) {
            tma_prefetch(&P.tmV);
            tma_prefetch(&P.tmPK);
            tma_prefetch(&P.tmPV);
        }
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState ab{abort_flag, P.status};

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(q_full, SM::kTile);
            for (int p = 0; p < SM::kPanels; ++p)
                tma_load_3d(smem + SM::kOffQ + p * 16384, &P.tmQ, p * 64, it.h, row0, q_full);
            int k_last[KS], v_last[VS];
            for (int i = 0; i < KS; ++i) k_last[i] = -1;
            for (int i = 0; i < VS; ++i) v_last[i] = -1;
            // K runs one tile ahead of V: S_{j+1} needs K_{j+1} before PV_j needs V_j.
            TileCursor kc, vc;
            bool live = true;
            auto load_k = [&](int j) -> bool {
                const int ks = j % KS;
                if (j >= KS && !mbar_wait(&k_empty[ks], ((j / KS) - 1) & 1, ab)) return false;
                mbar_expect_tx(&k_full[ks], SM::kTile);
                uint8_t *kd = smem + SM::kOffK + ks * SM::kTile;
                const Seg &s = segs[kc.seg];
                const int key0 = s.begin + kc.tile * kKeyTile;
                for (int p = 0; p < SM::kPanels; ++p) {
                    if (s.src == 0)
                        tma_load_3d(kd + p * 16384, &P.tmK, p * 64, g, key0, &k_full[ks]);
                    else
                        tma_load_3d(kd + p * 16384, &P.tmPK, p * 64, key0, g, &k_full[ks]);
                }
                k_last[ks] = j;
                kc.advance(segs);
                return true;
            };
            auto load_v = [&](int j) -> bool {
                const int vs = j % VS;
                if (j >= VS && !mbar_wait(&v_empty[vs], ((j / VS) - 1) & 1, ab)) return false;
                mbar_expect_tx(&v_full[vs], SM::kTile);
                uint8_t *vd = smem + SM::kOffV + vs * SM::kTile;
                const Seg &s = segs[vc.seg];
                const int key0 = s.begin + vc.tile * kKeyTile;
                for (int p = 0; p < SM::kPanels; ++p) {
                    if (s.src == 0)
                        tma_load_3d(vd + p * 16384, &P.tmV, p * 64, g, key0, &v_full[vs]);
                    else
                        tma_load_3d(vd + p * 16384, &P.tmPV, p * 64, key0, g, &v_full[vs]);
                }
                v_last[vs] = j;
                vc.advance(segs);
                return true;
            };
            if (T > 0) live = load_k(0);
            for (int j = 0; live && j < T; ++j) {
                if (j + 1 < T) live = load_k(j + 1);
                if (live && !STATS) live = load_v(j);
            }
            // Every load this thread issued has landed before the CTA may exit.
            mbar_wait_drain(q_full, 0);
            for (int i = 0; i < KS; ++i)
                if (k_last[i] >= 0) mbar_wait_drain(&k_full[i], (k_last[i] / KS) & 1);
            for (int i = 0; i < VS; ++i)
                if (v_last[i] >= 0) mbar_wait_drain(&v_full[i], (v_last[i] / VS) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // Descriptors are built once; a K-step or a ring stage only adds its
            // byte offset / 16 to the start-address field (addresses < 256 KiB, so
            // the 14-bit field never carries into the next one).  This keeps the
            // issuing thread down to a couple of instructions per MMA.
            constexpr int NK = D / 16;  // K-steps of S = Q K^T
            uint64_t qd[NK];            // A descriptors of the Q tile, one per K-step
            const uint64_t q_desc = sdesc_sw128(smem_u32(smem + SM::kOffQ), 16, 1024);
            const uint64_t k_desc = sdesc_sw128(smem_u32(smem + SM::kOffK), 16, 1024);
            const uint64_t v_desc = sdesc_sw128(smem_u32(smem + SM::kOffV), 16384, 1024);
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
            if (ok) ok = issue_s(0);
            if (ok && T > 1) ok = issue_s(1);
            for (int j = 0; ok && j < T; ++j) {
                if (!STATS) {
                    if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, ab)) break;
                    tc_fence_after();
                    const int vs = j % VS;
                    if (!mbar_wait(&v_full[vs], (j / VS) & 1, ab)) break;
                    tc_fence_after();
                    const uint32_t a_p = tmem + kColP + (j & 1) * (kKeyTile / 2);
                    const uint64_t vd = v_desc + static_cast<uint64_t>((vs * SM::kTile) >> 4);
                    // K-step kb covers keys 16kb..16kb+15: P columns +8kb, V rows +2048 B.
                    mma_ts_x4(tmem + kColO, a_p, a_p + 8, a_p + 16, a_p + 24, vd, vd + 128, vd + 256,
                              vd + 384, kIdescPV, j > 0);
                    mma_ts_x4(tmem + kColO, a_p + 32, a_p + 40, a_p + 48, a_p + 56, vd + 512, vd + 640,
                              vd + 768, vd + 896, kIdescPV, 1u);
                    tc_commit(&v_empty[vs]);
                    tc_commit(&pv_done[j & 1]);
                }
                if (j + 2 < T) {
                    // S buffer (j&1) is reused by S_{j+2}: the softmax has loaded S_j
                    // (s_free_j; in attention mode also implied by p_full_j above).
                    if (!mbar_wait(&s_free[j & 1], (j >> 1) & 1, ab)) break;
                    tc_fence_after();
                    if (!issue_s(j + 2)) break;
                }
            }
            // No MMA may still be running when TMEM is released.
            tc_commit(mma_drain);
            mbar_wait_drain(mma_drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        // Warps 0-7: warp w owns rows 32*(w%4) .. +31 (its TMEM lane quarter) and
        // the key half kh = w/4 of every tile (keys 64*kh .. +63).  The two warps
        // of a quarter exchange their partial row maxima through shared memory;
        // every abort decision is taken jointly with bar.red.and so that both
        // always reach the same named barriers.
        const int quarter = warp & 3, kh = warp >> 2;
        const int r = quarter * 32 + lane;  // row within the tile == TMEM lane
        const int t = row0 + r;
        const int pair_bar = 1 + quarter;   // named barrier of the two warps of a quarter
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        float *red = reinterpret_cast<float *>(smem + SM::kOffRed);  // [2][2][128]
        const float sl2 = L.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        int sg = 0, kt = 0;
        for (int j = 0; j < T; ++j) {
            const Seg &s = segs[sg];
            const int key0 = s.begin + kt * kKeyTile + kh * kHalf;
            int lim_end = s.end;
            if (s.causal && t + 1 < lim_end) lim_end = t + 1;
            const int lim = lim_end - key0;  // keys [0, lim) of this half-tile are valid for row r

            const bool got = __all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1, ab));
            tc_fence_after();
            float x[kHalf];
            {
                uint32_t u[kHalf];
#pragma unroll
                for (int c = 0; c < kHalf / 32; ++c)
                    tmem_ld32(lane_addr + (j & 1) * kKeyTile + kh * kHalf + c * 32,
                              *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < kHalf; ++e) x[e] = __uint_as_float(u[e]);
            }
            tc_fence_before();
            mbar_arrive(&s_free[j & 1]);
            // P_j overwrites the columns of P_{j-2}; S_j was issued after PV_{j-2},
            // so S_j's completion (seen above) implies PV_{j-2} has completed.
            const bool landed = true;
            if (lim < kHalf) {
#pragma unroll
                for (int c = 0; c < kHalf; ++c)
                    if (c >= lim) x[c] = -INFINITY;
            }
            // Partial row max (3-input max, 4 chains), then the pair's exchange.
            static_assert(kHalf == 64, "max64 covers one half tile");
            const float mx_mine = max64(x);
            red[((j & 1) * 2 + kh) * kRowTile + r] = mx_mine;
            ok = bar_red_and(pair_bar, 64, got && landed);
            if (!ok) break;
            const float mx = fmaxf(mx_mine, red[((j & 1) * 2 + (kh ^ 1)) * kRowTile + r]) * sl2;
            const float m_new = fmaxf(m_run, mx);
            const bool need = m_new > m_run + 8.0f;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(m_run - m_new);
                l_run *= alpha;
                m_run = m_new;
            }
            if (!STATS && j > 0 && __any_sync(0xffffffffu, need)) {
                // O holds the sum up to tile j-1 scaled by the old max: rescale this
                // warp's half of the O columns once PV_{j-1} has landed.  Both warps
                // of the quarter see the same rows' `need`, so both come here.
                const bool landed = __all_sync(
                    0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ab));
                ok = bar_red_and(pair_bar, 64, landed);
                if (!ok) break;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t u[32];
                    const uint32_t a = lane_addr + kColO + kh * (D / 2) + c * 32;
                    tmem_ld32(a, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
                    tmem_st32(a, u);
                }
                tmem_wait_st();
            }
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            // Probabilities: exponent arguments and partial sums in packed pairs.
            const float2 sl2v = make_float2(sl2, sl2), nmu = make_float2(-mu, -mu);
            float2 ps[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) ps[k] = make_float2(0.f, 0.f);
            uint32_t u[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float2 arg = ffma2(make_float2(x[2 * e], x[2 * e + 1]), sl2v, nmu);
                const float2 p = make_float2(ex2(arg.x), ex2(arg.y));
                ps[e & 3] = fadd2(ps[e & 3], p);
                if (!STATS) u[e] = pack_bf16x2(p.x, p.y);
            }
            if (STATS) {
                (void)u;
            } else {
                tmem_st32(lane_addr + kColP + (j & 1) * (kKeyTile / 2) + kh * 32, u);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[j & 1]);
            }
            const float2 pss = fadd2(fadd2(ps[0], ps[1]), fadd2(ps[2], ps[3]));
            l_run += pss.x + pss.y;
            if (s.begin + (kt + 1) * kKeyTile >= s.end) {
                ++sg;
                kt = 0;
            } else {
                ++kt;
            }
        }

        // ------------------------------------------------------------ epilogue
        // Row sum = the two halves' partial sums (same running max in both).
        float *lred = red + 4 * kRowTile;  // [2][128]
        lred[kh * kRowTile + r] = l_run;
        bar_sync(pair_bar, 64);
        const float l_tot = l_run + lred[(kh ^ 1) * kRowTile + r];
        const bool valid = ok && t < row_end;
        const float lse2 = (l_tot > 0.f) ? m_run + __log2f(l_tot) : -INFINITY;
        if (STATS) {
            if (valid && kh == 0) {
                const int i = t - (L.N - L.q);
                P.stats[(static_cast<size_t>(it.sub) * L.Hq + it.h) * L.q + i] = lse2;
            }
        } else if (ok && T > 0) {
            const bool landed = __all_sync(
                0xffffffffu, mbar_wait(&pv_done[(T - 1) & 1], ((T - 1) >> 1) & 1, ab));
            if (bar_red_and(pair_bar, 64, landed)) {
                tc_fence_after();
                const float inv = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
                const int c0 = kh * (D / 2);  // this warp's half of the O columns
                if (it.kind == kQueryPart) {
                    const int i = t - (L.N - L.q);
                    float *dst = P.part_O + ((static_cast<size_t>(it.sub) * L.Hq + it.h) * L.q + i) * D + c0;
#pragma unroll
                    for (int c = 0; c < D / 64; ++c) {
                        uint32_t u[32];
                        tmem_ld32(lane_addr + kColO + c0 + c * 32, u);
                        tmem_wait_ld();
                        if (valid) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4) {
                                float4 f = make_float4(__uint_as_float(u[e]) * inv,
                                                       __uint_as_float(u[e + 1]) * inv,
                                                       __uint_as_float(u[e + 2]) * inv,
                                                       __uint_as_float(u[e + 3]) * inv);
                                *reinterpret_cast<float4 *>(dst + c * 32 + e) = f;
                            }
                        }
                    }
                    if (valid && kh == 0)
                        P.part_lse[(static_cast<size_t>(it.sub) * L.Hq + it.h) * L.q + i] = lse2;
                } else {
                    __nv_bfloat16 *dst = P.O + (static_cast<size_t>(t) * L.Hq + it.h) * D + c0;
#pragma unroll
                    for (int c = 0; c < D / 64; ++c) {
                        uint32_t u[32];
                        tmem_ld32(lane_addr + kColO + c0 + c * 32, u);
                        tmem_wait_ld();
                        if (valid) {
#pragma unroll
                            for (int e = 0; e < 32; e += 8) {
                                uint4 w;
                                w.x = pack_bf16x2(__uint_as_float(u[e]) * inv, __uint_as_float(u[e + 1]) * inv);
                                w.y = pack_bf16x2(__uint_as_float(u[e + 2]) * inv, __uint_as_float(u[e + 3]) * inv);
                                w.z = pack_bf16x2(__uint_as_float(u[e + 4]) * inv, __uint_as_float(u[e + 5]) * inv);
                                w.w = pack_bf16x2(__uint_as_float(u[e + 6]) * inv, __uint_as_float(u[e + 7]) * inv);
                                *reinterpret_cast<uint4 *>(dst + c * 32 + e) = w;
                            }
                        }
                    }
                    if (valid && kh == 0 && P.lse)
                        P.lse[static_cast<size_t>(it.h) * L.N + t] = lse2 * 0.69314718055994531f;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace spava

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
//   warps 0-3  softmax: thread r owns row r (TMEM lane r); online softmax with
//              conditional rescaling (the running max is only moved when it
//              grows by more than 2^8), P written back into TMEM as bf16
//   warp  4    TMA producer: Q tile once, then K (and V) tiles through rings
//   warp  5    MMA issuer: S = Q K^T (SS, K-major/K-major) into one of two S
//              buffers in TMEM; O += P V (P from TMEM, V MN-major in smem)
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D).
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
    static constexpr int VS = STATS ? 1 : 3;        // STATS mode leaves V unused
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kTile;
    static constexpr int kOffV = kOffK + KS * kTile;
    static constexpr int kOffBar = kOffV + (STATS ? 0 : VS) * kTile;
    static constexpr int kNumBar = 1 + 2 * KS + 2 * VS + 8 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBar * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

constexpr int kAttnThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kColO = 256;

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
    const Item it = decode_item(P.groups, P.n_groups, blockIdx.x, L.Hq);
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
            mbar_init(&s_free[i], kRowTile);
            mbar_init(&p_full[i], kRowTile);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        tma_prefetch(&P.tmQ);
        tma_prefetch(&P.tmK);
        if (!STATS) {
            tma_prefetch(&P.tmV);
            tma_prefetch(&P.tmPK);
            tma_prefetch(&P.tmPV);
        }
    }
    if (warp == 5) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState ab{abort_flag, P.status};

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint32_t q_base = smem_u32(smem + SM::kOffQ);
            mbar_expect_tx(q_full, SM::kTile);
            for (int p = 0; p < SM::kPanels; ++p)
                tma_load_3d(smem + SM::kOffQ + p * 16384, &P.tmQ, p * 64, it.h, row0, q_full);
            (void)q_base;
            int k_last[KS], v_last[VS];
            for (int i = 0; i < KS; ++i) k_last[i] = -1;
            for (int i = 0; i < VS; ++i) v_last[i] = -1;
            int sg = 0, kt = 0;
            for (int j = 0; j < T; ++j) {
                const Seg &s = segs[sg];
                const int key0 = s.begin + kt * kKeyTile;
                const int ks = j % KS;
                if (j >= KS && !mbar_wait(&k_empty[ks], ((j / KS) - 1) & 1, ab)) break;
                mbar_expect_tx(&k_full[ks], SM::kTile);
                uint8_t *kd = smem + SM::kOffK + ks * SM::kTile;
                for (int p = 0; p < SM::kPanels; ++p) {
                    if (s.src == 0)
                        tma_load_3d(kd + p * 16384, &P.tmK, p * 64, g, key0, &k_full[ks]);
                    else
                        tma_load_3d(kd + p * 16384, &P.tmPK, p * 64, key0, g, &k_full[ks]);
                }
                k_last[ks] = j;
                if (!STATS) {
                    const int vs = j % VS;
                    if (j >= VS && !mbar_wait(&v_empty[vs], ((j / VS) - 1) & 1, ab)) break;
                    mbar_expect_tx(&v_full[vs], SM::kTile);
                    uint8_t *vd = smem + SM::kOffV + vs * SM::kTile;
                    for (int p = 0; p < SM::kPanels; ++p) {
                        if (s.src == 0)
                            tma_load_3d(vd + p * 16384, &P.tmV, p * 64, g, key0, &v_full[vs]);
                        else
                            tma_load_3d(vd + p * 16384, &P.tmPV, p * 64, key0, g, &v_full[vs]);
                    }
                    v_last[vs] = j;
                }
                if (s.begin + (kt + 1) * kKeyTile >= s.end) {
                    ++sg;
                    kt = 0;
                } else {
                    ++kt;
                }
            }
            // Every load this thread issued has landed before the CTA may exit.
            mbar_wait_drain(q_full, 0);
            for (int i = 0; i < KS; ++i)
                if (k_last[i] >= 0) mbar_wait_drain(&k_full[i], (k_last[i] / KS) & 1);
            for (int i = 0; i < VS; ++i)
                if (v_last[i] >= 0) mbar_wait_drain(&v_full[i], (v_last[i] / VS) & 1);
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t q_base = smem_u32(smem + SM::kOffQ);
            const uint32_t k_base = smem_u32(smem + SM::kOffK);
            const uint32_t v_base = smem_u32(smem + SM::kOffV);
            bool ok = mbar_wait(q_full, 0, ab);
            tc_fence_after();
            auto issue_s = [&](int j) -> bool {
                const int ks = j % KS;
                if (!mbar_wait(&k_full[ks], (j / KS) & 1, ab)) return false;
                tc_fence_after();
                const uint32_t d_s = tmem + (j & 1) * kKeyTile;
                const uint32_t kb = k_base + ks * SM::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(d_s, sdesc_sw128(q_base + off, 16, 1024),
                           sdesc_sw128(kb + off, 16, 1024), kIdescS, kk > 0);
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
                    const uint32_t a_p = tmem + (j & 1) * kKeyTile;
                    const uint32_t vb = v_base + vs * SM::kTile;
#pragma unroll
                    for (int kb = 0; kb < kKeyTile / 16; ++kb)
                        mma_ts(tmem + kColO, a_p + kb * 8, sdesc_sw128(vb + kb * 2048, 16384, 1024),
                               kIdescPV, (j > 0 || kb > 0) ? 1u : 0u);
                    tc_commit(&v_empty[vs]);
                    tc_commit(&pv_done[j & 1]);
                }
                if (j + 2 < T) {
                    // S buffer (j&1) is reused by S_{j+2}: its contents (S_j, then
                    // P_j) must have been consumed.
                    if (!STATS) {
                        if (!mbar_wait(&pv_done[j & 1], (j >> 1) & 1, ab)) break;
                    } else {
                        if (!mbar_wait(&s_free[j & 1], (j >> 1) & 1, ab)) break;
                    }
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
        const int r = threadIdx.x;  // row within the tile == TMEM lane
        const int t = row0 + r;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sl2 = L.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        int sg = 0, kt = 0;
        for (int j = 0; j < T; ++j) {
            const Seg &s = segs[sg];
            const int key0 = s.begin + kt * kKeyTile;
            int lim_end = s.end;
            if (s.causal && t + 1 < lim_end) lim_end = t + 1;
            const int lim = lim_end - key0;  // keys [0, lim) of this tile are valid for row r

            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1, ab));
            if (!ok) break;
            tc_fence_after();
            float x[kKeyTile];
            {
                uint32_t u[32];
#pragma unroll
                for (int c = 0; c < kKeyTile / 32; ++c) {
                    tmem_ld32(lane_addr + (j & 1) * kKeyTile + c * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(u[e]);
                }
            }
            if (STATS) {
                tc_fence_before();
                mbar_arrive(&s_free[j & 1]);
            }
            if (lim < kKeyTile) {
#pragma unroll
                for (int c = 0; c < kKeyTile; ++c)
                    if (c >= lim) x[c] = -INFINITY;
            }
            float mx = x[0];
#pragma unroll
            for (int c = 1; c < kKeyTile; ++c) mx = fmaxf(mx, x[c]);
            mx *= sl2;
            const float m_new = fmaxf(m_run, mx);
            const bool need = m_new > m_run + 8.0f;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(m_run - m_new);
                l_run *= alpha;
                m_run = m_new;
            }
            if (!STATS && j > 0 && __any_sync(0xffffffffu, need)) {
                // O holds the sum up to tile j-1 scaled by the old max: rescale it
                // once PV_{j-1} has landed.
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ab));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(lane_addr + kColO + c * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
                    tmem_st32(lane_addr + kColO + c * 32, u);
                }
                tmem_wait_st();
            }
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            float sum = 0.f;
            if (STATS) {
#pragma unroll
                for (int c = 0; c < kKeyTile; ++c) sum += ex2(fmaf(x[c], sl2, -mu));
            } else {
#pragma unroll
                for (int c = 0; c < kKeyTile / 64; ++c) {
                    uint32_t u[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float p0 = ex2(fmaf(x[c * 64 + 2 * e], sl2, -mu));
                        const float p1 = ex2(fmaf(x[c * 64 + 2 * e + 1], sl2, -mu));
                        sum += p0 + p1;
                        u[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(lane_addr + (j & 1) * kKeyTile + c * 32, u);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[j & 1]);
            }
            l_run += sum;
            if (s.begin + (kt + 1) * kKeyTile >= s.end) {
                ++sg;
                kt = 0;
            } else {
                ++kt;
            }
        }

        // ------------------------------------------------------------ epilogue
        const bool valid = ok && t < row_end;
        const float lse2 = (l_run > 0.f) ? m_run + __log2f(l_run) : -INFINITY;
        if (STATS) {
            if (valid) {
                const int i = t - (L.N - L.q);
                P.stats[(static_cast<size_t>(it.sub) * L.Hq + it.h) * L.q + i] = lse2;
            }
        } else if (ok && T > 0) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&pv_done[(T - 1) & 1], ((T - 1) >> 1) & 1, ab));
            if (ok) {
                tc_fence_after();
                const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
                if (it.kind == kQueryPart) {
                    const int i = t - (L.N - L.q);
                    float *dst = P.part_O + ((static_cast<size_t>(it.sub) * L.Hq + it.h) * L.q + i) * D;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t u[32];
                        tmem_ld32(lane_addr + kColO + c * 32, u);
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
                    if (valid) P.part_lse[(static_cast<size_t>(it.sub) * L.Hq + it.h) * L.q + i] = lse2;
                } else {
                    __nv_bfloat16 *dst = P.O + (static_cast<size_t>(t) * L.Hq + it.h) * D;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t u[32];
                        tmem_ld32(lane_addr + kColO + c * 32, u);
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
                    if (valid && P.lse) P.lse[static_cast<size_t>(it.h) * L.N + t] = lse2 * 0.69314718055994531f;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace spava

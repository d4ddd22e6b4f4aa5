// attn_kernel.cuh -- approximate attention, two query tiles per CTA, the
// tensor core working on one tile while the other tile's softmax runs.
//
// "Riepilogo Tecnico: APB-V", Metodologia, "Meccanismo di Attenzione
// Approssimata" / "Computazione": every row attends its key segments (anchor,
// passing blocks, partner chunk, own chunk; plan.cuh); "Forward Fuso di
// Contesto e Query": query rows are computed as per-segment partials carrying
// their log-sum-exp, merged later.
//
// One CTA = two adjacent 128-row tiles A (x = 0) and B (x = 1) of one head; B
// may be absent at the end of a region.  Both see the same key sequence, except
// that B sees one more tile (its own diagonal) when the sequence ends in a
// causal segment.  Warp roles:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: warp w owns the
//              TMEM lane quarter w % 4, i.e. 32 rows, and all 128 keys of every
//              key tile -- no exchange between warps.  Online softmax with
//              conditional rescaling (the running max only moves when it grows
//              by more than 2^8), P written back into TMEM as bf16.
//   warp  8    TMA producer: Q_A, Q_B once, then K (one tile ahead) and V rings
//   warp  9    MMA issuer (warps 10-11 only complete its warpgroup), per key tile j:
//                PV_A(j)  S_A(j+1)  PV_B(j)  S_B(j+1)
//              so S_X(j+1) enters the tensor pipe right behind PV_X(j) while the
//              other tile's softmax is running.  The whole warp runs the loop
//              (lane 0 issues): it meets tile X's softmax warps at the named
//              barrier that announces P_X(j).
// Hand-offs: TMA and MMA completions reach the other roles through mbarriers
// (bounded waits); P_X(j) reaches the MMA warp through a named barrier.
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [384,384+D).
// P_X(j) (bf16 pairs) goes to S_X's columns [0,64) once the softmax holds all of
// S_X(j) in registers.  The tcgen05.mma operations of one thread run in issue
// order, so S_X(j+1), issued right behind PV_X(j), overwrites P_X(j) only after
// PV_X(j) has read it (the order the CUTLASS Blackwell FMHA also relies on).
// The commit that announces S_X(j+1) tracks every earlier MMA of the thread,
// PV_X(j) included, so whenever the softmax of tile X sees a new S, O_X is
// stable and can be rescaled without a further wait.
//
// STATS = true is the statistics pass of the scoring ("Blocchi di Passaggio":
// each chunk's keys are scored by the query block's softmax over that chunk):
// the same key tiles, max and sum in the same order, but no V, no PV and no P;
// the item's per-row base-2 log-sum-exp goes to P.stats.  The running sum is
// the very arithmetic of the full kernel, so the statistics equal, bit for
// bit, the log-sum-exps the full kernel's query-row partials carry -- the
// scoring may take either.
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
    float *stats;       // STATS: [segments, Hq, q] log2-domain lse of the query rows
    int *status;        // workspace status word
    int *queue;         // work-item counter of the persistent attention grid (zeroed per launch)
    int32_t n_items;    // work items of the attention launch
};

// sm_100 allows at most 227 KiB of dynamic shared memory per CTA.
constexpr int kMaxDynSmem = 232448;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct AttnSmem {
    static constexpr int kPanels = D / 64;
    static constexpr int kTile = kRowTile * D * 2;  // one 128-row bf16 tile
    // Each K tile feeds two S MMAs and each V tile two PVs, so the rings turn
    // over half as often per MMA as with one query tile.
    static constexpr int KS = D == 128 ? 2 : 4;
    static constexpr int VS = D == 128 ? 2 : 3;
    static constexpr int kOffQ = 0;  // Q_A, Q_B
    static constexpr int kOffK = 2 * kTile;
    static constexpr int kOffV = kOffK + KS * kTile;
    static constexpr int kOffBar = kOffV + VS * kTile;
    static constexpr int kNumBar = 1 + 2 * KS + 2 * VS + 4 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBar * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(AttnSmem<128>::kAlloc <= kMaxDynSmem, "attention smem over budget");
static_assert(AttnSmem<64>::kAlloc <= kMaxDynSmem, "attention smem over budget");

// Three warpgroups: softmax of tile A, softmax of tile B, and one holding the
// TMA producer and the MMA issuer (its other two warps idle).  The third gives
// registers to the first two: launched at kLaunchRegs per thread, it drops to
// kRegsIo and the softmax warpgroups rise to kRegsSoftmax.
constexpr int kSoftWarps = 8;  // 4 per query tile
constexpr int kAttnThreads = 3 * 128;
constexpr int kProducerWarp = kSoftWarps;
constexpr int kMmaWarp = kSoftWarps + 1;
constexpr int kLaunchRegs = 168;  // 65536 / 384, rounded down to the allocation unit of 8
constexpr int kRegsIo = 80;
constexpr int kRegsSoftmax = 208;
static_assert(128 * kRegsIo + 256 * kRegsSoftmax <= kAttnThreads * kLaunchRegs,
              "register split above the CTA's pool");
constexpr int kColO = 256;  // O_A; O_B at kColO + 128
constexpr int kItemBar = 1;  // named barrier of all threads between work items
// P_X(j) is in TMEM (or, in the statistics pass, S_X(j) has been read): named
// barrier kPBar + X between tile X's four softmax warps (bar.arrive) and the
// whole MMA warp (bar.sync).  A hardware barrier hands off in ~130 cycles, an
// mbarrier's arrive-to-wake in ~350.  It has no timeout, so arrivals and syncs
// pair one for one by construction: the MMA warp syncs P_X(j) only after it has
// issued S_X(j), and the softmax warps arrive for step j only after S_X(j) has
// completed, waiting for it without regard to other roles' aborts (their own
// bounded wait gives up only if a committed MMA never completes).  At most one
// arrival is ever pending, since the next S needs the sync first.
constexpr int kPBar = 2;
constexpr int kPBarThreads = 4 * 32 + 32;

// Work items of a region (one group): row tiles 2p and 2p+1 of one query head;
// when the region has an odd number of row tiles, its last tile (the costliest,
// alone) is paired ACROSS query heads instead -- heads 2k and 2k+1 of a KV head
// share that tile's rows, key sequence and K/V, and differ only in Q -- so that
// at most one tile per KV head runs alone.  Inside a group: KV head by KV head,
// the cross-head items first (costliest), then the row pairs in descending
// cost, the query heads of a KV head adjacent.
__host__ __device__ inline int pair_items(int n_rt, int G) {
    return (n_rt / 2) * G + ((n_rt & 1) ? (G + 1) / 2 : 0);
}

// Item b: tile A = row tile it.rt of head it.h; tile B = row tile it.rt + 1 of
// the same head (*h_b = it.h), or the same row tile of head *h_b = it.h + 1
// (cross-head item), or none (*h_b = -1).
__host__ __device__ inline Item decode_pair_item(const Group *groups, int n_groups, int b, int G,
                                                 int *h_b) {
    int k = 0;
    while (k + 1 < n_groups && b >= groups[k + 1].item_begin) ++k;
    const Group &g = groups[k];
    const int i = b - g.item_begin;
    const int per_kv = pair_items(g.n_rt, G);
    const int kv = i / per_kv;
    int rem = i % per_kv;
    Item it;
    it.kind = g.kind;
    it.sub = g.sub;
    const int n_cross = (g.n_rt & 1) ? (G + 1) / 2 : 0;
    if (rem < n_cross) {
        it.rt = g.n_rt - 1;
        it.h = kv * G + 2 * rem;
        *h_b = (2 * rem + 1 < G) ? it.h + 1 : -1;
        return it;
    }
    rem -= n_cross;
    const int np = g.n_rt / 2;
    it.rt = 2 * (np - 1 - rem / G);  // first row tile of the pair
    it.h = kv * G + rem % G;
    *h_b = it.h;
    return it;
}

// Max of 128 values: four independent chains of 3-input max.
__device__ __forceinline__ float max128(const float (&x)[128]) {
    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = fmax3(x[k], x[4 + k], x[8 + k]);
#pragma unroll
    for (int c = 12; c + 8 <= 124; c += 8)
#pragma unroll
        for (int k = 0; k < 4; ++k) m[k] = fmax3(m[k], x[c + k], x[c + 4 + k]);
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = fmaxf(m[k], x[124 + k]);
    return fmaxf(fmax3(m[0], m[1], m[2]), m[3]);
}

// Everything about work item b that the roles need: rows of tiles A and B, the
// key segments and tile counts.
struct ItemPlan {
    Item it;
    int hB;  // query head of tile B
    int r0A, eA, r0B, eB;
    int rs;  // global position minus local row of the item's rows
    bool hasB;
    Seg segs[kMaxSegs];
    int ns, T, TA, TB, g;
};

__device__ __forceinline__ void plan_item(const Layer &L, const Group *groups, int n_groups, int b,
                                          ItemPlan &ip) {
    int h_b;
    ip.it = decode_pair_item(groups, n_groups, b, L.G, &h_b);
    item_rows(L, ip.it, ip.r0A, ip.eA);
    ip.g = ip.it.h / L.G;
    ip.rs = region_shift(L, item_region(L, ip.it));
    if (h_b != ip.it.h) {
        // Cross-head item (or a tile alone): B has A's rows and key sequence.
        ip.hasB = h_b >= 0;
        ip.hB = h_b;
        ip.r0B = ip.r0A, ip.eB = ip.eA;
        ip.ns = build_segments(L, ip.it, ip.segs);
        ip.T = count_tiles(ip.segs, ip.ns);
        ip.TA = ip.T;
        ip.TB = ip.hasB ? ip.T : 0;
        return;
    }
    Item it_b = ip.it;
    it_b.rt = ip.it.rt + 1;
    item_rows(L, it_b, ip.r0B, ip.eB);
    ip.hasB = ip.eB > ip.r0B;
    ip.hB = ip.it.h;
    ip.ns = build_segments(L, ip.hasB ? it_b : ip.it, ip.segs);
    ip.T = count_tiles(ip.segs, ip.ns);
    // A causal last segment starts on a tile boundary of the region, so its last
    // tile for B is B's diagonal, which lies beyond every row of A.
    ip.TA = (ip.hasB && ip.ns > 0 && ip.segs[ip.ns - 1].causal) ? ip.T - 1 : ip.T;
    ip.TB = ip.hasB ? ip.T : 0;
}

template <int D, bool STATS = false>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_kernel(const __grid_constant__ AttnParams P) {
    using SM = AttnSmem<D>;
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
    uint64_t *s_full = v_empty + VS;  // [2]: S_X(j) in TMEM
    uint64_t *o_done = s_full + 2;    // [2]: the last PV_X has completed
    uint64_t *mma_drain = o_done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layer &L = P.L;
    int *claim = reinterpret_cast<int *>(smem + SM::kOffMisc + 8);

    // Barriers start every item fresh: between items (nothing in flight any
    // more) they are invalidated and initialised again.
    auto init_bars = [&](bool again) {
        auto init = [&](uint64_t *bar, uint32_t count) {
            if (again) mbar_inval(bar);
            mbar_init(bar, count);
        };
        init(q_full, 1);
        for (int i = 0; i < KS; ++i) {
            init(&k_full[i], 1);
            init(&k_empty[i], 1);
        }
        for (int i = 0; i < VS; ++i) {
            init(&v_full[i], 1);
            init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            init(&s_full[i], 1);
            init(&o_done[i], 1);
        }
        init(mma_drain, 1);
        fence_mbar_init();
    };
    if (threadIdx.x == 0) {
        init_bars(false);
        *abort_flag = 0;
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch(&P.tmQ);
        tma_prefetch(&P.tmK);
        if (!STATS) {  // the statistics pass encodes only the Q and K maps
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

    // Persistent grid: each CTA claims work items one at a time from a queue in
    // the workspace, in the planner's order (costliest first), i.e. greedy
    // longest-processing-time-first over the SMs.  The claim happens between two
    // CTA-wide barriers, after every role is done with the previous item; a CTA
    // whose waits gave up claims nothing more.
    auto next_item = [&](int round) -> int {
        if (threadIdx.x == kProducerWarp * 32) {
            if (round > 0) init_bars(true);
            *claim = *abort_flag ? INT32_MAX : atomicAdd(P.queue, 1);
        }
        tc_fence_before();
        bar_sync(kItemBar, kAttnThreads);
        tc_fence_after();
        return *claim;
    };
    auto end_item = [&]() {
        tc_fence_before();
        bar_sync(kItemBar, kAttnThreads);
        tc_fence_after();
    };

    if (warp >= kSoftWarps) {
        reg_dealloc<kRegsIo>();
        for (int round = 0;; ++round) {
        const int b = next_item(round);
        if (b >= P.n_items) break;
        ItemPlan ip;
        plan_item(L, P.groups, P.n_groups, b, ip);
        const Item &it = ip.it;
        const int r0A = ip.r0A, r0B = ip.r0B, T = ip.T, TA = ip.TA, TB = ip.TB, g = ip.g;
        const bool hasB = ip.hasB;
        const Seg *segs = ip.segs;
        if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(q_full, hasB ? 2 * SM::kTile : SM::kTile);
            for (int p = 0; p < SM::kPanels; ++p)
                tma_load_3d(smem + SM::kOffQ + p * 16384, &P.tmQ, p * 64, it.h, r0A - ip.rs, q_full);
            if (hasB)
                for (int p = 0; p < SM::kPanels; ++p)
                    tma_load_3d(smem + SM::kOffQ + SM::kTile + p * 16384, &P.tmQ, p * 64, ip.hB,
                                r0B - ip.rs, q_full);
            int k_last[KS], v_last[VS];
            for (int i = 0; i < KS; ++i) k_last[i] = -1;
            for (int i = 0; i < VS; ++i) v_last[i] = -1;
            // K runs one tile ahead of V: S_X(j+1) needs K_{j+1} right behind PV_X(j).
            TileCursor kc, vc;
            auto load_k = [&](int j) -> bool {
                const int ks = j % KS;
                if (j >= KS && !mbar_wait(&k_empty[ks], ((j / KS) - 1) & 1, ab)) return false;
                mbar_expect_tx(&k_full[ks], SM::kTile);
                uint8_t *kd = smem + SM::kOffK + ks * SM::kTile;
                const Seg &s = segs[kc.seg];
                const int key0 = s.begin + kc.tile * kKeyTile;
                for (int p = 0; p < SM::kPanels; ++p) {
                    if (s.src == 0)
                        tma_load_3d(kd + p * 16384, &P.tmK, p * 64, g, key0 - s.shift, &k_full[ks]);
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
                        tma_load_3d(vd + p * 16384, &P.tmV, p * 64, g, key0 - s.shift, &v_full[vs]);
                    else
                        tma_load_3d(vd + p * 16384, &P.tmPV, p * 64, key0, g, &v_full[vs]);
                }
                v_last[vs] = j;
                vc.advance(segs);
                return true;
            };
            bool live = T > 0 ? load_k(0) : true;
            for (int j = 0; live && j < T; ++j) {
                if (j + 1 < T) live = load_k(j + 1);
                if (!STATS && live) live = load_v(j);
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
        // The whole warp runs the loop (it takes part in the P barriers, which
        // count whole warps); lane 0 alone issues the tcgen05 operations, and
        // every lane's wait result is combined so that the warp stays converged.
        {
            const bool leader = lane == 0;
            auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, ab));
            };
            auto commit = [&](uint64_t *bar) {
                if (leader) tc_commit(bar);
            };
            // Descriptors built once; a K-step or a ring stage adds its byte
            // offset / 16 to the start-address field.
            constexpr int NK = D / 16;
            uint64_t qd[2][NK];
            const uint64_t k_desc = sdesc_sw128(smem_u32(smem + SM::kOffK), 16, 1024);
            const uint64_t v_desc = sdesc_sw128(smem_u32(smem + SM::kOffV), 16384, 1024);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const uint64_t q_desc = sdesc_sw128(smem_u32(smem + SM::kOffQ + x * SM::kTile), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < NK; ++kk)
                    qd[x][kk] = q_desc + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            }
            // S_X(j) = Q_X K_j^T into TMEM columns [128x, 128x+128).
            auto mma_s = [&](int x, int j) {
                if (!leader) return;
                const uint64_t kd = k_desc + static_cast<uint64_t>(((j % KS) * SM::kTile) >> 4);
                const uint32_t d_s = tmem + x * kKeyTile;
#pragma unroll
                for (int g4 = 0; g4 < NK / 4; ++g4) {
                    const uint64_t kb = kd + static_cast<uint64_t>(g4 * (16384 >> 4));
                    mma_ss_x4(d_s, qd[x][4 * g4], qd[x][4 * g4 + 1], qd[x][4 * g4 + 2],
                              qd[x][4 * g4 + 3], kb, kb + 2, kb + 4, kb + 6, kIdescS, g4 > 0);
                }
                tc_commit(&s_full[x]);
            };
            // O_X += P_X(j) V_j.  K-step kb covers keys 16kb..16kb+15: P columns
            // +8kb inside S_X, V rows +2048 B.
            auto mma_pv = [&](int x, int j) {
                if (!leader) return;
                const uint32_t a_p = tmem + x * kKeyTile;
                const uint64_t vd = v_desc + static_cast<uint64_t>(((j % VS) * SM::kTile) >> 4);
                const uint32_t d_o = tmem + kColO + x * 128;
                mma_ts_x4(d_o, a_p, a_p + 8, a_p + 16, a_p + 24, vd, vd + 128, vd + 256, vd + 384,
                          kIdescPV, j > 0);
                mma_ts_x4(d_o, a_p + 32, a_p + 40, a_p + 48, a_p + 56, vd + 512, vd + 640, vd + 768,
                          vd + 896, kIdescPV, 1u);
            };
            bool ok = wait(q_full, 0) && (T == 0 || wait(&k_full[0], 0));
            tc_fence_after();
            if (ok && T > 0) {
                if (TA > 0) mma_s(0, 0);
                if (TB > 0) mma_s(1, 0);
                commit(&k_empty[0]);
            }
            // Statistics only: S_X(j+1) as soon as the softmax has read S_X(j).
            for (int j = 0; STATS && ok && j < T; ++j) {
                const int kn = j + 1, ks = kn % KS;
                bool k_seen = false;
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int TX = x ? TB : TA;
                    if (ok && j < TX) {
                        __syncwarp();
                        bar_sync(kPBar + x, kPBarThreads);
                        tc_fence_after();
                        if (kn < TX) {
                            if (!k_seen) {
                                ok = wait(&k_full[ks], (kn / KS) & 1);
                                if (!ok) break;
                                tc_fence_after();
                                k_seen = true;
                            }
                            mma_s(x, kn);
                        }
                    }
                }
                if (!ok) break;
                if (k_seen) commit(&k_empty[ks]);
            }
            for (int j = 0; !STATS && ok && j < T; ++j) {
                const int vs = j % VS, kn = j + 1, ks = kn % KS;
                if (!wait(&v_full[vs], (j / VS) & 1)) break;
                bool k_seen = false;
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int TX = x ? TB : TA;
                    if (ok && j < TX) {
                        __syncwarp();
                        bar_sync(kPBar + x, kPBarThreads);
                        tc_fence_after();
                        mma_pv(x, j);
                        if (j + 1 == TX) commit(&o_done[x]);
                        if (kn < TX) {
                            if (!k_seen) {
                                ok = wait(&k_full[ks], (kn / KS) & 1);
                                if (!ok) break;
                                tc_fence_after();
                                k_seen = true;
                            }
                            mma_s(x, kn);
                        }
                    }
                }
                if (!ok) break;
                commit(&v_empty[vs]);
                if (k_seen) commit(&k_empty[ks]);
            }
            // No MMA may still be running when TMEM is released.
            commit(mma_drain);
            mbar_wait_drain(mma_drain, 0);
        }
        __syncwarp();
        }
        end_item();
        }
    } else {
        reg_alloc<kRegsSoftmax>();
        for (int round = 0;; ++round) {
        const int b = next_item(round);
        if (b >= P.n_items) break;
        ItemPlan ip;
        plan_item(L, P.groups, P.n_groups, b, ip);
        const Item &it = ip.it;
        const int r0A = ip.r0A, r0B = ip.r0B, eA = ip.eA, eB = ip.eB, TA = ip.TA, TB = ip.TB;
        const Seg *segs = ip.segs;
        // ------------------------------------------------------------ softmax
        const int x = warp >> 2, quarter = warp & 3;
        const int hx = x ? ip.hB : it.h;  // query head of this warp's tile
        const int TX = x ? TB : TA;
        const int row0 = x ? r0B : r0A, row_end = x ? eB : eA;
        const int r = quarter * 32 + lane;  // row within the tile == TMEM lane
        const int t = row0 + r;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t col_s = x * kKeyTile, col_o = kColO + x * 128;
        const float sl2 = L.scale_log2;
        const float2 sl2v = make_float2(sl2, sl2);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        TileCursor cur;
        for (int j = 0; j < TX; ++j) {
            const Seg &s = segs[cur.seg];
            const int key0 = s.begin + cur.tile * kKeyTile;
            int lim_end = s.end;
            if (s.causal && t + 1 < lim_end) lim_end = t + 1;
            const int lim = lim_end - key0;  // keys [0, lim) of this tile are valid for row r
            cur.advance(segs);

            // Not cut short by another role's abort: once the MMA warp has issued
            // S_X(j) it will wait on this tile's P barrier, and only a completed
            // S_X(j) may be answered there (or the barrier would be left short).
            ok = __all_sync(0xffffffffu, mbar_wait_own(&s_full[x], j & 1, ab));
            if (!ok) break;
            tc_fence_after();
            float xs[kKeyTile];
            {
                uint32_t u[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + col_s + c * 32, u[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    reg_fence(u[c]);
#pragma unroll
                    for (int e = 0; e < 32; ++e) xs[c * 32 + e] = __uint_as_float(u[c][e]);
                }
            }
            if (STATS) {  // S_X(j) is in registers: the next S may overwrite it
                tc_fence_before();
                bar_arrive(kPBar + x, kPBarThreads);
            }
            if (lim < kKeyTile) {  // only tiles crossing a segment end or the diagonal
#pragma unroll
                for (int c = 0; c < kKeyTile; ++c)
                    if (c >= lim) xs[c] = -INFINITY;
            }
            // Rounded operations (never contracted into FMAs), so that the
            // statistics pass repeats this arithmetic exactly.
            const float mx = __fmul_rn(max128(xs), sl2);
            const float m_new = fmaxf(m_run, mx);
            const bool need = m_new > m_run + 8.0f;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(__fsub_rn(m_run, m_new));
                l_run = __fmul_rn(l_run, alpha);
                m_run = m_new;
            }
            if (!STATS && j > 0 && __any_sync(0xffffffffu, need)) {
                // O_X holds the sum up to tile j-1 scaled by the old max, and is
                // stable: PV_X(j-1) completed before S_X(j) was announced.
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    const uint32_t a = lane_addr + col_o + c * 32;
                    tmem_ld32(a, u);
                    tmem_wait_ld();
                    reg_fence(u);
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
                    tmem_st32(a, u);
                }
                tmem_wait_st();
            }
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            const float2 nmu = make_float2(-mu, -mu);
            float2 ps[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            // P, 32 keys (16 bf16-pair columns) at a time, over S columns this
            // warp has already read.
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 arg = ffma2(make_float2(xs[c * 32 + 2 * e], xs[c * 32 + 2 * e + 1]), sl2v, nmu);
                    const float2 p = make_float2(ex2(arg.x), ex2(arg.y));
                    ps[e & 1] = fadd2(ps[e & 1], p);
                    if (!STATS) pk[e] = pack_bf16x2(p.x, p.y);
                }
                if (!STATS) tmem_st16(lane_addr + col_s + c * 16, pk);
            }
            if (!STATS) {
                tmem_wait_st();
                tc_fence_before();
                bar_arrive(kPBar + x, kPBarThreads);
            }
            const float2 pss = fadd2(ps[0], ps[1]);
            l_run = __fadd_rn(l_run, __fadd_rn(pss.x, pss.y));
        }

        // ------------------------------------------------------------ epilogue
        if (STATS) {
            // The row's base-2 log-sum-exp over the item's keys (tile B may be
            // absent: TB = 0, no head).
            if (ok && TX > 0 && t < row_end) {
                const int i = t - (L.N - L.q);
                P.stats[(static_cast<size_t>(it.sub) * L.Hq + hx) * L.q + i] =
                    (l_run > 0.f) ? __fadd_rn(m_run, __log2f(l_run)) : -INFINITY;
            }
        } else if (ok && TX > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&o_done[x], 0, ab));
            if (ok) {
                tc_fence_after();
                const bool valid = t < row_end;
                const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
                const float lse2 = (l_run > 0.f) ? __fadd_rn(m_run, __log2f(l_run)) : -INFINITY;
                if (it.kind == kQueryPart) {
                    const int i = t - (L.N - L.q);
                    float *dst = P.part_O + ((static_cast<size_t>(it.sub) * L.Hq + hx) * L.q + i) * D;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t u[32];
                        tmem_ld32(lane_addr + col_o + c * 32, u);
                        tmem_wait_ld();
                        reg_fence(u);
                        if (valid) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4)
                                *reinterpret_cast<float4 *>(dst + c * 32 + e) =
                                    make_float4(__uint_as_float(u[e]) * inv, __uint_as_float(u[e + 1]) * inv,
                                                __uint_as_float(u[e + 2]) * inv, __uint_as_float(u[e + 3]) * inv);
                        }
                    }
                    if (valid) P.part_lse[(static_cast<size_t>(it.sub) * L.Hq + hx) * L.q + i] = lse2;
                } else {
                    const int tl = t - ip.rs;  // local row
                    __nv_bfloat16 *dst = P.O + (static_cast<size_t>(tl) * L.Hq + hx) * D;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t u[32];
                        tmem_ld32(lane_addr + col_o + c * 32, u);
                        tmem_wait_ld();
                        reg_fence(u);
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
                    if (valid && P.lse) P.lse[static_cast<size_t>(hx) * L.Nl + tl] = lse2 * 0.69314718055994531f;
                }
            }
        }
        end_item();
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

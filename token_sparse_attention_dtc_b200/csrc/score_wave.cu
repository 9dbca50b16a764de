// Dynamic Token Coverage scoring on the tensor cores, wave schedule (bf16, q = 16 recent
// queries, at most 4 query heads per KV head).
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 2 (the last q queries
// score all keys with a per-head softmax; column sums give s_h); bxzpzcl.cn post §2.1;
// gist.science §2 "Scoring".  The result is the same exact two-pass softmax as the
// single-wave kernel in score_tc.cu; what changes is the order of the work:
//
// - The B*Hkv KV groups are scored in W waves of gpw groups each, every CTA of the
//   cooperative grid taking one contiguous tile range of one group in every wave.  A wave
//   holds at most about 40 MB of K, so the K tiles a CTA read in pass 1 are still in L2
//   when pass 2 reads them again: K crosses HBM once.
// - Each CTA runs the phases P1(0), P1(1), P2(0), P1(2), P2(1), ..., P2(W-1).  The grid
//   barrier that separates pass 1 and pass 2 of wave w (every CTA has stored its
//   (max, sum) pairs of wave w and counted itself in) is waited for only after pass 1 of
//   wave w+1, so it costs little idle time.  Each CTA then merges its group's pairs in a
//   fixed order itself (no CTA does the others' merge, so none falls behind).
// - Both passes compute S^T = Ktile * Qblk^T with the 128 tokens on the TMEM lanes and
//   the N = 16*G query rows as columns (M = 128, N = 16*G).  Pass 1 therefore keeps a
//   running (max, sum) per query row in every thread over the tokens of its lane, and
//   reduces over lanes once per wave (shuffles inside a warp, shared memory across the 4
//   lane quadrants), instead of padding the query rows to M = 128 on every tile.
//
// Warp 0 streams K tiles by TMA through a 5-stage ring, warp 1 issues the MMAs into an
// 8-deep TMEM ring of 64-column accumulators, warp 2 loads the waves' Q rows by TMA into
// three shared-memory slots (wave w+2's rows land while waves w and w+1 run), warp 3
// stores each wave's per-row pairs and counts the CTA in, warps 4-19 run the epilogue:
// lane quadrant wq = warp % 4 (tokens wq*32 .. wq*32+31 of a tile, the TMEM lanes that
// warp may read) and column group cg = (warp - 4) / 4 (head cg of the group, its 16
// recent queries).  All waits are bounded.
#include <math.h>

#include <algorithm>

#include "sm100.cuh"

namespace tsa {
using namespace sm100;

int device_sm_count();  // score_tc.cu: SM count of the current device, cached per device

namespace {

constexpr int kThreads = 640, kStages = 5, kTile = 128, kQE = 16, kEpiWarps = 16;
constexpr int kEpi0 = 4;       // first epilogue warp: warps 4-19, warpgroups 1-4
constexpr int kStatsWarp = 3;
constexpr int kQRows = 64;     // Q slot rows: 16 recent queries x at most 4 heads
constexpr int kQSlots = 3;
// Pass-1 pair slots: wave w+4 reuses wave w's slot only after the wave-(w+2) barrier,
// which every CTA passes after its P2(w) merge has read the slot.
constexpr int kPartSlots = 4;
constexpr int kNbuf = 8, kLgb = 3, kBufCols = 64;  // TMEM ring: 8 x 64 columns
constexpr int kMaxCtas = 160;  // pair slots per wave: the grid never exceeds 160 CTAs
constexpr uint64_t kDrainNs = 1000000000ull;
constexpr float kNoMax = -1e30f;   // running max before any token (finite: no inf - inf)
constexpr float kRescale = 8.0f;   // a value this far (log2 units) above the max moves it

template <int D> struct WaveSmem {
    static constexpr int KT = kTile * D * 2;    // one K tile
    static constexpr int QS = kQRows * D * 2;   // one Q slot
    alignas(1024) uint8_t k[kStages][KT];
    alignas(1024) uint8_t q[kQSlots][QS];
    uint64_t k_full[kStages], k_empty[kStages], acc_full[kNbuf], acc_empty[kNbuf];
    uint64_t q_full[kQSlots], q_free[kQSlots], stats_full[2], drain;
    uint64_t stall;          // test hook: initialised, never completed
    float2 red[2][4][4][kQE];  // pass-1 pairs per [wave % 2][column group][quadrant][query]
    int team_ok[4];           // pass 2: the team leader's barrier wait succeeded
    alignas(16) float mlog[kQRows];  // pass 2: max + log2(sum) per query row
    float wsum[kEpiWarps];   // layer score: per epilogue warp partial sums
    uint32_t tmem_base;
    int abort, never, flag_ok;
};

// Phase p of the 2W phases: pass 1 or 2 of wave w, in the order P1(0), P1(1), P2(0),
// P1(2), P2(1), ..., P1(W-1), P2(W-2), P2(W-1).
__device__ inline void phase_of(int p, int W, int &pass, int &w) {
    if (p == 0) {
        pass = 1;
        w = 0;
    } else if (p == 2 * W - 1) {
        pass = 2;
        w = W - 1;
    } else if (p & 1) {
        pass = 1;
        w = (p + 1) / 2;
    } else {
        pass = 2;
        w = p / 2 - 1;
    }
}

// Merge (m2, l2) into (m1, l1): two sums of 2^(z - m) over disjoint token sets.
__device__ inline void merge_ml(float &m1, float &l1, float m2, float l2) {
    const float mx = fmaxf(m1, m2);
    l1 = l1 * ex2(m1 - mx) + l2 * ex2(m2 - mx);
    m1 = mx;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_score_wave(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
             int L, int H, int Hkv, int Bn, int S, int gpw, int W, float sl2, float2 *part,
             float *__restrict__ s_h, float *__restrict__ s_l, float *zp, unsigned int *sync,
             Control *ctl, uint64_t limit_ns, int stall) {
    // The kernel after this one in a layer (budget and selection) may start launching; it
    // waits for this grid to complete before it reads the scores.
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    WaveSmem<D> &sm = *reinterpret_cast<WaveSmem<D> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int KT = WaveSmem<D>::KT, NDB = D / 64;
    const int G = H / Hkv, N = G * kQE;  // N: query rows of a group (<= 64, multiple of 16)
    const unsigned nctas = gridDim.x;
    const int cta = blockIdx.x, gl = cta / S, split = cta % S;
    const int ntiles = (L + kTile - 1) / kTile;
    const int per = ntiles / S, rem = ntiles % S;
    const int first = split * per + min(split, rem), count = per + (split < rem ? 1 : 0);
    const int nphase = 2 * W;
    // sync[0] grid barrier, sync[1..kPartSlots] per-wave counts, sync[kPartSlots + 1] the
    // CTAs done; all zero at launch, and zero again when the last CTA is done.
    unsigned int *gbar = sync, *cnt = sync + 1, *done = sync + 1 + kPartSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int a = 0; a < kNbuf; ++a) {
            mbar_init(&sm.acc_full[a], 1);
            mbar_init(&sm.acc_empty[a], kEpiWarps);  // one arrival per epilogue warp
        }
        for (int s = 0; s < kQSlots; ++s) {
            mbar_init(&sm.q_full[s], 1);
            mbar_init(&sm.q_free[s], 1);
        }
        for (int s = 0; s < 2; ++s) mbar_init(&sm.stats_full[s], kEpiWarps);
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.stall, 1);
        sm.abort = 0;
        sm.never = 0;
        sm.flag_ok = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort = &sm.abort;
    bool ok = true;
    if (warp == 0) {
        // ---- producer: K tiles of every phase, pass 1 ascending, pass 2 descending
        if (lane == 0) {
            // Pass 1 keeps its tiles in L2 for pass 2's reread; pass 2 reads them last.
            const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
            int issued = 0;
            for (int p = 0; p < nphase && ok; ++p) {
                int pass, w;
                phase_of(p, W, pass, w);
                const int bg = w * gpw + gl, b = bg / Hkv, kv = bg % Hkv;
                for (int it = 0; it < count; ++it) {
                    const int gi = p * count + it, s = gi % kStages;
                    if (!(ok = mbar_wait(&sm.k_empty[s], ((gi / kStages) & 1) ^ 1, limit_ns, abort)))
                        break;
                    const int tile = pass == 1 ? first + it : first + count - 1 - it;
                    mbar_expect_tx(&sm.k_full[s], KT);
#pragma unroll
                    for (int db = 0; db < NDB; ++db)
                        tma_load_4d_hint(sm.k[s] + db * kTile * 128, &tmK, &sm.k_full[s], db * 64,
                                         tile * kTile, kv, b, pass == 1 ? keep : drop);
                    issued = gi + 1;
                }
            }
            for (int gi = (issued > kStages ? issued - kStages : 0); gi < issued; ++gi)
                mbar_wait(&sm.k_full[gi % kStages], (gi / kStages) & 1, kDrainNs, &sm.never);
        }
    } else if (warp == 1) {
        // ---- MMA issuer: S^T = Ktile * Qslot^T, M = 128 tokens, N = 16*G query rows
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, N, false);
            bool any = false;
            // Test hook: a wait that nothing completes, so it runs out after limit_ns.
            if (stall) ok = mbar_wait(&sm.stall, 0, limit_ns, abort);
            for (int p = 0; p < nphase && ok; ++p) {
                int pass, w;
                phase_of(p, W, pass, w);
                const int qslot = w % kQSlots;
                if (pass == 1 && !(ok = mbar_wait(&sm.q_full[qslot], (w / kQSlots) & 1, limit_ns, abort)))
                    break;
                const uint32_t qa = smem_u32(sm.q[qslot]);
                for (int it = 0; it < count; ++it) {
                    const int gi = p * count + it, s = gi % kStages, a = gi & (kNbuf - 1);
                    if (!(ok = mbar_wait(&sm.k_full[s], (gi / kStages) & 1, limit_ns, abort)))
                        break;
                    if (!(ok = mbar_wait(&sm.acc_empty[a], ((gi >> kLgb) & 1) ^ 1, limit_ns, abort)))
                        break;
                    tc_fence_after();
                    const uint32_t ka = smem_u32(sm.k[s]);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t kof = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
                        const uint32_t qof = (kk / 4) * (kQRows * 128) + (kk % 4) * 32;
                        mma_ss(tmem + a * kBufCols, sdesc_sw128(ka + kof, 16, 1024),
                               sdesc_sw128(qa + qof, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                    }
                    any = true;
                    mma_commit(&sm.k_empty[s]);
                    mma_commit(&sm.acc_full[a]);
                }
                if (ok && pass == 2) mma_commit(&sm.q_free[qslot]);  // free for wave w+3
            }
            if (any) {
                mma_commit(&sm.drain);
                mbar_wait(&sm.drain, 0, kDrainNs, &sm.never);
            }
        }
    } else if (warp == 2) {
        // ---- Q loader: wave w's recent-query rows into slot w % 3 by TMA, row
        // n = g*16 + i <- Q[b, L-16+i, kv*G+g, :] (one 16-row box per head and 64-column
        // block; each box lands 1024-byte aligned, so its 128-byte swizzle is the MMA's).
        if (lane == 0) {
            int issued = 0;
            for (int w = 0; w < W; ++w) {
                const int slot = w % kQSlots;
                if (w >= kQSlots &&
                    !(ok = mbar_wait(&sm.q_free[slot], (w / kQSlots - 1) & 1, limit_ns, abort)))
                    break;
                const int bg = w * gpw + gl, b = bg / Hkv, kv = bg % Hkv;
                mbar_expect_tx(&sm.q_full[slot], (uint32_t)(N * D * 2));
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int db = 0; db < NDB; ++db)
                        tma_load_4d(sm.q[slot] + db * (kQRows * 128) + g * kQE * 128, &tmQ,
                                    &sm.q_full[slot], db * 64, kv * G + g, L - kQE, b);
                issued = w + 1;
            }
            for (int w = (issued > kQSlots ? issued - kQSlots : 0); w < issued; ++w)
                mbar_wait(&sm.q_full[w % kQSlots], (w / kQSlots) & 1, kDrainNs, &sm.never);
        }
    } else if (warp == kStatsWarp) {
        // ---- statistics warp: for each wave, once the 16 epilogue warps have left their
        // lane-reduced pairs in red[w % 2], merge the 4 lane quadrants of each query row in
        // order, store the CTA's pair per row (row-major over the group's S splits), and
        // count the CTA in with a release add.
        for (int w = 0; w < W && ok; ++w) {
            const int slot = w % kPartSlots;
            if (!(ok = mbar_wait(&sm.stats_full[w & 1], (w >> 1) & 1, limit_ns, abort))) break;
            for (int n = lane; n < N; n += 32) {
                const int c2 = n / kQE, c = n % kQE;
                float2 acc = sm.red[w & 1][c2][0][c];
                for (int q2 = 1; q2 < 4; ++q2)
                    merge_ml(acc.x, acc.y, sm.red[w & 1][c2][q2][c].x, sm.red[w & 1][c2][q2][c].y);
                __stcg(&part[(((size_t)slot * gpw + gl) * kQRows + n) * S + split], acc);
            }
            __syncwarp();
            if (lane == 0)
                asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(cnt + slot) : "memory");
        }
    } else {
        // ---- epilogue
        const int wq = warp & 3, cg = (warp - kEpi0) >> 2, r = wq * 32 + lane;
        const uint32_t lo = (uint32_t)(wq * 32) << 16;
        const int et = threadIdx.x - kEpi0 * 32;  // 0..511
        const int ew = warp - kEpi0;              // 0..15
        const bool active = cg < G;               // this warp's head exists in the group
        const int pmin = L - kQE;                 // position of recent query 0
        const int tt = wq * 32 + lane;            // 0..127 within the head's team
        // Layer-score total: this warp's sum of its s_h values per batch element, kept
        // in zp[b][cta][ew] (zero for batch elements it never scores).
        float zrun = 0.0f;
        int zb = gl / Hkv;  // batch element of wave 0
        if (lane == 0)
            for (int bb = 0; bb < Bn; ++bb) zp[((size_t)bb * nctas + cta) * kEpiWarps + ew] = 0.0f;
        // Tile fetch: wait for the TMEM buffer of tile gi, start loading this thread's 16
        // columns (its head's 16 queries) of it.
        auto fetch = [&](int gi, uint32_t (&v)[16]) -> bool {
            const int a = gi & (kNbuf - 1);
            const bool good = mbar_wait(&sm.acc_full[a], (gi >> kLgb) & 1, limit_ns, abort);
            if (!__all_sync(0xffffffffu, good)) return false;
            tc_fence_after();
            if (active) tmem_ld16(tmem + a * kBufCols + cg * kQE + lo, v);
            return true;
        };
        // Finish the load of tile gi and hand its buffer back to the MMA warp (one
        // arrival per warp, once every lane's load is complete).
        auto release = [&](int gi, uint32_t (&v)[16]) {
            tmem_ld_wait_regs(v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[gi & (kNbuf - 1)]);
        };
        float m[kQE], l[kQE];
        for (int p = 0; p < nphase; ++p) {
            int pass, w;
            phase_of(p, W, pass, w);
            const int slot = w % kPartSlots, bg = w * gpw + gl, b = bg / Hkv, kv = bg % Hkv;
            uint32_t va[16];
            if (pass == 1) {
#pragma unroll
                for (int j = 0; j < kQE; ++j) {
                    m[j] = kNoMax;
                    l[j] = 0.0f;
                }
                for (int it = 0; it < count && ok; ++it) {
                    const int gi = p * count + it;
                    if (!(ok = fetch(gi, va))) break;
                    release(gi, va);
                    if (active) {
                        const int t0 = (first + it) * kTile, t = t0 + r;
                        if (t0 + kTile - 1 <= pmin) {  // every token precedes every recent query
                            if (it == 0) {
#pragma unroll
                                for (int j = 0; j < kQE; ++j) {
                                    m[j] = __uint_as_float(va[j]) * sl2;
                                    l[j] = 1.0f;
                                }
                            } else {  // m is finite here: tile 0 of the range set it
                                float x[kQE];
#pragma unroll
                                for (int j = 0; j < kQE; j += 2)
                                    fma2(x[j], x[j + 1], __uint_as_float(va[j]),
                                         __uint_as_float(va[j + 1]), sl2, sl2, -m[j], -m[j + 1]);
                                float mx = fmax3(x[0], x[1], x[2]);
#pragma unroll
                                for (int j = 3; j < kQE - 1; j += 2) mx = fmax3(mx, x[j], x[j + 1]);
                                mx = fmaxf(mx, x[kQE - 1]);
                                if (mx > kRescale) {  // rare: move the reference max of some rows
#pragma unroll
                                    for (int j = 0; j < kQE; ++j) {
                                        const float c = x[j] > kRescale ? x[j] : 0.0f;
                                        l[j] *= ex2(-c);
                                        m[j] += c;
                                        x[j] -= c;
                                    }
                                }
#pragma unroll
                                for (int j = 0; j < kQE; j += 2)
                                    add2(l[j], l[j + 1], l[j], l[j + 1], ex2(x[j]), ex2(x[j + 1]));
                            }
                        } else {  // causal: token t counts for query j only if t <= L-16+j
#pragma unroll
                            for (int j = 0; j < kQE; ++j) {
                                if (t > pmin + j) continue;
                                const float z = __uint_as_float(va[j]) * sl2;
                                if (z > m[j]) {
                                    l[j] *= ex2(m[j] - z);
                                    m[j] = z;
                                }
                                l[j] += ex2(z - m[j]);
                            }
                        }
                    }
                }
                // Reduce the 32 lanes' pairs: halve the held rows at each shuffle step
                // (lane bit set: keep the upper half), so lane pair (2c, 2c+1) ends with
                // row c; the even lane leaves the merged pair for the statistics warp.
                ok = __all_sync(0xffffffffu, ok) && !*abort;
                if (active && ok) {
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        const int o = 16 >> s, half = 8 >> s;
                        const bool up = (lane & o) != 0;
#pragma unroll
                        for (int k = 0; k < half; ++k) {
                            const float sm_ = up ? m[k] : m[k + half], sl_ = up ? l[k] : l[k + half];
                            float km = up ? m[k + half] : m[k], kl = up ? l[k + half] : l[k];
                            const float rm = __shfl_xor_sync(0xffffffffu, sm_, o);
                            const float rl = __shfl_xor_sync(0xffffffffu, sl_, o);
                            merge_ml(km, kl, rm, rl);
                            m[k] = km;
                            l[k] = kl;
                        }
                    }
                    const float rm = __shfl_xor_sync(0xffffffffu, m[0], 1);
                    const float rl = __shfl_xor_sync(0xffffffffu, l[0], 1);
                    if (!(lane & 1)) {
                        merge_ml(m[0], l[0], rm, rl);
                        sm.red[w & 1][cg][wq][lane >> 1] = make_float2(m[0], l[0]);
                    }
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&sm.stats_full[w & 1]);
            } else {
                // ---- pass 2: the team's leader waits until every CTA has stored its
                // wave-w pairs; then the team merges its head's 16 rows over the group's S
                // splits (8 threads per row; thread sub takes splits sub, sub+8, ...: max
                // first, then the rescaled sums, then a fixed shuffle tree), then s_h per
                // token.
                if (active && tt == 0) {
                    int good = 0;
                    if (ok && !*abort) {
                        const unsigned target = ((unsigned)(w / kPartSlots) + 1u) * nctas;
                        const uint64_t t0 = globaltimer_ns();
                        for (uint32_t k = 0;; ++k) {
                            unsigned v;
                            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];"
                                         : "=r"(v) : "l"(cnt + slot) : "memory");
                            if (v >= target) { good = 1; break; }
                            if ((k & 63) == 63 && (*abort || globaltimer_ns() - t0 > limit_ns)) break;
                            __nanosleep(32);
                        }
                    }
                    sm.team_ok[cg] = good;
                }
                named_barrier(2 + cg, 128);
                ok = ok && (!active || sm.team_ok[cg]);  // idle teams still free each buffer
                {
                    const int c = tt >> 3, sub = tt & 7;  // row cg*16 + c, eighth sub
                    float mm = kNoMax, ll = 0.0f;
                    if (ok && active && sub < S) {
                        const float2 *src =
                            part + (((size_t)slot * gpw + gl) * kQRows + cg * kQE + c) * S;
                        const int nu = (S - sub + 7) / 8;  // splits sub, sub+8, ... < S
                        float2 pv[kMaxCtas / 8];
#pragma unroll
                        for (int u = 0; u < kMaxCtas / 8; ++u)  // every load issued at once
                            pv[u] = __ldcg(src + sub + 8 * min(u, nu - 1));
#pragma unroll
                        for (int u = 0; u < kMaxCtas / 8; ++u)
                            if (u < nu) mm = fmaxf(mm, pv[u].x);
#pragma unroll
                        for (int u = 0; u < kMaxCtas / 8; ++u)
                            if (u < nu) ll = fmaf(pv[u].y, ex2(pv[u].x - mm), ll);
                    }
#pragma unroll
                    for (int o = 1; o < 8; o <<= 1) {
                        const float rm = __shfl_xor_sync(0xffffffffu, mm, o);
                        const float rl = __shfl_xor_sync(0xffffffffu, ll, o);
                        if (!(sub & o)) merge_ml(mm, ll, rm, rl);
                    }
                    if (ok && active && sub == 0) sm.mlog[cg * kQE + c] = mm + log2f(ll);
                }
                named_barrier(2 + cg, 128);
                float ml[kQE];
                if (ok && active) {
                    const float4 *src = reinterpret_cast<const float4 *>(sm.mlog + cg * kQE);
#pragma unroll
                    for (int u = 0; u < kQE / 4; ++u) {
                        const float4 f = src[u];
                        ml[4 * u] = f.x;
                        ml[4 * u + 1] = f.y;
                        ml[4 * u + 2] = f.z;
                        ml[4 * u + 3] = f.w;
                    }
                }
                if (b != zb) {  // a new batch element: keep the finished one's total
                    if (lane == 0) zp[((size_t)zb * nctas + cta) * kEpiWarps + ew] = zrun;
                    zrun = 0.0f;
                    zb = b;
                }
                float *dst = s_h + ((size_t)b * H + kv * G + cg) * L;
                float zs = 0.0f;
                for (int it = 0; it < count && ok; ++it) {
                    const int gi = p * count + it;
                    if (!(ok = fetch(gi, va))) break;
                    release(gi, va);
                    if (active) {
                        const int t0 = (first + count - 1 - it) * kTile, t = t0 + r;
                        float acc;
                        if (t0 + kTile - 1 <= pmin) {
                            float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
#pragma unroll
                            for (int j = 0; j < kQE; j += 4) {
                                float x0, x1, x2, x3;
                                fma2(x0, x1, __uint_as_float(va[j]), __uint_as_float(va[j + 1]), sl2,
                                     sl2, -ml[j], -ml[j + 1]);
                                fma2(x2, x3, __uint_as_float(va[j + 2]), __uint_as_float(va[j + 3]),
                                     sl2, sl2, -ml[j + 2], -ml[j + 3]);
                                add2(a0, a1, a0, a1, ex2(x0), ex2(x1));
                                add2(b0, b1, b0, b1, ex2(x2), ex2(x3));
                            }
                            acc = (a0 + a1) + (b0 + b1);
                        } else {
                            acc = 0.0f;
#pragma unroll
                            for (int j = 0; j < kQE; ++j)
                                if (t <= pmin + j) acc += ex2(fmaf(__uint_as_float(va[j]), sl2, -ml[j]));
                        }
                        if (t < L) {
                            dst[t] = acc;
                            zs += acc;
                        }
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
                zrun += zs;
            }
        }
        if (lane == 0) zp[((size_t)zb * nctas + cta) * kEpiWarps + ew] = zrun;
        // Grid barrier among the epilogue warps of every CTA on gbar (zero at launch),
        // which reaches `target` = nctas times the barrier's ordinal.
        auto grid_sync = [&](unsigned target) -> bool {
            __threadfence();
            named_barrier(1, kEpiWarps * 32);
            if (et == 0) {
                int good = 0;
                if (!*abort) {
                    atomicAdd(gbar, 1u);
                    const uint64_t t0 = globaltimer_ns();
                    for (uint32_t k = 0;; ++k) {
                        unsigned v;
                        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(gbar) : "memory");
                        if (v >= target) { good = 1; break; }
                        if ((k & 63) == 63 && (*abort || globaltimer_ns() - t0 > limit_ns)) break;
                        __nanosleep(32);
                    }
                }
                sm.flag_ok = good;
            }
            named_barrier(1, kEpiWarps * 32);
            return sm.flag_ok != 0;
        };
        if (s_l) {
            // ---- layer score: after one grid barrier (every s_h row and every warp's
            // total is stored), Z = the totals summed in a fixed order, and for this CTA's
            // token range s_l[t] = (sum_h s_h[h, t] in head order) / Z.
            const bool g1 = grid_sync(nctas);
            ok = ok && g1;
            const int cl = ceil_div(L, (int)nctas);
            const int t0 = min(L, cta * cl), t1 = min(L, t0 + cl);
            for (int bb = 0; bb < Bn; ++bb) {
                float z = 0.0f;
                if (ok)
                    for (int e = et; e < (int)nctas * kEpiWarps; e += kEpiWarps * 32)
                        z += __ldcg(zp + (size_t)bb * nctas * kEpiWarps + e);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                if (lane == 0) sm.wsum[ew] = z;
                named_barrier(1, kEpiWarps * 32);
                float Z = 0.0f;
                for (int w2 = 0; w2 < kEpiWarps; ++w2) Z += sm.wsum[w2];
                if (ok)
                    for (int t = t0 + et; t < t1; t += kEpiWarps * 32) {
                        const float *col = s_h + (size_t)bb * H * L + t;
                        float u = 0.0f;
                        for (int h0 = 0; h0 < H; h0 += 32) {  // 32 heads' loads in flight
                            float hv[32];
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                hv[k] = h0 + k < H ? __ldcg(col + (size_t)(h0 + k) * L) : 0.0f;
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                if (h0 + k < H) u += hv[k];
                        }
                        s_l[(size_t)bb * L + t] = u / Z;
                    }
                named_barrier(1, kEpiWarps * 32);  // wsum is free again
            }
        }
    }
    if (!ok) {
        *abort = 1;
        report_error(ctl, TSA_ERR_DEVICE_TIMEOUT, 300 + warp);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    // Every wait of this CTA on the counters is behind it (each one either succeeded or
    // gave up): the last CTA to get here returns them to zero for the next launch, so no
    // memset precedes a launch.
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(done, 1u) == nctas - 1u) {
            for (int i = 0; i < 1 + kPartSlots; ++i) atomicExch(sync + i, 0u);
            atomicExch(done, 0u);
            __threadfence();
        }
    }
}

int wave_sm_count() { return std::min(device_sm_count(), kMaxCtas); }

}  // namespace

bool score_wave_eligible(const tsa_dims &dm, int qe) {
    if (!(dm.dtype == TSA_BF16 && (dm.d == 64 || dm.d == 128) && qe == kQE &&
          dm.H % dm.Hkv == 0 && dm.H / dm.Hkv <= 4 && dm.L >= kQE))
        return false;
    return true;
}

// Every KV group in one wave: one CTA per split of every group, so at most one group
// per SM.
bool score_one_wave_fits(const tsa_dims &dm) { return dm.B * dm.Hkv <= wave_sm_count(); }

// The wave plan.  one_wave: every group in one wave (gpw = B*Hkv, W = 1).  Otherwise gpw
// groups per wave (the largest divisor of B*Hkv with at most ~40 MB of K per wave and,
// when there are two or more groups, at least two waves).  S splits per group,
// gpw * S <= SMs CTAs.
void score_wave_plan(const tsa_dims &dm, bool one_wave, int &gpw, int &S, int &W) {
    const int groups = dm.B * dm.Hkv, sms = wave_sm_count();
    const int ntiles = ceil_div(dm.L, kTile);
    if (one_wave) {
        gpw = groups;
        S = std::max(1, std::min(ntiles, sms / gpw));
        W = 1;
        return;
    }
    const double kg = (double)dm.L * dm.d * 2.0;
    int cap = (int)std::max(1.0, (40.0 * (1 << 20)) / kg);
    cap = std::min(cap, std::max(1, groups / 2));
    cap = std::min(cap, sms);
    if (score_wave_group_cap() > 0) cap = std::min(cap, score_wave_group_cap());
    gpw = 1;
    for (int d = cap; d >= 1; --d)
        if (groups % d == 0) {
            gpw = d;
            break;
        }
    S = std::max(1, std::min(ntiles, sms / gpw));
    W = groups / gpw;
}

template <int D>
static cudaError_t score_wave_impl(const tsa_dims &dm, const void *Q, const void *K,
                                   float scale, float *s_h, float *s_l, const WsLayout &w,
                                   char *ws, cudaStream_t st, uint32_t limit_us,
                                   bool one_wave) {
    CUtensorMap tk;
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)dm.L, (uint64_t)dm.Hkv, (uint64_t)dm.B};
    const uint64_t strides[3] = {(uint64_t)dm.Hkv * D * 2, (uint64_t)D * 2,
                                 (uint64_t)dm.L * dm.Hkv * D * 2};
    const uint32_t box[4] = {64, (uint32_t)kTile, 1, 1};
    if (!make_tmap_bf16_4d(&tk, K, dims, strides, box)) return cudaErrorInvalidValue;
    CUtensorMap tq;  // Q [B, L, H, D]: boxes of 16 tokens x 64 columns of one head
    const uint64_t qdims[4] = {(uint64_t)D, (uint64_t)dm.H, (uint64_t)dm.L, (uint64_t)dm.B};
    const uint64_t qstrides[3] = {(uint64_t)D * 2, (uint64_t)dm.H * D * 2,
                                  (uint64_t)dm.L * dm.H * D * 2};
    const uint32_t qbox[4] = {64, 1, (uint32_t)kQE, 1};
    if (!make_tmap_bf16_4d(&tq, Q, qdims, qstrides, qbox)) return cudaErrorInvalidValue;
    const size_t smem = std::max<size_t>(sizeof(WaveSmem<D>) + 1024, 116 * 1024);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_score_wave<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)))
        return e;
    int gpw, S, W;
    score_wave_plan(dm, one_wave, gpw, S, W);
    float sl2 = scale * 1.4426950408889634f;
    float2 *part = reinterpret_cast<float2 *>(ws + w.score_part);
    Control *ctl = reinterpret_cast<Control *>(ws);
    unsigned int *sync = reinterpret_cast<unsigned int *>(&ctl->pad[0]);
    float *zp = reinterpret_cast<float *>(ws + w.score_part + kScoreWavePartBytes);
    uint64_t lim = (uint64_t)limit_us * 1000ull;
    int stall = test_stall();
    int L = dm.L, H = dm.H, Hkv = dm.Hkv, Bn = dm.B;
    void *args[] = {&tk, &tq, &L, &H, &Hkv, &Bn, &S, &gpw, &W, &sl2, (void *)&part,
                    (void *)&s_h, (void *)&s_l, (void *)&zp, (void *)&sync,
                    (void *)&ctl, &lim, &stall};
    e = cudaLaunchCooperativeKernel((const void *)k_score_wave<D>, dim3(gpw * S),
                                    dim3(kThreads), args, smem, st);
    if (e == cudaSuccess) note_launches(1);
    return e;
}

// Scoring with the wave schedule (one_wave: every group in one wave); s_l may be NULL
// (s_h only).
cudaError_t launch_score_wave(const tsa_dims &dm, const void *Q, const void *K, float scale,
                              float *s_h, float *s_l, const WsLayout &w, char *ws,
                              cudaStream_t st, uint32_t limit_us, bool one_wave) {
    return dm.d == 64
               ? score_wave_impl<64>(dm, Q, K, scale, s_h, s_l, w, ws, st, limit_us, one_wave)
               : score_wave_impl<128>(dm, Q, K, scale, s_h, s_l, w, ws, st, limit_us, one_wave);
}

}  // namespace tsa

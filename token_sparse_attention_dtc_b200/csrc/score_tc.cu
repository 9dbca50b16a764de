// Dynamic Token Coverage scoring on the tensor cores (bf16 inputs), exact two-pass softmax
// in one cooperative kernel.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 2 (the last q queries
// score all keys with a per-head softmax; column sums give s_h); bxzpzcl.cn post §2.1;
// gist.science §2 "Scoring".  For KV group kv the N = G*qe recent-query rows of its G
// heads (row n = g*qe + i -> head kv*G+g, position L-qe+i) are scored against 128-token
// K tiles.  All logits are z2 = scale*log2(e)*<q, k> in fp32 (bf16 products, fp32
// accumulation in TMEM).
//
// Each CTA owns a contiguous range of K tiles of one group and walks it twice:
// Pass 1 (ascending): S = Qblk · Ktile^T with the query rows on the TMEM lanes (M = 128
//   query rows, zero-padded; two row blocks when N > 128).  Each epilogue thread keeps a
//   running (max, sum of 2^(z2-max)) of one query row over a quarter of each tile's
//   columns; the quarters are merged in a fixed order and the CTA writes one (max, sum)
//   per row.
// Grid barrier: the epilogue waits until every CTA has written its pass-1 pairs, then
//   merges the pairs of its group in split order into (max, 1/sum) per row.  The
//   producer and MMA warps do not wait: pass-2 MMAs need no statistics.
// Pass 2 (descending, so the first tiles are the ones pass 1 read last and are likely
//   still in L2): S^T = Ktile · Qblk^T with the tokens on the TMEM lanes (N = query rows
//   padded to 16).  Each thread owns one token and adds 2^(z2 - max_n) / sum_n over the
//   rows of the heads of its column group in row order, then stores s_h[b, h, t].
// Layer score (when one launch covers every group): each epilogue warp also sums the s_h
//   values it wrote; after one more grid barrier, Z = those sums of the batch element's
//   CTAs in a fixed order, and each CTA writes s_l = (sum over heads) / Z for its tokens.
// Warp 0 streams K tiles by TMA through a 4-stage ring, warp 1 issues the MMAs into a
// ring of TMEM accumulators (4 of 128 columns, or 2 of 256), warps 4-19 run the epilogue
// (4 TMEM lane quadrants x 4 column groups).  The grid is at most one CTA per SM and is
// launched cooperatively, so every CTA is resident for the grid barrier, whose word resets
// itself (no memset between launches).  All waits are bounded.
#include <math.h>

#include <algorithm>
#include <atomic>

#include "sm100.cuh"

namespace tsa {
using namespace sm100;

// The wave-scheduled kernel (score_wave.cu) takes the shapes it covers.
bool score_wave_eligible(const tsa_dims &dm, int qe);
bool score_one_wave_fits(const tsa_dims &dm);
cudaError_t launch_score_wave(const tsa_dims &dm, const void *Q, const void *K, float scale,
                              float *s_h, float *s_l, const WsLayout &w, char *ws,
                              cudaStream_t st, uint32_t limit_us, bool one_wave);

// From this many bytes of K on (1.5 x the L2 size), the automatic schedule scores every
// KV group in one wave of the wave-scheduled kernel (tokens on the TMEM lanes in both
// passes); with less K, pass 2 rereads most of K from L2 and the single-wave kernel here is
// as fast or faster.
constexpr double kOneWaveMinKBytes = 192.0 * (1 << 20);

namespace {

constexpr int kThreads = 640, kStages = 4, kTile = 128;
constexpr int kEpiWarps = 16;  // warps 4..19: 4 TMEM lane quadrants x 4 column groups
constexpr uint64_t kDrainNs = 1000000000ull;

template <int D> struct ScoreSmem {
    static constexpr int KT = kTile * D * 2;  // bytes of one K tile
    alignas(1024) uint8_t q[2 * 128 * D * 2];  // up to 256 query rows, swizzled, K-major
    alignas(1024) uint8_t k[kStages][KT];
    uint64_t k_full[kStages], k_empty[kStages], acc_full[4], acc_empty[4], drain;
    uint64_t stall;     // test hook: initialised, never completed
    alignas(16) float mlog[256];  // pass 2: max + log2(sum) per query row (log2 units)
    float2 red[4][256]; // pass 1: per column group (max, sum) per query row
    float wsum[16];     // layer score: per epilogue warp partial sums
    uint32_t tmem_base;
    int abort, never, gbar_ok;
};

// Copy the N recent-query rows of group (b, kv) into shared memory in the 128-byte swizzled
// K-major layout the MMA descriptors expect; rows N..nrows-1 are zero.
template <int D>
__device__ inline void load_q_block(uint8_t *qs, const __nv_bfloat16 *__restrict__ Q, int b,
                                    int kv, int L, int H, int G, int qe, int N, int nrows) {
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    const int block_bytes = nrows * 128;
    for (int e = threadIdx.x; e < nrows * CPR; e += kThreads) {
        const int n = e / CPR, ch = e % CPR;
        const int db = ch / 8, c8 = ch % 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < N) {
            const int g = n / qe, i = n % qe;
            const size_t off = (((size_t)b * L + (L - qe + i)) * H + kv * G + g) * D + ch * 8;
            v = *reinterpret_cast<const uint4 *>(Q + off);
        }
        *reinterpret_cast<uint4 *>(qs + db * block_bytes + n * 128 + ((c8 ^ (n & 7)) * 16)) = v;
    }
}

// Tile range [first, first + count) of this CTA among the group's ntiles tiles.
__device__ inline void tile_range(int ntiles, int nsplit, int split, int &first, int &count) {
    const int per = ntiles / nsplit, rem = ntiles % nsplit;
    first = split * per + min(split, rem);
    count = per + (split < rem ? 1 : 0);
}

__device__ inline void online_merge(float &m, float &l, float m2, float l2) {
    const float mx = fmaxf(m, m2);
    const float a = (m == -INFINITY) ? 0.0f : l * ex2(m - mx);
    const float c = (m2 == -INFINITY) ? 0.0f : l2 * ex2(m2 - mx);
    m = mx;
    l = a + c;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_score_tc(const __grid_constant__ CUtensorMap tmK, const __nv_bfloat16 *__restrict__ Q, int L,
           int H, int Hkv, int qe, float sl2, int nsplit, int group0, float2 *part,
           float *__restrict__ s_h, float *__restrict__ s_l, float *__restrict__ norm_part,
           unsigned int *gbar, Control *ctl, uint64_t limit_ns, int stall) {
    // The kernel after this one in a layer (budget and selection) may start launching; it
    // waits for this grid to complete before it reads the scores.
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    ScoreSmem<D> &sm = *reinterpret_cast<ScoreSmem<D> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int KT = ScoreSmem<D>::KT, NDB = D / 64;
    const int split = blockIdx.x, bg = group0 + blockIdx.y;
    const int b = bg / Hkv, kv = bg % Hkv, G = H / Hkv, N = G * qe;
    const int RB = (N + 127) / 128;   // pass 1 row blocks
    // TMEM accumulator ring: 4 buffers of 128 columns when one row block (and <= 128
    // query columns in pass 2) suffices, else 2 of 256; the MMA runs nbuf - 1 tiles ahead.
    const int lgb = RB == 1 ? 2 : 1, nbuf = 1 << lgb;
    const uint32_t bstride = 512u >> lgb;
    const int Npad = (N + 15) & ~15;  // pass 2 MMA N
    const int nrows = RB * 128;       // query rows held in shared memory
    const int ntiles = (L + kTile - 1) / kTile;
    int first, count;
    tile_range(ntiles, nsplit, split, first, count);
    const int total = 2 * count;  // iterations over both passes
    const unsigned nctas = gridDim.x * gridDim.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int a = 0; a < 4; ++a) {
            mbar_init(&sm.acc_full[a], 1);
            mbar_init(&sm.acc_empty[a], kEpiWarps * 32);
        }
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.stall, 1);
        sm.abort = 0;
        sm.never = 0;
        sm.gbar_ok = 0;
        fence_mbar_init();
    }
    load_q_block<D>(sm.q, Q, b, kv, L, H, G, qe, N, nrows);
    fence_proxy_async_smem();  // make the generic-proxy Q writes visible to the MMA
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
    // Tile of iteration it: pass 1 ascending, pass 2 descending within the CTA's range.
    auto tile_at = [&](int it) { return it < count ? first + it : first + total - 1 - it; };

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < total; ++it) {
                const int s = it % kStages;
                if (!(ok = mbar_wait(&sm.k_empty[s], ((it / kStages) & 1) ^ 1, limit_ns, abort)))
                    break;
                mbar_expect_tx(&sm.k_full[s], KT);
#pragma unroll
                for (int db = 0; db < NDB; ++db)
                    tma_load_4d(sm.k[s] + db * kTile * 128, &tmK, &sm.k_full[s], db * 64,
                                tile_at(it) * kTile, kv, b);
                issued = it + 1;
            }
            for (int it = (issued > kStages ? issued - kStages : 0); it < issued; ++it)
                mbar_wait(&sm.k_full[it % kStages], (it / kStages) & 1, kDrainNs, &sm.never);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t qa = smem_u32(sm.q);
            const uint32_t id1 = idesc_bf16(128, kTile, false);
            const uint32_t id2 = idesc_bf16(128, Npad, false);
            bool any = false;
            // Test hook: a wait that nothing completes, so it runs out after limit_ns.
            if (stall) ok = mbar_wait(&sm.stall, 0, limit_ns, abort);
            for (int it = 0; it < total && ok; ++it) {
                const int s = it % kStages, a = it & (nbuf - 1);
                if (!(ok = mbar_wait(&sm.k_full[s], (it / kStages) & 1, limit_ns, abort))) break;
                if (!(ok = mbar_wait(&sm.acc_empty[a], ((it >> lgb) & 1) ^ 1, limit_ns, abort)))
                    break;
                tc_fence_after();
                const uint32_t ka = smem_u32(sm.k[s]);
                const uint32_t dacc = tmem + a * bstride;
                if (it < count) {
                    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t kof = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
                            const uint32_t qof =
                                (kk / 4) * (nrows * 128) + rb * 128 * 128 + (kk % 4) * 32;
                            mma_ss(dacc + rb * 128, sdesc_sw128(qa + qof, 16, 1024),
                                   sdesc_sw128(ka + kof, 16, 1024), id1, kk > 0 ? 1u : 0u);
                        }
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t kof = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
                        const uint32_t qof = (kk / 4) * (nrows * 128) + (kk % 4) * 32;
                        mma_ss(dacc, sdesc_sw128(ka + kof, 16, 1024),
                               sdesc_sw128(qa + qof, 16, 1024), id2, kk > 0 ? 1u : 0u);
                    }
                }
                any = true;
                mma_commit(&sm.k_empty[s]);
                mma_commit(&sm.acc_full[a]);
            }
            if (any) {
                mma_commit(&sm.drain);
                mbar_wait(&sm.drain, 0, kDrainNs, &sm.never);
            }
        }
    } else if (warp >= 4) {
        // Epilogue warp (wq, cg): TMEM lane quadrant wq = warp % 4 (the lanes this warp may
        // read), column group cg = (warp - 4) / 4.
        const int wq = warp & 3, cg = (warp - 4) >> 2, r = wq * 32 + lane;
        const uint32_t lo = (uint32_t)(wq * 32) << 16;
        const int pmin = L - qe;           // first recent-query position
        const int et = threadIdx.x - 128;  // 0..511 among the epilogue threads
        // ---- pass 1: thread owns query row r (+128) over tile columns [cg*32, cg*32+32)
        {
            float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
            int pr[2];
            for (int rb = 0; rb < 2; ++rb) {
                const int n = rb * 128 + r;
                pr[rb] = n < N ? L - qe + (n % qe) : -1;  // -1: padding row, never valid
            }
            for (int it = 0; it < count; ++it) {
                const int a = it & (nbuf - 1);
                ok = mbar_wait(&sm.acc_full[a], (it >> lgb) & 1, limit_ns, abort);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                const int tc0 = tile_at(it) * kTile + cg * 32;  // token of column 0 here
                const bool tail = tc0 + 31 > pmin;  // some token may follow a query
                for (int rb = 0; rb < RB; ++rb) {
                    if (rb * 128 + wq * 32 >= N) continue;  // whole warp on padding rows
                    uint32_t v[32];
                    tmem_ld32(tmem + a * bstride + rb * 128 + cg * 32 + lo, v);
                    tmem_ld_wait();
                    if (pr[rb] < 0) continue;
                    float cm;
                    if (!tail) {  // every token here precedes every recent query
                        float c0 = __uint_as_float(v[0]), c1 = __uint_as_float(v[1]);
#pragma unroll
                        for (int e = 2; e < 30; e += 4) {
                            c0 = fmax3(c0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                            c1 = fmax3(c1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                        }
                        cm = fmax3(c0, c1, fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31])));
                    } else {
                        cm = -INFINITY;
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            float z = __uint_as_float(v[e]);
                            if (tc0 + e > pr[rb]) z = -INFINITY;
                            v[e] = __float_as_uint(z);
                            cm = fmaxf(cm, z);
                        }
                        if (cm == -INFINITY) continue;
                    }
                    cm *= sl2;
                    if (cm > m[rb]) {
                        l[rb] = (m[rb] == -INFINITY) ? 0.0f : l[rb] * ex2(m[rb] - cm);
                        m[rb] = cm;
                    }
                    const float nm = -m[rb];
                    float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {  // paired fp32: two columns per FMA / add
                        float x0, x1, x2, x3;
                        fma2(x0, x1, __uint_as_float(v[e]), __uint_as_float(v[e + 1]), sl2, sl2,
                             nm, nm);
                        fma2(x2, x3, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]), sl2,
                             sl2, nm, nm);
                        add2(a0, a1, a0, a1, ex2(x0), ex2(x1));
                        add2(b0, b1, b0, b1, ex2(x2), ex2(x3));
                    }
                    l[rb] += (a0 + a1) + (b0 + b1);
                }
                tc_fence_before();
                mbar_arrive(&sm.acc_empty[a]);
            }
            for (int rb = 0; rb < RB; ++rb) sm.red[cg][rb * 128 + r] = make_float2(m[rb], l[rb]);
        }
        named_barrier(1, kEpiWarps * 32);
        ok = __all_sync(0xffffffffu, ok) && !*abort;
        if (ok && cg == 0)
            for (int rb = 0; rb < RB; ++rb) {
                const int n = rb * 128 + r;
                if (n >= N) continue;
                float mm = -INFINITY, ll = 0.0f;
                for (int g2 = 0; g2 < 4; ++g2)  // fixed merge order
                    online_merge(mm, ll, sm.red[g2][n].x, sm.red[g2][n].y);
                __stcg(&part[((size_t)bg * nsplit + split) * N + n], make_float2(mm, ll));
            }
        // Grid barrier among the epilogue warps of every CTA, on a word that returns to its
        // initial state by itself (no reset between launches): CTA 0 adds
        // 2^31 - (nctas - 1), every other CTA adds 1, so bit 31 flips exactly when the
        // last CTA arrives and the low 31 bits are back at zero.  A CTA waits until bit 31
        // differs from the value its own add returned.  Every epilogue thread must call it
        // (named barriers inside); it returns false when the wait ran out or the CTA
        // aborted.  A launch that fails part-way can leave the word off its initial state:
        // its error word is set, and reading the error (tsa_get_device_status) resets
        // the control block.
        const unsigned bar_add =
            (blockIdx.x == 0 && blockIdx.y == 0) ? 0x80000000u - (nctas - 1u) : 1u;
        auto grid_sync = [&]() -> bool {
            __threadfence();
            named_barrier(1, kEpiWarps * 32);
            if (et == 0) {
                int good = 0;
                if (!*abort) {
                    const unsigned old = atomicAdd(gbar, bar_add);
                    const uint64_t t0 = globaltimer_ns();
                    for (uint32_t k = 0;; ++k) {
                        unsigned v;
                        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(gbar) : "memory");
                        if ((v ^ old) & 0x80000000u) { good = 1; break; }
                        if ((k & 63) == 63 && (*abort || globaltimer_ns() - t0 > limit_ns)) break;
                        __nanosleep(64);
                    }
                }
                sm.gbar_ok = good;
            }
            named_barrier(1, kEpiWarps * 32);
            return sm.gbar_ok != 0;
        };
        // ---- grid barrier: every CTA's pass-1 pairs are in global memory
        {
            const bool g1 = grid_sync();
            ok = ok && g1;
        }
        // ---- merge the pass-1 pairs of this group in split order: (max, 1/sum) per row
        if (ok && et < N) {
            float mm = -INFINITY, ll = 0.0f;
            for (int s = 0; s < nsplit; ++s) {
                const float2 p = __ldcg(&part[((size_t)bg * nsplit + s) * N + et]);
                online_merge(mm, ll, p.x, p.y);
            }
            sm.mlog[et] = mm + log2f(ll);  // exp2(z - m) / l = exp2(z - (m + log2 l))
        }
        named_barrier(1, kEpiWarps * 32);
        // ---- pass 2: thread owns token r of the tile and the heads g = cg, cg + 4, ...;
        // head g's query rows are the columns [g*qe, (g+1)*qe), summed in row order.
        // zs: this thread's sum of the s_h values it writes (for the layer score's total).
        float zs = 0.0f;
        for (int it = count; it < total && ok; ++it) {
            const int a = it & (nbuf - 1);
            ok = mbar_wait(&sm.acc_full[a], (it >> lgb) & 1, limit_ns, abort);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const int t = tile_at(it) * kTile + r;
            const bool early = tile_at(it) * kTile + kTile - 1 <= pmin;  // no query follows
            for (int g = cg; g < G; g += 4) {
                const int c0 = g * qe, c1 = c0 + qe;
                float acc = 0.0f, a0 = 0.0f, a1 = 0.0f;
                for (int cs = c0 & ~15; cs < c1; cs += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem + a * bstride + cs + lo, v);
                    tmem_ld_wait();
                    if (early && cs >= c0 && cs + 16 <= c1) {  // all 16 columns count
                        const float4 *ml = reinterpret_cast<const float4 *>(sm.mlog + cs);
#pragma unroll
                        for (int e = 0; e < 16; e += 4) {
                            const float4 mq = ml[e / 4];
                            float x0, x1, x2, x3;
                            fma2(x0, x1, __uint_as_float(v[e]), __uint_as_float(v[e + 1]), sl2,
                                 sl2, -mq.x, -mq.y);
                            fma2(x2, x3, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]), sl2,
                                 sl2, -mq.z, -mq.w);
                            add2(a0, a1, a0, a1, ex2(x0), ex2(x1));
                            add2(a0, a1, a0, a1, ex2(x2), ex2(x3));
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int n = cs + e;
                            if (n < c0 || n >= c1) continue;
                            if (t <= pmin + (n - c0))
                                acc += ex2(fmaf(__uint_as_float(v[e]), sl2, -sm.mlog[n]));
                        }
                    }
                }
                acc += a0 + a1;
                if (t < L) {
                    s_h[((size_t)b * H + kv * G + g) * L + t] = acc;
                    zs += acc;
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.acc_empty[a]);
        }
        if (s_l) {
            // ---- layer score in the same launch (it covers every KV group of every batch
            // element): each epilogue warp stores the sum of the s_h values it wrote; after
            // one grid barrier, Z_b = those totals of batch element b's CTAs summed in a
            // fixed order, and s_l[t] = (sum_h s_h[h, t] in head order) / Z_b over this
            // CTA's token range.
            const int cta = blockIdx.y * gridDim.x + blockIdx.x, Bn = gridDim.y / Hkv;
            const int ew = warp - 4;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
            if (lane == 0) __stcg(norm_part + (size_t)cta * kEpiWarps + ew, zs);
            const bool g2 = grid_sync();  // every s_h row and warp total is stored
            ok = ok && g2;
            const int cl = ceil_div(L, (int)nctas);
            const int t0 = min(L, cta * cl), t1 = min(L, t0 + cl);
            const int per_b = (int)gridDim.x * Hkv * kEpiWarps;  // totals of one batch element
            for (int bb = 0; bb < Bn; ++bb) {
                float z = 0.0f;
                if (ok)
                    for (int e = et; e < per_b; e += kEpiWarps * 32)
                        z += __ldcg(norm_part + (size_t)bb * per_b + e);
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
        report_error(ctl, TSA_ERR_DEVICE_TIMEOUT, 200 + warp);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

// SM count of the current device, cached per device (the cooperative grid is sized from
// it, so it must be the count of the device the launch goes to).
int device_sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    if (dev < 0 || dev >= 64) {
        int n = 0;
        return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
                       n > 0 ? n : 148;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

namespace {

int sm_count() { return device_sm_count(); }

}  // namespace

// Splits per KV group of the tensor-core scoring: about one CTA per SM in total (one
// cooperative launch covers at most sm_count() groups).
int score_tc_splits(const tsa_dims &dm) {
    const int ntiles = ceil_div(dm.L, kTile);
    const int groups = std::min(dm.B * dm.Hkv, sm_count());
    const int n = std::max(1, std::min(ntiles, sm_count() / groups));
    return std::min(n, score_split_cap(dm));  // never more than the workspace holds
}

template <int D>
static cudaError_t score_tc_impl(const tsa_dims &dm, const void *Q, const void *K, int qe,
                                 float scale, float *s_h, float *s_l, const WsLayout &w, char *ws,
                                 cudaStream_t st, uint32_t limit_us, bool &fused) {
    CUtensorMap tk;
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)dm.L, (uint64_t)dm.Hkv, (uint64_t)dm.B};
    const uint64_t strides[3] = {(uint64_t)dm.Hkv * D * 2, (uint64_t)D * 2,
                                 (uint64_t)dm.L * dm.Hkv * D * 2};
    const uint32_t box[4] = {64, (uint32_t)kTile, 1, 1};
    if (!make_tmap_bf16_4d(&tk, K, dims, strides, box)) return cudaErrorInvalidValue;
    // At least 116 KB so that one CTA holds an SM (and all 512 TMEM columns) at a time.
    const size_t smem = std::max<size_t>(sizeof(ScoreSmem<D>) + 1024, 116 * 1024);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_score_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)))
        return e;
    int nsplit = score_tc_splits(dm);
    float sl2 = scale * 1.4426950408889634f;
    float2 *part = reinterpret_cast<float2 *>(ws + w.score_part);
    Control *ctl = reinterpret_cast<Control *>(ws);
    // pad[0..4] belong to the wave-scheduled kernel, which resets them before each launch.
    unsigned int *gbar = reinterpret_cast<unsigned int *>(&ctl->pad[16]);
    uint64_t lim = (uint64_t)limit_us * 1000ull;
    int stall = test_stall();
    const __nv_bfloat16 *Qb = (const __nv_bfloat16 *)Q;
    int L = dm.L, H = dm.H, Hkv = dm.Hkv;
    const int groups = dm.B * dm.Hkv, per_launch = std::min(groups, sm_count());
    // One launch covering every group also computes the layer score.
    fused = per_launch == groups && s_l != nullptr;
    float *sl = fused ? s_l : nullptr;
    float *np = reinterpret_cast<float *>(ws + w.norm_part);
    for (int g0 = 0; g0 < groups; g0 += per_launch) {
        int group0 = g0;
        const int gc = std::min(per_launch, groups - g0);
        void *args[] = {&tk, (void *)&Qb, &L, &H, &Hkv, &qe, &sl2, &nsplit, &group0,
                        (void *)&part, (void *)&s_h, (void *)&sl, (void *)&np, (void *)&gbar,
                        (void *)&ctl, &lim, &stall};
        e = cudaLaunchCooperativeKernel((const void *)k_score_tc<D>, dim3(nsplit, gc),
                                        dim3(kThreads), args, smem, st);
        if (e != cudaSuccess) return e;
        note_launches(1);
    }
    return cudaSuccess;
}

// s_l may be NULL (no layer score); `fused` tells the caller whether s_l was written.
cudaError_t launch_score_tc(const tsa_dims &dm, const void *Q, const void *K, int qe,
                            float scale, float *s_h, float *s_l, const WsLayout &w, char *ws,
                            cudaStream_t st, uint32_t limit_us, bool &fused) {
    const int mode = score_schedule();
    if (score_wave_eligible(dm, qe)) {
        const double kbytes = 2.0 * dm.B * dm.L * dm.Hkv * dm.d;
        const bool one = mode == 0 && kbytes >= kOneWaveMinKBytes && score_one_wave_fits(dm);
        if (mode == 1 || one) {
            fused = s_l != nullptr;
            return launch_score_wave(dm, Q, K, scale, s_h, s_l, w, ws, st, limit_us, one);
        }
    }
    return dm.d == 64
               ? score_tc_impl<64>(dm, Q, K, qe, scale, s_h, s_l, w, ws, st, limit_us, fused)
               : score_tc_impl<128>(dm, Q, K, qe, scale, s_h, s_l, w, ws, st, limit_us, fused);
}

}  // namespace tsa

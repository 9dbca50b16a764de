// Causal flash attention on the 5th-generation tensor cores (tcgen05 + TMEM), bf16 in,
// fp32 accumulate, for the compressed L'×L' problem of each head and for the dense GQA
// layer.
//
// Method: "Token Sparse Attention" papernotes.org notes, 整体框架 (dense attention on the
// compressed problem, complexity O(L'^2 d)); bxzpzcl.cn post §1.1 (softmax(Q̂K̂ᵀ/√d)V̂).
// The causal mask j <= i in compressed order is the mask on original positions because
// the index lists are ascending.
//
// One CTA per pair of 128-row query tiles (A = 2p, B = 2p+1) of one head; every K/V
// tile is loaded once and used by both.  CTAs run head by head, heaviest pairs first.
// Warp roles (320 threads):
//   warp 0      TMA producer: both Q tiles once, then K and V tiles through a 2-stage ring.
//   warp 1      TMEM owner and MMA issuer.  Order per key tile j:
//                 PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)
//               so that the softmax of one tile overlaps the MMAs of the other.  S = Q K^T
//               goes to the tile's TMEM S buffer; O += P V reads P (bf16, written over S)
//               from TMEM and V from shared memory.
//   warps 2-5   softmax of tile A, warps 6-9 softmax of tile B: thread r owns query row r.
//               Online max/sum in log2 units; O is rescaled only when the running max grows
//               by more than 2^8 (so P <= 2^8); P is written back to TMEM; the epilogue
//               writes O / l as bf16.
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256, 256+d), O_B [384, 384+d).
// Because S_X(j+1) is issued after PV_X(j), its completion also means PV_X(j) is done:
// the softmax may rescale O_X right after S_X(j+1) arrives.
// Every wait is bounded in time; a wait that runs out records TSA_ERR_DEVICE_TIMEOUT,
// the CTA drains its in-flight copies and MMAs, frees TMEM and exits.
#include <math.h>
#include <string.h>

#include <algorithm>

#include "sm100.cuh"

namespace tsa {
using namespace sm100;

namespace {

constexpr int kBM = 128, kBN = 128, kStages = 2, kThreads = 320;
// Direct-gather mode: warps 10 and 11 join warp 0 as copy producers (384 threads).
constexpr int kGatherWarps = 3, kGatherThreads = kThreads + 64;
constexpr uint64_t kDrainNs = 1000000000ull;  // drain waits: 1 s

template <int D> struct AttnSmem {
    static constexpr int TILE = kBM * D * 2;  // bytes of a 128-row tile
    alignas(1024) uint8_t q[2][TILE];
    alignas(1024) uint8_t k[kStages][TILE];
    alignas(1024) uint8_t v[kStages][TILE];
    uint64_t q_full, k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2], o_final[2], drain;
    uint64_t stall;  // test hook: initialised, never completed
    int64_t goff[kGatherWarps][2][kBM];  // direct-gather mode: each producer's row offsets
    uint32_t tmem_base;
    int abort;
    int never;  // stays 0: drain waits ignore the abort flag
};

// Direct-gather mode: rows are read through the index lists from the original tensors,
// and the epilogue writes Y = X + Ô into the kept rows (no compressed copies).
struct GatherArgs {
    const __nv_bfloat16 *Q, *K, *V;  // [B, L, H, d], [B, L, Hkv, d]
    const int32_t *idx;              // [B, H, L]: kept tokens ascending, then the rest
    const __nv_bfloat16 *X;          // [B, L, H*d]
    __nv_bfloat16 *Y;                // [B, L, H*d], may be X
};

// Producer of the direct-gather mode: producer warp pw (0..kGatherWarps-1, all 32 lanes)
// copies its share of every tile.  A 128-row tile of positions p0..p0+127 is copied with
// 16-byte cp.async into the 128-byte-swizzle layout the MMA descriptors read (16-byte
// chunk k of row r at r*128 + ((k ^ (r & 7)) * 16) in each 64-column block), row p taken
// from token idx[p] (p clamped to L - 1; rows past L' are masked or never stored); warp pw
// takes the row groups pw, pw + kGatherWarps, ... of 32/CPR rows.  After issuing its share
// of a tile each lane hands its arrival on the tile's full barrier to the copy engine
// (cp.async.mbarrier.arrive: the arrival lands with the lane's copies; 32 per producer
// warp), so no producer waits for its own copies; the MMA thread fences generic -> async
// proxy after the barrier completes.
template <int D>
__device__ __forceinline__ bool gather_producer(AttnSmem<D> &sm, const GatherArgs &ga, int pw,
                                                int b, int h, int kvh, int L, int H, int Hkv,
                                                int i0, bool hasB, int nkv, int lane, Control *ctl,
                                                uint64_t limit_ns, volatile int *abort) {
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    const int32_t *S = ga.idx + ((size_t)b * H + h) * L;
    bool bad = false;
    // Token indices of rows p0 + 4*lane .. p0 + 4*lane + 3 (clamped to L - 1), loaded in
    // one round trip; staged in shared memory as element offsets of the rows
    // ((b * L + t) * heads + head) * D, so the copy loop has no global dependence and no
    // index arithmetic (K and V share the offsets of a step).
    auto load_idx = [&](int p0, int (&v)[4]) {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = __ldg(S + min(p0 + 4 * lane + e, L - 1));
    };
    auto stage_idx = [&](int slot, const int (&v)[4], int heads, int head) {
        __syncwarp();  // the previous copy loop has read this slot
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int t = v[e];
            if ((unsigned)t >= (unsigned)L) {
                bad = true;
                t = 0;
            }
            sm.goff[pw][slot][4 * lane + e] = (((int64_t)b * L + t) * heads + head) * D;
        }
        __syncwarp();
    };
    auto tile = [&](uint8_t *dst, const __nv_bfloat16 *src, int slot) {
        const uint32_t d0 = smem_u32(dst);
        const int c = lane % CPR;
        const uint32_t coff = (uint32_t)(c / 8) * (kBM * 128);
        const __nv_bfloat16 *base = src + c * 8;
        constexpr int RPI = 32 / CPR;  // rows per warp iteration
#pragma unroll 4
        for (int r = pw * RPI + lane / CPR; r < kBM; r += kGatherWarps * RPI)
            cp_async16(d0 + coff + r * 128 + (((c % 8) ^ (r & 7)) << 4), base + sm.goff[pw][slot][r]);
    };

    int va[4], vb[4];
    load_idx(i0, va);
    if (hasB) load_idx(i0 + kBM, vb);
    stage_idx(0, va, H, h);
    tile(sm.q[0], ga.Q, 0);
    if (hasB) {
        stage_idx(1, vb, H, h);
        tile(sm.q[1], ga.Q, 1);
    }
    cp_async_mbar_arrive(&sm.q_full);
    int nxt[4];
    if (nkv > 0) load_idx(0, nxt);
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
        const int s = j % kStages, slot = j & 1;
        const uint32_t ph = ((j / kStages) & 1) ^ 1;
        stage_idx(slot, nxt, Hkv, kvh);
        if (j + 1 < nkv) load_idx((j + 1) * kBN, nxt);  // in flight during this step's copies
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.k_empty[s], ph, limit_ns, abort));
        if (!ok) break;
        tile(sm.k[s], ga.K, slot);
        cp_async_mbar_arrive(&sm.k_full[s]);
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.v_empty[s], ph, limit_ns, abort));
        if (!ok) break;
        tile(sm.v[s], ga.V, slot);
        cp_async_mbar_arrive(&sm.v_full[s]);
    }
    // Drain: every copy of this lane lands before the CTA can exit.
    cp_async_wait_all();
    if (__any_sync(0xffffffffu, bad) && lane == 0) report_error(ctl, TSA_ERR_INVALID_ARG, 31);
    return ok;
}

// P = 2^(S*sl2 - mu) of one row, packed to bf16x2 over sr[0..63]; returns the row sum of
// the fp32 values.  Paired fp32 instructions for the scale-subtract and the sums.
// kDiag: the diagonal tile, whose masked entries are -inf and give exactly 0.  (The two
// instantiations compile to the same arithmetic; keeping the diagonal step separate lets
// the register allocator treat the common step on its own.)
template <bool kDiag>
__device__ __forceinline__ float exp_pack_row(uint32_t (&sr)[128], float sl2, float mu) {
    const float nmu = -mu;
    float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
#pragma unroll
    for (int c = 0; c < 64; c += 2) {  // columns 2c .. 2c+3 (pairs c and c+1)
        float x0, x1, x2, x3, p0, p1, p2, p3;
        fma2(x0, x1, __uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]), sl2, sl2, nmu,
             nmu);
        fma2(x2, x3, __uint_as_float(sr[2 * c + 2]), __uint_as_float(sr[2 * c + 3]), sl2, sl2,
             nmu, nmu);
        p0 = ex2(x0);
        p1 = ex2(x1);
        p2 = ex2(x2);
        p3 = ex2(x3);
        add2(a0, a1, a0, a1, p0, p1);
        add2(b0, b1, b0, b1, p2, p3);
        sr[c] = pack_bf16(p0, p1);  // in place: sr[c] and sr[c+1] were already read
        sr[c + 1] = pack_bf16(p2, p3);
    }
    return (a0 + a1) + (b0 + b1);
}

// Softmax of one query tile (this warpgroup), steps j = 0..n-1; the last step is the
// diagonal key tile.  Returns false if a wait ran out.
template <int D>
__device__ __forceinline__ bool softmax_tile(AttnSmem<D> &sm, int X, int n, uint32_t tS,
                                             uint32_t tO, int r, uint32_t lo, float sl2,
                                             uint64_t limit_ns, volatile int *abort, float &l_out) {
    float m = -INFINITY, l = 0.0f;
    for (int j = 0; j < n; ++j) {
        bool ok = mbar_wait(&sm.s_full[X], j & 1, limit_ns, abort);
        if (!__all_sync(0xffffffffu, ok)) return false;
        tc_fence_after();
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
            tmem_ld32(tS + lo + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_ld_wait();
        if (j == n - 1) {  // diagonal tile: key c is visible to row r iff c <= r
#pragma unroll
            for (int c = 0; c < 128; ++c)
                if (c > r) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
#pragma unroll
        for (int c = 2; c < 126; c += 4) {
            mx0 = fmax3(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
            mx1 = fmax3(mx1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
        }
        const float mt =
            fmax3(mx0, mx1, fmaxf(__uint_as_float(sr[126]), __uint_as_float(sr[127]))) * sl2;
        float mu = m, factor = 1.0f;
        bool resc = false;
        if (m == -INFINITY) {
            mu = mt;
            factor = 0.0f;
        } else if (mt > m + 8.0f) {
            mu = mt;
            factor = ex2(m - mt);
            resc = true;
        }
        m = mu;
        l = l * factor +
            (j == n - 1 ? exp_pack_row<true>(sr, sl2, mu) : exp_pack_row<false>(sr, sl2, mu));
        if (__any_sync(0xffffffffu, resc)) {
            // S_X(j) was issued after PV_X(j-1), so O_X is complete here.
            const float f = resc ? factor : 1.0f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + lo + c * 32, o);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                tmem_st32(tO + lo + c * 32, o);
            }
        }
        tmem_st32(tS + lo, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_st32(tS + lo + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();  // every lane's P is in TMEM: one arrival per warp
        if ((r & 31) == 0) mbar_arrive(&sm.p_full[X]);
    }
    l_out = l;
    return true;
}

template <int D, bool kGather>
__global__ void __launch_bounds__(kGather ? kGatherThreads : kThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ Lkeep, int dense,
          int L, int H, int Hkv, float sl2, __nv_bfloat16 *__restrict__ O, GatherArgs ga,
          const uint32_t *__restrict__ bmask, int hgroup, Control *ctl, uint64_t limit_ns,
          int stall) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<D> &sm = *reinterpret_cast<AttnSmem<D> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int TILE = AttnSmem<D>::TILE, NDB = D / 64;
    // CTA order: groups of `hgroup` heads whose K/V fit in L2 together, one group after
    // the other; inside a group the heaviest pairs of all its heads come first.  The CTAs in
    // flight share their heads' K/V tiles in L2, and the light pairs fill the tail.
    pdl_wait();  // Q, K, V and the kept counts are the previous kernels'
    pdl_trigger();
    const int npairs = ceil_div(L, 2 * kBM), B_H = gridDim.x / npairs;
    const int grp = blockIdx.x / (hgroup * npairs), r = blockIdx.x % (hgroup * npairs);
    const int ghead = min(hgroup, B_H - grp * hgroup);  // heads in this group
    const int bh = grp * hgroup + r % ghead, pair = npairs - 1 - r / ghead;
    const int b = bh / H, h = bh % H;
    // A kept count outside [0, L] is clamped (and reported): rows past L are never
    // read or written.
    const int lk_in = dense ? L : __ldg(Lkeep + b);
    const int Lk = min(max(lk_in, 0), L);
    if (lk_in != Lk && pair == 0 && threadIdx.x == 0) report_error(ctl, TSA_ERR_INVALID_ARG, 30);
    const int i0 = pair * 2 * kBM;  // first row of tile A
    if (i0 >= Lk) return;
    const bool hasB = i0 + kBM < Lk;
    // Key blocks of this pair: all of 0..2p+1, or the kept ones of the block-sparse mask
    // (ascending; block 0 and the diagonal blocks 2p, 2p+1 are always kept).
    const int NW = ceil_div(ceil_div(L, kBN), 32);
    const uint32_t *bm = bmask ? bmask + ((size_t)bh * npairs + pair) * NW : nullptr;
    int nA = 2 * pair + 1, nB = hasB ? 2 * pair + 2 : 0;
    if (bm) {
        int below = 0, all = 0;  // kept blocks <= 2p, and in total
        for (int w = 0; w < NW; ++w) {
            const uint32_t word = __ldg(bm + w);
            all += __popc(word);
            const int lo = 2 * pair + 1 - 32 * w;  // bits [0, lo) of this word are <= 2p
            below += __popc(lo >= 32 ? word : (lo > 0 ? word & ((1u << lo) - 1u) : 0u));
        }
        nA = below;
        nB = hasB ? all : 0;
    }
    const int nkv = hasB ? nB : nA;
    const int kvh = (dense || kGather) ? h / (H / Hkv) : h;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        const uint32_t nfill = kGather ? 32 * kGatherWarps : 1;  // cp.async lanes, or one TMA thread
        mbar_init(&sm.q_full, nfill);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], nfill);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], nfill);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sm.s_full[x], 1);
            mbar_init(&sm.p_full[x], 4);  // the 4 warps of the softmax warpgroup
            mbar_init(&sm.o_final[x], 1);
        }
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.stall, 1);
        sm.abort = 0;
        sm.never = 0;
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
    if (kGather && (warp == 0 || warp >= 10)) {
        ok = gather_producer<D>(sm, ga, warp == 0 ? 0 : warp - 9, b, h, kvh, L, H, Hkv, i0, hasB,
                                nkv, lane, ctl, limit_ns, abort);
    } else if (warp == 0) {
        if (lane == 0) {
            int issued = 0;  // K/V tiles issued (negative: K of tile -issued-1 only)
            int cw = 0;      // block-sparse: current mask word and its unvisited bits
            uint32_t cur = bm ? __ldg(bm) : 0u;
            auto next_block = [&](int j) -> int {
                if (!bm) return j;
                while (cur == 0u) cur = __ldg(bm + (++cw));
                const int e = __ffs(cur) - 1;
                cur &= cur - 1u;
                return cw * 32 + e;
            };
            mbar_expect_tx(&sm.q_full, 2 * TILE);
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int db = 0; db < NDB; ++db)
                    tma_load_4d(sm.q[x] + db * kBM * 128, &tmQ, &sm.q_full, db * 64,
                                i0 + x * kBM, h, b);
            for (int j = 0; j < nkv; ++j) {
                const int s = j % kStages;
                const uint32_t ph = ((j / kStages) & 1) ^ 1;
                const int kb = next_block(j);  // key block of step j
                if (!(ok = mbar_wait(&sm.k_empty[s], ph, limit_ns, abort))) break;
                mbar_expect_tx(&sm.k_full[s], TILE);
#pragma unroll
                for (int db = 0; db < NDB; ++db)
                    tma_load_4d(sm.k[s] + db * kBN * 128, &tmK, &sm.k_full[s], db * 64, kb * kBN,
                                kvh, b);
                if (!(ok = mbar_wait(&sm.v_empty[s], ph, limit_ns, abort))) {
                    issued = -(j + 1);
                    break;
                }
                mbar_expect_tx(&sm.v_full[s], TILE);
#pragma unroll
                for (int db = 0; db < NDB; ++db)
                    tma_load_4d(sm.v[s] + db * kBN * 128, &tmV, &sm.v_full[s], db * 64, kb * kBN,
                                kvh, b);
                issued = j + 1;
            }
            // Drain: wait (bounded) for every copy this thread started to land.
            mbar_wait(&sm.q_full, 0, kDrainNs, &sm.never);
            const int nk = issued >= 0 ? issued : -issued, nv = issued >= 0 ? issued : -issued - 1;
            for (int j = (nk > kStages ? nk - kStages : 0); j < nk; ++j)
                mbar_wait(&sm.k_full[j % kStages], (j / kStages) & 1, kDrainNs, &sm.never);
            for (int j = (nv > kStages ? nv - kStages : 0); j < nv; ++j)
                mbar_wait(&sm.v_full[j % kStages], (j / kStages) & 1, kDrainNs, &sm.never);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(kBM, kBN, false);
            constexpr uint32_t idO = idesc_bf16(kBM, D, true);
            bool any = false;
            auto S_mma = [&](int x, int j) {
                const uint32_t qa = smem_u32(sm.q[x]), ka = smem_u32(sm.k[j % kStages]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * (kBM * 128) + (kk % 4) * 32;
                    mma_ss(tmem + x * 128, sdesc_sw128(qa + off, 16, 1024),
                           sdesc_sw128(ka + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.s_full[x]);
                any = true;
            };
            auto PV_mma = [&](int x, int j) {
                const uint32_t va = smem_u32(sm.v[j % kStages]);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8,
                           sdesc_sw128(va + kk * 2048, kBN * 128, 1024), idO,
                           (j > 0 || kk > 0) ? 1u : 0u);
            };
            // Test hook: a wait that nothing completes, so it runs out after limit_ns.
            if (stall) ok = mbar_wait(&sm.stall, 0, limit_ns, abort);
            ok = ok && mbar_wait(&sm.q_full, 0, limit_ns, abort) &&
                 mbar_wait(&sm.k_full[0], 0, limit_ns, abort);
            if (ok) {
                if (kGather) fence_proxy_async_smem();  // cp.async writes -> the MMA's reads
                tc_fence_after();
                S_mma(0, 0);
                if (hasB) S_mma(1, 0);
                mma_commit(&sm.k_empty[0]);
            }
            for (int j = 0; j < nkv && ok; ++j) {
                const bool next = j + 1 < nkv;
                if (!(ok = mbar_wait(&sm.v_full[j % kStages], (j / kStages) & 1, limit_ns, abort)))
                    break;
                if (next && !(ok = mbar_wait(&sm.k_full[(j + 1) % kStages],
                                             ((j + 1) / kStages) & 1, limit_ns, abort)))
                    break;
                if (kGather) fence_proxy_async_smem();  // cp.async writes -> the MMA's reads
                for (int x = 0; x < 2; ++x) {
                    const int nx = x ? nB : nA;
                    if (j >= nx) continue;
                    if (!(ok = mbar_wait(&sm.p_full[x], j & 1, limit_ns, abort))) break;
                    tc_fence_after();
                    PV_mma(x, j);
                    if (j == nx - 1) mma_commit(&sm.o_final[x]);
                    else S_mma(x, j + 1);
                }
                if (!ok) break;
                mma_commit(&sm.v_empty[j % kStages]);
                if (next) mma_commit(&sm.k_empty[(j + 1) % kStages]);
            }
            if (any) {  // every MMA issued here has completed before TMEM is freed
                mma_commit(&sm.drain);
                mbar_wait(&sm.drain, 0, kDrainNs, &sm.never);
            }
        }
    } else {
        // 0: tile A (warps 2-5), 1: tile B (warps 6-9).  A warp reaches only the TMEM lane
        // quadrant warp % 4, and any four consecutive warps cover all four.
        const int X = (warp - 2) >> 2;
        const int wq = warp & 3, r = wq * 32 + lane;
        const uint32_t lo = (uint32_t)(wq * 32) << 16;
        const int n = X ? nB : nA;
        if (n > 0) {
            const uint32_t tS = tmem + X * 128, tO = tmem + 256 + X * 128;
            float l = 1.0f;
            ok = softmax_tile<D>(sm, X, n, tS, tO, r, lo, sl2, limit_ns, abort, l);
            if (ok) ok = mbar_wait(&sm.o_final[X], 0, limit_ns, abort);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                const int i = i0 + X * kBM + r;
                const float inv = 1.0f / l;
                __nv_bfloat16 *orow = dense ? O + (((size_t)b * L + i) * H + h) * D
                                            : O + ((size_t)bh * L + i) * D;
                if (kGather) {  // Y[t] = X[t] + bf16(O / l) for token t = idx[i]
                    const int t = i < Lk ? __ldg(ga.idx + (size_t)bh * L + i) : -1;
                    const bool st = (unsigned)t < (unsigned)L;
                    const size_t seg = st ? (((size_t)b * L + t) * H + h) * D : 0;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + lo + c * 32, o);
                        tmem_ld_wait();
                        if (st) {
                            const uint4 *xs = reinterpret_cast<const uint4 *>(ga.X + seg + c * 32);
                            uint4 *ys = reinterpret_cast<uint4 *>(ga.Y + seg + c * 32);
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4) {
                                const uint4 xv = xs[q4];
                                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                                uint32_t yw[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const uint32_t ob = pack_bf16(
                                        __uint_as_float(o[q4 * 8 + 2 * e]) * inv,
                                        __uint_as_float(o[q4 * 8 + 2 * e + 1]) * inv);
                                    yw[e] = pack_bf16(
                                        __uint_as_float(xw[e] << 16) + __uint_as_float(ob << 16),
                                        __uint_as_float(xw[e] & 0xffff0000u) +
                                            __uint_as_float(ob & 0xffff0000u));
                                }
                                ys[q4] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
                            }
                        }
                    }
                } else {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + lo + c * 32, o);
                    tmem_ld_wait();
                    if (i < Lk) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 w;
                            w.x = pack_bf16(__uint_as_float(o[q4 * 8 + 0]) * inv,
                                            __uint_as_float(o[q4 * 8 + 1]) * inv);
                            w.y = pack_bf16(__uint_as_float(o[q4 * 8 + 2]) * inv,
                                            __uint_as_float(o[q4 * 8 + 3]) * inv);
                            w.z = pack_bf16(__uint_as_float(o[q4 * 8 + 4]) * inv,
                                            __uint_as_float(o[q4 * 8 + 5]) * inv);
                            w.w = pack_bf16(__uint_as_float(o[q4 * 8 + 6]) * inv,
                                            __uint_as_float(o[q4 * 8 + 7]) * inv);
                            dst[q4] = w;
                        }
                    }
                }
                }
            } else {
                ok = false;
            }
        }
    }
    if (!ok) {
        *abort = 1;
        report_error(ctl, TSA_ERR_DEVICE_TIMEOUT, 100 + warp);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

template <int D, bool kGather>
static cudaError_t attn_tc_impl(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                                const int32_t *Lkeep, int dense, float scale, void *O,
                                const GatherArgs &ga, const uint32_t *bmask, Control *ctl,
                                cudaStream_t st, uint32_t limit_us, bool pdl = false) {
    CUtensorMap tq, tk, tv;
    memset(&tq, 0, sizeof tq);  // the direct-gather mode reads no tensor map
    memset(&tk, 0, sizeof tk);
    memset(&tv, 0, sizeof tv);
    const uint64_t B = dm.B, L = dm.L, H = dm.H, Hkv = dm.Hkv;
    const uint32_t box[4] = {64, (uint32_t)kBM, 1, 1};
    bool okm = true;
    if (kGather) {
    } else if (dense) {
        const uint64_t dq[4] = {(uint64_t)D, L, H, B}, dk[4] = {(uint64_t)D, L, Hkv, B};
        const uint64_t sq[3] = {H * D * 2, (uint64_t)D * 2, L * H * D * 2};
        const uint64_t sk[3] = {Hkv * D * 2, (uint64_t)D * 2, L * Hkv * D * 2};
        okm = make_tmap_bf16_4d(&tq, Q, dq, sq, box) && make_tmap_bf16_4d(&tk, K, dk, sk, box) &&
              make_tmap_bf16_4d(&tv, V, dk, sk, box);
    } else {
        const uint64_t dd[4] = {(uint64_t)D, L, H, B};
        const uint64_t sd[3] = {(uint64_t)D * 2, L * D * 2, H * L * D * 2};
        okm = make_tmap_bf16_4d(&tq, Q, dd, sd, box) && make_tmap_bf16_4d(&tk, K, dd, sd, box) &&
              make_tmap_bf16_4d(&tv, V, dd, sd, box);
    }
    if (!okm) return cudaErrorInvalidValue;
    // At least 116 KB so that one CTA holds an SM (and all 512 TMEM columns) at a time.
    const size_t smem = std::max<size_t>(sizeof(AttnSmem<D>) + 1024, 116 * 1024);
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc<D, kGather>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long nblocks = (long)ceil_div(dm.L, 2 * kBM) * dm.B * dm.H;
    // Heads per scheduling group: as many as have K and V (2 * L * D bf16 each, counted
    // without GQA sharing) within kL2Share bytes.
    constexpr size_t kL2Share = 64u << 20;
    const size_t kv_head = (size_t)4 * dm.L * D;
    const int hgroup = (int)std::max<size_t>(1, std::min<size_t>((size_t)dm.B * dm.H, kL2Share / kv_head));
    e = launch_k(k_attn_tc<D, kGather>, dim3((unsigned)nblocks),
                 dim3(kGather ? kGatherThreads : kThreads), smem, st, pdl, tq, tk, tv, Lkeep,
                 dense, dm.L, dm.H, dm.Hkv, scale * 1.4426950408889634f, (__nv_bfloat16 *)O, ga,
                 bmask, hgroup, ctl, (uint64_t)limit_us * 1000ull, test_stall());
    note_launches(1);
    return e;
}

cudaError_t launch_attn_tc(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                           const int32_t *Lkeep, int dense, float scale, void *O, Control *ctl,
                           cudaStream_t st, uint32_t limit_us, const uint32_t *bmask, bool pdl) {
    const GatherArgs none{};
    return dm.d == 64 ? attn_tc_impl<64, false>(dm, Q, K, V, Lkeep, dense, scale, O, none, bmask,
                                                ctl, st, limit_us, pdl)
                      : attn_tc_impl<128, false>(dm, Q, K, V, Lkeep, dense, scale, O, none, bmask,
                                                 ctl, st, limit_us, pdl);
}

// Compressed attention reading Q, K, V rows through idx, with Y = X + Ô written into the
// kept rows (the unselected rows of Y are the caller's: equal to X in place).
cudaError_t launch_attn_gather(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                               const int32_t *idx, const int32_t *Lkeep, float scale,
                               const void *X, void *Y, Control *ctl, cudaStream_t st,
                               uint32_t limit_us) {
    GatherArgs ga;
    ga.Q = (const __nv_bfloat16 *)Q;
    ga.K = (const __nv_bfloat16 *)K;
    ga.V = (const __nv_bfloat16 *)V;
    ga.idx = idx;
    ga.X = (const __nv_bfloat16 *)X;
    ga.Y = (__nv_bfloat16 *)Y;
    return dm.d == 64
               ? attn_tc_impl<64, true>(dm, Q, K, V, Lkeep, 0, scale, nullptr, ga, nullptr, ctl, st,
                                        limit_us)
               : attn_tc_impl<128, true>(dm, Q, K, V, Lkeep, 0, scale, nullptr, ga, nullptr, ctl, st,
                                         limit_us);
}

}  // namespace tsa

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

#include <algorithm>

#include "sm100.cuh"

namespace tsa {
using namespace sm100;

namespace {

constexpr int kBM = 128, kBN = 128, kStages = 2, kThreads = 320;
constexpr uint64_t kDrainNs = 1000000000ull;  // drain waits: 1 s

template <int D> struct AttnSmem {
    static constexpr int TILE = kBM * D * 2;  // bytes of a 128-row tile
    alignas(1024) uint8_t q[2][TILE];
    alignas(1024) uint8_t k[kStages][TILE];
    alignas(1024) uint8_t v[kStages][TILE];
    uint64_t q_full, k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2], o_final[2], drain;
    uint64_t stall;  // test hook: initialised, never completed
    uint32_t tmem_base;
    int abort;
    int never;  // stays 0: drain waits ignore the abort flag
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
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
        mbar_arrive(&sm.p_full[X]);
    }
    l_out = l;
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ Lkeep, int dense,
          int L, int H, int Hkv, float sl2, __nv_bfloat16 *__restrict__ O, Control *ctl,
          uint64_t limit_ns, int stall) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<D> &sm = *reinterpret_cast<AttnSmem<D> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int TILE = AttnSmem<D>::TILE, NDB = D / 64;
    // Head-major order: the CTAs in flight together work on the same head (heaviest pairs
    // first), so they walk the same K/V tiles at the same pace and share them in L2.
    const int npairs = ceil_div(L, 2 * kBM);
    const int bh = blockIdx.x / npairs, pair = npairs - 1 - (int)(blockIdx.x % npairs);
    const int b = bh / H, h = bh % H;
    const int Lk = dense ? L : __ldg(Lkeep + b);
    const int i0 = pair * 2 * kBM;  // first row of tile A
    if (i0 >= Lk) return;
    const bool hasB = i0 + kBM < Lk;
    const int nA = 2 * pair + 1, nB = hasB ? 2 * pair + 2 : 0;
    const int nkv = hasB ? nB : nA;
    const int kvh = dense ? h / (H / Hkv) : h;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sm.s_full[x], 1);
            mbar_init(&sm.p_full[x], 128);
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
    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;  // K/V tiles issued (negative: K of tile -issued-1 only)
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
                if (!(ok = mbar_wait(&sm.k_empty[s], ph, limit_ns, abort))) break;
                mbar_expect_tx(&sm.k_full[s], TILE);
#pragma unroll
                for (int db = 0; db < NDB; ++db)
                    tma_load_4d(sm.k[s] + db * kBN * 128, &tmK, &sm.k_full[s], db * 64, j * kBN,
                                kvh, b);
                if (!(ok = mbar_wait(&sm.v_empty[s], ph, limit_ns, abort))) {
                    issued = -(j + 1);
                    break;
                }
                mbar_expect_tx(&sm.v_full[s], TILE);
#pragma unroll
                for (int db = 0; db < NDB; ++db)
                    tma_load_4d(sm.v[s] + db * kBN * 128, &tmV, &sm.v_full[s], db * 64, j * kBN,
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

template <int D>
static cudaError_t attn_tc_impl(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                                const int32_t *Lkeep, int dense, float scale, void *O,
                                Control *ctl, cudaStream_t st, uint32_t limit_us) {
    CUtensorMap tq, tk, tv;
    const uint64_t B = dm.B, L = dm.L, H = dm.H, Hkv = dm.Hkv;
    const uint32_t box[4] = {64, (uint32_t)kBM, 1, 1};
    bool okm;
    if (dense) {
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
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const long nblocks = (long)ceil_div(dm.L, 2 * kBM) * dm.B * dm.H;
    k_attn_tc<D><<<(unsigned)nblocks, kThreads, smem, st>>>(
        tq, tk, tv, Lkeep, dense, dm.L, dm.H, dm.Hkv, scale * 1.4426950408889634f,
        (__nv_bfloat16 *)O, ctl, (uint64_t)limit_us * 1000ull, test_stall());
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_attn_tc(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                           const int32_t *Lkeep, int dense, float scale, void *O, Control *ctl,
                           cudaStream_t st, uint32_t limit_us) {
    return dm.d == 64 ? attn_tc_impl<64>(dm, Q, K, V, Lkeep, dense, scale, O, ctl, st, limit_us)
                      : attn_tc_impl<128>(dm, Q, K, V, Lkeep, dense, scale, O, ctl, st, limit_us);
}

}  // namespace tsa

// Causal flash attention on the 5th-generation tensor cores (tcgen05 + TMEM), bf16 in,
// fp32 accumulate, for the compressed L'×L' problem of each head and for the dense GQA
// layer.  One CTA per 128-row query tile, heaviest (longest causal) tiles first.
//
// Method: "Token Sparse Attention" papernotes.org notes, 整体框架 (dense attention on the
// compressed problem, complexity O(L'^2 d)); bxzpzcl.cn post §1.1 (softmax(Q̂K̂ᵀ/√d)V̂).
// The causal mask j <= i in compressed order is the mask on original positions because
// the index lists are ascending.
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q tile once, then K and V tiles through a 2-stage ring.
//   warp 1      TMEM owner and MMA issuer: S_j = Q K_j^T into one of two TMEM S buffers,
//               then O += P_j V_j with P_j read from TMEM (bf16, written over S_j).
//   warps 4-7   softmax: thread r owns query row r.  Online max/sum in log2 units with a
//               lazy O rescale (only when the running max grows by more than 2^8), P
//               written back to TMEM, then the epilogue O / l -> bf16 -> global.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+d).
// Every wait is bounded in time; a wait that runs out records TSA_ERR_DEVICE_TIMEOUT,
// the CTA drains its in-flight copies and MMAs, frees TMEM and exits.
#include <math.h>

#include <algorithm>

#include "sm100.cuh"

namespace tsa {
using namespace sm100;

namespace {

constexpr int kBM = 128, kBN = 128, kStages = 2, kThreads = 256;
constexpr uint64_t kDrainNs = 1000000000ull;  // drain waits: 1 s

template <int D> struct AttnSmem {
    static constexpr int TILE = kBM * D * 2;  // bytes of a 128-row tile
    alignas(1024) uint8_t q[TILE];
    alignas(1024) uint8_t k[kStages][TILE];
    alignas(1024) uint8_t v[kStages][TILE];
    uint64_t q_full, k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2], pv_done, o_final, drain;
    uint32_t tmem_base;
    int abort;
    int never;  // stays 0: drain waits ignore the abort flag
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ Lkeep, int dense,
          int L, int H, int Hkv, float sl2, __nv_bfloat16 *__restrict__ O, Control *ctl,
          uint64_t limit_ns) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<D> &sm = *reinterpret_cast<AttnSmem<D> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int TILE = AttnSmem<D>::TILE, NDB = D / 64;
    const int ntiles = ceil_div(L, kBM);
    const int BH = gridDim.x / ntiles;
    const int tile = ntiles - 1 - (int)(blockIdx.x / BH), bh = blockIdx.x % BH;
    const int b = bh / H, h = bh % H;
    const int Lk = dense ? L : __ldg(Lkeep + b);
    const int i0 = tile * kBM;
    if (i0 >= Lk) return;
    const int n_kv = tile + 1;
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
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 128);
        }
        mbar_init(&sm.pv_done, 1);
        mbar_init(&sm.o_final, 1);
        mbar_init(&sm.drain, 1);
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
    const uint32_t tS0 = tmem, tS1 = tmem + 128, tO = tmem + 256;
    volatile int *abort = &sm.abort;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;  // K/V tiles issued
            mbar_expect_tx(&sm.q_full, TILE);
#pragma unroll
            for (int db = 0; db < NDB; ++db)
                tma_load_4d(sm.q + db * kBM * 128, &tmQ, &sm.q_full, db * 64, i0, h, b);
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % kStages;
                const uint32_t ph = ((j / kStages) & 1) ^ 1;
                if (!(ok = mbar_wait(&sm.k_empty[s], ph, limit_ns, abort))) break;
                mbar_expect_tx(&sm.k_full[s], TILE);
#pragma unroll
                for (int db = 0; db < NDB; ++db)
                    tma_load_4d(sm.k[s] + db * kBN * 128, &tmK, &sm.k_full[s], db * 64, j * kBN,
                                kvh, b);
                if (!(ok = mbar_wait(&sm.v_empty[s], ph, limit_ns, abort))) {
                    issued = -(j + 1);  // K_j in flight, V_j not issued
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
            const uint32_t qa = smem_u32(sm.q);
            bool any = false;
            auto issue_S = [&](int j) -> bool {
                const int s = j % kStages;
                if (!mbar_wait(&sm.k_full[s], (j / kStages) & 1, limit_ns, abort)) return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(sm.k[s]);
                const uint32_t dS = (j & 1) ? tS1 : tS0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * (kBM * 128) + (kk % 4) * 32;
                    mma_ss(dS, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                }
                any = true;
                mma_commit(&sm.k_empty[s]);
                mma_commit(&sm.s_full[j & 1]);
                return true;
            };
            ok = mbar_wait(&sm.q_full, 0, limit_ns, abort);
            if (ok) ok = issue_S(0);
            if (ok && n_kv > 1) ok = issue_S(1);
            for (int j = 0; j < n_kv && ok; ++j) {
                const int s = j % kStages;
                if (!(ok = mbar_wait(&sm.p_full[j & 1], (j >> 1) & 1, limit_ns, abort))) break;
                if (!(ok = mbar_wait(&sm.v_full[s], (j / kStages) & 1, limit_ns, abort))) break;
                tc_fence_after();
                const uint32_t va = smem_u32(sm.v[s]);
                const uint32_t aP = (j & 1) ? tS1 : tS0;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tO, aP + kk * 8, sdesc_sw128(va + kk * 2048, kBN * 128, 1024), idO,
                           (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&sm.v_empty[s]);
                mma_commit(&sm.pv_done);
                if (j == n_kv - 1) mma_commit(&sm.o_final);
                if (j + 2 < n_kv) ok = issue_S(j + 2);
            }
            if (any) {  // every MMA issued here has completed before TMEM is freed
                mma_commit(&sm.drain);
                mbar_wait(&sm.drain, 0, kDrainNs, &sm.never);
            }
        }
    } else if (warp >= 4) {
        const int wq = warp & 3, r = wq * 32 + lane;
        const uint32_t lo = (uint32_t)(wq * 32) << 16;
        float m = -INFINITY, l = 0.0f;
        for (int j = 0; j < n_kv; ++j) {
            ok = mbar_wait(&sm.s_full[j & 1], (j >> 1) & 1, limit_ns, abort);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = ((j & 1) ? tS1 : tS0) + lo;
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            tmem_ld_wait();
            const bool diag = (j == n_kv - 1);
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                float v = __uint_as_float(sr[c]);
                if (diag && c > r) v = -INFINITY;
                sr[c] = __float_as_uint(v);
                mt = fmaxf(mt, v);
            }
            mt *= sl2;
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
            float sum = 0.0f;
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = ex2(fmaf(__uint_as_float(sr[2 * c]), sl2, -mu));
                const float p1 = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -mu));
                sum += p0 + p1;
                pk[c] = pack_bf16(p0, p1);
            }
            l = l * factor + sum;
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                // PV_{j-2} is complete (S_j was issued after it and has completed), so the
                // parity of phase j-1 identifies PV_{j-1} unambiguously.
                ok = mbar_wait(&sm.pv_done, (j - 1) & 1, limit_ns, abort);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
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
                tmem_st_wait();
            }
            tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sm.p_full[j & 1]);
        }
        // O is final once the last O += P V has completed.  (A parity wait on pv_done
        // cannot tell that phase from the one before it, which may still be pending.)
        if (ok) ok = mbar_wait(&sm.o_final, 0, limit_ns, abort);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const int i = i0 + r;
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
                        w.x = pack_bf16(__uint_as_float(o[q4 * 8 + 0]) * inv, __uint_as_float(o[q4 * 8 + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[q4 * 8 + 2]) * inv, __uint_as_float(o[q4 * 8 + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[q4 * 8 + 4]) * inv, __uint_as_float(o[q4 * 8 + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[q4 * 8 + 6]) * inv, __uint_as_float(o[q4 * 8 + 7]) * inv);
                        dst[q4] = w;
                    }
                }
            }
        } else {
            ok = false;
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
    const long nblocks = (long)ceil_div(dm.L, kBM) * dm.B * dm.H;
    k_attn_tc<D><<<(unsigned)nblocks, kThreads, smem, st>>>(
        tq, tk, tv, Lkeep, dense, dm.L, dm.H, dm.Hkv, scale * 1.4426950408889634f,
        (__nv_bfloat16 *)O, ctl, (uint64_t)limit_us * 1000ull);
    return cudaGetLastError();
}

cudaError_t launch_attn_tc(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                           const int32_t *Lkeep, int dense, float scale, void *O, Control *ctl,
                           cudaStream_t st, uint32_t limit_us) {
    return dm.d == 64 ? attn_tc_impl<64>(dm, Q, K, V, Lkeep, dense, scale, O, ctl, st, limit_us)
                      : attn_tc_impl<128>(dm, Q, K, V, Lkeep, dense, scale, O, ctl, st, limit_us);
}

}  // namespace tsa

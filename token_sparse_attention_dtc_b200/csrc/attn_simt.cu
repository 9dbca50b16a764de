// Causal attention on CUDA cores for fp32 inputs (the fp32 path keeps full fp32
// products; tensor-core tf32 would not meet a 1e-4 output tolerance).  bf16 inputs run on
// the tensor cores (attn_tc.cu).  Flash-style
// online softmax over 64-key tiles, one block per (16-row query tile, batch, head).
//
// Method: "Token Sparse Attention" papernotes.org notes, 整体框架 (dense attention on
// the compressed L'×L' problem); bxzpzcl.cn post §1.1 (softmax(Q̂K̂ᵀ/√d)V̂).  The causal
// mask j <= i in compressed order equals the mask on original positions because the
// index lists are ascending.
//
// 16-row query tiles (16 threads per row, each 4 key columns of S and D/16 output
// columns), so that short rows still spread over many blocks.
#include <math.h>

#include "common.cuh"

namespace tsa {

constexpr int kAttnSimtThreads = 256;
constexpr int kBM = 16, kBN = 64;
constexpr int kTPR = kAttnSimtThreads / kBM;  // threads per query row
constexpr int kSC = kBN / kTPR;               // key columns of S per thread

template <int D> struct SimtSmem {
    float q[kBM][D + 1];
    float k[kBN][D + 1];
    float v[kBN][D];
    float p[kBM][kBN + 1];
};

// Linear block id -> (query tile, b*H + h), heaviest causal tiles first.
template <typename T, int D>
__global__ void __launch_bounds__(kAttnSimtThreads)
k_attn_simt(const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
            const int32_t *__restrict__ Lkeep, int dense, int L, int H, int Hkv, float sl2,
            T *__restrict__ O) {
    extern __shared__ float smem_raw[];
    SimtSmem<D> &sm = *reinterpret_cast<SimtSmem<D> *>(smem_raw);
    const int BH = gridDim.x / ceil_div(L, kBM);
    const int ntiles = ceil_div(L, kBM);
    const int tile = ntiles - 1 - (int)(blockIdx.x / BH), bh = blockIdx.x % BH;
    const int b = bh / H, h = bh % H, kv = h / (H / Hkv);
    const int Lk = dense ? L : min(max(Lkeep[b], 0), L);  // clamped: rows past L untouched
    const int i0 = tile * kBM;
    if (i0 >= Lk) return;
    size_t qbase, kbase, qstride, kstride;
    if (dense) {
        qbase = ((size_t)b * L * H + h) * D;
        kbase = ((size_t)b * L * Hkv + kv) * D;
        qstride = (size_t)H * D;
        kstride = (size_t)Hkv * D;
    } else {
        qbase = kbase = (size_t)bh * L * D;
        qstride = kstride = D;
    }
    const int tid = threadIdx.x, r = tid / kTPR, cg = tid % kTPR;
    constexpr int OC = D / kTPR;  // output columns per thread
    for (int e = tid; e < kBM * D; e += kAttnSimtThreads) {
        const int rr = e / D, c = e % D, i = i0 + rr;
        sm.q[rr][c] = i < Lk ? Elem<T>::load(Q, qbase + (size_t)i * qstride + c) : 0.0f;
    }
    float o[OC];
#pragma unroll
    for (int c = 0; c < OC; ++c) o[c] = 0.0f;
    float m = -INFINITY, l = 0.0f;
    const int i = i0 + r;
    const int jend = min(i0 + kBM, Lk);
    for (int j0 = 0; j0 < jend; j0 += kBN) {
        __syncthreads();
        for (int e = tid; e < kBN * D; e += kAttnSimtThreads) {
            const int rr = e / D, c = e % D, j = j0 + rr;
            const bool ok = j < Lk;
            sm.k[rr][c] = ok ? Elem<T>::load(K, kbase + (size_t)j * kstride + c) : 0.0f;
            sm.v[rr][c] = ok ? Elem<T>::load(V, kbase + (size_t)j * kstride + c) : 0.0f;
        }
        __syncthreads();
        float s[kSC];
#pragma unroll
        for (int c = 0; c < kSC; ++c) s[c] = 0.0f;
        for (int k = 0; k < D; ++k) {
            const float qv = sm.q[r][k];
#pragma unroll
            for (int c = 0; c < kSC; ++c) s[c] = fmaf(qv, sm.k[cg * kSC + c][k], s[c]);
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kSC; ++c) {
            const int j = j0 + cg * kSC + c;
            s[c] = (j <= i && j < Lk) ? s[c] * sl2 : -INFINITY;
            mx = fmaxf(mx, s[c]);
        }
#pragma unroll
        for (int o = 1; o < kTPR; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mnew = fmaxf(m, mx);
        const float corr = (m == -INFINITY) ? 0.0f : exp2f(m - mnew);
        float ps = 0.0f;
#pragma unroll
        for (int c = 0; c < kSC; ++c) {
            const float p = (s[c] == -INFINITY) ? 0.0f : exp2f(s[c] - mnew);
            sm.p[r][cg * kSC + c] = p;
            ps += p;
        }
#pragma unroll
        for (int o = 1; o < kTPR; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l = l * corr + ps;
        m = mnew;
#pragma unroll
        for (int c = 0; c < OC; ++c) o[c] *= corr;
        __syncthreads();
        for (int j = 0; j < kBN; ++j) {
            const float p = sm.p[r][j];
#pragma unroll
            for (int c = 0; c < OC; ++c) o[c] = fmaf(p, sm.v[j][cg * OC + c], o[c]);
        }
    }
    if (i < Lk) {
        const float inv = 1.0f / l;
        T *orow = O + qbase + (size_t)i * qstride + cg * OC;
#pragma unroll
        for (int c = 0; c < OC; ++c) orow[c] = Elem<T>::from_f(o[c] * inv);
    }
}

template <typename T, int D>
static cudaError_t attn_simt_impl(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                                  const int32_t *Lkeep, int dense, float scale, void *O,
                                  cudaStream_t st) {
    const size_t smem = sizeof(SimtSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(k_attn_simt<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long nblocks = (long)ceil_div(dm.L, kBM) * dm.B * dm.H;
    if (nblocks > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    k_attn_simt<T, D><<<(unsigned)nblocks, kAttnSimtThreads, smem, st>>>(
        (const T *)Q, (const T *)K, (const T *)V, Lkeep, dense, dm.L, dm.H, dm.Hkv,
        scale * 1.4426950408889634f, (T *)O);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_attn_simt(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                             const int32_t *Lkeep, int dense, float scale, void *O,
                             cudaStream_t st) {
    if (dm.dtype != TSA_F32) return cudaErrorInvalidValue;  // bf16 runs on the tensor cores
    return dm.d == 64 ? attn_simt_impl<float, 64>(dm, Q, K, V, Lkeep, dense, scale, O, st)
                      : attn_simt_impl<float, 128>(dm, Q, K, V, Lkeep, dense, scale, O, st);
}

}  // namespace tsa

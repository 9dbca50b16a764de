// Compress (gather of Q, K, V rows through the per-head index lists) and decompress
// (scatter of the attention rows back to their tokens, fused with the residual add).
// Both are pure HBM traffic: 16-byte vector loads and stores, one index read per row.
//
// Method: "Token Sparse Attention" papernotes.org notes, 整体框架 and 关键设计 1
// (gather Q̂, K̂, V̂ by S_h; scatter Ô into a zero L×d tensor; X_{l+1} = X_l +
// Decompress(Ô)); bxzpzcl.cn post §1.1; gist.science §2 "Core Architecture".
#include <algorithm>

#include "common.cuh"

namespace tsa {

constexpr int kMoveThreads = 256;
constexpr int kGatherRows = 32;  // rows of one (b, h) per block

// Rows of one (b, h) per gather block: every thread owns kQkvRows * VPR / kMoveThreads
// vectors, and issues all their loads (index, then Q, K and V) before its first store.
constexpr int kQkvRows = 64;

// grid (B*H, ceil(L / kQkvRows)).  VPR = 16-byte vectors per row.  Heads vary fastest
// across blocks, so the G heads that share a KV row read it close in time.
template <int VPR>
__global__ void __launch_bounds__(kMoveThreads)
k_gather_qkv(const uint4 *__restrict__ Q, const uint4 *__restrict__ K, const uint4 *__restrict__ V,
             const int32_t *__restrict__ idx, const int32_t *__restrict__ Lkeep, int L, int H,
             int Hkv, uint4 *__restrict__ Qh, uint4 *__restrict__ Kh, uint4 *__restrict__ Vh,
             Control *ctl) {
    constexpr int kPer = kQkvRows * VPR / kMoveThreads;
    static_assert(kPer * kMoveThreads == kQkvRows * VPR, "whole vectors per thread");
    pdl_wait();  // the index lists and counts are the previous kernels'
    pdl_trigger();
    const int bh = blockIdx.x, b = bh / H, h = bh % H, kv = h / (H / Hkv);
    const int Lk = min(max(Lkeep[b], 0), L);  // a count outside [0, L] is clamped
    const int pad_end = min(L, (Lk + 127) & ~127);
    const int i0 = blockIdx.y * kQkvRows;
    if (i0 >= pad_end) return;
    const int32_t *S = idx + (size_t)bh * L;
    int t[kPer];  // token of each vector's row; -1: a zero row of the padding
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int i = i0 + (threadIdx.x + u * kMoveThreads) / VPR;
        t[u] = i < Lk ? __ldg(S + i) : -1;
    }
    uint4 q[kPer], k[kPer], w[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int v = (threadIdx.x + u * kMoveThreads) % VPR;
        if ((unsigned)t[u] < (unsigned)L) {
            const size_t qs = (((size_t)b * L + t[u]) * H + h) * VPR + v;
            const size_t ks = (((size_t)b * L + t[u]) * Hkv + kv) * VPR + v;
            q[u] = __ldg(Q + qs);
            k[u] = __ldg(K + ks);
            w[u] = __ldg(V + ks);
        } else {
            q[u] = k[u] = w[u] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int e = threadIdx.x + u * kMoveThreads, i = i0 + e / VPR;
        if (i >= pad_end) break;
        if (t[u] >= L || t[u] < -1 || (t[u] == -1 && i < Lk)) {  // not an index of this sequence
            report_error(ctl, TSA_ERR_INVALID_ARG, 20);
            continue;
        }
        const size_t dst = ((size_t)bh * L + i) * VPR + e % VPR;
        Qh[dst] = q[u];
        Kh[dst] = k[u];
        Vh[dst] = w[u];
    }
}

template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int n = 4;
    static __device__ inline void unpack(const uint4 &u, float *f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    static __device__ inline uint4 pack(const float *f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int n = 8;
    static __device__ inline void unpack(const uint4 &u, float *f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ inline uint4 pack(const float *f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&p);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename T>
__device__ inline uint4 add_vec(const uint4 &x, const uint4 &o) {
    float a[Vec<T>::n], c[Vec<T>::n];
    Vec<T>::unpack(x, a);
    Vec<T>::unpack(o, c);
#pragma unroll
    for (int i = 0; i < Vec<T>::n; ++i) a[i] = a[i] + c[i];
    return Vec<T>::pack(a);
}

// Sparse decompress + residual.  grid (B*H, ceil(L / kGatherRows)).
// in_place: only the kept segments, Y[seg] += Oh[row].  Otherwise every segment of Y is
// written once: kept ones X + Oh, the complement (idx[Lk:L]) copies X.
template <typename T, int VPR, bool in_place>
__global__ void __launch_bounds__(kMoveThreads)
k_scatter_residual(const uint4 *__restrict__ Oh, const int32_t *__restrict__ idx,
                   const int32_t *__restrict__ Lkeep, const uint4 *X, uint4 *Y, int L, int H) {
    pdl_wait();  // Ô is the previous kernel's
    pdl_trigger();
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int Lk = min(max(Lkeep[b], 0), L);  // a count outside [0, L] is clamped
    const int i0 = blockIdx.y * kGatherRows;
    const int iend = in_place ? Lk : L;
    if (i0 >= iend) return;
    const int32_t *S = idx + (size_t)bh * L;
    for (int e = threadIdx.x; e < kGatherRows * VPR; e += kMoveThreads) {
        const int i = i0 + e / VPR, v = e % VPR;
        if (i >= iend) break;
        const int t = S[i];
        if ((unsigned)t >= (unsigned)L) continue;  // not a token of this sequence: skipped
        const size_t seg = (((size_t)b * L + t) * H + h) * VPR + v;
        const uint4 x = X[seg];
        if (i < Lk) Y[seg] = add_vec<T>(x, Oh[((size_t)bh * L + i) * VPR + v]);
        else Y[seg] = x;
    }
}

// The unselected segments of an out-of-place layer whose kept segments the attention
// epilogue writes itself: Y[seg] = X[seg] for idx[Lk:L].  grid (B*H, ceil(L / kGatherRows)).
template <int VPR>
__global__ void __launch_bounds__(kMoveThreads)
k_copy_rest(const int32_t *__restrict__ idx, const int32_t *__restrict__ Lkeep, const uint4 *X,
            uint4 *Y, int L, int H) {
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int Lk = min(max(Lkeep[b], 0), L);
    const int i0 = max(blockIdx.y * kGatherRows, Lk), i1 = min(L, (blockIdx.y + 1) * kGatherRows);
    const int32_t *S = idx + (size_t)bh * L;
    for (int e = threadIdx.x; e < (i1 - i0) * VPR; e += kMoveThreads) {
        const int i = i0 + e / VPR, v = e % VPR;
        const int t = S[i];
        if ((unsigned)t >= (unsigned)L) continue;  // a bad list is reported by the attention
        const size_t seg = (((size_t)b * L + t) * H + h) * VPR + v;
        Y[seg] = X[seg];
    }
}

// Dense residual: Y = X + O elementwise over [B, L, H*d].
template <typename T>
__global__ void __launch_bounds__(kMoveThreads)
k_residual_dense(const uint4 *__restrict__ O, const uint4 *X, uint4 *Y, size_t nvec) {
    for (size_t e = (size_t)blockIdx.x * kMoveThreads + threadIdx.x; e < nvec;
         e += (size_t)gridDim.x * kMoveThreads)
        Y[e] = add_vec<T>(X[e], O[e]);
}

cudaError_t launch_gather(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                          const int32_t *idx, const int32_t *Lkeep, void *Qh, void *Kh, void *Vh,
                          Control *ctl, cudaStream_t st, bool pdl) {
    const int esz = dm.dtype == TSA_F32 ? 4 : 2;
    const int vpr = dm.d * esz / 16;
    dim3 grid(dm.B * dm.H, ceil_div(dm.L, kQkvRows));
    cudaError_t e;
#define TSA_GATHER(V_)                                                                       \
    e = launch_k(k_gather_qkv<V_>, grid, dim3(kMoveThreads), 0, st, pdl, (const uint4 *)Q,  \
                 (const uint4 *)K, (const uint4 *)V, idx, Lkeep, dm.L, dm.H, dm.Hkv,          \
                 (uint4 *)Qh, (uint4 *)Kh, (uint4 *)Vh, ctl)
    switch (vpr) {
        case 8: TSA_GATHER(8); break;
        case 16: TSA_GATHER(16); break;
        case 32: TSA_GATHER(32); break;
        default: return cudaErrorInvalidValue;
    }
#undef TSA_GATHER
    note_launches(1);
    return e;
}

template <typename T>
static cudaError_t scatter_impl(const tsa_dims &dm, const void *Oh, const int32_t *idx,
                                const int32_t *Lkeep, const void *X, void *Y, cudaStream_t st,
                                bool pdl) {
    const int vpr = dm.d * (int)sizeof(T) / 16;
    if (!idx) {
        const size_t nvec = (size_t)dm.B * dm.L * dm.H * vpr;
        const int blocks = (int)std::min<size_t>((nvec + kMoveThreads - 1) / kMoveThreads,
                                                 (size_t)148 * 16);
        k_residual_dense<T><<<blocks, kMoveThreads, 0, st>>>((const uint4 *)Oh, (const uint4 *)X,
                                                            (uint4 *)Y, nvec);
        note_launches(1);
        return cudaGetLastError();
    }
    dim3 grid(dm.B * dm.H, ceil_div(dm.L, kGatherRows));
    const bool ip = (X == Y);
    cudaError_t e;
#define TSA_SCATTER(V_)                                                                     \
    e = ip ? launch_k(k_scatter_residual<T, V_, true>, grid, dim3(kMoveThreads), 0, st, pdl, \
                      (const uint4 *)Oh, idx, Lkeep, (const uint4 *)X, (uint4 *)Y, dm.L,     \
                      dm.H)                                                                  \
           : launch_k(k_scatter_residual<T, V_, false>, grid, dim3(kMoveThreads), 0, st,     \
                      pdl, (const uint4 *)Oh, idx, Lkeep, (const uint4 *)X, (uint4 *)Y,      \
                      dm.L, dm.H)
    switch (vpr) {
        case 8: TSA_SCATTER(8); break;
        case 16: TSA_SCATTER(16); break;
        case 32: TSA_SCATTER(32); break;
        default: return cudaErrorInvalidValue;
    }
#undef TSA_SCATTER
    note_launches(1);
    return e;
}

cudaError_t launch_scatter(const tsa_dims &dm, const void *Oh, const int32_t *idx,
                           const int32_t *Lkeep, const void *X, void *Y, cudaStream_t st,
                           bool pdl) {
    return dm.dtype == TSA_F32 ? scatter_impl<float>(dm, Oh, idx, Lkeep, X, Y, st, pdl)
                               : scatter_impl<__nv_bfloat16>(dm, Oh, idx, Lkeep, X, Y, st, pdl);
}

cudaError_t launch_copy_rest(const tsa_dims &dm, const int32_t *idx, const int32_t *Lkeep,
                             const void *X, void *Y, cudaStream_t st) {
    const int vpr = dm.d * (dm.dtype == TSA_F32 ? 4 : 2) / 16;
    dim3 grid(dm.B * dm.H, ceil_div(dm.L, kGatherRows));
    switch (vpr) {
        case 8: k_copy_rest<8><<<grid, kMoveThreads, 0, st>>>(idx, Lkeep, (const uint4 *)X, (uint4 *)Y, dm.L, dm.H); break;
        case 16: k_copy_rest<16><<<grid, kMoveThreads, 0, st>>>(idx, Lkeep, (const uint4 *)X, (uint4 *)Y, dm.L, dm.H); break;
        case 32: k_copy_rest<32><<<grid, kMoveThreads, 0, st>>>(idx, Lkeep, (const uint4 *)X, (uint4 *)Y, dm.L, dm.H); break;
        default: return cudaErrorInvalidValue;
    }
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace tsa

// Dynamic Token Coverage scoring on CUDA cores for fp32 inputs (tf32 tensor cores would
// not meet the 1e-5 score tolerance; bf16 inputs score on the tensor cores in
// score_tc.cu), the split combine, and the layer-score normalisation shared by every
// dtype.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 2 (recent queries
// score all keys; column sums give s_h; their normalised sum gives s_l); bxzpzcl.cn
// post §2.1.  The softmax of each recent query row is exact, in two passes over K:
// pass 1 finds each row's max and normaliser, pass 2 sums the normalised weights per
// (head, token).  All arithmetic is fp32 in log2 units: z2 = scale*log2(e)*<q, k>,
// weight = 2^(z2 - max2) / sum.
#include <math.h>

#include "common.cuh"

namespace tsa {

constexpr int kSimtThreads = 256;
constexpr int kSimtChunk = 32;  // query columns per register block

__device__ inline void online_push(float &m, float &l, float z) {
    if (z > m) {
        l = l * exp2f(m - z) + 1.0f;
        m = z;
    } else {
        l += exp2f(z - m);
    }
}

__device__ inline void online_merge(float &m, float &l, float m2, float l2) {
    const float mm = fmaxf(m, m2);
    const float a = (m == -INFINITY) ? 0.0f : l * exp2f(m - mm);
    const float b = (m2 == -INFINITY) ? 0.0f : l2 * exp2f(m2 - mm);
    m = mm;
    l = a + b;
}

// Pass 1.  grid (nsplit, B*Hkv, G), 256 threads.  Block (split, group, g) covers the
// qe recent-query columns of head h = kv*G + g over tokens [split*split_len, ...).
// part[(bg*nsplit + split)*N + g*qe + i] = (max, sum) of that split.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_score_stats_simt(const T *__restrict__ Q, const T *__restrict__ K, int L, int H, int Hkv,
                   int qe, float sl2, int split_len, int nsplit, float2 *__restrict__ part) {
    const int split = blockIdx.x, bg = blockIdx.y, g = blockIdx.z;
    const int b = bg / Hkv, kv = bg % Hkv, G = H / Hkv, h = kv * G + g, N = G * qe;
    __shared__ float Qs[kSimtChunk][D];
    __shared__ float red_m[kSimtThreads / 32][kSimtChunk], red_l[kSimtThreads / 32][kSimtChunk];
    const int t0 = split * split_len, t1 = min(L, t0 + split_len);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int c0 = 0; c0 < qe; c0 += kSimtChunk) {
        const int nc = min(kSimtChunk, qe - c0);
        for (int e = threadIdx.x; e < kSimtChunk * D; e += blockDim.x) {
            const int r = e / D, c = e % D;
            float v = 0.0f;
            if (r < nc) v = Elem<T>::load(Q, (((size_t)b * L + (L - qe + c0 + r)) * H + h) * D + c);
            Qs[r][c] = v;
        }
        __syncthreads();
        float m[kSimtChunk], l[kSimtChunk];
#pragma unroll
        for (int r = 0; r < kSimtChunk; ++r) { m[r] = -INFINITY; l[r] = 0.0f; }
        for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
            const T *kr = K + (((size_t)b * L + t) * Hkv + kv) * D;
            float acc[kSimtChunk];
#pragma unroll
            for (int r = 0; r < kSimtChunk; ++r) acc[r] = 0.0f;
            for (int c = 0; c < D; c += 4) {
                float kf[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) kf[u] = Elem<T>::load(kr, c + u);
#pragma unroll
                for (int r = 0; r < kSimtChunk; ++r)
#pragma unroll
                    for (int u = 0; u < 4; ++u) acc[r] = fmaf(Qs[r][c + u], kf[u], acc[r]);
            }
#pragma unroll
            for (int r = 0; r < kSimtChunk; ++r)
                if (r < nc && t <= L - qe + c0 + r) online_push(m[r], l[r], acc[r] * sl2);
        }
        // Fixed-order block reduction of the per-thread (max, sum) pairs.
#pragma unroll
        for (int r = 0; r < kSimtChunk; ++r) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m[r], o);
                const float l2 = __shfl_xor_sync(0xffffffffu, l[r], o);
                online_merge(m[r], l[r], m2, l2);
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < kSimtChunk; ++r) { red_m[warp][r] = m[r]; red_l[warp][r] = l[r]; }
        }
        __syncthreads();
        if (warp == 0 && lane < nc) {
            float mm = red_m[0][lane], ll = red_l[0][lane];
            for (int w = 1; w < kSimtThreads / 32; ++w) online_merge(mm, ll, red_m[w][lane], red_l[w][lane]);
            part[((size_t)bg * nsplit + split) * N + g * qe + c0 + lane] = make_float2(mm, ll);
        }
        __syncthreads();
    }
}

// Combine the per-split pairs in split order: stat[bg*N + n] = (max, 1/sum).
__global__ void k_score_combine(const float2 *__restrict__ part, int nsplit, int N,
                                float2 *__restrict__ stat) {
    const int bg = blockIdx.x;
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
        float m = -INFINITY, l = 0.0f;
        for (int s = 0; s < nsplit; ++s) {
            const float2 p = part[((size_t)bg * nsplit + s) * N + n];
            online_merge(m, l, p.x, p.y);
        }
        stat[(size_t)bg * N + n] = make_float2(m, 1.0f / l);
    }
}

// Pass 2.  Same grid as pass 1.  s_h[b,h,t] = sum_i 2^(z2_i - max_i) / sum_i over the
// recent queries i whose position is >= t, summed in i order.
template <typename T, int D, int TPT>
__global__ void __launch_bounds__(kSimtThreads)
k_score_colsum_simt(const T *__restrict__ Q, const T *__restrict__ K, int L, int H, int Hkv,
                    int qe, float sl2, int split_len, const float2 *__restrict__ stat,
                    float *__restrict__ s_h) {
    const int split = blockIdx.x, bg = blockIdx.y, g = blockIdx.z;
    const int b = bg / Hkv, kv = bg % Hkv, G = H / Hkv, h = kv * G + g, N = G * qe;
    __shared__ float Qs[kSimtChunk][D];
    __shared__ float2 St[kSimtChunk];
    const int t0 = split * split_len;
    float s[TPT];
#pragma unroll
    for (int j = 0; j < TPT; ++j) s[j] = 0.0f;
    for (int c0 = 0; c0 < qe; c0 += kSimtChunk) {
        const int nc = min(kSimtChunk, qe - c0);
        for (int e = threadIdx.x; e < kSimtChunk * D; e += blockDim.x) {
            const int r = e / D, c = e % D;
            float v = 0.0f;
            if (r < nc) v = Elem<T>::load(Q, (((size_t)b * L + (L - qe + c0 + r)) * H + h) * D + c);
            Qs[r][c] = v;
        }
        if (threadIdx.x < kSimtChunk)
            St[threadIdx.x] = threadIdx.x < nc ? stat[(size_t)bg * N + g * qe + c0 + threadIdx.x]
                                               : make_float2(0.0f, 0.0f);
        __syncthreads();
#pragma unroll
        for (int j = 0; j < TPT; ++j) {
            const int t = t0 + j * kSimtThreads + threadIdx.x;
            if (t >= L) break;
            const T *kr = K + (((size_t)b * L + t) * Hkv + kv) * D;
            float acc[kSimtChunk];
#pragma unroll
            for (int r = 0; r < kSimtChunk; ++r) acc[r] = 0.0f;
            for (int c = 0; c < D; c += 4) {
                float kf[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) kf[u] = Elem<T>::load(kr, c + u);
#pragma unroll
                for (int r = 0; r < kSimtChunk; ++r)
#pragma unroll
                    for (int u = 0; u < 4; ++u) acc[r] = fmaf(Qs[r][c + u], kf[u], acc[r]);
            }
            float sj = s[j];
#pragma unroll
            for (int r = 0; r < kSimtChunk; ++r)
                if (r < nc && t <= L - qe + c0 + r) sj += exp2f(acc[r] * sl2 - St[r].x) * St[r].y;
            s[j] = sj;
        }
        __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < TPT; ++j) {
        const int t = t0 + j * kSimtThreads + threadIdx.x;
        if (t < L) s_h[((size_t)b * H + h) * L + t] = s[j];
    }
}

// u[b,t] = sum_h s_h[b,h,t] in head order, stored in s_l; per-block partial sums of u
// (fixed tree) into part[b*nblk + blk].  grid (nblk, B), 256 threads.
__global__ void __launch_bounds__(256)
k_norm_u(const float *__restrict__ s_h, int L, int H, int nblk, float *__restrict__ s_l,
         float *__restrict__ part) {
    const int b = blockIdx.y, t = blockIdx.x * 256 + threadIdx.x;
    float u = 0.0f;
    if (t < L) {
        for (int h = 0; h < H; ++h) u += s_h[((size_t)b * H + h) * L + t];
        s_l[(size_t)b * L + t] = u;
    }
    __shared__ float red[256];
    red[threadIdx.x] = u;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[(size_t)b * nblk + blockIdx.x] = red[0];
}

// Z = sum of the partials (same fixed order in every block); s_l = u / Z.
__global__ void __launch_bounds__(256)
k_norm_div(float *__restrict__ s_l, int L, int nblk, const float *__restrict__ part) {
    const int b = blockIdx.y, t = blockIdx.x * 256 + threadIdx.x;
    float z = 0.0f;
    for (int i = threadIdx.x; i < nblk; i += 256) z += part[(size_t)b * nblk + i];
    __shared__ float red[256];
    red[threadIdx.x] = z;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    const float Z = red[0];
    if (t < L) s_l[(size_t)b * L + t] = s_l[(size_t)b * L + t] / Z;
}

// ---------------------------------------------------------------- launchers ---

template <typename T, int D>
static cudaError_t score_simt_impl(const tsa_dims &dm, const void *Q, const void *K, int qe,
                                   float scale, float *s_h, const WsLayout &w, char *ws,
                                   cudaStream_t st) {
    const float sl2 = scale * 1.4426950408889634f;
    const int split_len = score_simt_split(dm.L);
    const int nsplit = ceil_div(dm.L, split_len);
    const int G = dm.H / dm.Hkv;
    float2 *part = reinterpret_cast<float2 *>(ws + w.score_part);
    float2 *stat = reinterpret_cast<float2 *>(ws + w.score_stat);
    dim3 grid(nsplit, dm.B * dm.Hkv, G);
    k_score_stats_simt<T, D><<<grid, kSimtThreads, 0, st>>>(
        (const T *)Q, (const T *)K, dm.L, dm.H, dm.Hkv, qe, sl2, split_len, nsplit, part);
    k_score_combine<<<dm.B * dm.Hkv, 256, 0, st>>>(part, nsplit, G * qe, stat);
#define TSA_COLSUM(TPT)                                                                    \
    k_score_colsum_simt<T, D, TPT><<<grid, kSimtThreads, 0, st>>>(                          \
        (const T *)Q, (const T *)K, dm.L, dm.H, dm.Hkv, qe, sl2, split_len, stat, s_h)
    switch (split_len / kSimtThreads) {  // tokens per thread
        case 16: TSA_COLSUM(16); break;
        case 4: TSA_COLSUM(4); break;
        default: TSA_COLSUM(1); break;
    }
#undef TSA_COLSUM
    note_launches(3);
    return cudaGetLastError();
}

cudaError_t launch_score_simt(const tsa_dims &dm, const void *Q, const void *K, int qe,
                              float scale, float *s_h, const WsLayout &w, char *ws,
                              cudaStream_t st) {
    if (dm.dtype != TSA_F32) return cudaErrorInvalidValue;  // bf16 scores on the tensor cores
    return dm.d == 64 ? score_simt_impl<float, 64>(dm, Q, K, qe, scale, s_h, w, ws, st)
                      : score_simt_impl<float, 128>(dm, Q, K, qe, scale, s_h, w, ws, st);
}

cudaError_t launch_combine(const float2 *part, int nsplit, int N, float2 *stat, int groups,
                           cudaStream_t st) {
    k_score_combine<<<groups, 256, 0, st>>>(part, nsplit, N, stat);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_norm(const tsa_dims &dm, const float *s_h, float *s_l, const WsLayout &w,
                        char *ws, cudaStream_t st) {
    float *part = reinterpret_cast<float *>(ws + w.norm_part);
    dim3 grid(w.nblk_norm, dm.B);
    k_norm_u<<<grid, 256, 0, st>>>(s_h, dm.L, dm.H, w.nblk_norm, s_l, part);
    k_norm_div<<<grid, 256, 0, st>>>(s_l, dm.L, w.nblk_norm, part);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace tsa

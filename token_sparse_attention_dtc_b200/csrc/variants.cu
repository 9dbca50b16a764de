// Budget and score variants of the layer: a fixed-ratio budget and token-axis pooling of
// the head scores.
//
// Method: "Token Sparse Attention" papernotes.org notes, 消融实验 (the dynamic coverage
// budget against a fixed ratio s = 0.3 / 0.5; s is the fraction of tokens pruned, so
// L' = L - floor(s L)) and 关键设计 2 (the recent-query column sums are pooled into the
// head score s_h before the layer score).  The pages name no pooling kind or window; both
// plain ones are provided: the max or the mean over [t - r, t + r] clipped to [0, L), the
// mean dividing by the number of tokens in range.
#include "common.cuh"

namespace tsa {

namespace {

constexpr int kPoolTile = 2048, kPoolThreads = 256;

__global__ void k_fill_lkeep(int32_t *Lkeep, int B, int32_t value) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) Lkeep[b] = value;
}

// grid (ceil(L / kPoolTile), B*H); the tile and a halo of r tokens on each side are
// staged in shared memory.  kMax: max pooling, else mean (fp32 sum in token order, then
// one division by the count).
template <bool kMax>
__global__ void __launch_bounds__(kPoolThreads)
k_pool(const float *__restrict__ s_h, int L, int r, float *__restrict__ out) {
    extern __shared__ float buf[];
    const size_t row = blockIdx.y;
    const int t0 = blockIdx.x * kPoolTile;
    const int lo = t0 - r, n = kPoolTile + 2 * r;
    const float *in = s_h + row * L;
    for (int i = threadIdx.x; i < n; i += kPoolThreads) {
        const int t = lo + i;
        buf[i] = (t >= 0 && t < L) ? in[t] : 0.0f;  // out-of-range slots are never read
    }
    __syncthreads();
    const int t1 = min(L, t0 + kPoolTile);
    for (int t = t0 + threadIdx.x; t < t1; t += kPoolThreads) {
        const int a = max(0, t - r), b = min(L - 1, t + r);
        float acc = buf[a - lo];
        for (int u = a + 1; u <= b; ++u) acc = kMax ? fmaxf(acc, buf[u - lo]) : acc + buf[u - lo];
        out[row * L + t] = kMax ? acc : acc / (float)(b - a + 1);
    }
}

}  // namespace

cudaError_t launch_fill_lkeep(int B, int32_t value, int32_t *Lkeep, cudaStream_t st) {
    k_fill_lkeep<<<ceil_div(B, 128), 128, 0, st>>>(Lkeep, B, value);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_pool(const tsa_dims &dm, const float *s_h, int kind, int width, float *out,
                        cudaStream_t st) {
    const int r = width / 2;
    dim3 grid(ceil_div(dm.L, kPoolTile), dm.B * dm.H);
    const size_t smem = sizeof(float) * (kPoolTile + 2 * r);
    if (kind == TSA_POOL_MAX)
        k_pool<true><<<grid, kPoolThreads, smem, st>>>(s_h, dm.L, r, out);
    else
        k_pool<false><<<grid, kPoolThreads, smem, st>>>(s_h, dm.L, r, out);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace tsa

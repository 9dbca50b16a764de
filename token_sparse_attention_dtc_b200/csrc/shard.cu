// One layer sharded by KV group across GPUs: the partial layer score of a shard's heads
// and the fixed-order combination of every shard's partial.
//
// Method: "Token Sparse Attention" bxzpzcl.cn post §2.1 层级预算分配 and papernotes.org
// notes 关键设计 2: the layer score is the normalised sum over all heads of the head
// scores, s_l = u / sum_t u with u[t] = sum_h s_h[h, t], and every head keeps the same
// number of tokens.  u is the only quantity that couples the heads, so a GPU that holds
// some of the heads computes its partial sum over them, the partials are exchanged, and
// every GPU sums them in the same (rank) order: each GPU then holds the same s_l bit for
// bit and derives the same budget.
#include "common.cuh"

namespace tsa {

constexpr int kShardThreads = 256;

// u_part[b, t] = sum over the shard's heads h (in head order) of s_h[b, h, t].
// grid (ceil(L / 256), B).
__global__ void __launch_bounds__(kShardThreads)
k_head_sum(const float *__restrict__ s_h, int L, int H, float *__restrict__ u_part) {
    const int b = blockIdx.y, t = blockIdx.x * kShardThreads + threadIdx.x;
    if (t >= L) return;
    const float *col = s_h + (size_t)b * H * L + t;
    float u = 0.0f;
    for (int h = 0; h < H; ++h) u += __ldg(col + (size_t)h * L);
    u_part[(size_t)b * L + t] = u;
}

// u[b, t] = sum over r = 0, 1, ... (in that order) of u_parts[r, b, t], written to s_l
// unnormalised; part[b, block] = the block's sum of u in a fixed tree order.
// grid (nblk = ceil(L / 256), B).
__global__ void __launch_bounds__(kShardThreads)
k_combine_parts(const float *__restrict__ u_parts, int nparts, int B, int L, int nblk,
                float *__restrict__ s_l, float *__restrict__ part) {
    const int b = blockIdx.y, t = blockIdx.x * kShardThreads + threadIdx.x;
    float u = 0.0f;
    if (t < L) {
        for (int r = 0; r < nparts; ++r) u += __ldg(u_parts + ((size_t)r * B + b) * L + t);
        s_l[(size_t)b * L + t] = u;
    }
    __shared__ float red[kShardThreads];
    red[threadIdx.x] = u;
    __syncthreads();
    for (int o = kShardThreads / 2; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[(size_t)b * nblk + blockIdx.x] = red[0];
}

// Z_b = the block sums in a fixed order (the same in every block); s_l = u / Z_b.
__global__ void __launch_bounds__(kShardThreads)
k_combine_div(float *__restrict__ s_l, int L, int nblk, const float *__restrict__ part) {
    const int b = blockIdx.y, t = blockIdx.x * kShardThreads + threadIdx.x;
    float z = 0.0f;
    for (int i = threadIdx.x; i < nblk; i += kShardThreads) z += part[(size_t)b * nblk + i];
    __shared__ float red[kShardThreads];
    red[threadIdx.x] = z;
    __syncthreads();
    for (int o = kShardThreads / 2; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (t < L) s_l[(size_t)b * L + t] = s_l[(size_t)b * L + t] / red[0];
}

cudaError_t launch_head_sum(const tsa_dims &dm, const float *s_h, float *u_part,
                            cudaStream_t st) {
    k_head_sum<<<dim3(ceil_div(dm.L, kShardThreads), dm.B), kShardThreads, 0, st>>>(
        s_h, dm.L, dm.H, u_part);
    note_launches(1);
    return cudaGetLastError();
}

// Scratch: B * ceil(L / 256) floats at `part`.
cudaError_t launch_combine_parts(int B, int L, int nparts, const float *u_parts, float *s_l,
                                 float *part, cudaStream_t st) {
    const int nblk = ceil_div(L, kShardThreads);
    const dim3 grid(nblk, B);
    k_combine_parts<<<grid, kShardThreads, 0, st>>>(u_parts, nparts, B, L, nblk, s_l, part);
    k_combine_div<<<grid, kShardThreads, 0, st>>>(s_l, L, nblk, part);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace tsa

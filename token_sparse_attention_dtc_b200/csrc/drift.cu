// Choice of the sparse layers by inter-layer representation drift, on calibration hidden
// states.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 3:
//   R_l = E_t[ ||h_{l+1,t} - h_{l,t}||_2 / (||h_{l,t}||_2 + eps) ],
// the layers ranked by R, and { l : R^_l <= delta } made sparse (delta = 0.5: the half with
// the smallest drift); bxzpzcl.cn post §2 (only the layers below the median drift).
// R^_l = rank_l / N with rank_l the 1-based position in ascending R, ties to the lower
// layer; the mean runs over all T tokens.
//
// HBM-bound: every state row is read from DRAM once.  A warp owns one token and walks
// the layers in order, keeping the row of h_l in registers while it loads h_{l+1} (the
// generic kernel, for widths that are not 512 * 2^k bytes, re-reads h_l from cache); per token the two squared norms are summed in
// fp32 (lanes, then a fixed butterfly), the ratio is accumulated in fp64 in the warp's own
// shared-memory row, and the blocks' partials are summed in a fixed order, so R does not
// depend on scheduling.
#include "sm100.cuh"

namespace tsa {
using namespace sm100;

namespace {

// One token per warp: with 16-byte loads of both rows in flight for every warp of every
// resident block, the walk over the layers is not latency-bound.
constexpr int kDriftWarps = 8, kDriftTokensPerWarp = 1;
constexpr int kDriftTokensPerBlock = kDriftWarps * kDriftTokensPerWarp;

// Adds |b - a|^2 and |a|^2 of one 16-byte vector into the pairs (dd[0], dd[1]) and
// (hh[0], hh[1]) (even and odd elements), with paired fp32 instructions.
__device__ inline void acc_pair(const uint4 &a, const uint4 &b, float (&dd)[2], float (&hh)[2],
                                float) {
    const float *x = reinterpret_cast<const float *>(&a), *y = reinterpret_cast<const float *>(&b);
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
        float d0, d1;
        sub2(d0, d1, y[i], y[i + 1], x[i], x[i + 1]);
        fma2(dd[0], dd[1], d0, d1, d0, d1, dd[0], dd[1]);
        fma2(hh[0], hh[1], x[i], x[i + 1], x[i], x[i + 1], hh[0], hh[1]);
    }
}
// bf16: the low element of a word is its low 16 bits shifted up, the high one its high 16
// bits masked (exact conversions).
__device__ inline void acc_pair(const uint4 &a, const uint4 &b, float (&dd)[2], float (&hh)[2],
                                __nv_bfloat16) {
    const uint32_t xa[4] = {a.x, a.y, a.z, a.w}, yb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float x0 = __uint_as_float(xa[i] << 16), x1 = __uint_as_float(xa[i] & 0xffff0000u);
        const float y0 = __uint_as_float(yb[i] << 16), y1 = __uint_as_float(yb[i] & 0xffff0000u);
        float d0, d1;
        sub2(d0, d1, y0, y1, x0, x1);
        fma2(dd[0], dd[1], d0, d1, d0, d1, dd[0], dd[1]);
        fma2(hh[0], hh[1], x0, x1, x0, x1, hh[0], hh[1]);
    }
}

// grid ceil(T / kDriftTokensPerBlock); dynamic shared memory kDriftWarps * N doubles.
template <typename T>
__global__ void __launch_bounds__(kDriftWarps * 32)
k_drift_partial(const uint4 *__restrict__ h, int N, long long Ttok, int vec_per_row, float eps,
                double *__restrict__ partial) {
    extern __shared__ double acc[];  // [kDriftWarps][N]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kDriftWarps * N; i += blockDim.x) acc[i] = 0.0;
    __syncthreads();
    const size_t state = (size_t)Ttok * vec_per_row;  // uint4 per state
    for (int k = 0; k < kDriftTokensPerWarp; ++k) {
        const long long t = (long long)blockIdx.x * kDriftTokensPerBlock + k * kDriftWarps + warp;
        if (t >= Ttok) break;
        for (int l = 0; l < N; ++l) {
            const uint4 *a = h + (size_t)l * state + (size_t)t * vec_per_row;
            const uint4 *b = a + state;
            float d2[2] = {0.0f, 0.0f}, h2[2] = {0.0f, 0.0f};
#pragma unroll 4
            for (int v = lane; v < vec_per_row; v += 32) acc_pair(a[v], b[v], d2, h2, T());
            float dd = d2[0] + d2[1], hh = h2[0] + h2[1];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                dd += __shfl_xor_sync(0xffffffffu, dd, o);
                hh += __shfl_xor_sync(0xffffffffu, hh, o);
            }
            if (lane == 0) acc[warp * N + l] += (double)(sqrtf(dd) / (sqrtf(hh) + eps));
        }
    }
    __syncthreads();
    for (int l = threadIdx.x; l < N; l += blockDim.x) {
        double s = 0.0;
        for (int w = 0; w < kDriftWarps; ++w) s += acc[w * N + l];
        partial[(size_t)blockIdx.x * N + l] = s;
    }
}

// Same, with the row of h_l kept in registers (V uint4 per lane, d_model * esize =
// 512 * V bytes, V <= 16): each row is loaded once, all V loads of the next row in flight at once.
template <typename T, int V>
__global__ void __launch_bounds__(kDriftWarps * 32)
k_drift_partial_reg(const uint4 *__restrict__ h, int N, long long Ttok, float eps,
                    double *__restrict__ partial) {
    extern __shared__ double acc[];  // [kDriftWarps][N]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kDriftWarps * N; i += blockDim.x) acc[i] = 0.0;
    __syncthreads();
    const size_t state = (size_t)Ttok * V * 32;
    const long long t = (long long)blockIdx.x * kDriftTokensPerBlock + warp;
    if (t < Ttok) {
        const uint4 *row = h + (size_t)t * V * 32 + lane;
        uint4 cur[V];
#pragma unroll
        for (int v = 0; v < V; ++v) cur[v] = __ldcs(row + v * 32);
        for (int l = 0; l < N; ++l) {
            row += state;
            uint4 nxt[V];
#pragma unroll
            for (int v = 0; v < V; ++v) nxt[v] = __ldcs(row + v * 32);
            float d2[2] = {0.0f, 0.0f}, h2[2] = {0.0f, 0.0f};
#pragma unroll
            for (int v = 0; v < V; ++v) acc_pair(cur[v], nxt[v], d2, h2, T());
            float dd = d2[0] + d2[1], hh = h2[0] + h2[1];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                dd += __shfl_xor_sync(0xffffffffu, dd, o);
                hh += __shfl_xor_sync(0xffffffffu, hh, o);
            }
            if (lane == 0) acc[warp * N + l] += (double)(sqrtf(dd) / (sqrtf(hh) + eps));
#pragma unroll
            for (int v = 0; v < V; ++v) cur[v] = nxt[v];
        }
    }
    __syncthreads();
    for (int l = threadIdx.x; l < N; l += blockDim.x) {
        double s = 0.0;
        for (int w = 0; w < kDriftWarps; ++w) s += acc[w * N + l];
        partial[(size_t)blockIdx.x * N + l] = s;
    }
}

// One block: R_l = sum of the partials in block order / T, then the rank mask.
__global__ void k_drift_final(const double *__restrict__ partial, int nblk, int N, long long Ttok,
                              double delta, double *__restrict__ R, int32_t *__restrict__ mask) {
    extern __shared__ double r[];
    for (int l = threadIdx.x; l < N; l += blockDim.x) {
        double s = 0.0;
        for (int b = 0; b < nblk; ++b) s += partial[(size_t)b * N + l];
        r[l] = s / (double)Ttok;
        R[l] = r[l];
    }
    __syncthreads();
    for (int l = threadIdx.x; l < N; l += blockDim.x) {
        int rank = 1;
        for (int m = 0; m < N; ++m) rank += (r[m] < r[l] || (r[m] == r[l] && m < l)) ? 1 : 0;
        mask[l] = ((double)rank / (double)N <= delta) ? 1 : 0;
    }
}

}  // namespace

size_t drift_workspace_bytes(int N, long long Ttok) {
    const long long nblk = (Ttok + kDriftTokensPerBlock - 1) / kDriftTokensPerBlock;
    return align256(sizeof(Control)) + align256((size_t)nblk * N * sizeof(double));
}

cudaError_t launch_drift(int N, long long Ttok, int d_model, int dtype, const void *h, double eps,
                         double delta, double *R, int32_t *mask, char *ws, cudaStream_t st) {
    const long long nblk = (Ttok + kDriftTokensPerBlock - 1) / kDriftTokensPerBlock;
    double *partial = reinterpret_cast<double *>(ws + align256(sizeof(Control)));
    const int esz = dtype == TSA_F32 ? 4 : 2, vpr = d_model * esz / 16;
    const size_t smem = sizeof(double) * kDriftWarps * N;
    const unsigned g = (unsigned)nblk, nt = kDriftWarps * 32;
#define TSA_DRIFT_REG(TT, VV) \
    k_drift_partial_reg<TT, VV><<<g, nt, smem, st>>>((const uint4 *)h, N, Ttok, (float)eps, partial)
    const bool bf = dtype != TSA_F32;
    if (vpr % 32 == 0 && vpr / 32 <= 16 && (vpr / 32 & (vpr / 32 - 1)) == 0) {
        switch (vpr / 32) {
            case 1: if (bf) TSA_DRIFT_REG(__nv_bfloat16, 1); else TSA_DRIFT_REG(float, 1); break;
            case 2: if (bf) TSA_DRIFT_REG(__nv_bfloat16, 2); else TSA_DRIFT_REG(float, 2); break;
            case 4: if (bf) TSA_DRIFT_REG(__nv_bfloat16, 4); else TSA_DRIFT_REG(float, 4); break;
            case 8: if (bf) TSA_DRIFT_REG(__nv_bfloat16, 8); else TSA_DRIFT_REG(float, 8); break;
            default: if (bf) TSA_DRIFT_REG(__nv_bfloat16, 16); else TSA_DRIFT_REG(float, 16); break;
        }
    } else if (dtype == TSA_F32)
        k_drift_partial<float><<<(unsigned)nblk, kDriftWarps * 32, smem, st>>>(
            (const uint4 *)h, N, Ttok, vpr, (float)eps, partial);
    else
        k_drift_partial<__nv_bfloat16><<<(unsigned)nblk, kDriftWarps * 32, smem, st>>>(
            (const uint4 *)h, N, Ttok, vpr, (float)eps, partial);
    k_drift_final<<<1, 256, sizeof(double) * N, st>>>(partial, (int)nblk, N, Ttok, delta, R, mask);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace tsa

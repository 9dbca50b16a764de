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
// HBM-bound: every state row is read from DRAM once.  A warp owns one token at a time and
// walks the layers in order over slices of the row (4 KB, or less for narrower rows), one
// slice after another, with a ring of three register buffers: the loads of rows l + 1 and
// l + 2 are in flight while rows l and l + 1 are compared.  Rows that are not a multiple of
// 512 bytes take a generic walk that re-reads h_l from cache.  Per token the two squared
// norms are summed in fp32 (lanes, then a fixed butterfly, then the slices in order), and
// the ratio is accumulated in fp64 into one of a fixed number of token slots (token t into
// slot t mod P); the slots are summed in a fixed order, so R depends neither on scheduling
// nor on the grid.
#include "sm100.cuh"

namespace tsa {
using namespace sm100;

namespace {

// Two warps per block, persistent grid (as many blocks as fit at once).  The widest walk
// (a ring of three 4 KB buffers) takes 128 registers: 16 warps per SM, each with up to
// 8 KB of loads in flight.
constexpr int kDriftWarps = 2;
// Partial sums per layer: token t goes to slot t mod min(T, kDriftSlots).
constexpr int kDriftSlots = 4096;
// Slice width (uint4 per lane; 8 = 4 KB) and depth of the register ring.
constexpr int kSliceV = 8, kRing = 3;

long long drift_slots(long long Ttok) { return Ttok < kDriftSlots ? Ttok : kDriftSlots; }

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

// Sums |b - a|^2 and |a|^2 over the lanes of a warp (fixed butterfly; every lane ends
// with the same values).
__device__ inline void warp_sum2(float (&d2)[2], float (&h2)[2], float &dd, float &hh) {
    dd = d2[0] + d2[1];
    hh = h2[0] + h2[1];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        dd += __shfl_xor_sync(0xffffffffu, dd, o);
        hh += __shfl_xor_sync(0xffffffffu, hh, o);
    }
}

// Lane 0: slice s of S of layer l gave the sums (dd, hh); the last slice adds the token's
// ratio to the slot.
__device__ inline void drift_note(double *acc, float2 *part, int l, int s, int S, float dd,
                                  float hh, float eps) {
    if (S > 1) {
        if (s > 0) {
            dd += part[l].x;
            hh += part[l].y;
        }
        if (s < S - 1) {
            part[l] = make_float2(dd, hh);
            return;
        }
    }
    acc[l] += (double)(sqrtf(dd) / (sqrtf(hh) + eps));
}

// One step of a walk with a ring of R register buffers: the loads of row l + R - 1 go
// into fut, then rows l (cur) and l + 1 (nxt) are compared.
template <typename T, int V, int R>
__device__ __forceinline__ void ring_step(const uint4 (&cur)[V], const uint4 (&nxt)[V],
                                          uint4 (&fut)[V], const uint4 *row0, size_t state,
                                          int l, int N, int s, int S, int lane, double *acc,
                                          float2 *part, float eps) {
    if (l + R - 1 <= N) {
        const uint4 *r = row0 + (size_t)(l + R - 1) * state;
#pragma unroll
        for (int v = 0; v < V; ++v) fut[v] = __ldcs(r + v * 32);
    }
    float d2[2] = {0.0f, 0.0f}, h2[2] = {0.0f, 0.0f};
#pragma unroll
    for (int v = 0; v < V; ++v) acc_pair(cur[v], nxt[v], d2, h2, T());
    float dd, hh;
    warp_sum2(d2, h2, dd, hh);
    if (lane == 0) drift_note(acc, part, l, s, S, dd, hh, eps);
}

// Register cap for a ring of R buffers of V uint4 (the buffers and 32 more).
constexpr int drift_regs(int V, int R) {
    return R * V * 4 + 32 < 64 ? 64 : (R * V * 4 + 32 > 232 ? 232 : (R * V * 4 + 39) / 8 * 8);
}

// Persistent grid; warp w of the grid owns the slots w, w + (warps in the grid), ...; per
// slot it walks the tokens t = slot, slot + P, ... and writes the slot's sums to
// partial[l * P + slot].  V > 0: a row is S slices of V uint4 per lane (vpr = 32 * V * S),
// walked with a ring of R register buffers.  V == 0: the generic walk over vpr uint4 (S ==
// 1).  Dynamic shared memory: kDriftWarps * N doubles, then kDriftWarps * N float2.
template <typename T, int V, int R>
__global__ void __maxnreg__(drift_regs(V, R))
k_drift_walk(const uint4 *__restrict__ h, int N, long long Ttok, int vpr, int S, int P,
             float eps, double *__restrict__ partial) {
    extern __shared__ double sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double *acc = sm + (size_t)warp * N;
    float2 *part = reinterpret_cast<float2 *>(sm + (size_t)kDriftWarps * N) + (size_t)warp * N;
    const size_t state = (size_t)Ttok * vpr;  // uint4 per state
    const int nw = gridDim.x * kDriftWarps;
    for (int p = blockIdx.x * kDriftWarps + warp; p < P; p += nw) {
        for (int l = lane; l < N; l += 32) acc[l] = 0.0;
        __syncwarp();
        for (long long t = p; t < Ttok; t += P) {
            if constexpr (V == 0) {
                for (int l = 0; l < N; ++l) {
                    const uint4 *a = h + (size_t)l * state + (size_t)t * vpr;
                    const uint4 *b = a + state;
                    float d2[2] = {0.0f, 0.0f}, h2[2] = {0.0f, 0.0f};
#pragma unroll 4
                    for (int v = lane; v < vpr; v += 32) acc_pair(a[v], b[v], d2, h2, T());
                    float dd, hh;
                    warp_sum2(d2, h2, dd, hh);
                    if (lane == 0) drift_note(acc, part, l, 0, 1, dd, hh, eps);
                }
            } else {
                for (int s = 0; s < S; ++s) {
                    const uint4 *row0 = h + (size_t)t * vpr + s * V * 32 + lane;
                    uint4 b[R][V];
#pragma unroll
                    for (int j = 0; j < R - 1; ++j)
                        if (j <= N) {
#pragma unroll
                            for (int v = 0; v < V; ++v)
                                b[j][v] = __ldcs(row0 + (size_t)j * state + v * 32);
                        }
                    for (int l0 = 0; l0 < N; l0 += R) {
#pragma unroll
                        for (int j = 0; j < R; ++j)
                            if (l0 + j < N)
                                ring_step<T, V, R>(b[j], b[(j + 1) % R], b[(j + R - 1) % R], row0,
                                                   state, l0 + j, N, s, S, lane, acc, part, eps);
                    }
                }
            }
        }
        __syncwarp();
        for (int l = lane; l < N; l += 32) partial[(size_t)l * P + p] = acc[l];
        __syncwarp();
    }
}

// One block: warp w sums layers w, w + (warps), ... over the P slots (lanes in a strided
// order, then a fixed butterfly), R_l = sum / T; then the rank mask.
__global__ void __launch_bounds__(1024)
k_drift_final(const double *__restrict__ partial, int P, int N, long long Ttok, double delta,
              double *__restrict__ R, int32_t *__restrict__ mask) {
    extern __shared__ double r[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
    for (int l = warp; l < N; l += nwarp) {
        const double *q = partial + (size_t)l * P;
        double s = 0.0;
        for (int p = lane; p < P; p += 32) s += q[p];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) {
            r[l] = s / (double)Ttok;
            R[l] = r[l];
        }
    }
    __syncthreads();
    for (int l = threadIdx.x; l < N; l += blockDim.x) {
        int rank = 1;
        for (int m = 0; m < N; ++m) rank += (r[m] < r[l] || (r[m] == r[l] && m < l)) ? 1 : 0;
        mask[l] = ((double)rank / (double)N <= delta) ? 1 : 0;
    }
}

template <typename T, int V>
cudaError_t drift_walk(const uint4 *h, int N, long long Ttok, int vpr, int S, int P, float eps,
                       double *partial, cudaStream_t st) {
    const size_t smem = kDriftWarps * N * (sizeof(double) + sizeof(float2));
    auto *k = k_drift_walk<T, V, kRing>;
    int dev = 0, nsm = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kDriftWarps * 32, smem);
    if (e != cudaSuccess) return e;
    const long long need = (P + kDriftWarps - 1) / kDriftWarps;
    const long long fit = (long long)nsm * (per_sm > 0 ? per_sm : 1);
    k<<<(unsigned)(need < fit ? need : fit), kDriftWarps * 32, smem, st>>>(h, N, Ttok, vpr, S, P,
                                                                          eps, partial);
    return cudaGetLastError();
}

}  // namespace

size_t drift_workspace_bytes(int N, long long Ttok) {
    return align256(sizeof(Control)) + align256((size_t)drift_slots(Ttok) * N * sizeof(double));
}

cudaError_t launch_drift(int N, long long Ttok, int d_model, int dtype, const void *h, double eps,
                         double delta, double *R, int32_t *mask, char *ws, cudaStream_t st) {
    const int P = (int)drift_slots(Ttok);
    double *partial = reinterpret_cast<double *>(ws + align256(sizeof(Control)));
    const int esz = dtype == TSA_F32 ? 4 : 2, vpr = d_model * esz / 16;
    const uint4 *hv = static_cast<const uint4 *>(h);
    const float e = (float)eps;
    const bool bf = dtype != TSA_F32;
    // A row of vpr uint4 is S slices of V uint4 per lane, V the largest of 8, 4, 2, 1
    // dividing vpr / 32; rows that are not a multiple of 512 bytes take the generic walk.
    const int w = vpr % 32 == 0 ? vpr / 32 : 0;
    const int V = w == 0 ? 0 : w % kSliceV == 0 ? kSliceV : w % 4 == 0 ? 4 : w % 2 == 0 ? 2 : 1;
    const int S = V > 0 ? w / V : 1;
    cudaError_t err;
#define TSA_DRIFT(VV)                                                                       \
    (bf ? drift_walk<__nv_bfloat16, VV>(hv, N, Ttok, vpr, S, P, e, partial, st)             \
        : drift_walk<float, VV>(hv, N, Ttok, vpr, S, P, e, partial, st))
    switch (V) {
        case kSliceV: err = TSA_DRIFT(kSliceV); break;
        case 4: err = TSA_DRIFT(4); break;
        case 2: err = TSA_DRIFT(2); break;
        case 1: err = TSA_DRIFT(1); break;
        default: err = TSA_DRIFT(0); break;
    }
#undef TSA_DRIFT
    if (err != cudaSuccess) return err;
    const int nt = N >= 32 ? 1024 : 32 * N;
    k_drift_final<<<1, nt, sizeof(double) * N, st>>>(partial, P, N, Ttok, delta, R, mask);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace tsa

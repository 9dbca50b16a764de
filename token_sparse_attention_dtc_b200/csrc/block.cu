// Block-sparse pattern inside the compressed space.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键发现 (token sparsity stacked on
// block-level sparsity is the most valuable pairing) and the bxzpzcl.cn post §3.2
// 与现有方案的兼容性 ("token selection first, then block-sparse computation").  The block
// choice is this project's own definition (the pages give none):
//   query pair p = compressed rows [256p, 256p + 256), key block j = rows [128j, 128j + 128);
//   z[p][j] = scale * < mean of the pair's Q̂ rows, mean of block j's K̂ rows > for j < 2p;
//   kept: j = 0, the diagonal blocks 2p and 2p + 1, and every j < 2p with
//   z[p][j] >= max_j z[p][j] - theta (one fp32 subtraction, fp32 comparison).
// Means are fp32 sums in a fixed order; each dot product is an fp32 FMA chain over the
// columns in order, so logits and masks do not depend on scheduling.
#include "common.cuh"

namespace tsa {

namespace {

constexpr int kBlockThreads = 256;

// grid (B*H, NB): the mean of block j's K̂ rows (full blocks only) and, for even j, the
// mean of pair j/2's Q̂ rows.  256 threads = 16 row lanes x 16 column groups of 8 (16-byte
// loads): row lane r sums rows r, r+16, ... of its 8 columns, then the 16 partial sums
// are added in row-lane order (a fixed order).
template <typename T>
__global__ void __launch_bounds__(kBlockThreads)
k_block_means(const T *__restrict__ Qh, const T *__restrict__ Kh, const int32_t *__restrict__ Lkeep,
              int L, int H, int d, int NP, int NB, float *__restrict__ qbar,
              float *__restrict__ kbar) {
    constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte load
    __shared__ float part[16][16 * EPV];
    const int bh = blockIdx.x, j = blockIdx.y, b = bh / H;
    const int Lk = min(max(Lkeep[b], 0), L);  // clamped: rows past L untouched
    const int rl = threadIdx.x / 16, cg = threadIdx.x % 16;
    const size_t base = (size_t)bh * L * d;
    auto mean_rows = [&](const T *src, int r0, int r1, float *dst) {
        for (int cb = 0; cb < d; cb += 16 * EPV) {  // one pass per 16 * EPV columns
            const int c0 = cb + cg * EPV;
            const bool active = c0 < d;
            float acc[EPV];
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[e] = 0.0f;
            if (active)
                for (int i = r0 + rl; i < r1; i += 16) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(src + base + (size_t)i * d + c0);
                    const T *x = reinterpret_cast<const T *>(&v);
#pragma unroll
                    for (int e = 0; e < EPV; ++e) acc[e] += Elem<T>::to_f(x[e]);
                }
            __syncthreads();
            if (active)
#pragma unroll
                for (int e = 0; e < EPV; ++e) part[rl][c0 - cb + e] = acc[e];
            __syncthreads();
            for (int c = threadIdx.x; c < min(16 * EPV, d - cb); c += kBlockThreads) {
                float t = 0.0f;
                for (int r = 0; r < 16; ++r) t += part[r][c];
                dst[cb + c] = t / (float)(r1 - r0);
            }
        }
    };
    if (128 * j + 128 <= Lk) mean_rows(Kh, 128 * j, 128 * j + 128, kbar + ((size_t)bh * NB + j) * d);
    if ((j & 1) == 0 && 128 * j < Lk) {
        const int p = j / 2;
        mean_rows(Qh, 256 * p, min(Lk, 256 * p + 256), qbar + ((size_t)bh * NP + p) * d);
    }
}

// grid (ceil(NP / kPairsPerCta), B*H), 256 threads: 32 pairs per CTA, 4 per warp.  Key
// means are staged 32 blocks at a time (a chunk = one mask word); lane j of a warp
// computes the logit of its pair against block 32w + j.  Pass 1 takes each pair's max,
// pass 2 recomputes the logits, writes them if asked, and forms each mask word with a
// ballot.
constexpr int kPairsPerCta = 32, kPairsPerWarp = kPairsPerCta / (kBlockThreads / 32);

__global__ void __launch_bounds__(kBlockThreads)
k_block_select(const float *__restrict__ qbar, const float *__restrict__ kbar,
               const int32_t *__restrict__ Lkeep, int L, int H, int d, int NP, int NB, int NW,
               float scale, float theta, float *__restrict__ logits, uint32_t *__restrict__ mask) {
    extern __shared__ float4 sm4[];  // qs[kPairsPerCta][d], ks[32][d + 4] (16-byte aligned)
    float *qs = reinterpret_cast<float *>(sm4), *ks = qs + kPairsPerCta * d;
    const int kst = d + 4;  // 16-byte loads of 8 consecutive lanes hit distinct banks
    const int bh = blockIdx.y, b = bh / H, p0 = blockIdx.x * kPairsPerCta;
    const int Lk = min(max(Lkeep[b], 0), L);  // clamped: rows past L untouched
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int npair = max(0, min(kPairsPerCta, min(NP, ceil_div(Lk, 256)) - p0));
    for (int e = threadIdx.x; e < kPairsPerCta * d; e += kBlockThreads)
        qs[e] = e < npair * d ? qbar[((size_t)bh * NP + p0) * d + e] : 0.0f;
    const int nchunk_dot = ceil_div(2 * (p0 + npair - 1), 32);  // chunks with candidates
    float mx[kPairsPerWarp];
#pragma unroll
    for (int k = 0; k < kPairsPerWarp; ++k) mx[k] = -INFINITY;
    auto stage = [&](int w) {
        __syncthreads();
        const int j0 = 32 * w, nj = min(32, NB - j0);
        for (int e = threadIdx.x; e < 32 * d; e += kBlockThreads) {
            const int jj = e / d, c = e % d;
            ks[jj * kst + c] = jj < nj ? kbar[((size_t)bh * NB + j0 + jj) * d + c] : 0.0f;
        }
        __syncthreads();
    };
    // Logits of this warp's pairs against block 32w + lane (staged): one 16-byte load of
    // the key mean feeds all kPairsPerWarp pairs.  Each dot runs over c in order.
    auto logits4 = [&](float (&z)[kPairsPerWarp]) {
        float acc[kPairsPerWarp];
#pragma unroll
        for (int k = 0; k < kPairsPerWarp; ++k) acc[k] = 0.0f;
        const float4 *kr = reinterpret_cast<const float4 *>(ks + lane * kst);
        for (int c4 = 0; c4 < d / 4; ++c4) {
            const float4 kv = kr[c4];
#pragma unroll
            for (int k = 0; k < kPairsPerWarp; ++k) {
                const float4 qv = reinterpret_cast<const float4 *>(qs + (warp * kPairsPerWarp + k) * d)[c4];
                acc[k] = fmaf(qv.x, kv.x, acc[k]);
                acc[k] = fmaf(qv.y, kv.y, acc[k]);
                acc[k] = fmaf(qv.z, kv.z, acc[k]);
                acc[k] = fmaf(qv.w, kv.w, acc[k]);
            }
        }
#pragma unroll
        for (int k = 0; k < kPairsPerWarp; ++k) z[k] = scale * acc[k];
    };
    for (int w = 0; w < nchunk_dot; ++w) {  // pass 1: max over the candidates j < 2p
        stage(w);
        float z[kPairsPerWarp];
        logits4(z);
#pragma unroll
        for (int k = 0; k < kPairsPerWarp; ++k) {
            const int pl = warp * kPairsPerWarp + k, p = p0 + pl, j = 32 * w + lane;
            if (pl < npair && j < 2 * p) mx[k] = fmaxf(mx[k], z[k]);
        }
    }
#pragma unroll
    for (int k = 0; k < kPairsPerWarp; ++k)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], o));
    for (int w = 0; w < NW; ++w) {  // pass 2: logits and mask words
        const bool dots = w < nchunk_dot;
        float zz[kPairsPerWarp] = {};
        if (dots) {
            stage(w);
            logits4(zz);
        }
#pragma unroll
        for (int k = 0; k < kPairsPerWarp; ++k) {
            const int pl = warp * kPairsPerWarp + k, p = p0 + pl, j = 32 * w + lane;
            if (p0 + pl >= NP) continue;
            if (pl >= npair) {  // pair past L': nothing kept
                if (lane == 0) mask[((size_t)bh * NP + p) * NW + w] = 0u;
                if (logits && j < NB) logits[((size_t)bh * NP + p) * NB + j] = __int_as_float(0x7fc00000);
                continue;
            }
            const bool cand = j < 2 * p;
            const float z = zz[k];
            bool keep = j == 0 || j == 2 * p || (j == 2 * p + 1 && 256 * p + 128 < Lk);
            if (cand && j > 0 && z >= mx[k] - theta) keep = true;
            const uint32_t bits = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) mask[((size_t)bh * NP + p) * NW + w] = bits;
            if (logits && j < NB)
                logits[((size_t)bh * NP + p) * NB + j] = cand ? z : __int_as_float(0x7fc00000);
        }
    }
}

}  // namespace

size_t block_scratch_bytes(const tsa_dims &dm) {
    const size_t NP = ceil_div(dm.L, 256), NB = ceil_div(dm.L, 128);
    return align256((size_t)dm.B * dm.H * (NP + NB) * dm.d * sizeof(float));
}

size_t block_mask_words(const tsa_dims &dm) {
    const size_t NP = ceil_div(dm.L, 256), NB = ceil_div(dm.L, 128);
    return (size_t)dm.B * dm.H * NP * ceil_div((int)NB, 32);
}

cudaError_t launch_block_select(const tsa_dims &dm, const void *Qh, const void *Kh,
                                const int32_t *Lkeep, float scale, float theta, float *logits,
                                uint32_t *mask, char *scratch, cudaStream_t st) {
    const int NP = ceil_div(dm.L, 256), NB = ceil_div(dm.L, 128), NW = ceil_div(NB, 32);
    float *qbar = reinterpret_cast<float *>(scratch);
    float *kbar = qbar + (size_t)dm.B * dm.H * NP * dm.d;
    dim3 g1(dm.B * dm.H, NB);
    if (dm.dtype == TSA_F32)
        k_block_means<float><<<g1, kBlockThreads, 0, st>>>((const float *)Qh, (const float *)Kh,
                                                           Lkeep, dm.L, dm.H, dm.d, NP, NB, qbar, kbar);
    else
        k_block_means<__nv_bfloat16><<<g1, kBlockThreads, 0, st>>>(
            (const __nv_bfloat16 *)Qh, (const __nv_bfloat16 *)Kh, Lkeep, dm.L, dm.H, dm.d, NP, NB,
            qbar, kbar);
    const size_t zsm = sizeof(float) * (kPairsPerCta * dm.d + 32 * (dm.d + 4));
    if (zsm > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            k_block_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)zsm);
        if (e != cudaSuccess) return e;
    }
    k_block_select<<<dim3(ceil_div(NP, kPairsPerCta), dm.B * dm.H), kBlockThreads, zsm, st>>>(
        qbar, kbar, Lkeep, dm.L, dm.H, dm.d, NP, NB, NW, scale, theta, logits, mask);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace tsa

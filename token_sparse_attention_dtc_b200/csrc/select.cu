// Per-head top-L' selection: block-wide radix selection over the IEEE bits of the
// (non-negative) fp32 head scores, with integer histograms only, so the results do not
// depend on thread scheduling; then an ordered compaction.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 2 (each head keeps its
// own top-k_keep tokens); gist.science §2 "Head-Wise Selection".
#include "common.cuh"

namespace tsa {

constexpr int kSelThreads = 1024;

// Exclusive block-wide prefix count of a 0/1 flag; returns the prefix, sets total.
__device__ inline int block_scan_flag(bool f, int *warp_tot, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    const int in_warp = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
        const int v = warp_tot[lane];
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        warp_tot[lane] = x - v;     // exclusive
        warp_tot[32 + lane] = x;    // inclusive
    }
    __syncthreads();
    const int r = warp_tot[warp] + in_warp;
    total = warp_tot[32 + 31];
    __syncthreads();
    return r;
}

// One block per (b, h).  Threshold key v* and the number of tokens equal to v* to take
// (the lowest-index ones) by descending radix selection, then an ordered compaction
// that writes kept tokens ascending followed by the rest ascending.
__global__ void __launch_bounds__(kSelThreads)
k_select(const float *__restrict__ s_h, int L, int H, const int32_t *__restrict__ Lkeep,
         int32_t *__restrict__ idx, Control *ctl) {
    const int bh = blockIdx.x, b = bh / H;
    const float *s = s_h + (size_t)bh * L;
    int32_t *out = idx + (size_t)bh * L;
    const int keep = Lkeep[b];
    __shared__ unsigned int cnt[256];
    __shared__ int warp_tot[64];
    __shared__ uint32_t s_prefix, s_mask;
    __shared__ int s_need;
    if (keep <= 0 || keep >= L) {  // nothing or everything kept: identity order
        for (int t = threadIdx.x; t < L; t += blockDim.x) out[t] = t;
        if (keep < 0 || keep > L) report_error(ctl, TSA_ERR_INVALID_ARG, 2);
        return;
    }
    if (threadIdx.x == 0) { s_prefix = 0; s_mask = 0; s_need = keep; }
    bool bad = false;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) cnt[i] = 0;
        __syncthreads();
        const uint32_t prefix = s_prefix, mask = s_mask;
        for (int t = threadIdx.x; t < L; t += blockDim.x) {
            const uint32_t key = score_key<kHeadScoreMax>(s[t], bad);
            if ((key & mask) == prefix) atomicAdd(&cnt[(key >> shift) & 255], 1u);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int need = s_need, dg = 0;
            for (int i = 255; i >= 0; --i) {
                if ((int)cnt[i] >= need) { dg = i; break; }
                need -= cnt[i];
            }
            s_need = need;
            s_prefix = prefix | ((uint32_t)dg << shift);
            s_mask = mask | (255u << shift);
        }
        __syncthreads();
    }
    const uint32_t thr = s_prefix;
    const int take_eq = s_need;  // tokens equal to thr that are kept, lowest index first
    int base_sel = 0, base_rest = keep, base_eq = 0;
    for (int t0 = 0; t0 < L; t0 += blockDim.x) {
        const int t = t0 + threadIdx.x;
        bool dummy = false;
        const uint32_t key = t < L ? score_key<kHeadScoreMax>(s[t], dummy) : 0u;
        const bool eq = t < L && key == thr;
        int n_eq;
        const int eq_rank = base_eq + block_scan_flag(eq, warp_tot, n_eq);
        const bool sel = t < L && (key > thr || (eq && eq_rank < take_eq));
        int n_sel;
        const int pos = block_scan_flag(sel, warp_tot, n_sel);
        if (t < L) {
            if (sel) out[base_sel + pos] = t;
            else out[base_rest + (t - t0 - pos)] = t;
        }
        base_sel += n_sel;
        base_rest += min((int)blockDim.x, L - t0) - n_sel;
        base_eq += n_eq;
    }
    if (bad) report_error(ctl, TSA_ERR_NONFINITE, 3);
}

cudaError_t launch_select(const tsa_dims &dm, const float *s_h, const int32_t *Lkeep,
                          int32_t *idx, Control *ctl, cudaStream_t st) {
    k_select<<<dm.B * dm.H, kSelThreads, 0, st>>>(s_h, dm.L, dm.H, Lkeep, idx, ctl);
    return cudaGetLastError();
}

}  // namespace tsa

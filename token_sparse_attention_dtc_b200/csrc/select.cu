// Per-head top-L' selection over the whole GPU.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 2 (each head keeps its
// own top-k_keep tokens); gist.science §2 "Head-Wise Selection".  Ties go to the lower
// token index and the kept tokens are listed in ascending order.
//
// No sort: the threshold key (the L'-th largest score of the row, as the IEEE bits of a
// non-negative float, which order like the values) is found digit by digit with three
// grid-wide count histograms (12, 12 and 8 bits; shared-memory privatised, global
// integer atomics), each followed by a one-block scan per row.  Then an ordered
// compaction: per 4096-token chunk count the tokens above the threshold and equal to it,
// scan the chunk counts per row, and write every chunk's kept tokens and the rest in
// token order.  All state is integer, so the result does not depend on scheduling.
#include "common.cuh"

namespace tsa {

namespace {

constexpr int kHistThreads = 256, kHistPerThread = 16;  // 4096 tokens per histogram block
constexpr int kScanThreads = 1024;
constexpr int kChunk = 4096, kWriteThreads = 1024;

__host__ __device__ constexpr int level_shift(int lv) { return lv == 0 ? 20 : (lv == 1 ? 8 : 0); }
__host__ __device__ constexpr int level_bits(int lv) { return lv == 2 ? 8 : 12; }

struct ChunkInfo {
    int32_t n_gt, n_eq;  // tokens above / equal to the threshold in the chunk
    int32_t sel_base;    // kept tokens before the chunk
    int32_t eq_before;   // tokens equal to the threshold before the chunk
};

// Exclusive block-wide prefix count of a 0/1 flag (token order = thread order).
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
        warp_tot[lane] = x - v;   // exclusive
        warp_tot[32 + lane] = x;  // inclusive
    }
    __syncthreads();
    const int r = warp_tot[warp] + in_warp;
    total = warp_tot[32 + 31];
    __syncthreads();
    return r;
}

// Exclusive block-wide prefix sum of an int over kScanThreads threads; returns the total.
__device__ inline int block_scan_int(int v, int &total) {
    __shared__ int wt[32];
    __shared__ int s_tot;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wt[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int w0 = wt[lane];
        int w = w0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane == 31) s_tot = w;
        wt[lane] = w - w0;
    }
    __syncthreads();
    const int r = wt[warp] + x - v;
    total = s_tot;
    __syncthreads();
    return r;
}

__global__ void k_sel_init(const int32_t *__restrict__ Lkeep, int L, int H, int rows,
                           SelectState *st, Control *ctl) {
    const int row = blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    const int keep = Lkeep[row / H];
    SelectState s{};
    s.need = keep;
    s.identity = (keep <= 0 || keep >= L) ? 1 : 0;  // nothing or everything kept
    st[row] = s;
    if (keep < 0 || keep > L) report_error(ctl, TSA_ERR_INVALID_ARG, 2);
}

// grid (ceil(L / 4096), rows), 256 threads, shared memory 4 bytes per digit.
__global__ void __launch_bounds__(kHistThreads)
k_sel_hist(const float *__restrict__ s_h, int L, int lv, const SelectState *__restrict__ st,
           unsigned int *hist, Control *ctl) {
    extern __shared__ unsigned int hcnt[];
    const int row = blockIdx.y;
    const SelectState S = st[row];
    if (S.identity) return;
    const int shift = level_shift(lv), nb = 1 << level_bits(lv);
    for (int i = threadIdx.x; i < nb; i += kHistThreads) hcnt[i] = 0;
    __syncthreads();
    const uint32_t hi_mask = lv == 0 ? 0u : (0xffffffffu << (shift + level_bits(lv)));
    const float *s = s_h + (size_t)row * L;
    bool bad = false;
    const int t0 = blockIdx.x * kHistThreads * kHistPerThread + threadIdx.x;
#pragma unroll 4
    for (int u = 0; u < kHistPerThread; ++u) {
        const int t = t0 + u * kHistThreads;
        if (t >= L) break;
        const uint32_t key = score_key<kHeadScoreMax>(s[t], bad);
        if ((key & hi_mask) == (S.prefix & hi_mask)) atomicAdd(&hcnt[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    unsigned int *g = hist + (size_t)row * 4096;
    for (int i = threadIdx.x; i < nb; i += kHistThreads)
        if (hcnt[i]) atomicAdd(&g[i], hcnt[i]);
    if (bad && lv == 0) report_error(ctl, TSA_ERR_NONFINITE, 3);
}

// One block per row: the digit of level LV that holds the need-th largest key among the
// keys with the chosen prefix.  Thread t owns the digits of ranks t*per .. t*per+per-1
// counted from the top digit (rank r is digit nb-1-r); ranks past nb own nothing.
template <int LV>
__global__ void __launch_bounds__(kScanThreads)
k_sel_scan(SelectState *st, const unsigned int *__restrict__ hist) {
    constexpr int nb = 1 << level_bits(LV);
    constexpr int per = (nb + kScanThreads - 1) / kScanThreads;  // 4 or 1
    const int row = blockIdx.x;
    __shared__ SelectState S;
    if (threadIdx.x == 0) S = st[row];
    __syncthreads();
    if (S.identity) return;
    const unsigned int *g = hist + (size_t)row * 4096;
    const int r0 = (int)threadIdx.x * per;
    int cnt[per];
    int mine = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
        cnt[i] = r0 + i < nb ? (int)g[nb - 1 - (r0 + i)] : 0;
        mine += cnt[i];
    }
    int tot;
    const int above = block_scan_int(mine, tot);  // tokens in higher digits
    if (mine > 0 && above < S.need && above + mine >= S.need) {  // exactly one thread
        int acc = above;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            if (acc + cnt[i] >= S.need) {
                SelectState n = S;
                n.prefix = S.prefix | ((uint32_t)(nb - 1 - (r0 + i)) << level_shift(LV));
                n.need = S.need - acc;
                st[row] = n;
                break;
            }
            acc += cnt[i];
        }
    }
}

// grid (nchunks, rows): tokens above and equal to the threshold per chunk.
__global__ void __launch_bounds__(256)
k_sel_count(const float *__restrict__ s_h, int L, int nchunks, const SelectState *__restrict__ st,
            ChunkInfo *ci) {
    const int row = blockIdx.y, chunk = blockIdx.x;
    const SelectState S = st[row];
    if (S.identity) return;
    const float *s = s_h + (size_t)row * L;
    int gt = 0, eq = 0;
    bool dummy = false;
    for (int t = chunk * kChunk + threadIdx.x; t < min(L, (chunk + 1) * kChunk); t += 256) {
        const uint32_t key = score_key<kHeadScoreMax>(s[t], dummy);
        gt += key > S.prefix;
        eq += key == S.prefix;
    }
    __shared__ int rg[256], re[256];
    rg[threadIdx.x] = gt;
    re[threadIdx.x] = eq;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) {
            rg[threadIdx.x] += rg[threadIdx.x + o];
            re[threadIdx.x] += re[threadIdx.x + o];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        ci[(size_t)row * nchunks + chunk].n_gt = rg[0];
        ci[(size_t)row * nchunks + chunk].n_eq = re[0];
    }
}

// One block per row: chunk offsets of the kept tokens and of the equal-key ranks.
__global__ void __launch_bounds__(kScanThreads)
k_sel_offsets(int nchunks, const SelectState *__restrict__ st, ChunkInfo *ci) {
    const int row = blockIdx.x;
    const SelectState S = st[row];
    if (S.identity) return;
    ChunkInfo *c = ci + (size_t)row * nchunks;
    const int k = threadIdx.x;  // one chunk per thread (nchunks <= 1024)
    const int n_eq = k < nchunks ? c[k].n_eq : 0, n_gt = k < nchunks ? c[k].n_gt : 0;
    int tot;
    const int eq_before = block_scan_int(n_eq, tot);
    const int taken = max(0, min(n_eq, S.need - eq_before));
    const int sel_base = block_scan_int(n_gt + taken, tot);
    if (k < nchunks) {
        c[k].eq_before = eq_before;
        c[k].sel_base = sel_base;
    }
}

// grid (nchunks, rows), 1024 threads: ordered compaction of one chunk.
__global__ void __launch_bounds__(kWriteThreads)
k_sel_write(const float *__restrict__ s_h, int L, int H, int nchunks,
            const int32_t *__restrict__ Lkeep, const SelectState *__restrict__ st,
            const ChunkInfo *__restrict__ ci, int32_t *__restrict__ idx, Control *ctl) {
    const int row = blockIdx.y, chunk = blockIdx.x;
    const SelectState S = st[row];
    int32_t *out = idx + (size_t)row * L;
    const int c0 = chunk * kChunk, c1 = min(L, c0 + kChunk);
    if (S.identity) {  // nothing or everything kept: identity order
        for (int t = c0 + threadIdx.x; t < c1; t += kWriteThreads) out[t] = t;
        return;
    }
    const int keep = Lkeep[row / H];
    const ChunkInfo info = ci[(size_t)row * nchunks + chunk];
    const float *s = s_h + (size_t)row * L;
    __shared__ int warp_tot[64];
    int base_sel = info.sel_base, base_eq = info.eq_before;
    int base_rest = keep + (c0 - info.sel_base);  // unselected tokens before the chunk
    bool dummy = false;
    for (int r0 = c0; r0 < c1; r0 += kWriteThreads) {
        const int t = r0 + threadIdx.x;
        const uint32_t key = t < c1 ? score_key<kHeadScoreMax>(s[t], dummy) : 0u;
        const bool eq = t < c1 && key == S.prefix;
        int n_eq;
        const int eq_rank = base_eq + block_scan_flag(eq, warp_tot, n_eq);
        const bool sel = t < c1 && (key > S.prefix || (eq && eq_rank < S.need));
        int n_sel;
        const int pos = block_scan_flag(sel, warp_tot, n_sel);
        if (t < c1) {
            const int at = sel ? base_sel + pos : base_rest + (t - r0 - pos);
            if ((unsigned)at < (unsigned)L) out[at] = t;
            else report_error(ctl, TSA_ERR_INVALID_ARG, 10);  // inconsistent counts
        }
        base_sel += n_sel;
        base_rest += min(kWriteThreads, c1 - r0) - n_sel;
        base_eq += n_eq;
    }
}

struct SelectLayout {
    size_t states, hist, chunks, end;
};

SelectLayout select_layout(int B, int H, int L) {
    const size_t rows = (size_t)B * H, nchunks = (size_t)ceil_div(L, kChunk);
    SelectLayout y;
    y.states = 256;  // after the control block
    y.hist = align256(y.states + sizeof(SelectState) * rows);
    y.chunks = align256(y.hist + 4096 * 4 * rows);
    y.end = align256(y.chunks + sizeof(ChunkInfo) * rows * nchunks);
    return y;
}

}  // namespace

size_t select_end(int B, int H, int L) { return select_layout(B, H, L).end; }

cudaError_t launch_select(const tsa_dims &dm, const float *s_h, const int32_t *Lkeep,
                          int32_t *idx, char *ws, cudaStream_t stream) {
    const int rows = dm.B * dm.H, nchunks = ceil_div(dm.L, kChunk);
    const SelectLayout y = select_layout(dm.B, dm.H, dm.L);
    Control *ctl = reinterpret_cast<Control *>(ws);
    if (radix_cluster_fits(dm.L)) return launch_select_cluster(dm, s_h, Lkeep, idx, ctl, stream);
    SelectState *st = reinterpret_cast<SelectState *>(ws + y.states);
    unsigned int *hist = reinterpret_cast<unsigned int *>(ws + y.hist);
    ChunkInfo *ci = reinterpret_cast<ChunkInfo *>(ws + y.chunks);
    k_sel_init<<<ceil_div(rows, 256), 256, 0, stream>>>(Lkeep, dm.L, dm.H, rows, st, ctl);
    note_launches(1 + 3 * 2 + 3);  // init, (histogram, scan) per level, count/offsets/write
    dim3 hg(ceil_div(dm.L, kHistThreads * kHistPerThread), rows);
    for (int lv = 0; lv < 3; ++lv) {
        cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)4096 * 4 * rows, stream);
        if (e != cudaSuccess) return e;
        k_sel_hist<<<hg, kHistThreads, (size_t)4 << level_bits(lv), stream>>>(s_h, dm.L, lv, st,
                                                                             hist, ctl);
        if (lv == 0) k_sel_scan<0><<<rows, kScanThreads, 0, stream>>>(st, hist);
        else if (lv == 1) k_sel_scan<1><<<rows, kScanThreads, 0, stream>>>(st, hist);
        else k_sel_scan<2><<<rows, kScanThreads, 0, stream>>>(st, hist);
    }
    k_sel_count<<<dim3(nchunks, rows), 256, 0, stream>>>(s_h, dm.L, nchunks, st, ci);
    k_sel_offsets<<<rows, kScanThreads, 0, stream>>>(nchunks, st, ci);
    k_sel_write<<<dim3(nchunks, rows), kWriteThreads, 0, stream>>>(s_h, dm.L, dm.H, nchunks, Lkeep,
                                                                   st, ci, idx, ctl);
    return cudaGetLastError();
}

}  // namespace tsa

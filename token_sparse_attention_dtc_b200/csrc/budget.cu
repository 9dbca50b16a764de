// Coverage budget: the smallest k such that the k smallest layer scores carry mass >= tau.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 2 (sort s_l ascending,
// smallest k whose cumulative mass reaches tau, keep L - k); bxzpzcl.cn post §2.1
// 层级预算分配; gist.science §2 "Budget Allocation".
//
// No sort is needed: the answer is found digit by digit (a radix selection) over the IEEE
// bits of the non-negative fp32 scores, which order like the values.  Each score's mass
// is floor(s * 2^62) as a uint64, so every sum is an exact integer and the result does
// not depend on the order of the atomics.  Three levels of 12, 12 and 8 bits, each a
// grid-wide histogram (count and mass per digit, global integer atomics) followed by a
// one-block scan that picks the digit where the running mass crosses the threshold.
#include "common.cuh"

namespace tsa {

namespace {

constexpr int kHistThreads = 256, kHistPerThread = 16;
constexpr int kScanThreads = 1024;

__device__ inline unsigned long long mass62(uint32_t key) {
    return __double2ull_rz((double)__uint_as_float(key) * 4611686018427387904.0);
}

// Level geometry: bits of the key consumed before this level, and this level's width.
__host__ __device__ constexpr int level_shift(int lv) { return lv == 0 ? 20 : (lv == 1 ? 8 : 0); }
__host__ __device__ constexpr int level_bits(int lv) { return lv == 2 ? 8 : 12; }

struct Hist {  // one level of one batch element
    unsigned int *cnt;
    unsigned long long *mass;
};

__device__ inline Hist hist_of(char *base, int b, int lv) {
    char *p = base + (size_t)b * kBudgetHistBytes;
    if (lv >= 1) p += 4096 * 12;
    if (lv >= 2) p += 4096 * 12;
    const int nb = 1 << level_bits(lv);
    return Hist{reinterpret_cast<unsigned int *>(p),
                reinterpret_cast<unsigned long long *>(p + 4 * nb)};
}

// grid (ceil(L / 4096), B), 256 threads, dynamic shared memory 12 bytes per digit.
// Histogram of digit `lv` over the scores whose higher digits equal the prefix chosen so
// far (level 0: all scores), gathered per block in shared memory, then added to the
// global histogram with one atomic per non-empty digit.
__global__ void __launch_bounds__(kHistThreads)
k_budget_hist(const float *__restrict__ s_l, int L, int lv, const BudgetState *__restrict__ st,
              char *hist_base, Control *ctl) {
    extern __shared__ __align__(16) unsigned char hsm[];
    const int b = blockIdx.y;
    const BudgetState S = st[b];
    if (S.done) return;
    const int shift = level_shift(lv), nb = 1 << level_bits(lv);
    unsigned int *cnt = reinterpret_cast<unsigned int *>(hsm);
    unsigned long long *mass = reinterpret_cast<unsigned long long *>(hsm + 4 * nb);
    for (int i = threadIdx.x; i < nb; i += kHistThreads) { cnt[i] = 0; mass[i] = 0; }
    __syncthreads();
    const uint32_t hi_mask = lv == 0 ? 0u : (0xffffffffu << (shift + level_bits(lv)));
    const float *s = s_l + (size_t)b * L;
    bool bad = false;
    const int t0 = blockIdx.x * kHistThreads * kHistPerThread + threadIdx.x;
#pragma unroll 4
    for (int u = 0; u < kHistPerThread; ++u) {
        const int t = t0 + u * kHistThreads;
        if (t >= L) break;
        const uint32_t key = score_key<kLayerScoreMax>(s[t], bad);
        if ((key & hi_mask) != (S.prefix & hi_mask)) continue;
        const int dg = (key >> shift) & (nb - 1);
        atomicAdd(&cnt[dg], 1u);
        const unsigned long long m = mass62(key);
        if (m) atomicAdd(&mass[dg], m);
    }
    __syncthreads();
    const Hist hh = hist_of(hist_base, b, lv);
    for (int i = threadIdx.x; i < nb; i += kHistThreads) {
        if (cnt[i]) {
            atomicAdd(&hh.cnt[i], cnt[i]);
            if (mass[i]) atomicAdd(&hh.mass[i], mass[i]);
        }
    }
    if (bad && lv == 0) report_error(ctl, TSA_ERR_NONFINITE, 1);
}

// Exclusive block-wide scan of a uint64 and an int over kScanThreads (1024) threads;
// also returns the totals.
__device__ inline void block_scan2(unsigned long long v, int c, unsigned long long &excl_v,
                                   int &excl_c, unsigned long long &tot_v, int &tot_c) {
    __shared__ unsigned long long wv[32], s_tv;
    __shared__ int wc[32], s_tc;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long x = v;
    int y = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long xv = __shfl_up_sync(0xffffffffu, x, o);
        const int yv = __shfl_up_sync(0xffffffffu, y, o);
        if (lane >= o) { x += xv; y += yv; }
    }
    if (lane == 31) { wv[warp] = x; wc[warp] = y; }
    __syncthreads();
    if (warp == 0) {
        const unsigned long long a0 = wv[lane];
        const int b0 = wc[lane];
        unsigned long long a = a0;
        int bq = b0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long av = __shfl_up_sync(0xffffffffu, a, o);
            const int bv = __shfl_up_sync(0xffffffffu, bq, o);
            if (lane >= o) { a += av; bq += bv; }
        }
        if (lane == 31) { s_tv = a; s_tc = bq; }
        wv[lane] = a - a0;
        wc[lane] = bq - b0;
    }
    __syncthreads();
    excl_v = wv[warp] + (x - v);
    excl_c = wc[warp] + (y - c);
    tot_v = s_tv;
    tot_c = s_tc;
    __syncthreads();
}

// One block per batch element: find the digit of level `lv` where the running mass
// (mass of all smaller scores) first reaches T.  At the last level also finish k.
__global__ void __launch_bounds__(kScanThreads)
k_budget_scan(int L, int lv, unsigned long long T, BudgetState *__restrict__ st,
              char *hist_base, int32_t *__restrict__ Lkeep) {
    const int b = blockIdx.x;
    __shared__ BudgetState S;
    if (threadIdx.x == 0) S = st[b];
    __syncthreads();
    if (S.done) {
        if (lv == 2 && threadIdx.x == 0) Lkeep[b] = L - S.k;
        return;
    }
    const Hist hh = hist_of(hist_base, b, lv);
    const int nb = 1 << level_bits(lv);
    const int per = (nb + kScanThreads - 1) / kScanThreads;  // 4 or 1
    const int d0 = threadIdx.x * per;
    unsigned long long mv = 0;
    int mc = 0;
    for (int i = 0; i < per; ++i)
        if (d0 + i < nb) { mv += hh.mass[d0 + i]; mc += hh.cnt[d0 + i]; }
    unsigned long long ev, tv;
    int ec, tc;
    block_scan2(mv, mc, ev, ec, tv, tc);
    __shared__ int found;
    if (threadIdx.x == 0) found = 0;
    __syncthreads();
    const unsigned long long base = S.before;
    if (mv > 0 && base + ev < T && base + ev + mv >= T) {  // exactly one thread
        unsigned long long acc = base + ev;
        int c = S.cbefore + ec;
        for (int i = 0; i < per; ++i) {
            const unsigned long long m = hh.mass[d0 + i];
            if (acc + m >= T) {
                BudgetState n = S;
                n.prefix = S.prefix | ((uint32_t)(d0 + i) << level_shift(lv));
                n.before = acc;
                n.cbefore = c;
                if (lv == 2) {  // the exact key: take j copies of its mass
                    const unsigned long long a = mass62(n.prefix);
                    n.k = c + (int)((T - acc + a - 1) / a);
                    n.done = 1;
                    Lkeep[b] = L - n.k;
                }
                st[b] = n;
                found = 1;
                break;
            }
            acc += m;
            c += hh.cnt[d0 + i];
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && !found) {  // total mass below T: prune everything
        BudgetState n = S;
        n.done = 1;
        n.k = L;
        st[b] = n;
        if (lv == 2) Lkeep[b] = 0;
    }
}

__global__ void k_budget_init(BudgetState *st, int B, unsigned long long T, int32_t *Lkeep,
                              int L) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    BudgetState s{};
    if (T == 0ull) {  // tau = 0: nothing is pruned
        s.done = 1;
        s.k = 0;
    }
    st[b] = s;
    (void)Lkeep;
    (void)L;
}

}  // namespace

cudaError_t launch_budget(const tsa_dims &dm, const float *s_l, double tau, int32_t *Lkeep,
                          char *ws, cudaStream_t stream) {
    const unsigned long long T = (unsigned long long)ceil(tau * 4611686018427387904.0);
    Control *ctl = reinterpret_cast<Control *>(ws);
    if (radix_cluster_fits(dm.L)) return launch_budget_cluster(dm, s_l, T, Lkeep, ctl, stream);
    BudgetState *st = reinterpret_cast<BudgetState *>(ws + kBudgetStateOffset);
    char *hist = ws + budget_hist_offset(dm.B);
    cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)dm.B * kBudgetHistBytes, stream);
    if (e != cudaSuccess) return e;
    k_budget_init<<<ceil_div(dm.B, 128), 128, 0, stream>>>(st, dm.B, T, Lkeep, dm.L);
    note_launches(1 + 3 * 2);  // init, (histogram, scan) per level
    dim3 hg(ceil_div(dm.L, kHistThreads * kHistPerThread), dm.B);
    for (int lv = 0; lv < 3; ++lv) {
        const size_t smem = (size_t)12 << level_bits(lv);
        k_budget_hist<<<hg, kHistThreads, smem, stream>>>(s_l, dm.L, lv, st, hist, ctl);
        k_budget_scan<<<dm.B, kScanThreads, 0, stream>>>(dm.L, lv, T, st, hist, Lkeep);
    }
    return cudaGetLastError();
}

}  // namespace tsa

// Coverage budget and per-head top-L' selection in one launch each, for rows of up to
// 8 x 32768 scores: the row lives in the shared memory of one thread-block cluster.
//
// Method: "Token Sparse Attention" papernotes.org notes, 关键设计 2 (ascending sort of
// s_l, smallest k whose cumulative mass reaches tau, keep L - k; each head keeps its own
// top tokens); bxzpzcl.cn post §2.1 层级预算分配; gist.science §2 "Budget Allocation" and
// "Head-Wise Selection".
//
// The arithmetic is the grid-wide path's: the answer is found digit by digit over the
// IEEE key of a non-negative fp32 score (which orders like the value), the budget adds
// fixed-point masses floor(s * 2^62) and selection counts keys, so every histogram is an
// exact integer.  The digits are the exponent, then 12 and 11 mantissa bits.  What
// changes is where the data sits.  Each CTA of a cluster of C <= 8 CTAs loads one slice
// of the row into shared memory once; every level builds a shared-memory histogram per
// CTA, and after a cluster barrier every CTA sums the C histograms through distributed
// shared memory and scans them itself, so all CTAs reach the same digit without another
// exchange.  Selection then writes its slice of the ordered index list, each warp one
// contiguous segment: kept tokens (above the threshold key, then the lowest-index ties)
// and the rest, both in token order.  One launch replaces the grid-wide path's histogram,
// scan, count, offset and write kernels and their memsets.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace tsa {

namespace {

constexpr int kThreads = 1024;          // 32 warps; the block scans assume this
constexpr int kWarps = kThreads / 32;
constexpr int kMaxKeysPerCta = 32768;   // 128 KB of keys
constexpr int kMaxCluster = 8;          // portable cluster size
constexpr int kBins = 4096;             // widest level
constexpr int kRound = 4 * kThreads;    // keys per histogram round (4 per thread)
constexpr int kCopies = 16;             // private first-level histograms (one per warp pair)
// Rows of up to this many tokens take budget and selection in one launch, the budget
// recomputed by every (b, h) CTA (cheaper than a second launch at these lengths).
constexpr int kFusedMaxTokens = 8192;

// Levels: bits 31..23 (sign and exponent), 22..11 and 10..0 of the key.  Scores crowd
// into a few exponents, so the first level's atomics go to kCopies private histograms
// (warp w adds to copy w % kCopies) that are folded before the cluster exchange.
__host__ __device__ constexpr int lv_shift(int lv) { return lv == 0 ? 23 : (lv == 1 ? 11 : 0); }
__host__ __device__ constexpr int lv_bits(int lv) { return lv == 0 ? 9 : (lv == 1 ? 12 : 11); }
constexpr int kBins0 = 1 << lv_bits(0);

__device__ inline unsigned long long mass62(uint32_t key) {
    return __double2ull_rz((double)__uint_as_float(key) * 4611686018427387904.0);
}

// floor(s * 2^62) for s = M * 2^(E - 150) (E the biased exponent, M the 24-bit mantissa
// with its leading one) is M << (E - 88) when E >= 88 and M >> (88 - E) below.  Every key
// of one histogram bin has the same exponent (the first level's digit is it), so the
// bin's mass is (sum of the per-key units) << max(E - 88, 0), with units below 2^24.
// The units are added as two 12-bit halves in 32-bit counters, which stay exact for up
// to 2^20 keys per CTA.
__device__ inline uint32_t mass_units(uint32_t key) {
    const int E = (int)((key >> 23) & 0xffu);
    if (E == 0) return 0;  // zero or subnormal: below 2^-126, so no mass
    const uint32_t M = (key & 0x7fffffu) | 0x800000u;
    const int sh = E - 88;
    return sh >= 0 ? M : (sh > -24 ? M >> -sh : 0u);
}
__device__ inline int mass_shift(uint32_t key) { return max((int)((key >> 23) & 0xffu) - 88, 0); }

// Exclusive prefix over the block (token order = thread order); `tot` gets the block
// total.  `wt` is 32 words of shared memory that no other thread touches until the next
// __syncthreads after this returns.
template <typename T>
__device__ inline T block_excl(T v, T &tot, T *wt) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    T x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wt[warp] = x;
    __syncthreads();
    const T w = wt[lane];
    T before = lane < warp ? w : T(0), all = w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        before += __shfl_xor_sync(0xffffffffu, before, o);
        all += __shfl_xor_sync(0xffffffffu, all, o);
    }
    tot = all;
    return before + x - v;
}

// Exclusive prefix over the 32 lanes of a warp.
__device__ inline int warp_excl(int v) {
    const int lane = threadIdx.x & 31;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x - v;
}

// Block-wide sum added into a shared counter that starts at 0.
__device__ inline void block_add(int v, int *dst) {
    v = __reduce_add_sync(0xffffffffu, (unsigned)v);
    if ((threadIdx.x & 31) == 0 && v) atomicAdd(dst, v);
}

// Bins d0 .. d0+PER-1 of the histogram at `a` (the same offset in every CTA), summed
// over the C CTAs of the cluster.  d0 is a multiple of PER, so the reads are vectors.
template <int PER>
__device__ inline void cluster_bins(const cg::cluster_group &cl, int C, const uint32_t *a, int d0,
                                    uint32_t (&out)[PER]) {
#pragma unroll
    for (int i = 0; i < PER; ++i) out[i] = 0;
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c) {
        if (c >= C) break;
        const uint32_t *p = cl.map_shared_rank(a, c) + d0;
        if constexpr (PER == 4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(p);
            out[0] += v.x;
            out[1] += v.y;
            out[2] += v.z;
            out[3] += v.w;
        } else if constexpr (PER == 2) {
            const uint2 v = *reinterpret_cast<const uint2 *>(p);
            out[0] += v.x;
            out[1] += v.y;
        } else {
            out[0] += *p;
        }
    }
}

// Barrier over the CTAs that share histograms: the whole cluster, or this CTA alone when
// kOne (a one-CTA launch, where a cluster barrier would only add its cost).
template <bool kOne>
__device__ inline void csync(const cg::cluster_group &cl) {
    if constexpr (kOne) __syncthreads();
    else cl.sync();
}

// cluster_bins for one CTA: plain shared-memory reads.
template <bool kOne, int PER>
__device__ inline void bins_of(const cg::cluster_group &cl, int C, const uint32_t *a, int d0,
                               uint32_t (&out)[PER]) {
    if constexpr (kOne) {
#pragma unroll
        for (int i = 0; i < PER; ++i) out[i] = a[d0 + i];
    } else {
        cluster_bins<PER>(cl, C, a, d0, out);
    }
}

__device__ inline void zero_words(uint32_t *p, int n) {  // n a multiple of 4, p 16-byte aligned
    for (int i = threadIdx.x * 4; i < n; i += kThreads * 4)
        *reinterpret_cast<uint4 *>(p + i) = make_uint4(0, 0, 0, 0);
}

// Private first-level copies folded into copy 0: thread t owns words 4t .. 4t+3 of every
// copy; copy c starts at word c * stride.
__device__ inline void fold_copies(uint32_t *h, int words, int stride) {
    for (int i = threadIdx.x * 4; i < words; i += kThreads * 4) {
        uint4 a = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < kCopies; ++c) {
            const uint4 v = *reinterpret_cast<const uint4 *>(h + c * stride + i);
            a.x += v.x;
            a.y += v.y;
            a.z += v.z;
            a.w += v.w;
        }
        *reinterpret_cast<uint4 *>(h + i) = a;
    }
}

// Slice of the row owned by this CTA: tokens [t0, t0 + n).
struct Slice {
    int t0, n;
};
__device__ inline Slice slice_of(int rank, int per_cta, int L) {
    const int t0 = rank * per_cta;
    return Slice{t0, max(0, min(per_cta, L - t0))};
}

// Keys of the slice into shared memory; true if a score was out of range.  `src` is the
// row.  t0 is a multiple of 4, so when L is too the slice is 16-byte aligned.
template <uint32_t kMax>
__device__ inline bool load_keys(uint32_t *keys, const float *__restrict__ src, int L, Slice s) {
    bool bad = false;
    int done = 0;
    if ((L & 3) == 0) {
        const float4 *s4 = reinterpret_cast<const float4 *>(src + s.t0);
        const int n4 = s.n >> 2;
#pragma unroll 4
        for (int i = threadIdx.x; i < n4; i += kThreads) {
            const float4 v = __ldg(s4 + i);
            *reinterpret_cast<uint4 *>(keys + 4 * i) =
                make_uint4(score_key<kMax>(v.x, bad), score_key<kMax>(v.y, bad),
                           score_key<kMax>(v.z, bad), score_key<kMax>(v.w, bad));
        }
        done = n4 << 2;
    }
    for (int i = done + threadIdx.x; i < s.n; i += kThreads) keys[i] = score_key<kMax>(src[s.t0 + i], bad);
    return bad;
}

struct BudgetShared {
    unsigned long long wt[32];
    unsigned long long before;  // mass of the keys below the chosen digits
    uint32_t prefix;            // digits chosen so far
    int found;                  // the last level that found its digit, plus one
    int below;                  // keys of this CTA below the threshold key
    int keep;                   // the result, for every thread of the CTA
};

// One level of the budget search.  Returns false when the row's mass stays below T.
template <int LV, bool kOne>
__device__ inline bool budget_level(const cg::cluster_group &cl, int C, uint32_t *hist0,
                                    const uint32_t *keys, int n, unsigned long long T,
                                    BudgetShared &S) {
    constexpr int shift = lv_shift(LV), nb = 1 << lv_bits(LV);
    constexpr int per = nb >= kThreads ? nb / kThreads : 1;  // 1, 4, 2
    constexpr uint32_t hi_mask = LV == 0 ? 0u : (0xffffffffu << (shift + lv_bits(LV)));
    const int tid = threadIdx.x;
    // The level's (high, low) histogram; at the first level copy 0 of the private ones,
    // copy c at hist0 + c * 2 * kBins0 (all copies fit in the two buffers).
    uint32_t *hh = LV == 0 ? hist0 : hist0 + (LV & 1) * 2 * kBins;
    uint32_t *hl = hh + (LV == 0 ? kBins0 : kBins);
    uint32_t *ph = LV == 0 ? hist0 + (tid >> 5) % kCopies * 2 * kBins0 : hh;
    uint32_t *pl = ph + (LV == 0 ? kBins0 : kBins);
    zero_words(hh, LV == 0 ? kCopies * 2 * kBins0 : 2 * kBins);
    __syncthreads();  // zeroed bins; the keys and the state of the last level
    const uint32_t pre = S.prefix & hi_mask;
    const unsigned long long base = S.before;
    for (int i = tid * 4; i < n; i += kRound) {
        const uint4 k4 = *reinterpret_cast<const uint4 *>(keys + i);
        const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t u = mass_units(kk[j]);
            if (i + j < n && (kk[j] & hi_mask) == pre && u != 0) {
                const uint32_t dg = (kk[j] >> shift) & (nb - 1);
                atomicAdd(&ph[dg], u >> 12);
                atomicAdd(&pl[dg], u & 0xfffu);
            }
        }
    }
    if (LV == 0) {
        __syncthreads();
        fold_copies(hist0, 2 * kBins0, 2 * kBins0);
    }
    csync<kOne>(cl);  // every CTA's histogram of this level is complete
    // Thread t owns digits t*per .. t*per+per-1 (ascending key order).
    const int d0 = tid * per;
    unsigned long long mv[per], mine = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) mv[i] = 0;
    if (d0 < nb) {
        uint32_t uh[per], ul[per];
        bins_of<kOne, per>(cl, C, hh, d0, uh);
        bins_of<kOne, per>(cl, C, hl, d0, ul);
#pragma unroll
        for (int i = 0; i < per; ++i) {
            // The bin's exponent: its own digit at the first level, else the prefix's.
            const int sh = mass_shift(LV == 0 ? (uint32_t)(d0 + i) << shift : pre);
            mv[i] = (((unsigned long long)uh[i] << 12) + ul[i]) << sh;
            mine += mv[i];
        }
    }
    unsigned long long tot;
    const unsigned long long ex = block_excl(mine, tot, S.wt);
    if (mine > 0 && base + ex < T && base + ex + mine >= T) {  // exactly one thread
        unsigned long long acc = base + ex;
        bool hit = false;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            if (!hit && acc + mv[i] >= T) {
                S.prefix = pre | ((uint32_t)(d0 + i) << shift);
                S.before = acc;
                S.found = LV + 1;
                hit = true;
            }
            acc += mv[i];
        }
    }
    __syncthreads();
    return S.found == LV + 1;
}

// Coverage budget of one row of layer scores, on a cluster of C CTAs that each hold one
// slice of the row's keys: the number of tokens kept (0 when the row's mass stays below T).
// Every CTA of the cluster returns the same value.
template <bool kOne>
__device__ inline int budget_row(const cg::cluster_group &cl, int C, uint32_t *hist0,
                                 const uint32_t *keys, Slice sl, int L, unsigned long long T,
                                 BudgetShared &S) {
    const int tid = threadIdx.x;
    if (T == 0ull) return L;  // tau = 0: nothing is pruned (no shared memory was shared yet)
    if (tid == 0) {
        S.prefix = 0;
        S.before = 0;
        S.found = 0;
        S.below = 0;
    }
    // Every CTA takes the same branch: they scan the same summed histograms.
    if (!budget_level<0, kOne>(cl, C, hist0, keys, sl.n, T, S) ||
        !budget_level<1, kOne>(cl, C, hist0, keys, sl.n, T, S) ||
        !budget_level<2, kOne>(cl, C, hist0, keys, sl.n, T, S)) {
        csync<kOne>(cl);  // peers may still be reading this CTA's histogram
        return 0;         // the whole row's mass is below tau: prune everything
    }
    // k = (scores below the threshold key) + the copies of that key that reach tau.
    const uint32_t P = S.prefix;
    int below = 0;
    for (int i = tid; i < sl.n; i += kThreads) below += keys[i] < P;
    block_add(below, &S.below);
    csync<kOne>(cl);
    if (tid == 0) {
        int cnt = 0;
        if constexpr (kOne) cnt = S.below;
        else
            for (int c = 0; c < C; ++c) cnt += cl.map_shared_rank(&S, c)->below;
        const unsigned long long a = mass62(P);
        S.keep = L - (cnt + (int)((T - S.before + a - 1) / a));
    }
    csync<kOne>(cl);  // every CTA has read every CTA's count; S.keep is visible to the CTA
    return S.keep;
}

// grid (C, B), cluster (C, 1, 1), 1024 threads.  Dynamic shared memory: two histogram
// buffers of 4096 (high, low) pairs of 32-bit mass-unit sums, then the slice's keys.
__global__ void __launch_bounds__(kThreads, 1)
k_budget_cluster(const float *__restrict__ s_l, int L, int per_cta, unsigned long long T,
                 int32_t *__restrict__ Lkeep, Control *ctl) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *hist0 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + 2 * kBins * 8);
    __shared__ BudgetShared S;
    cg::cluster_group cl = cg::this_cluster();
    const int C = (int)cl.num_blocks(), cr = (int)cl.block_rank();
    const int b = blockIdx.y;
    const Slice sl = slice_of(cr, per_cta, L);
    if (load_keys<kLayerScoreMax>(keys, s_l + (size_t)b * L, L, sl))
        report_error(ctl, TSA_ERR_NONFINITE, 1);
    const int keep = budget_row<false>(cl, C, hist0, keys, sl, L, T, S);
    if (cr == 0 && threadIdx.x == 0) Lkeep[b] = keep;
}

struct SelectShared {
    int wt[32];
    int wgt[kWarps], weq[kWarps];  // per warp: keys above / equal to the threshold
    uint32_t prefix;               // digits chosen so far; the threshold key at the end
    int need;                      // keys still to take from the chosen digit range
    int gt, eq;                    // per CTA (read by the peers)
    int sel_base, eq_before;       // kept / equal keys of the row before this slice
};

// One level of the top-k search: narrows S.prefix and S.need.
template <int LV, bool kOne>
__device__ inline void select_level(const cg::cluster_group &cl, int C, uint32_t *hist0,
                                    const uint32_t *keys, int n, SelectShared &S) {
    constexpr int shift = lv_shift(LV), nb = 1 << lv_bits(LV);
    constexpr int per = nb >= kThreads ? nb / kThreads : 1;
    constexpr uint32_t hi_mask = LV == 0 ? 0u : (0xffffffffu << (shift + lv_bits(LV)));
    const int tid = threadIdx.x;
    // The level's histogram; at the first level copy 0 of the private ones, copy c at
    // hist0 + c * kBins0 (all copies fit in the two buffers).
    uint32_t *h = LV == 0 ? hist0 : hist0 + (LV & 1) * kBins;
    uint32_t *ph = LV == 0 ? hist0 + (tid >> 5) % kCopies * kBins0 : h;
    zero_words(h, LV == 0 ? kCopies * kBins0 : kBins);
    __syncthreads();
    const uint32_t pre = S.prefix & hi_mask;
    const int need = S.need;
    for (int i = tid * 4; i < n; i += kRound) {
        const uint4 k4 = *reinterpret_cast<const uint4 *>(keys + i);
        const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (i + j < n && (kk[j] & hi_mask) == pre) atomicAdd(&ph[(kk[j] >> shift) & (nb - 1)], 1u);
    }
    if (LV == 0) {
        __syncthreads();
        fold_copies(hist0, kBins0, kBins0);
    }
    csync<kOne>(cl);
    // Thread t sums digits t*per .. t*per+per-1; threads past the digits own none.
    const int d0 = tid * per;
    uint32_t cnt[per];
#pragma unroll
    for (int i = 0; i < per; ++i) cnt[i] = 0;
    if (d0 < nb) bins_of<kOne, per>(cl, C, h, d0, cnt);
    int mine = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) mine += (int)cnt[i];
    // Keys in higher digits = total - (keys up to and including this thread's digits).
    int tot;
    const int below = block_excl(mine, tot, S.wt);
    const int above = tot - below - mine;
    if (mine > 0 && above < need && above + mine >= need) {  // exactly one thread
        int acc = above;
        bool hit = false;
#pragma unroll
        for (int i = per - 1; i >= 0; --i) {  // digits from the top down
            if (!hit && acc + (int)cnt[i] >= need) {
                S.prefix = pre | ((uint32_t)(d0 + i) << shift);
                S.need = need - acc;
                hit = true;
            }
            acc += (int)cnt[i];
        }
    }
    __syncthreads();
}

// Top-`keep` selection of one row of head scores on a cluster of C CTAs (each holding
// one slice of the row): writes the row's index list `out`.  `keys` must have room for the
// slice; the keys are loaded here.
template <bool kOne>
__device__ inline void select_row(const cg::cluster_group &cl, int C, int cr, uint32_t *hist0,
                                  uint32_t *keys, Slice sl, const float *__restrict__ src,
                                  int L, int keep, int32_t *__restrict__ out, Control *ctl,
                                  SelectShared &S) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (keep <= 0 || keep >= L) {  // nothing or everything kept: the identity order
        for (int i = tid; i < sl.n; i += kThreads) out[sl.t0 + i] = sl.t0 + i;
        if ((keep < 0 || keep > L) && cr == 0 && tid == 0) report_error(ctl, TSA_ERR_INVALID_ARG, 2);
        return;
    }
    if (load_keys<kHeadScoreMax>(keys, src, L, sl))
        report_error(ctl, TSA_ERR_NONFINITE, 3);
    if (tid == 0) {
        S.prefix = 0;
        S.need = keep;
    }
    select_level<0, kOne>(cl, C, hist0, keys, sl.n, S);
    select_level<1, kOne>(cl, C, hist0, keys, sl.n, S);
    select_level<2, kOne>(cl, C, hist0, keys, sl.n, S);
    // Threshold key P; the first `take` keys equal to P (in token order) are kept.
    const uint32_t P = S.prefix;
    const int take = S.need;
    // Warp w owns the contiguous segment [w0, w1) of the slice.
    const int seg = (ceil_div(sl.n, kWarps) + 31) & ~31;
    const int w0 = min(warp * seg, sl.n), w1 = min(w0 + seg, sl.n);
    const unsigned lt = (1u << lane) - 1u;
    int gt = 0, eq = 0;
    for (int i = w0; i < w1; i += 32) {  // warp-uniform bounds
        const int t = i + lane;
        const bool v = t < w1;
        const uint32_t k = v ? keys[t] : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, v && k > P));
        eq += __popc(__ballot_sync(0xffffffffu, v && k == P));
    }
    if (lane == 0) {
        S.wgt[warp] = gt;
        S.weq[warp] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        const int g = (int)__reduce_add_sync(0xffffffffu, (unsigned)S.wgt[lane]);
        const int e = (int)__reduce_add_sync(0xffffffffu, (unsigned)S.weq[lane]);
        if (lane == 0) {
            S.gt = g;
            S.eq = e;
        }
    }
    csync<kOne>(cl);  // every CTA's counts are final
    if (tid == 0) {
        int eq_before = 0, sel_base = 0;
        for (int c = 0; c < cr; ++c) {
            const SelectShared *o = cl.map_shared_rank(&S, c);
            const int g = o->gt, e = o->eq;
            sel_base += g + max(0, min(e, take - eq_before));
            eq_before += e;
        }
        S.sel_base = sel_base;
        S.eq_before = eq_before;
    }
    __syncthreads();
    // Per-warp bases: lane l works out warp l's, then each warp takes its own.
    const int e_l = S.weq[lane], g_l = S.wgt[lane];
    const int eqb_l = S.eq_before + warp_excl(e_l);
    const int sel_l = g_l + max(0, min(e_l, take - eqb_l));
    const int selb_l = S.sel_base + warp_excl(sel_l);
    int eqb = __shfl_sync(0xffffffffu, eqb_l, warp);
    int selb = __shfl_sync(0xffffffffu, selb_l, warp);
    int restb = keep + (sl.t0 + w0 - selb);  // unselected tokens before the segment
    for (int i = w0; i < w1; i += 32) {
        const int t = i + lane;
        const bool v = t < w1;
        const uint32_t k = v ? keys[t] : 0u;
        const unsigned em = __ballot_sync(0xffffffffu, v && k == P);
        const bool s = v && (k > P || (k == P && eqb + __popc(em & lt) < take));
        const unsigned sm = __ballot_sync(0xffffffffu, s);
        const unsigned rm = __ballot_sync(0xffffffffu, v) & ~sm;
        if (v) {
            const int at = s ? selb + __popc(sm & lt) : restb + __popc(rm & lt);
            if ((unsigned)at < (unsigned)L) out[at] = sl.t0 + t;
            else report_error(ctl, TSA_ERR_INVALID_ARG, 10);  // inconsistent counts
        }
        eqb += __popc(em);
        selb += __popc(sm);
        restb += __popc(rm);
    }
    csync<kOne>(cl);  // peers have read this CTA's counts
}

// grid (C, B*H), cluster (C, 1, 1), 1024 threads.  Dynamic shared memory: two 4096-bin
// uint32 count histograms, then the slice's keys.
__global__ void __launch_bounds__(kThreads, 1)
k_select_cluster(const float *__restrict__ s_h, int L, int H, int per_cta,
                 const int32_t *__restrict__ Lkeep, int32_t *__restrict__ idx, Control *ctl) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *hist0 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + 2 * kBins * 4);
    __shared__ SelectShared S;
    cg::cluster_group cl = cg::this_cluster();
    const int C = (int)cl.num_blocks(), cr = (int)cl.block_rank();
    const int row = blockIdx.y;
    const Slice sl = slice_of(cr, per_cta, L);
    select_row<false>(cl, C, cr, hist0, keys, sl, s_h + (size_t)row * L, L, Lkeep[row / H],
                      idx + (size_t)row * L, ctl, S);
}

// Budget and selection in one launch for short rows (the whole row in one CTA): CTA
// (b, h) computes batch element b's budget from s_l (every CTA of b gets the same, exact
// integer result; head 0's CTA stores it), then selects head h's tokens with it.
// grid (1, B*H), cluster (1, 1, 1), 1024 threads.  Dynamic shared memory: two histogram
// buffers of 4096 (high, low) 32-bit pairs, then one row of keys (s_l's, then s_h's).
__global__ void __launch_bounds__(kThreads, 1)
k_budget_select(const float *__restrict__ s_l, const float *__restrict__ s_h, int L, int H,
                unsigned long long T, int32_t *__restrict__ Lkeep, int32_t *__restrict__ idx,
                Control *ctl) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *hist0 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + 2 * kBins * 8);
    __shared__ BudgetShared SB;
    __shared__ SelectShared SS;
    cg::cluster_group cl = cg::this_cluster();
    const int row = blockIdx.y, b = row / H;
    pdl_wait();  // the scores are the previous kernel's
    pdl_trigger();
    const Slice sl = slice_of(0, L, L);
    if (load_keys<kLayerScoreMax>(keys, s_l + (size_t)b * L, L, sl))
        report_error(ctl, TSA_ERR_NONFINITE, 1);
    const int keep = budget_row<true>(cl, 1, hist0, keys, sl, L, T, SB);
    if (row % H == 0 && threadIdx.x == 0) Lkeep[b] = keep;
    __syncthreads();  // the budget is done with the keys and the histograms
    select_row<true>(cl, 1, 0, hist0, keys, sl, s_h + (size_t)row * L, L, keep,
                     idx + (size_t)row * L, ctl, SS);
}

// Selection: the smallest cluster whose slices fit (the rows already fill the GPU).
// Budget: one cluster per batch element, so up to 8 CTAs of at least 4096 scores each.
// 0 when the row is too long for this path.
int cluster_size(int L) {
    for (int c = 1; c <= kMaxCluster; c *= 2)
        if (ceil_div(L, c) <= kMaxKeysPerCta) return c;
    return 0;
}
int budget_cluster_size(int L) {
    int c = cluster_size(L);
    while (c > 0 && c < kMaxCluster && ceil_div(L, 2 * c) >= 4096) c *= 2;
    return c;
}

int slice_tokens(int L, int C) { return (ceil_div(L, C) + 3) & ~3; }

size_t keys_bytes(int per_cta) { return (size_t)4 * ceil_div(per_cta, kRound) * kRound; }

template <typename Kernel, typename... Args>
cudaError_t launch_cluster(Kernel k, int C, int rows, size_t smem, cudaStream_t stream, bool pdl,
                           Args... args) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(C, rows);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 2 : 1;
    note_launches(1);
    return cudaLaunchKernelEx(&cfg, k, args...);
}

}  // namespace

bool radix_cluster_fits(int L) { return cluster_size(L) > 0; }

cudaError_t launch_budget_cluster(const tsa_dims &dm, const float *s_l, unsigned long long T,
                                  int32_t *Lkeep, Control *ctl, cudaStream_t stream) {
    const int C = budget_cluster_size(dm.L), per = slice_tokens(dm.L, C);
    const size_t smem = (size_t)2 * kBins * 8 + keys_bytes(per);
    return launch_cluster(k_budget_cluster, C, dm.B, smem, stream, false, s_l, dm.L, per, T, Lkeep,
                          ctl);
}

bool budget_select_fused_fits(int L) { return L <= kFusedMaxTokens; }

cudaError_t launch_budget_select(const tsa_dims &dm, const float *s_l, const float *s_h,
                                 unsigned long long T, int32_t *Lkeep, int32_t *idx,
                                 Control *ctl, cudaStream_t stream, bool pdl) {
    const size_t smem = (size_t)2 * kBins * 8 + keys_bytes(dm.L);
    return launch_cluster(k_budget_select, 1, dm.B * dm.H, smem, stream, pdl, s_l, s_h, dm.L,
                          dm.H, T, Lkeep, idx, ctl);
}

cudaError_t launch_select_cluster(const tsa_dims &dm, const float *s_h, const int32_t *Lkeep,
                                  int32_t *idx, Control *ctl, cudaStream_t stream) {
    const int C = cluster_size(dm.L), per = slice_tokens(dm.L, C);
    const size_t smem = (size_t)2 * kBins * 4 + keys_bytes(per);
    return launch_cluster(k_select_cluster, C, dm.B * dm.H, smem, stream, false, s_h, dm.L, dm.H,
                          per, Lkeep, idx, ctl);
}

}  // namespace tsa

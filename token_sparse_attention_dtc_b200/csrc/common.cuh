// Shared device/host helpers of the CUDA library (not used by the CPU oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tsa.h"

namespace tsa {

// Workspace control block: the first 256 bytes of every workspace.
struct Control {
    int32_t err;        // first device error (tsa_status), 0 when none
    int32_t err_where;  // kernel-specific detail of that error
    int32_t pad[62];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

// Tokens per scoring split of the CUDA-core path: 4096, fewer for shorter rows so that a
// row still spans several blocks.
inline int score_simt_split(int L) { return L >= 32768 ? 4096 : (L >= 4096 ? 1024 : 256); }
// Scratch of the wave-scheduled tensor-core scoring: float2 per-CTA (max, sum) pairs of
// 4 wave slots x up to 160 CTAs x 64 query rows, then float per-warp layer-score totals
// [B][up to 160 CTAs][16 warps].
constexpr size_t kScoreWavePartBytes = size_t(4) * 160 * 64 * 8;
inline size_t score_wave_bytes(int B) { return kScoreWavePartBytes + size_t(B) * 160 * 16 * 4; }

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialisation may start while the kernel before it in the stream is still running:
// pdl_wait() returns once that kernel has completed and its writes are visible, and
// pdl_trigger() lets the next such kernel start launching.  Kernels call pdl_trigger()
// only after pdl_wait(), so every kernel of a chain sees the writes of all the kernels
// before it.  Both are no-ops in a kernel launched the ordinary way.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch of `k` on `st`; with pdl, the launch may overlap the tail of the kernel before it
// (the kernel must begin with pdl_wait()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    if (pdl) {
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...);
}

// Device error reporting: the first error wins.
__device__ inline void report_error(Control *c, int code, int where) {
    if (atomicCAS(&c->err, 0, code) == 0) c->err_where = where;
}

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ inline float load(const float *p, size_t i) { return p[i]; }
    static __device__ inline float to_f(float x) { return x; }
    static __device__ inline float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ inline float load(const __nv_bfloat16 *p, size_t i) {
        return __bfloat162float(p[i]);
    }
    static __device__ inline float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ inline __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Scores are non-negative floats: their IEEE bits order like the values.  -0.0 maps
// to +0.0; a value above `max_bits` (the bits of the largest legal score), a negative
// value, an infinity or a NaN is flagged and treated as 0.
template <uint32_t max_bits>
__device__ inline uint32_t score_key(float v, bool &bad) {
    uint32_t k = __float_as_uint(v);
    if (k == 0x80000000u) k = 0;
    if (k > max_bits) { bad = true; k = 0; }
    return k;
}
constexpr uint32_t kLayerScoreMax = 0x3f800000u;  // s_l <= 1
constexpr uint32_t kHeadScoreMax = 0x7f7fffffu;   // s_h <= q: any finite non-negative

// Coverage-budget search state of one batch element (workspace, after the control block).
struct BudgetState {
    uint32_t prefix;            // key digits chosen so far
    int32_t done;               // 1 once k is known
    int32_t k;                  // tokens pruned (valid when done)
    int32_t cbefore;            // count of scores below the current digit range
    unsigned long long before;  // their fixed-point mass
    unsigned long long pad;
};
static_assert(sizeof(BudgetState) == 32, "budget state is 32 bytes");
constexpr size_t kBudgetStateOffset = 256;
// Per batch element: two 4096-digit levels and one 256-digit level of (uint32 count,
// uint64 mass).
constexpr size_t kBudgetHistBytes = 4096 * 12 * 2 + 256 * 12;
__host__ __device__ inline size_t budget_hist_offset(int B) {
    return align256(kBudgetStateOffset + sizeof(BudgetState) * (size_t)B);
}
__host__ __device__ inline size_t budget_end(int B) {
    return align256(budget_hist_offset(B) + kBudgetHistBytes * (size_t)B);
}

// Top-k search state of one (batch, head) row of the selection.
struct SelectState {
    uint32_t prefix;   // key digits chosen so far; the threshold key at the end
    int32_t need;      // tokens still to take from the current digit range
    int32_t identity;  // 1 when L' is 0 or L (the index list is the identity)
    int32_t pad;
};
static_assert(sizeof(SelectState) == 16, "select state is 16 bytes");
size_t select_end(int B, int H, int L);

// Budget and selection on rows that fit in one thread-block cluster's shared memory
// (up to 8 x 32768 scores): one launch each.  Longer rows take the grid-wide kernels.
bool radix_cluster_fits(int L);
cudaError_t launch_budget_cluster(const tsa_dims &dm, const float *s_l, unsigned long long T,
                                  int32_t *Lkeep, Control *ctl, cudaStream_t stream);
cudaError_t launch_select_cluster(const tsa_dims &dm, const float *s_h, const int32_t *Lkeep,
                                  int32_t *idx, Control *ctl, cudaStream_t stream);
// Short rows: the coverage budget and the selection in one launch (the same results as
// launch_budget + launch_select, bit for bit).
bool budget_select_fused_fits(int L);
cudaError_t launch_budget_select(const tsa_dims &dm, const float *s_l, const float *s_h,
                                 unsigned long long T, int32_t *Lkeep, int32_t *idx,
                                 Control *ctl, cudaStream_t stream, bool pdl = false);

// Host-side count of kernels this library has launched (read by tsa_kernel_launches).
void note_launches(int n);

// Every stage's scratch starts right after the 256-byte control block: the stages of a
// layer run one after another on one stream and keep their results outside the scratch,
// so their scratch regions may overlap.
// Layout of the workspace regions used by the scoring kernels.
struct WsLayout {
    size_t control = 0;     // Control
    size_t score_part = 0;  // float2 [B*Hkv][nsplit][N]  per-split (max, sum) in log2 units
    size_t score_stat = 0;  // float2 [B*Hkv][N]          combined (max, 1/sum)
    size_t norm_part = 0;   // float  [B][nblk]            partial sums of u
    size_t total = 0;
    int nsplit = 0, N = 0, qe = 0, nblk_norm = 0;
};

WsLayout ws_layout(const tsa_dims &dm, int q);

// Capacity, per KV group, of the workspace's scoring splits: the CUDA-core path (fp32)
// uses ceil(L / score_simt_split(L)) splits, the tensor-core path at most
// ceil(256 / (B*Hkv)) (and no more than the number of 128-token tiles).
inline int score_split_cap(const tsa_dims &dm) {
    const int groups = dm.B * dm.Hkv;
    const int tc = ceil_div(256, groups) < ceil_div(dm.L, 128) ? ceil_div(256, groups)
                                                              : ceil_div(dm.L, 128);
    const int simt = dm.dtype == TSA_F32 ? ceil_div(dm.L, score_simt_split(dm.L)) : 0;
    return simt > tc ? simt : tc;
}

// Host: the failure-path test hook set by tsa_set_test_stall (0 or 1).
int test_stall();
// Host: the scoring schedule set by tsa_set_score_schedule: 0 automatic (the default),
// 1 the wave-scheduled kernel wherever it applies, 2 the single-wave kernel everywhere.
int score_schedule();
// Host: the cap on KV groups per wave set by tsa_set_score_schedule (0: none).
int score_wave_group_cap();

}  // namespace tsa

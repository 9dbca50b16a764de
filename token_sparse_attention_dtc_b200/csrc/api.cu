// C ABI of libtsa: argument checks, workspace layout, stage dispatch and the fused layer.
// Every entry point only enqueues kernels on the caller's stream.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <string>

#include "common.cuh"

namespace tsa {

cudaError_t launch_score_simt(const tsa_dims &, const void *, const void *, int, float, float *,
                              const WsLayout &, char *, cudaStream_t);
cudaError_t launch_score_tc(const tsa_dims &, const void *, const void *, int, float, float *,
                            float *, const WsLayout &, char *, cudaStream_t, uint32_t, bool &);
cudaError_t launch_fill_lkeep(int, int32_t, int32_t *, cudaStream_t);
size_t drift_workspace_bytes(int, long long);
size_t block_scratch_bytes(const tsa_dims &);
size_t block_mask_words(const tsa_dims &);
cudaError_t launch_block_select(const tsa_dims &, const void *, const void *, const int32_t *,
                                float, float, float *, uint32_t *, char *, cudaStream_t);
cudaError_t launch_attn_gather(const tsa_dims &, const void *, const void *, const void *,
                               const int32_t *, const int32_t *, float, const void *, void *,
                               Control *, cudaStream_t, uint32_t);
cudaError_t launch_copy_rest(const tsa_dims &, const int32_t *, const int32_t *, const void *,
                             void *, cudaStream_t);
cudaError_t launch_drift(int, long long, int, int, const void *, double, double, double *,
                         int32_t *, char *, cudaStream_t);
cudaError_t launch_pool(const tsa_dims &, const float *, int, int, float *, cudaStream_t);
cudaError_t launch_norm(const tsa_dims &, const float *, float *, const WsLayout &, char *,
                        cudaStream_t);
cudaError_t launch_budget(const tsa_dims &, const float *, double, int32_t *, char *,
                          cudaStream_t);
cudaError_t launch_select(const tsa_dims &, const float *, const int32_t *, int32_t *, char *,
                          cudaStream_t);
cudaError_t launch_gather(const tsa_dims &, const void *, const void *, const void *,
                          const int32_t *, const int32_t *, void *, void *, void *, Control *,
                          cudaStream_t, bool = false);
cudaError_t launch_attn_simt(const tsa_dims &, const void *, const void *, const void *,
                             const int32_t *, int, float, void *, cudaStream_t);
cudaError_t launch_attn_tc(const tsa_dims &, const void *, const void *, const void *,
                           const int32_t *, int, float, void *, Control *, cudaStream_t,
                           uint32_t, const uint32_t * = nullptr, bool = false);
cudaError_t launch_scatter(const tsa_dims &, const void *, const int32_t *, const int32_t *,
                           const void *, void *, cudaStream_t, bool = false);
cudaError_t launch_head_sum(const tsa_dims &, const float *, float *, cudaStream_t);
cudaError_t launch_combine_parts(int, int, int, const float *, float *, float *, cudaStream_t);

static thread_local std::string g_last_error;
static uint32_t g_wait_limit_us = 2000000;  // 2 s
static int g_test_stall = 0;
static int g_score_wave = 0, g_score_wave_cap = 0;

int test_stall() { return g_test_stall; }
int score_schedule() { return g_score_wave; }  // 0 = automatic (the default)
int score_wave_group_cap() { return g_score_wave_cap; }

static std::atomic<uint64_t> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static tsa_status fail(tsa_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

tsa_status set_error(tsa_status s, const char *msg) {
    g_last_error = msg;
    return s;
}

static tsa_status cuda_status(cudaError_t e, const char *where) {
    if (e == cudaSuccess) return TSA_OK;
    return fail(TSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define TSA_TRY(expr)                        \
    do {                                     \
        const tsa_status s_ = (expr);        \
        if (s_ != TSA_OK) return s_;         \
    } while (0)

static size_t esize(const tsa_dims &dm) { return dm.dtype == TSA_F32 ? 4 : 2; }

static tsa_status check_dims(const tsa_dims *dm) {
    if (!dm) return fail(TSA_ERR_INVALID_ARG, "dims is NULL");
    if (dm->B < 1 || dm->L < 1 || dm->H < 1 || dm->Hkv < 1)
        return fail(TSA_ERR_INVALID_ARG, "B, L, H, Hkv must be >= 1 (got %d, %d, %d, %d)",
                    dm->B, dm->L, dm->H, dm->Hkv);
    if (dm->L > (1 << 21)) return fail(TSA_ERR_UNSUPPORTED, "L = %d exceeds 2^21", dm->L);
    if (dm->H % dm->Hkv) return fail(TSA_ERR_INVALID_ARG, "H %% Hkv != 0 (%d, %d)", dm->H, dm->Hkv);
    if (dm->d != 64 && dm->d != 128) return fail(TSA_ERR_UNSUPPORTED, "d = %d (64 or 128)", dm->d);
    if (dm->dtype != TSA_F32 && dm->dtype != TSA_BF16)
        return fail(TSA_ERR_UNSUPPORTED, "dtype %d", dm->dtype);
    if ((long long)dm->B * dm->H * dm->L > (1ll << 31))
        return fail(TSA_ERR_UNSUPPORTED, "B*H*L exceeds 2^31");
    return TSA_OK;
}

static tsa_status check_q(const tsa_dims *dm, int q) {
    if (q < 1) return fail(TSA_ERR_INVALID_ARG, "q = %d must be >= 1", q);
    const int qe = q < dm->L ? q : dm->L;
    if ((dm->H / dm->Hkv) * qe > 256)
        return fail(TSA_ERR_UNSUPPORTED, "G * min(q, L) = %d exceeds 256", (dm->H / dm->Hkv) * qe);
    return TSA_OK;
}

static tsa_status check_ptr(const void *p, const char *name) {
    if (!p) return fail(TSA_ERR_INVALID_ARG, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) & 15)
        return fail(TSA_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
    return TSA_OK;
}

static tsa_status check_scale(float scale) {
    if (!(scale > 0.0f) || !isfinite(scale))
        return fail(TSA_ERR_INVALID_ARG, "scale must be finite and > 0");
    return TSA_OK;
}

WsLayout ws_layout(const tsa_dims &dm, int q) {
    WsLayout w;
    w.qe = q < dm.L ? q : dm.L;
    w.N = (dm.H / dm.Hkv) * w.qe;
    w.nsplit = score_split_cap(dm);
    w.nblk_norm = ceil_div(dm.L, 256);
    // also 16 warp totals per scoring CTA (<= 160 CTAs) of the fused layer score
    const int norm_slots = std::max(w.nblk_norm, 160 * 16);
    size_t off = align256(sizeof(Control));  // scoring scratch after the control block
    const bool wave = dm.dtype == TSA_BF16;  // room for the wave-scheduled scoring too
    w.score_part = off;
    off = align256(off + std::max(sizeof(float2) * (size_t)dm.B * dm.Hkv * w.nsplit * w.N,
                                  wave ? score_wave_bytes(dm.B) : size_t(0)));
    w.score_stat = off;
    off = align256(off + sizeof(float2) * (size_t)dm.B * dm.Hkv * w.N);
    w.norm_part = off;
    off = align256(off + sizeof(float) * (size_t)dm.B * norm_slots);
    // the budget and selection scratch overlap the scoring scratch (stages run in order)
    w.total = std::max(off, std::max(budget_end(dm.B), select_end(dm.B, dm.H, dm.L)));
    return w;
}

struct LayerLayout {
    size_t s_h, s_hp, s_l, lkeep, idx, blk_scratch, blk_mask, qh, kh, vh, oh, total;
};

static LayerLayout layer_layout(const tsa_dims &dm, int q) {
    LayerLayout y;
    size_t off = ws_layout(dm, q).total;
    const size_t BHL = (size_t)dm.B * dm.H * dm.L;
    y.s_h = off; off = align256(off + 4 * BHL);
    y.s_hp = off; off = align256(off + 4 * BHL);  // pooled head scores (score variant)
    y.s_l = off; off = align256(off + 4 * (size_t)dm.B * dm.L);
    y.lkeep = off; off = align256(off + 4 * (size_t)dm.B);
    y.idx = off; off = align256(off + 4 * BHL);
    y.blk_scratch = off; off = align256(off + block_scratch_bytes(dm));  // block-sparse means
    y.blk_mask = off; off = align256(off + 4 * block_mask_words(dm));
    const size_t t = align256(BHL * dm.d * esize(dm));
    y.qh = off; off += t;
    y.kh = off; off += t;
    y.vh = off; off += t;
    y.oh = off; off += t;
    y.total = off;
    return y;
}

static tsa_status check_ws(const void *ws, size_t have, size_t need) {
    if (!ws) return fail(TSA_ERR_WORKSPACE, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255)
        return fail(TSA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
    if (have < need)
        return fail(TSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", have, need);
    return TSA_OK;
}

// ---------------------------------------------------------------- stages ---

static tsa_status do_score(const tsa_dims &dm, const void *Q, const void *K, int q, float scale,
                           float *s_h, float *s_l, char *ws, cudaStream_t st) {
    const WsLayout w = ws_layout(dm, q);
    cudaError_t e;
    bool fused = false;  // the tensor-core scoring also wrote s_l
    if (dm.dtype == TSA_BF16)
        e = launch_score_tc(dm, Q, K, w.qe, scale, s_h, s_l, w, ws, st, g_wait_limit_us, fused);
    else
        e = launch_score_simt(dm, Q, K, w.qe, scale, s_h, w, ws, st);
    TSA_TRY(cuda_status(e, "tsa_score"));
    if (fused) return TSA_OK;
    return cuda_status(launch_norm(dm, s_h, s_l, w, ws, st), "tsa_score (normalise)");
}

static tsa_status do_attn(const tsa_dims &dm, const void *Q, const void *K, const void *V,
                          const int32_t *Lkeep, int dense, float scale, void *O, char *ws,
                          cudaStream_t st, const uint32_t *bmask = nullptr, bool pdl = false) {
    cudaError_t e;
    if (dm.dtype == TSA_BF16)
        e = launch_attn_tc(dm, Q, K, V, Lkeep, dense, scale, O, reinterpret_cast<Control *>(ws),
                           st, g_wait_limit_us, bmask, pdl);
    else
        e = launch_attn_simt(dm, Q, K, V, Lkeep, dense, scale, O, st);
    return cuda_status(e, "tsa_attn");
}

}  // namespace tsa

using namespace tsa;

extern "C" {

size_t tsa_workspace_size(const tsa_dims *dims, int32_t q) {
    if (check_dims(dims) != TSA_OK || check_q(dims, q) != TSA_OK) return 0;
    return ws_layout(*dims, q).total;
}

size_t tsa_layer_workspace_size(const tsa_dims *dims, int32_t q) {
    if (check_dims(dims) != TSA_OK || check_q(dims, q) != TSA_OK) return 0;
    return layer_layout(*dims, q).total;
}

tsa_status tsa_score(const tsa_dims *dims, const void *Q, const void *K, int32_t q, float scale,
                     float *s_h, float *s_l, void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_q(dims, q));
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_ptr(Q, "Q"));
    TSA_TRY(check_ptr(K, "K"));
    TSA_TRY(check_ptr(s_h, "s_h"));
    TSA_TRY(check_ptr(s_l, "s_l"));
    TSA_TRY(check_ws(ws, ws_bytes, ws_layout(*dims, q).total));
    return do_score(*dims, Q, K, q, scale, s_h, s_l, (char *)ws, (cudaStream_t)stream);
}

tsa_status tsa_score_partial(const tsa_dims *dims, const void *Q, const void *K, int32_t q,
                             float scale, float *s_h, float *u_part, void *ws, size_t ws_bytes,
                             void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_q(dims, q));
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_ptr(Q, "Q"));
    TSA_TRY(check_ptr(K, "K"));
    TSA_TRY(check_ptr(s_h, "s_h"));
    TSA_TRY(check_ptr(u_part, "u_part"));
    const tsa_dims &dm = *dims;
    const WsLayout w = ws_layout(dm, q);
    TSA_TRY(check_ws(ws, ws_bytes, w.total));
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    bool fused = false;  // no layer score here: s_l is not passed
    if (dm.dtype == TSA_BF16)
        e = launch_score_tc(dm, Q, K, w.qe, scale, s_h, nullptr, w, (char *)ws, st,
                            g_wait_limit_us, fused);
    else
        e = launch_score_simt(dm, Q, K, w.qe, scale, s_h, w, (char *)ws, st);
    TSA_TRY(cuda_status(e, "tsa_score_partial"));
    return cuda_status(launch_head_sum(dm, s_h, u_part, st), "tsa_score_partial (head sum)");
}

tsa_status tsa_layer_score_combine(const tsa_dims *dims, int32_t nparts, const float *u_parts,
                                   float *s_l, void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    if (nparts < 1 || nparts > 1024) return fail(TSA_ERR_INVALID_ARG, "nparts must be in [1, 1024]");
    TSA_TRY(check_ptr(u_parts, "u_parts"));
    TSA_TRY(check_ptr(s_l, "s_l"));
    const size_t bytes = (size_t)4 * nparts * dims->B * dims->L;
    const char *a = (const char *)u_parts, *o = (const char *)s_l;
    if (a < o + (size_t)4 * dims->B * dims->L && o < a + bytes)
        return fail(TSA_ERR_INVALID_ARG, "s_l overlaps u_parts");
    const WsLayout w = ws_layout(*dims, 1);
    TSA_TRY(check_ws(ws, ws_bytes, w.total));
    return cuda_status(launch_combine_parts(dims->B, dims->L, nparts, u_parts, s_l,
                                            (float *)((char *)ws + w.norm_part),
                                            (cudaStream_t)stream),
                       "tsa_layer_score_combine");
}

tsa_status tsa_budget(const tsa_dims *dims, const float *s_l, double tau, int32_t *Lkeep,
                      void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    if (!(tau >= 0.0 && tau < 1.0)) return fail(TSA_ERR_INVALID_ARG, "tau must be in [0, 1)");
    TSA_TRY(check_ptr(s_l, "s_l"));
    TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    TSA_TRY(check_ws(ws, ws_bytes, budget_end(dims->B)));
    return cuda_status(launch_budget(*dims, s_l, tau, Lkeep, (char *)ws, (cudaStream_t)stream),
                       "tsa_budget");
}

tsa_status tsa_select(const tsa_dims *dims, const float *s_h, const int32_t *Lkeep, int32_t *idx,
                      void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_ptr(s_h, "s_h"));
    TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    TSA_TRY(check_ptr(idx, "idx"));
    TSA_TRY(check_ws(ws, ws_bytes, select_end(dims->B, dims->H, dims->L)));
    return cuda_status(launch_select(*dims, s_h, Lkeep, idx, (char *)ws, (cudaStream_t)stream),
                       "tsa_select");
}

tsa_status tsa_gather_qkv(const tsa_dims *dims, const void *Q, const void *K, const void *V,
                          const int32_t *idx, const int32_t *Lkeep, void *Qh, void *Kh, void *Vh,
                          void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_ptr(Q, "Q"));
    TSA_TRY(check_ptr(K, "K"));
    TSA_TRY(check_ptr(V, "V"));
    TSA_TRY(check_ptr(idx, "idx"));
    TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    TSA_TRY(check_ptr(Qh, "Qh"));
    TSA_TRY(check_ptr(Kh, "Kh"));
    TSA_TRY(check_ptr(Vh, "Vh"));
    TSA_TRY(check_ws(ws, ws_bytes, sizeof(Control)));
    return cuda_status(launch_gather(*dims, Q, K, V, idx, Lkeep, Qh, Kh, Vh, (Control *)ws,
                                     (cudaStream_t)stream),
                       "tsa_gather_qkv");
}

tsa_status tsa_attn(const tsa_dims *dims, const void *Qh, const void *Kh, const void *Vh,
                    const int32_t *Lkeep, int32_t dense, float scale, void *Oh, void *ws,
                    size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_ptr(Qh, "Qh"));
    TSA_TRY(check_ptr(Kh, "Kh"));
    TSA_TRY(check_ptr(Vh, "Vh"));
    TSA_TRY(check_ptr(Oh, "Oh"));
    if (!dense) TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    TSA_TRY(check_ws(ws, ws_bytes, sizeof(Control)));
    return do_attn(*dims, Qh, Kh, Vh, Lkeep, dense ? 1 : 0, scale, Oh, (char *)ws,
                   (cudaStream_t)stream);
}

tsa_status tsa_scatter_residual(const tsa_dims *dims, const void *Oh, const int32_t *idx,
                                const int32_t *Lkeep, const void *X, void *Y, void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_ptr(Oh, "Oh"));
    TSA_TRY(check_ptr(X, "X"));
    TSA_TRY(check_ptr(Y, "Y"));
    if (idx) {
        TSA_TRY(check_ptr(idx, "idx"));
        TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    }
    return cuda_status(launch_scatter(*dims, Oh, idx, Lkeep, X, Y, (cudaStream_t)stream),
                       "tsa_scatter_residual");
}

static tsa_status check_pool(int32_t kind, int32_t width) {
    if (kind != TSA_POOL_MAX && kind != TSA_POOL_MEAN)
        return fail(TSA_ERR_INVALID_ARG, "pool kind must be TSA_POOL_MAX or TSA_POOL_MEAN");
    if (width < 1 || (width & 1) == 0) return fail(TSA_ERR_INVALID_ARG, "pool width must be odd");
    if (width > 255) return fail(TSA_ERR_UNSUPPORTED, "pool width above 255");
    return TSA_OK;
}

static tsa_status check_sparsity(double s) {
    if (!(s >= 0.0 && s <= 1.0)) return fail(TSA_ERR_INVALID_ARG, "sparsity must be in [0, 1]");
    return TSA_OK;
}

// L' of the fixed-ratio budget: L - floor(s * L), the product in double.
static int32_t fixed_keep(int L, double s) { return L - (int32_t)floor(s * (double)L); }

tsa_status tsa_budget_fixed(const tsa_dims *dims, double sparsity, int32_t *Lkeep,
                            void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_sparsity(sparsity));
    TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    return cuda_status(launch_fill_lkeep(dims->B, fixed_keep(dims->L, sparsity), Lkeep,
                                         (cudaStream_t)stream),
                       "tsa_budget_fixed");
}

tsa_status tsa_pool_scores(const tsa_dims *dims, const float *s_h, int32_t kind, int32_t width,
                           float *s_h_out, float *s_l_out, void *ws, size_t ws_bytes,
                           void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_pool(kind, width));
    TSA_TRY(check_ptr(s_h, "s_h"));
    TSA_TRY(check_ptr(s_h_out, "s_h_out"));
    TSA_TRY(check_ptr(s_l_out, "s_l_out"));
    const size_t bytes = (size_t)4 * dims->B * dims->H * dims->L;
    const char *a = (const char *)s_h, *o = (const char *)s_h_out;
    if (a < o + bytes && o < a + bytes) return fail(TSA_ERR_INVALID_ARG, "s_h_out overlaps s_h");
    const WsLayout w = ws_layout(*dims, 1);
    TSA_TRY(check_ws(ws, ws_bytes, w.total));
    cudaStream_t st = (cudaStream_t)stream;
    TSA_TRY(cuda_status(launch_pool(*dims, s_h, kind, width, s_h_out, st), "tsa_pool_scores"));
    return cuda_status(launch_norm(*dims, s_h_out, s_l_out, w, (char *)ws, st),
                       "tsa_pool_scores (normalise)");
}

// Fused compress + attention + decompress: rows through idx, Y = X + Ô in the kept rows,
// Y = X in the others (copied when Y != X).
static tsa_status do_attn_gather(const tsa_dims &dm, const void *Q, const void *K,
                                 const void *V, const int32_t *idx, const int32_t *Lkeep,
                                 float scale, const void *X, void *Y, char *ws, cudaStream_t st) {
    if (X != Y)
        TSA_TRY(cuda_status(launch_copy_rest(dm, idx, Lkeep, X, Y, st), "tsa_attn_gather (rest)"));
    return cuda_status(launch_attn_gather(dm, Q, K, V, idx, Lkeep, scale, X, Y, (Control *)ws, st,
                                          g_wait_limit_us),
                       "tsa_attn_gather");
}

size_t tsa_block_workspace_size(const tsa_dims *dims) {
    if (check_dims(dims) != TSA_OK) return 0;
    return block_scratch_bytes(*dims);
}

static tsa_status check_theta(double theta) {
    if (!(theta >= 0.0 && theta <= 3.0e38))
        return fail(TSA_ERR_INVALID_ARG, "theta must be in [0, 3e38] (use 3e38 for every block)");
    return TSA_OK;
}

tsa_status tsa_block_select(const tsa_dims *dims, const void *Qh, const void *Kh,
                            const int32_t *Lkeep, float scale, double theta, float *logits,
                            uint32_t *mask, void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_theta(theta));
    TSA_TRY(check_ptr(Qh, "Qh"));
    TSA_TRY(check_ptr(Kh, "Kh"));
    TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    TSA_TRY(check_ptr(mask, "mask"));
    if (logits) TSA_TRY(check_ptr(logits, "logits"));
    TSA_TRY(check_ws(ws, ws_bytes, block_scratch_bytes(*dims)));
    return cuda_status(launch_block_select(*dims, Qh, Kh, Lkeep, scale, (float)theta, logits, mask,
                                           (char *)ws, (cudaStream_t)stream),
                       "tsa_block_select");
}

tsa_status tsa_attn_block(const tsa_dims *dims, const void *Qh, const void *Kh, const void *Vh,
                          const int32_t *Lkeep, const uint32_t *mask, float scale, void *Oh,
                          void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    if (dims->dtype != TSA_BF16)
        return fail(TSA_ERR_UNSUPPORTED, "block-sparse attention runs the bf16 tensor-core path only");
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_ptr(Qh, "Qh"));
    TSA_TRY(check_ptr(Kh, "Kh"));
    TSA_TRY(check_ptr(Vh, "Vh"));
    TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    TSA_TRY(check_ptr(mask, "mask"));
    TSA_TRY(check_ptr(Oh, "Oh"));
    TSA_TRY(check_ws(ws, ws_bytes, sizeof(Control)));
    return do_attn(*dims, Qh, Kh, Vh, Lkeep, 0, scale, Oh, (char *)ws, (cudaStream_t)stream, mask);
}

tsa_status tsa_attn_gather(const tsa_dims *dims, const void *Q, const void *K, const void *V,
                           const int32_t *idx, const int32_t *Lkeep, float scale, const void *X,
                           void *Y, void *ws, size_t ws_bytes, void *stream) {
    TSA_TRY(check_dims(dims));
    if (dims->dtype != TSA_BF16)
        return fail(TSA_ERR_UNSUPPORTED, "tsa_attn_gather runs the bf16 tensor-core path only");
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_ptr(Q, "Q"));
    TSA_TRY(check_ptr(K, "K"));
    TSA_TRY(check_ptr(V, "V"));
    TSA_TRY(check_ptr(idx, "idx"));
    TSA_TRY(check_ptr(Lkeep, "Lkeep"));
    TSA_TRY(check_ptr(X, "X"));
    TSA_TRY(check_ptr(Y, "Y"));
    TSA_TRY(check_ws(ws, ws_bytes, sizeof(Control)));
    return do_attn_gather(*dims, Q, K, V, idx, Lkeep, scale, X, Y, (char *)ws, (cudaStream_t)stream);
}

static tsa_status layer_impl(const tsa_dims *dims, const void *Q, const void *K, const void *V,
                             const void *X, void *Y, int32_t is_sparse, int32_t q,
                             const tsa_layer_opts &o, float scale, float *s_h_out,
                             float *s_l_out, int32_t *Lkeep_out, int32_t *idx_out, void *ws,
                             size_t ws_bytes, void *stream, void *const *stage_events) {
    TSA_TRY(check_dims(dims));
    TSA_TRY(check_q(dims, q));
    TSA_TRY(check_scale(scale));
    if (o.budget == TSA_BUDGET_COVERAGE) {
        if (!(o.tau >= 0.0 && o.tau < 1.0)) return fail(TSA_ERR_INVALID_ARG, "tau must be in [0, 1)");
    } else if (o.budget == TSA_BUDGET_FIXED) {
        TSA_TRY(check_sparsity(o.sparsity));
    } else {
        return fail(TSA_ERR_INVALID_ARG, "unknown budget kind");
    }
    if (o.pool != TSA_POOL_NONE) TSA_TRY(check_pool(o.pool, o.pool_width));
    if (o.direct_gather && dims->dtype != TSA_BF16)
        return fail(TSA_ERR_UNSUPPORTED, "direct gather runs the bf16 tensor-core path only");
    const bool blocks = o.block_theta >= 0.0;  // NaN or negative: every block
    if (blocks) {
        TSA_TRY(check_theta(o.block_theta));
        if (dims->dtype != TSA_BF16 || o.direct_gather)
            return fail(TSA_ERR_UNSUPPORTED, "block sparsity runs the bf16 staged path only");
    }
    TSA_TRY(check_ptr(Q, "Q"));
    TSA_TRY(check_ptr(K, "K"));
    TSA_TRY(check_ptr(V, "V"));
    TSA_TRY(check_ptr(X, "X"));
    TSA_TRY(check_ptr(Y, "Y"));
    for (const void *p : {(const void *)s_h_out, (const void *)s_l_out, (const void *)Lkeep_out,
                          (const void *)idx_out})
        if (p) TSA_TRY(check_ptr(p, "optional output"));
    const tsa_dims &dm = *dims;
    const LayerLayout y = layer_layout(dm, q);
    TSA_TRY(check_ws(ws, ws_bytes, y.total));
    char *w = (char *)ws;
    cudaStream_t st = (cudaStream_t)stream;
    auto rec = [&](int i) -> tsa_status {
        if (!stage_events) return TSA_OK;
        return cuda_status(cudaEventRecord((cudaEvent_t)stage_events[i], st), "event record");
    };
    const bool pooled = o.pool != TSA_POOL_NONE;
    // The kernels after the scoring are launched as a programmatic-dependent chain (each
    // may launch while the one before it finishes, and waits for it before reading its
    // results) unless stage events are recorded between them.
    const bool pdl = !stage_events;
    // Scores used by budget and selection: the raw ones, or the pooled ones.
    float *s_raw = (s_h_out && !pooled) ? s_h_out : (float *)(w + y.s_h);
    float *s_h = !pooled ? s_raw : (s_h_out ? s_h_out : (float *)(w + y.s_hp));
    float *s_l = s_l_out ? s_l_out : (float *)(w + y.s_l);
    int32_t *Lk = Lkeep_out ? Lkeep_out : (int32_t *)(w + y.lkeep);
    int32_t *idx = idx_out ? idx_out : (int32_t *)(w + y.idx);
    void *Qh = w + y.qh, *Kh = w + y.kh, *Vh = w + y.vh, *Oh = w + y.oh;
    if (!is_sparse) {
        for (int i = 0; i < 5; ++i) TSA_TRY(rec(i));
        TSA_TRY(do_attn(dm, Q, K, V, nullptr, 1, scale, Oh, w, st));
        TSA_TRY(rec(5));
        TSA_TRY(cuda_status(launch_scatter(dm, Oh, nullptr, nullptr, X, Y, st), "tsa_layer"));
        return rec(6);
    }
    TSA_TRY(rec(0));
    TSA_TRY(do_score(dm, Q, K, q, scale, s_raw, s_l, w, st));
    if (pooled) {
        TSA_TRY(cuda_status(launch_pool(dm, s_raw, o.pool, o.pool_width, s_h, st),
                            "tsa_layer pool"));
        TSA_TRY(cuda_status(launch_norm(dm, s_h, s_l, ws_layout(dm, q), w, st),
                            "tsa_layer pool (normalise)"));
    }
    TSA_TRY(rec(1));
    if (o.budget == TSA_BUDGET_COVERAGE && budget_select_fused_fits(dm.L)) {
        // short rows: budget and selection in one launch (both stage events after it)
        const unsigned long long T = (unsigned long long)ceil(o.tau * 4611686018427387904.0);
        TSA_TRY(cuda_status(launch_budget_select(dm, s_l, s_h, T, Lk, idx, (Control *)w, st,
                                                 pdl && !pooled),
                            "tsa_layer budget and select"));
        TSA_TRY(rec(2));
    } else {
        if (o.budget == TSA_BUDGET_COVERAGE)
            TSA_TRY(cuda_status(launch_budget(dm, s_l, o.tau, Lk, w, st), "tsa_layer budget"));
        else
            TSA_TRY(cuda_status(launch_fill_lkeep(dm.B, fixed_keep(dm.L, o.sparsity), Lk, st),
                                "tsa_layer budget"));
        TSA_TRY(rec(2));
        TSA_TRY(cuda_status(launch_select(dm, s_h, Lk, idx, w, st), "tsa_layer select"));
    }
    TSA_TRY(rec(3));
    if (o.direct_gather) {  // no compressed copies: one fused attention pass
        TSA_TRY(rec(4));
        TSA_TRY(do_attn_gather(dm, Q, K, V, idx, Lk, scale, X, Y, w, st));
        TSA_TRY(rec(5));
        return rec(6);
    }
    TSA_TRY(cuda_status(launch_gather(dm, Q, K, V, idx, Lk, Qh, Kh, Vh, (Control *)w, st, pdl),
                        "tsa_layer gather"));
    TSA_TRY(rec(4));
    uint32_t *bm = nullptr;
    if (blocks) {  // block-sparse pattern of the compressed problem (part of the attention)
        bm = (uint32_t *)(w + y.blk_mask);
        TSA_TRY(cuda_status(launch_block_select(dm, Qh, Kh, Lk, scale, (float)o.block_theta,
                                                nullptr, bm, w + y.blk_scratch, st),
                            "tsa_layer block select"));
    }
    TSA_TRY(do_attn(dm, Qh, Kh, Vh, Lk, 0, scale, Oh, w, st, bm, pdl && !blocks));
    TSA_TRY(rec(5));
    TSA_TRY(cuda_status(launch_scatter(dm, Oh, idx, Lk, X, Y, st, pdl), "tsa_layer scatter"));
    return rec(6);
}

tsa_status tsa_layer(const tsa_dims *dims, const void *Q, const void *K, const void *V,
                     const void *X, void *Y, int32_t is_sparse, int32_t q, double tau,
                     float scale, float *s_h_out, float *s_l_out, int32_t *Lkeep_out,
                     int32_t *idx_out, void *ws, size_t ws_bytes, void *stream,
                     void *const *stage_events) {
    tsa_layer_opts o{TSA_BUDGET_COVERAGE, tau, 0.0, TSA_POOL_NONE, 1, 0, -1.0};
    return layer_impl(dims, Q, K, V, X, Y, is_sparse, q, o, scale, s_h_out, s_l_out, Lkeep_out,
                      idx_out, ws, ws_bytes, stream, stage_events);
}

tsa_status tsa_layer_ex(const tsa_dims *dims, const void *Q, const void *K, const void *V,
                        const void *X, void *Y, int32_t is_sparse, int32_t q,
                        const tsa_layer_opts *opts, float scale, float *s_h_out,
                        float *s_l_out, int32_t *Lkeep_out, int32_t *idx_out, void *ws,
                        size_t ws_bytes, void *stream, void *const *stage_events) {
    const tsa_layer_opts o = opts ? *opts
                                  : tsa_layer_opts{TSA_BUDGET_COVERAGE, 0.005, 0.0, TSA_POOL_NONE, 1, 0,
                                                   -1.0};
    return layer_impl(dims, Q, K, V, X, Y, is_sparse, q, o, scale, s_h_out, s_l_out, Lkeep_out,
                      idx_out, ws, ws_bytes, stream, stage_events);
}

static tsa_status check_drift(int32_t n_layers, int64_t tokens, int32_t d_model, int32_t dtype) {
    if (n_layers < 1 || n_layers > 512)
        return fail(TSA_ERR_INVALID_ARG, "n_layers must be in [1, 512]");
    if (tokens < 1 || tokens > ((int64_t)1 << 36)) return fail(TSA_ERR_INVALID_ARG, "bad token count");
    if (dtype != TSA_F32 && dtype != TSA_BF16) return fail(TSA_ERR_UNSUPPORTED, "dtype");
    const int esz = dtype == TSA_F32 ? 4 : 2;
    if (d_model < 1 || d_model > 65536 || (d_model * esz) % 16)
        return fail(TSA_ERR_UNSUPPORTED, "d_model * element size must be a multiple of 16 bytes");
    return TSA_OK;
}

size_t tsa_drift_workspace_size(int32_t n_layers, int64_t tokens) {
    if (n_layers < 1 || n_layers > 512 || tokens < 1 || tokens > ((int64_t)1 << 36)) return 0;
    return drift_workspace_bytes(n_layers, tokens);
}

tsa_status tsa_drift(int32_t n_layers, int64_t tokens, int32_t d_model, int32_t dtype,
                     const void *h, double eps, double delta, double *R, int32_t *mask, void *ws,
                     size_t ws_bytes, void *stream) {
    TSA_TRY(check_drift(n_layers, tokens, d_model, dtype));
    if (!(eps >= 0.0 && eps < 1e30)) return fail(TSA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (!(delta >= 0.0 && delta <= 1.0)) return fail(TSA_ERR_INVALID_ARG, "delta must be in [0, 1]");
    TSA_TRY(check_ptr(h, "h"));
    TSA_TRY(check_ptr(R, "R"));
    TSA_TRY(check_ptr(mask, "mask"));
    TSA_TRY(check_ws(ws, ws_bytes, drift_workspace_bytes(n_layers, tokens)));
    return cuda_status(launch_drift(n_layers, tokens, d_model, dtype, h, eps, delta, R, mask,
                                    (char *)ws, (cudaStream_t)stream),
                       "tsa_drift");
}

tsa_status tsa_get_device_status(void *ws, void *stream) {
    if (!ws) return fail(TSA_ERR_WORKSPACE, "workspace is NULL");
    cudaStream_t st = (cudaStream_t)stream;
    TSA_TRY(cuda_status(cudaStreamSynchronize(st), "tsa_get_device_status"));
    Control c;
    TSA_TRY(cuda_status(cudaMemcpy(&c, ws, sizeof c, cudaMemcpyDeviceToHost),
                        "tsa_get_device_status read"));
    if (c.err != 0) {
        // The whole control block: the error word and the grid-barrier words, which a
        // launch that failed part-way can leave off their initial state.
        const Control zero{};
        TSA_TRY(cuda_status(cudaMemcpy(ws, &zero, sizeof zero, cudaMemcpyHostToDevice),
                            "tsa_get_device_status clear"));
        return fail((tsa_status)c.err, "device error %d (detail %d)", c.err, c.err_where);
    }
    return TSA_OK;
}

void tsa_set_wait_limit(uint32_t microseconds) { g_wait_limit_us = microseconds; }

void tsa_set_test_stall(int32_t on) { g_test_stall = on ? 1 : 0; }

void tsa_set_score_schedule(int32_t wave, int32_t max_groups_per_wave) {
    g_score_wave = (wave == 1 || wave == 2) ? wave : 0;
    g_score_wave_cap = max_groups_per_wave > 0 ? max_groups_per_wave : 0;
}

uint64_t tsa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char *tsa_status_string(tsa_status s) {
    switch (s) {
        case TSA_OK: return "TSA_OK";
        case TSA_ERR_INVALID_ARG: return "TSA_ERR_INVALID_ARG";
        case TSA_ERR_ALIGNMENT: return "TSA_ERR_ALIGNMENT";
        case TSA_ERR_UNSUPPORTED: return "TSA_ERR_UNSUPPORTED";
        case TSA_ERR_WORKSPACE: return "TSA_ERR_WORKSPACE";
        case TSA_ERR_CUDA: return "TSA_ERR_CUDA";
        case TSA_ERR_DEVICE_TIMEOUT: return "TSA_ERR_DEVICE_TIMEOUT";
        case TSA_ERR_NONFINITE: return "TSA_ERR_NONFINITE";
    }
    return "TSA_ERR_UNKNOWN";
}

const char *tsa_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"

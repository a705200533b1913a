// api.cu -- the C ABI declared in include/hybattn.h: argument validation on
// the host, workspace carve-up and kernel launches on the caller's stream.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace hyb {

// An NVTX range around each entry point (host side), so that a profiler's
// timeline names the stage that launched each kernel.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};



cudaError_t launch_block_merge(const void *x, int B, int L, int H, int dx, int m, const float *w,
                               void *out, cudaStream_t stream, int num_sms);
cudaError_t launch_index_scores_simt(const void *qi, const float *wi, const void *kic, float *scores,
                                     int B, int Lq, int Hi, int di, int Nc, int m, int W,
                                     const int32_t *q_pos, cudaStream_t stream);
cudaError_t launch_index_scores_tc(const void *qi, const float *wi, const void *kic, float *scores,
                                   int B, int Lq, int Hi, int di, int Nc, int m, int W,
                                   const int32_t *q_pos, cudaStream_t stream);
cudaError_t launch_topk_radix(const float *scores, int B, int Lq, int Nc, int m, int W, int K,
                              const int32_t *q_pos, int32_t *idx, float *sel_scores,
                              cudaStream_t stream);
bool index_fused_supported(int Lq, int Hi, int di, int Nc, int K);
cudaError_t launch_index_topk_fused(const void *qi, const float *wi, const void *kic, int32_t *idx,
                                    float *sel, int B, int Lq, int Hi, int di, int Nc, int m, int W, int K,
                                    const int32_t *q_pos, cudaStream_t stream);
cudaError_t launch_hca_attn(int B, int L, int Lkv, int Hq, int Hkv, int d, int Nc, int m, int W,
                            float scale, const void *q, const void *kc, const void *vc, const void *kr,
                            const void *vr, void *o, float *lse, cudaStream_t stream, int num_sms);
cudaError_t launch_csa_attn(int B, int Lq, int Lkv, int Hq, int Hkv, int Nc, int m, int W, int topk,
                            float scale, const int32_t *q_pos, const int32_t *kv_pos0, const void *q,
                            const void *kc, const void *vc, const int32_t *idx, const void *kr,
                            const void *vr, void *o, float *lse, cudaStream_t stream, int num_sms,
                            int pregathered);
cudaError_t launch_fp4_quantize(const void *x, long long rows, int dx, uint8_t *codes, float *qp,
                                cudaStream_t stream, int num_sms);
cudaError_t launch_fp4_dequantize(const uint8_t *codes, const float *qp, long long rows, int dx,
                                  void *out, cudaStream_t stream, int num_sms);
cudaError_t launch_fp4_gather(const uint8_t *kcodes, const float *kqp, const uint8_t *vcodes,
                              const float *vqp, const int32_t *idx, void *kout, void *vout, int B, int Lq,
                              int topk, int Hkv, int Nc, int d, cudaStream_t stream, int num_sms);
cudaError_t launch_index_dec_fp4(const void *qi, const float *wi, const uint8_t *kic_codes,
                                 const float *kic_qp, float *scores, int B, int Lq, int Hi, int di, int Nc,
                                 int m, int W, const int32_t *q_pos, cudaStream_t stream);
cudaError_t launch_hybrid_attn(int B, int Lq, int Lkv, int Hq, int Hkv, int d, int Nc, int m, int W,
                               int topk, float scale, const int32_t *q_pos, const int32_t *kv_pos0,
                               const void *q, const void *kc, const void *vc, const int32_t *idx,
                               const void *kr, const void *vr, void *o, float *lse,
                               cudaStream_t stream);

cudaError_t launch_decode_append(const AppendParams &p, cudaStream_t stream);
cudaError_t launch_attn_bwd(const BwdParams &p, cudaStream_t stream);
cudaError_t launch_block_merge_bwd(const void *x, int B, int L, int H, int D, int m, const float *w,
                                   const float *dc, float *dx, float *dw, float *G, cudaStream_t stream,
                                   int num_sms);
cudaError_t launch_gated_combine(const void *o1, const void *o2, const void *o3, const float *gate,
                                 void *o, long long rows, int d, cudaStream_t stream, int num_sms);

static int num_sms_current()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

static bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// With HYB_VERBOSE set in the environment, failed CUDA calls are reported on stderr.
static hyb_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess)
        return HYB_OK;
    static const bool verbose = getenv("HYB_VERBOSE") != nullptr;
    if (verbose)
        fprintf(stderr, "hybattn: CUDA error %d: %s\n", (int)e, cudaGetErrorString(e));
    return HYB_ERR_CUDA;
}

// Largest shared-memory footprint of one top-K row (keys) + static tables.
static constexpr size_t kTopkSmemLimit = 227 * 1024 - 20 * 1024;

static hyb_status check_problem(const hyb_problem *p, bool need_indexer)
{
    if (!p)
        return HYB_ERR_INVALID_ARG;
    if (p->B <= 0 || p->Lq <= 0 || p->Lkv < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->m <= 0 ||
        p->W < 0 || p->Nc < 0)
        return HYB_ERR_INVALID_ARG;
    if (p->Hq % p->Hkv != 0)
        return HYB_ERR_INVALID_ARG;
    if (p->d != 64 && p->d != 128)
        return HYB_ERR_UNSUPPORTED;
    if (p->topk > 0) {
        if (p->Hq / p->Hkv > 64 || p->topk > 2048)
            return HYB_ERR_UNSUPPORTED;
    }
    if (need_indexer) {
        if (p->topk <= 0 || p->Hi <= 0 || p->di <= 0)
            return HYB_ERR_INVALID_ARG;
        if (p->di != 32 && p->di != 64)
            return HYB_ERR_UNSUPPORTED;
        if (p->Hi > 16 || (size_t)p->Nc * 4 > kTopkSmemLimit)
            return HYB_ERR_UNSUPPORTED;
    }
    if (p->Lkv >= (1 << 30) || p->Lq >= (1 << 30) || p->Nc >= (1 << 30))
        return HYB_ERR_UNSUPPORTED;
    return HYB_OK;
}

// Stage 2 into a caller-chosen score buffer of B * Lq * Nc floats: tensor
// cores where the shape allows, CUDA cores otherwise, then the exact top-K.
static cudaError_t index_topk_into(const hyb_problem *p, const void *qi, const float *wi,
                                   const void *kic, int32_t *idx, float *sel_scores, float *scores,
                                   cudaStream_t stream)
{
    cudaError_t e = launch_index_scores_tc(qi, wi, kic, scores, p->B, p->Lq, p->Hi, p->di, p->Nc,
                                           p->m, p->W, p->q_pos, stream);
    if (e == cudaErrorNotSupported)
        e = launch_index_scores_simt(qi, wi, kic, scores, p->B, p->Lq, p->Hi, p->di, p->Nc, p->m,
                                     p->W, p->q_pos, stream);
    if (e != cudaSuccess)
        return e;
    return launch_topk_radix(scores, p->B, p->Lq, p->Nc, p->m, p->W, p->topk, p->q_pos, idx,
                             sel_scores, stream);
}

// Bytes of the two-kernel path's score rows (B * Lq * Nc fp32), 256-byte rounded.
static size_t index_scores_bytes(const hyb_problem *p)
{
    const size_t scores = (size_t)p->B * p->Lq * p->Nc * sizeof(float);
    return (scores + 255) & ~(size_t)255;
}

// Stage 2 in one kernel (scores recomputed on chip, no score rows stored), or
// the two-kernel path above.  Where both take the shape, the two kernels
// finish first as long as the score rows stay small (measured on one B200 at
// L = 1024 to 16384 with up to 256 MB of rows: 0.034 against 0.089 ms at
// L = 1024, 0.28 against 0.44 ms at L = 16384; at L = 32768, 1 GB of rows,
// the two are within 5% and the one kernel stores nothing), so they run when
// the rows take at most kIndexScoresMaxBytes and `ws_avail` bytes hold them.
constexpr size_t kIndexScoresMaxBytes = (size_t)256 << 20;

static bool index_topk_fused_path(const hyb_problem *p, size_t ws_avail)
{
    if (!index_fused_supported(p->Lq, p->Hi, p->di, p->Nc, p->topk))
        return false;
    const size_t need = index_scores_bytes(p);
    return need > kIndexScoresMaxBytes || ws_avail < need;
}

static float softmax_scale(const hyb_problem *p)
{
    return p->scale != 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
}

// 4-bit caches.  Attention: when a query batch selects fewer rows than the
// cache holds (decode), only those are dequantized, in slot order (the CSA
// kernel then reads them as its "pre-gathered" rows); otherwise the whole K
// and V caches are dequantized once.  The workspace holds the bf16 K rows,
// then the V rows.
static bool fp4_attn_pregather(const hyb_problem *p)
{
    return p->topk > 0 && p->d == 128 && (long long)p->Lq * p->topk < (long long)p->Nc;
}

static size_t fp4_attn_bytes(const hyb_problem *p)
{
    const long long rows = fp4_attn_pregather(p) ? (long long)p->B * p->Lq * p->topk * p->Hkv
                                                 : (long long)p->B * p->Nc * p->Hkv;
    const size_t one = ((size_t)rows * p->d * 2 + 255) & ~(size_t)255;
    return 2 * one;
}

// Indexer: the decode form (few query rows, di = 64) dequantizes key tiles
// on chip; other shapes dequantize the indexer-key cache into the workspace
// after the score buffer.
static bool fp4_index_in_kernel(const hyb_problem *p)
{
    return p->di == 64 && p->Lq < 64 && p->Hi <= 16;
}

// Checks shared by the two decode-append entry points (the caches are
// checked by each); fills everything but the cache pointers.
static hyb_status append_common(const hyb_problem *p, const int32_t *t_new, const void *k_new,
                                const void *v_new, const void *ki_new, const float *wk, const float *wv,
                                const float *wib, void *k_ring, void *v_ring, void *ki_ring,
                                int32_t *kv_pos0, AppendParams &a)
{
    if (!p || p->B <= 0 || p->Hkv <= 0 || p->d <= 0 || p->m <= 0 || p->W <= 0 || p->Nc <= 0)
        return HYB_ERR_INVALID_ARG;
    if (p->d % 8 != 0 || p->Lkv != 2 * p->W)
        return HYB_ERR_INVALID_ARG;
    if (p->m > p->W)
        return HYB_ERR_UNSUPPORTED;   // a block must still be in the window when it completes
    const bool csa = p->topk > 0;
    if (!t_new || !k_new || !v_new || !wk || !wv || !k_ring || !v_ring || !kv_pos0)
        return HYB_ERR_INVALID_ARG;
    if (csa && (!ki_new || !wib || !ki_ring || p->di <= 0 || p->di % 8 != 0))
        return HYB_ERR_INVALID_ARG;
    const void *ptrs[] = {k_new, v_new, wk, wv, k_ring, v_ring};
    for (const void *q : ptrs)
        if (!aligned16(q))
            return HYB_ERR_INVALID_ARG;
    if (csa && (!aligned16(ki_new) || !aligned16(wib) || !aligned16(ki_ring)))
        return HYB_ERR_INVALID_ARG;
    a = AppendParams{};
    a.B = p->B;
    a.Hkv = p->Hkv;
    a.d = p->d;
    a.di = csa ? p->di : 0;
    a.m = p->m;
    a.W = p->W;
    a.Nc = p->Nc;
    a.t_new = t_new;
    a.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    a.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    a.ki_new = csa ? static_cast<const __nv_bfloat16 *>(ki_new) : nullptr;
    a.wk = wk;
    a.wv = wv;
    a.wib = csa ? wib : nullptr;
    a.k_ring = static_cast<__nv_bfloat16 *>(k_ring);
    a.v_ring = static_cast<__nv_bfloat16 *>(v_ring);
    a.ki_ring = csa ? static_cast<__nv_bfloat16 *>(ki_ring) : nullptr;
    a.kv_pos0 = kv_pos0;
    return HYB_OK;
}

}  // namespace hyb

using namespace hyb;

extern "C" {

size_t hyb_workspace_size(const hyb_problem *p)
{
    if (!p || p->topk <= 0 || p->B <= 0 || p->Lq <= 0 || p->Nc <= 0)
        return 0;
    // an unlimited workspace picks the path the shape runs fastest on
    if (index_topk_fused_path(p, ~(size_t)0))
        return 0;
    return index_scores_bytes(p);
}

hyb_status hyb_hca_compress(const void *x, int B, int L, int H, int dx, int m, const float *w,
                            void *out, cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_hca_compress");
    if (!x || !w || !out || B <= 0 || L < 0 || H <= 0 || dx <= 0 || m <= 0)
        return HYB_ERR_INVALID_ARG;
    if (dx % 8 != 0 || !aligned16(x) || !aligned16(out) || !aligned16(w))
        return HYB_ERR_INVALID_ARG;
    if (m > 256 || (size_t)m * dx > 32768)
        return HYB_ERR_UNSUPPORTED;
    return cuda_status(launch_block_merge(x, B, L, H, dx, m, w, out, stream, num_sms_current()));
}

hyb_status hyb_csa_index_topk(const hyb_problem *p, const void *qi, const float *wi, const void *kic,
                              int32_t *idx, float *sel_scores, void *ws, size_t ws_bytes,
                              cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_csa_index_topk");
    hyb_status st = check_problem(p, true);
    if (st != HYB_OK)
        return st;
    if (!qi || !wi || !kic || !idx || !aligned16(qi) || !aligned16(kic))
        return HYB_ERR_INVALID_ARG;
    const size_t avail = ws && !(reinterpret_cast<uintptr_t>(ws) & 255u) ? ws_bytes : 0;
    if (index_topk_fused_path(p, avail))
        return cuda_status(launch_index_topk_fused(qi, wi, kic, idx, sel_scores, p->B, p->Lq, p->Hi, p->di,
                                                   p->Nc, p->m, p->W, p->topk, p->q_pos, stream));
    if (avail < index_scores_bytes(p))
        return HYB_ERR_WORKSPACE;
    return cuda_status(index_topk_into(p, qi, wi, kic, idx, sel_scores, static_cast<float *>(ws),
                                       stream));
}

hyb_status hyb_attn_fwd(const hyb_problem *p, const void *q, const void *kc, const void *vc,
                        const int32_t *idx, const void *k_raw, const void *v_raw, void *o, float *lse,
                        cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_attn_fwd");
    hyb_status st = check_problem(p, false);
    if (st != HYB_OK)
        return st;
    if (!q || !o || !k_raw || !v_raw)
        return HYB_ERR_INVALID_ARG;
    if (p->Nc > 0 && (!kc || !vc))
        return HYB_ERR_INVALID_ARG;
    if (idx && p->topk <= 0)
        return HYB_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o) || !aligned16(k_raw) || !aligned16(v_raw) ||
        (kc && !aligned16(kc)) || (vc && !aligned16(vc)))
        return HYB_ERR_INVALID_ARG;
    if (p->Lkv <= 0 && p->W > 0)
        return HYB_ERR_INVALID_ARG;
    const int Lkv = p->Lkv > 0 ? p->Lkv : 1;
    if (!idx && !p->q_pos && !p->kv_pos0 && p->Lq == p->Lkv) {
        // prefill HCA: persistent two-tile kernel
        return cuda_status(launch_hca_attn(p->B, p->Lq, Lkv, p->Hq, p->Hkv, p->d, p->Nc, p->m, p->W,
                                           softmax_scale(p), q, kc, vc, k_raw, v_raw, o, lse, stream,
                                           num_sms_current()));
    }
    if (idx && p->d == 128 && p->Nc > 0) {
        // CSA: per-token selections, transposed tcgen05 kernel
        return cuda_status(launch_csa_attn(p->B, p->Lq, Lkv, p->Hq, p->Hkv, p->Nc, p->m, p->W,
                                           p->topk, softmax_scale(p), p->q_pos, p->kv_pos0, q, kc, vc,
                                           idx, k_raw, v_raw, o, lse, stream, num_sms_current(), 0));
    }
    cudaError_t e = launch_hybrid_attn(p->B, p->Lq, Lkv, p->Hq, p->Hkv, p->d, p->Nc, p->m, p->W,
                                       p->topk, softmax_scale(p), p->q_pos, p->kv_pos0, q, kc, vc, idx,
                                       k_raw, v_raw, o, lse, stream);
    return cuda_status(e);
}

hyb_status hyb_fused_fwd(const hyb_problem *p, const void *q, const void *k_raw, const void *v_raw,
                         const float *wk, const float *wv, const void *qi, const float *wi,
                         const void *ki_raw, const float *wib, void *kc, void *vc, void *kic,
                         int32_t *idx, void *o, float *lse, void *ws, size_t ws_bytes,
                         cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_fused_fwd");
    const bool csa = p && p->topk > 0;
    hyb_status st = check_problem(p, csa);
    if (st != HYB_OK)
        return st;
    if (!kc || !vc || (csa && (!kic || !idx || !qi || !wi)))
        return HYB_ERR_INVALID_ARG;
    if (wk) {  // prefill: build the compressed caches from the raw rows
        if (!wv || (csa && (!ki_raw || !wib)))
            return HYB_ERR_INVALID_ARG;
        if (p->Nc != p->Lkv / p->m)
            return HYB_ERR_INVALID_ARG;
        st = hyb_hca_compress(k_raw, p->B, p->Lkv, p->Hkv, p->d, p->m, wk, kc, stream);
        if (st != HYB_OK)
            return st;
        st = hyb_hca_compress(v_raw, p->B, p->Lkv, p->Hkv, p->d, p->m, wv, vc, stream);
        if (st != HYB_OK)
            return st;
        if (csa) {
            st = hyb_hca_compress(ki_raw, p->B, p->Lkv, 1, p->di, p->m, wib, kic, stream);
            if (st != HYB_OK)
                return st;
        }
    }
    if (csa) {
        st = hyb_csa_index_topk(p, qi, wi, kic, idx, nullptr, ws, ws_bytes, stream);
        if (st != HYB_OK)
            return st;
    }
    return hyb_attn_fwd(p, q, kc, vc, csa ? idx : nullptr, k_raw, v_raw, o, lse, stream);
}

hyb_status hyb_decode_append(const hyb_problem *p, const int32_t *t_new, const void *k_new,
                             const void *v_new, const void *ki_new, const float *wk, const float *wv,
                             const float *wib, void *k_ring, void *v_ring, void *ki_ring, void *kc,
                             void *vc, void *kic, int32_t *kv_pos0, cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_decode_append");
    AppendParams a;
    hyb_status st = append_common(p, t_new, k_new, v_new, ki_new, wk, wv, wib, k_ring, v_ring, ki_ring,
                                  kv_pos0, a);
    if (st != HYB_OK)
        return st;
    const bool csa = p->topk > 0;
    if (!kc || !vc || !aligned16(kc) || !aligned16(vc) || (csa && (!kic || !aligned16(kic))))
        return HYB_ERR_INVALID_ARG;
    a.kc = static_cast<__nv_bfloat16 *>(kc);
    a.vc = static_cast<__nv_bfloat16 *>(vc);
    a.kic = csa ? static_cast<__nv_bfloat16 *>(kic) : nullptr;
    return cuda_status(launch_decode_append(a, stream));
}

hyb_status hyb_decode_append_fp4(const hyb_problem *p, const int32_t *t_new, const void *k_new,
                                 const void *v_new, const void *ki_new, const float *wk, const float *wv,
                                 const float *wib, void *k_ring, void *v_ring, void *ki_ring,
                                 uint8_t *kc_codes, float *kc_qp, uint8_t *vc_codes, float *vc_qp,
                                 uint8_t *kic_codes, float *kic_qp, int32_t *kv_pos0, cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_decode_append_fp4");
    AppendParams a;
    hyb_status st = append_common(p, t_new, k_new, v_new, ki_new, wk, wv, wib, k_ring, v_ring, ki_ring,
                                  kv_pos0, a);
    if (st != HYB_OK)
        return st;
    const bool csa = p->topk > 0;
    if (p->d > 256 || (csa && p->di > 256))
        return HYB_ERR_UNSUPPORTED;
    if (!kc_codes || !kc_qp || !vc_codes || !vc_qp || (csa && (!kic_codes || !kic_qp)))
        return HYB_ERR_INVALID_ARG;
    if (!aligned16(kc_codes) || !aligned16(kc_qp) || !aligned16(vc_codes) || !aligned16(vc_qp) ||
        (csa && (!aligned16(kic_codes) || !aligned16(kic_qp))))
        return HYB_ERR_INVALID_ARG;
    a.kcq = kc_codes;
    a.vcq = vc_codes;
    a.kicq = csa ? kic_codes : nullptr;
    a.kqp = reinterpret_cast<float2 *>(kc_qp);
    a.vqp = reinterpret_cast<float2 *>(vc_qp);
    a.kiqp = csa ? reinterpret_cast<float2 *>(kic_qp) : nullptr;
    return cuda_status(launch_decode_append(a, stream));
}

hyb_status hyb_fp4_quantize(const void *x, long long rows, int dx, uint8_t *codes, float *qp,
                            cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_fp4_quantize");
    if (!x || !codes || !qp || rows < 0)
        return HYB_ERR_INVALID_ARG;
    if (dx != 64 && dx != 128 && dx != 256)
        return HYB_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(qp))
        return HYB_ERR_INVALID_ARG;
    return cuda_status(launch_fp4_quantize(x, rows, dx, codes, qp, stream, num_sms_current()));
}

hyb_status hyb_fp4_dequantize(const uint8_t *codes, const float *qp, long long rows, int dx, void *out,
                              cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_fp4_dequantize");
    if (!codes || !qp || !out || rows < 0 || dx <= 0 || dx % 8 != 0)
        return HYB_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(codes) || !aligned16(qp))
        return HYB_ERR_INVALID_ARG;
    return cuda_status(launch_fp4_dequantize(codes, qp, rows, dx, out, stream, num_sms_current()));
}

size_t hyb_fp4_workspace_size(const hyb_problem *p)
{
    if (!p || p->B <= 0 || p->Lq <= 0 || p->Hkv <= 0 || p->d <= 0 || p->Nc < 0)
        return 0;
    const size_t attn = fp4_attn_bytes(p);
    size_t index = 0;
    if (p->topk > 0 && p->Hi > 0 && p->di > 0) {
        index = hyb_workspace_size(p);
        if (!fp4_index_in_kernel(p))
            index += ((size_t)p->B * p->Nc * p->di * 2 + 255) & ~(size_t)255;
    }
    return attn > index ? attn : index;
}

hyb_status hyb_csa_index_topk_fp4(const hyb_problem *p, const void *qi, const float *wi,
                                  const uint8_t *kic_codes, const float *kic_qp, int32_t *idx,
                                  float *sel_scores, void *ws, size_t ws_bytes, cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_csa_index_topk_fp4");
    hyb_status st = check_problem(p, true);
    if (st != HYB_OK)
        return st;
    if (!qi || !wi || !kic_codes || !kic_qp || !idx || !aligned16(qi) || !aligned16(kic_codes) ||
        !aligned16(kic_qp))
        return HYB_ERR_INVALID_ARG;
    if (!ws || ws_bytes < hyb_fp4_workspace_size(p) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return HYB_ERR_WORKSPACE;
    float *scores = static_cast<float *>(ws);
    if (fp4_index_in_kernel(p)) {
        // decode: the indexer dequantizes key tiles on chip
        cudaError_t e = launch_index_dec_fp4(qi, wi, kic_codes, kic_qp, scores, p->B, p->Lq, p->Hi,
                                             p->di, p->Nc, p->m, p->W, p->q_pos, stream);
        if (e != cudaSuccess)
            return cuda_status(e);
        return cuda_status(launch_topk_radix(scores, p->B, p->Lq, p->Nc, p->m, p->W, p->topk, p->q_pos,
                                             idx, sel_scores, stream));
    }
    // otherwise the whole indexer-key cache is dequantized once
    uint8_t *kic = static_cast<uint8_t *>(ws) + hyb_workspace_size(p);
    cudaError_t e = launch_fp4_dequantize(kic_codes, kic_qp, (long long)p->B * p->Nc, p->di, kic, stream,
                                          num_sms_current());
    if (e != cudaSuccess)
        return cuda_status(e);
    if (index_topk_fused_path(p, hyb_workspace_size(p)))
        return cuda_status(launch_index_topk_fused(qi, wi, kic, idx, sel_scores, p->B, p->Lq, p->Hi, p->di,
                                                   p->Nc, p->m, p->W, p->topk, p->q_pos, stream));
    return cuda_status(index_topk_into(p, qi, wi, kic, idx, sel_scores, scores, stream));
}

hyb_status hyb_attn_fwd_fp4(const hyb_problem *p, const void *q, const uint8_t *kc_codes,
                            const float *kc_qp, const uint8_t *vc_codes, const float *vc_qp,
                            const int32_t *idx, const void *k_raw, const void *v_raw, void *o, float *lse,
                            void *ws, size_t ws_bytes, cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_attn_fwd_fp4");
    hyb_status st = check_problem(p, false);
    if (st != HYB_OK)
        return st;
    if (p->Nc <= 0 || !kc_codes || !kc_qp || !vc_codes || !vc_qp)
        return HYB_ERR_INVALID_ARG;
    if (!aligned16(kc_codes) || !aligned16(kc_qp) || !aligned16(vc_codes) || !aligned16(vc_qp))
        return HYB_ERR_INVALID_ARG;
    if (idx && p->topk <= 0)
        return HYB_ERR_INVALID_ARG;
    if (!ws || ws_bytes < fp4_attn_bytes(p) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return HYB_ERR_WORKSPACE;
    uint8_t *wk = static_cast<uint8_t *>(ws);
    const int n = num_sms_current();
    if (idx && fp4_attn_pregather(p)) {
        // decode: only the selected rows, dequantized in slot order
        if (!q || !o || !k_raw || !v_raw || !aligned16(q) || !aligned16(o) || !aligned16(k_raw) ||
            !aligned16(v_raw) || (p->Lkv <= 0 && p->W > 0))
            return HYB_ERR_INVALID_ARG;
        const size_t half = fp4_attn_bytes(p) / 2;
        cudaError_t e = launch_fp4_gather(kc_codes, kc_qp, vc_codes, vc_qp, idx, wk, wk + half, p->B, p->Lq,
                                          p->topk, p->Hkv, p->Nc, p->d, stream, n);
        if (e != cudaSuccess)
            return cuda_status(e);
        const int Lkv = p->Lkv > 0 ? p->Lkv : 1;
        return cuda_status(launch_csa_attn(p->B, p->Lq, Lkv, p->Hq, p->Hkv, p->Nc, p->m, p->W, p->topk,
                                           softmax_scale(p), p->q_pos, p->kv_pos0, q, wk, wk + half, idx,
                                           k_raw, v_raw, o, lse, stream, n, 1));
    }
    // otherwise the whole K / V caches are dequantized once
    const long long rows = (long long)p->B * p->Nc * p->Hkv;
    const size_t half = fp4_attn_bytes(p) / 2;
    cudaError_t e = launch_fp4_dequantize(kc_codes, kc_qp, rows, p->d, wk, stream, n);
    if (e == cudaSuccess)
        e = launch_fp4_dequantize(vc_codes, vc_qp, rows, p->d, wk + half, stream, n);
    if (e != cudaSuccess)
        return cuda_status(e);
    return hyb_attn_fwd(p, q, wk, wk + half, idx, k_raw, v_raw, o, lse, stream);
}

hyb_status hyb_attn_bwd(const hyb_problem *p, const void *q, const void *kc, const void *vc,
                        const int32_t *idx, const void *k_raw, const void *v_raw, const void *o,
                        const float *lse, const void *dout, float *dq, float *dkc, float *dvc,
                        float *dk_raw, float *dv_raw, cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_attn_bwd");
    hyb_status st = check_problem(p, false);
    if (st != HYB_OK)
        return st;
    if (!q || !o || !lse || !dout || !dq || !dk_raw || !dv_raw || !k_raw || !v_raw)
        return HYB_ERR_INVALID_ARG;
    if (p->Nc > 0 && (!kc || !vc || !dkc || !dvc))
        return HYB_ERR_INVALID_ARG;
    if (idx && p->topk <= 0)
        return HYB_ERR_INVALID_ARG;
    if (p->Lkv <= 0)
        return HYB_ERR_INVALID_ARG;
    // every kernel of the pass moves whole 16-byte pieces of these rows
    if (!aligned16(q) || !aligned16(k_raw) || !aligned16(v_raw) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk_raw) || !aligned16(dv_raw) ||
        (p->Nc > 0 && (!aligned16(kc) || !aligned16(vc) || !aligned16(dkc) || !aligned16(dvc))))
        return HYB_ERR_INVALID_ARG;
    const float scale = softmax_scale(p);
    if (attn_bwd_tc_ok(idx != nullptr, p->d, p->q_pos, p->kv_pos0, p->Lq, p->Lkv, p->Nc, p->m, p->W))
        return cuda_status(launch_attn_bwd_tc(p->B, p->Lq, p->Hq, p->Hkv, p->Nc, p->m, p->W, scale, q, kc, vc,
                                              k_raw, v_raw, o, lse, dout, dq, dkc, dvc, dk_raw, dv_raw, stream,
                                              num_sms_current()));
    // CSA prefill with a window and d = 128: the tensor-core passes take the
    // window keys (they zero dkc / dvc, store dk_raw / dv_raw and write dq's
    // window part), then the CUDA-core pass adds the selected entries' part
    const bool split = idx && attn_bwd_tc_window_ok(p->d, p->q_pos, p->kv_pos0, p->Lq, p->Lkv, p->W);
    cudaError_t e = cudaSuccess;
    if (split) {
        e = launch_attn_bwd_tc(p->B, p->Lq, p->Hq, p->Hkv, p->Nc, p->m, p->W, scale, q, kc, vc, k_raw, v_raw, o,
                               lse, dout, dq, dkc, dvc, dk_raw, dv_raw, stream, num_sms_current(), true);
    } else {
        const size_t ck = (size_t)p->B * p->Nc * p->Hkv * p->d * sizeof(float);
        const size_t rk = (size_t)p->B * p->Lkv * p->Hkv * p->d * sizeof(float);
        if (ck) {
            e = cudaMemsetAsync(dkc, 0, ck, stream);
            if (e == cudaSuccess)
                e = cudaMemsetAsync(dvc, 0, ck, stream);
        }
        if (e == cudaSuccess)
            e = cudaMemsetAsync(dk_raw, 0, rk, stream);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(dv_raw, 0, rk, stream);
    }
    if (e != cudaSuccess)
        return cuda_status(e);
    BwdParams b;
    b.comp_only = split ? 1 : 0;
    b.B = p->B;
    b.Lq = p->Lq;
    b.Lkv = p->Lkv;
    b.Hq = p->Hq;
    b.Hkv = p->Hkv;
    b.g = p->Hq / p->Hkv;
    b.d = p->d;
    b.Nc = p->Nc;
    b.m = p->m;
    b.W = p->W;
    b.topk = idx ? p->topk : 0;
    b.scale = scale;
    b.q_pos = p->q_pos;
    b.kv_pos0 = p->kv_pos0;
    b.idx = idx;
    b.q = static_cast<const __nv_bfloat16 *>(q);
    b.kc = static_cast<const __nv_bfloat16 *>(kc);
    b.vc = static_cast<const __nv_bfloat16 *>(vc);
    b.kr = static_cast<const __nv_bfloat16 *>(k_raw);
    b.vr = static_cast<const __nv_bfloat16 *>(v_raw);
    b.o = static_cast<const __nv_bfloat16 *>(o);
    b.dout = static_cast<const __nv_bfloat16 *>(dout);
    b.lse = lse;
    b.dq = dq;
    b.dkc = dkc;
    b.dvc = dvc;
    b.dkr = dk_raw;
    b.dvr = dv_raw;
    return cuda_status(launch_attn_bwd(b, stream));
}

size_t hyb_hca_compress_bwd_workspace_size(int dx, int m)
{
    if (dx <= 0 || m <= 0)
        return 0;
    return ((size_t)m * dx * sizeof(float) + 255) & ~(size_t)255;
}

hyb_status hyb_hca_compress_bwd(const void *x, int B, int L, int H, int dx, int m, const float *w,
                                const float *dc, float *dx_acc, float *dw, void *ws, size_t ws_bytes,
                                cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_hca_compress_bwd");
    if (!x || !w || !dc || !dx_acc || !dw || B <= 0 || L < 0 || H <= 0 || dx <= 0 || m <= 0)
        return HYB_ERR_INVALID_ARG;
    if (dx % 32 != 0)
        return HYB_ERR_UNSUPPORTED;
    if (m > 256)
        return HYB_ERR_UNSUPPORTED;
    const size_t need = hyb_hca_compress_bwd_workspace_size(dx, m);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return HYB_ERR_WORKSPACE;
    float *G = static_cast<float *>(ws);
    cudaError_t e = cudaMemsetAsync(G, 0, (size_t)m * dx * sizeof(float), stream);
    if (e != cudaSuccess)
        return cuda_status(e);
    return cuda_status(launch_block_merge_bwd(x, B, L, H, dx, m, w, dc, dx_acc, dw, G, stream, num_sms_current()));
}

size_t hyb_gated_workspace_size(const hyb_problem *p)
{
    if (!p || p->B <= 0 || p->Lq <= 0 || p->Hq <= 0 || p->d <= 0)
        return 0;
    const size_t one = ((size_t)p->B * p->Lq * p->Hq * p->d * 2 + 255) & ~(size_t)255;
    return 3 * one;
}

hyb_status hyb_gated_fwd(const hyb_problem *p, const void *q, const void *kc, const void *vc,
                         const int32_t *idx, const void *k_raw, const void *v_raw, const float *gate,
                         void *o, void *ws, size_t ws_bytes, cudaStream_t stream)
{
    NvtxRange nvtx_range("hyb_gated_fwd");
    hyb_status st = check_problem(p, false);
    if (st != HYB_OK)
        return st;
    if (!idx || p->topk <= 0 || !gate || !o || !q || p->Nc <= 0 || p->W <= 0 || p->d % 8 != 0)
        return HYB_ERR_INVALID_ARG;
    const size_t need = hyb_gated_workspace_size(p);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return HYB_ERR_WORKSPACE;
    const size_t one = need / 3;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    // branch 1: every compressed block that ends at or before t (no window)
    hyb_problem p1 = *p;
    p1.W = 0;
    p1.topk = 0;
    st = hyb_attn_fwd(&p1, q, kc, vc, nullptr, k_raw, v_raw, w8, nullptr, stream);
    if (st != HYB_OK)
        return st;
    // branch 2: the selected blocks among those (no window)
    hyb_problem p2 = *p;
    p2.W = 0;
    st = hyb_attn_fwd(&p2, q, kc, vc, idx, k_raw, v_raw, w8 + one, nullptr, stream);
    if (st != HYB_OK)
        return st;
    // branch 3: the raw window only
    hyb_problem p3 = *p;
    p3.Nc = 0;
    p3.topk = 0;
    st = hyb_attn_fwd(&p3, q, nullptr, nullptr, nullptr, k_raw, v_raw, w8 + 2 * one, nullptr, stream);
    if (st != HYB_OK)
        return st;
    return cuda_status(launch_gated_combine(w8, w8 + one, w8 + 2 * one, gate, o,
                                            (long long)p->B * p->Lq * p->Hq, p->d, stream,
                                            num_sms_current()));
}

hyb_status hyb_get_device_status(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return HYB_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess)
        return HYB_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess)
        return HYB_ERR_CUDA;
    return (hyb_status)v;
}

hyb_status hyb_set_wait_limit_ns(unsigned long long ns)
{
    const uint64_t v = ns ? (uint64_t)ns : kWaitLimitNs;
    return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

hyb_status hyb_trace_attach(void *buf, size_t bytes)
{
    unsigned long long *b = static_cast<unsigned long long *>(buf);
    unsigned int cap = 0;
    if (b) {
        if ((reinterpret_cast<uintptr_t>(buf) & 15u) || bytes < 96)
            return HYB_ERR_INVALID_ARG;
        const size_t recs = (bytes / 8 - 4) / 8;   // records per role region
        cap = recs > 0xFFFFFFFFull ? 0xFFFFFFFFu : (unsigned int)recs;
    }
    if (cudaMemcpyToSymbol(g_trace_cap, &cap, sizeof(cap)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_trace_buf, &b, sizeof(b)) != cudaSuccess)
        return HYB_ERR_CUDA;
    return HYB_OK;
}

const char *hyb_error_string(hyb_status s)
{
    switch (s) {
    case HYB_OK: return "ok";
    case HYB_ERR_INVALID_ARG: return "invalid argument";
    case HYB_ERR_UNSUPPORTED: return "unsupported shape or option";
    case HYB_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case HYB_ERR_CUDA: return "CUDA runtime error";
    case HYB_ERR_DEVICE_TIMEOUT: return "device wait exceeded its bound";
    case HYB_ERR_DEVICE_BOUNDS: return "device met an out-of-range index";
    }
    return "unknown status";
}

}  // extern "C"

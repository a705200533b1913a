/*
 * hybattn.h -- C ABI of the B200 (sm_100a) library for the forward pass of
 * DeepSeek-V4-style hybrid attention: compressed sparse attention (CSA),
 * heavily compressed attention (HCA) and a raw sliding window (SWA) under one
 * softmax.
 *
 * Sources of the operations (web pages on DeepSeek-V4 hybrid attention):
 *   "deepseek-v4" blog (s1mplewind), section 1 "hybrid attn": CSA (4:1
 *     compression, lightning indexer, top-K per query, sparse attention), HCA
 *     (m = 128, dense attention over the compressed history) and SWA (raw KV of
 *     the latest 128 tokens plus the compressed history, fed to one attention).
 *   CSDN "DeepSeek-V4 CSA / HCA mechanism" code page, section 1 (block_merge:
 *     per-channel softmax of a [m, d] weight over the block positions, then a
 *     weighted sum) and section 2 (block_compress).
 *   CS336 lecture notes, "Attention Heads variants" (MQA / GQA head sharing)
 *     and "Attention Alternatives" (FlashAttention; DSA lightning indexer).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major
 *     and contiguous in the stated shape.  bf16 tensors are passed as void*.
 *   - Every call is asynchronous on `stream`.  Argument errors are detected on
 *     the host and returned before anything is launched.  Errors found by a
 *     kernel (an index out of range, a wait that timed out) are recorded in a
 *     per-device status word that hyb_get_device_status() reads and clears.
 *   - The library never allocates device memory.  Scratch space comes from
 *     the caller's workspace, sized by hyb_workspace_size().
 *   - Supported shapes: head dim d in {64, 128}; indexer dim di in {32, 64};
 *     Hq % Hkv == 0; sparse (top-K) attention needs Hq / Hkv <= 64 and
 *     topk <= 2048; block size 1 <= m <= 256 with m * dx <= 32768.
 *   - Visibility: compressed entry j (raw positions j*m .. j*m+m-1) is visible
 *     to a query at position t iff (j + 1) * m - 1 < t - W + 1, i.e. it lies
 *     entirely before the query's raw window [max(0, t-W+1), t].
 */
#ifndef HYBATTN_H
#define HYBATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hyb_status {
    HYB_OK = 0,
    HYB_ERR_INVALID_ARG = -1,     /* null pointer, bad size, inconsistent shape   */
    HYB_ERR_UNSUPPORTED = -2,     /* a valid shape this build does not implement  */
    HYB_ERR_WORKSPACE = -3,       /* workspace missing or smaller than required   */
    HYB_ERR_CUDA = -4,            /* a CUDA runtime call failed                   */
    HYB_ERR_DEVICE_TIMEOUT = -5,  /* a kernel wait exceeded its bound (device)    */
    HYB_ERR_DEVICE_BOUNDS = -6    /* a kernel met an out-of-range index (device)  */
} hyb_status;

/* Problem description shared by the indexer, the attention and the fused
 * entry point.  Prefill: Lq == Lkv == L, q_pos == NULL, kv_pos0 == NULL.
 * Decode: Lq == 1, q_pos[b] = absolute position of the query, raw rows are the
 * last Lkv tokens with kv_pos0[b] = position of raw row 0, and the compressed
 * caches hold Nc entries per sequence. */
typedef struct hyb_problem {
    int B;          /* sequences                                              */
    int Lq;         /* query tokens per sequence                              */
    int Lkv;        /* raw K/V rows per sequence                              */
    int Hq;         /* query heads                                            */
    int Hkv;        /* KV heads; query head h uses KV head h / (Hq / Hkv)     */
    int d;          /* head dim (64 or 128)                                   */
    int m;          /* compression block size (CSA 4, HCA 128)                */
    int W;          /* sliding-window length in tokens (0 disables the window)*/
    int topk;       /* K of the per-query top-K; <= 0 selects HCA (dense)     */
    int Hi;         /* indexer heads (CSA only)                               */
    int di;         /* indexer dim (CSA only)                                 */
    int Nc;         /* compressed entries per sequence (cache capacity)       */
    float scale;    /* softmax scale; 0 means 1/sqrt(d)                       */
    const int32_t *q_pos;    /* [B, Lq] absolute query positions, or NULL (t) */
    const int32_t *kv_pos0;  /* [B] position of raw row 0, or NULL (0)        */
} hyb_problem;

/* Bytes of device workspace for the fastest path of hyb_csa_index_topk /
 * hyb_fused_fwd on `p`: 0 for HCA; for CSA, B * Lq * Nc fp32 score rows
 * (256-byte rounded), except 0 where the selection runs in one kernel that
 * recomputes the scores on chip and stores none: problems of Lq >= 64 query
 * rows per sequence, Hi <= 4, di 32 or 64, Nc <= 65535 and topk <= 2048 whose
 * score rows would exceed 256 MiB.  Such one-kernel problems with smaller
 * rows also run without the workspace (ws NULL or too small), in the one
 * kernel, only more slowly.  A workspace must be 256-byte aligned. */
size_t hyb_workspace_size(const hyb_problem *p);

/* Stage 1, block_merge (CSDN code page, section 1):
 *   out[b, j, h, c] = sum_{i<m} P[i, c] * x[b, j*m + i, h, c],
 *   P[i, c] = exp(w[i, c]) / sum_{i'} exp(w[i', c]),  j < floor(L / m).
 * x: [B, L, H, dx] bf16; w: [m, dx] fp32; out: [B, floor(L/m), H, dx] bf16
 * (fp32 accumulation, rounded to nearest even).  A trailing partial block is
 * ignored.  Used for the K and V caches (d) and the indexer keys (di, H = 1). */
hyb_status hyb_hca_compress(const void *x, int B, int L, int H, int dx, int m,
                            const float *w, void *out, cudaStream_t stream);

/* Stage 2, lightning indexer + exact per-query top-K (deepseek-v4 blog,
 * section 1, CSA; formula: ReLU-weighted head sum):
 *   I[t, s] = sum_h wi[t, h] * max(0, qi[t, h, :] . kic[s, :])   (fp32)
 * over the entries s visible to query t, then the K largest, ties to the
 * lower s.  idx[b, t, :] receives the chosen entries in ascending order, -1
 * padded when fewer than K are visible.  sel_scores (nullable) receives the
 * fp32 score of each idx slot (-inf for padding).
 * qi: [B, Lq, Hi, di] bf16; wi: [B, Lq, Hi] fp32; kic: [B, Nc, di] bf16;
 * idx: [B, Lq, topk] int32; ws: workspace of hyb_workspace_size(p) bytes.
 * Two paths: score rows written to the workspace by a tensor-core kernel,
 * then one CTA per row selecting from them; or one kernel that scores and
 * selects on chip with only per-row histograms (the one-kernel shapes of
 * hyb_workspace_size).  The two kernels run when the workspace holds the
 * score rows and they take at most 256 MiB; the one kernel otherwise.  Both
 * give the same selection.  HYB_ERR_WORKSPACE when neither can run. */
hyb_status hyb_csa_index_topk(const hyb_problem *p, const void *qi, const float *wi,
                              const void *kic, int32_t *idx, float *sel_scores,
                              void *ws, size_t ws_bytes, cudaStream_t stream);

/* Bytes of the fixed device scratch behind hyb_csa_index_topk_noalloc. */
#define HYB_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* Stage 2 without a workspace (the pages have no counterpart: this is a
 * service of the library, not a step of the method).  Same inputs, outputs
 * and results as hyb_csa_index_topk, but the score rows live in a fixed
 * 8 MiB device array inside the library, so the call allocates nothing and
 * needs no workspace.  Meant for callers that may not allocate device memory
 * themselves: an engine whose memory planner owns every buffer, or a decode
 * loop where cudaMalloc / cudaFree would synchronise the device.
 *   - Problems the one-kernel selection takes (see hyb_workspace_size) run
 *     there when their B * Lq * Nc * 4 bytes of score rows exceed
 *     HYB_NOALLOC_SCRATCH_BYTES; any other problem must fit its rows in it,
 *     otherwise the call returns HYB_ERR_UNSUPPORTED and launches nothing
 *     (the decode shape 64 x 16384 entries uses 4 MiB).
 *   - Every GPU that loads the library holds the array until the process
 *     exits.  The first call on a device looks up the array's address with
 *     that device current; make that first call before any stream capture.
 *     The address is kept for the life of the process: do not use this entry
 *     point after cudaDeviceReset() on that device, or from a CUDA context
 *     other than the device's primary context (the library's copy of the
 *     array lives at another address there).
 *   - All calls share the array: calls whose kernels overlap on the GPU (for
 *     example on different streams) race and must be serialised by the
 *     caller.  Nothing in it needs clearing between calls. */
hyb_status hyb_csa_index_topk_noalloc(const hyb_problem *p, const void *qi, const float *wi,
                                      const void *kic, int32_t *idx, float *sel_scores,
                                      cudaStream_t stream);

/* Stage 3, hybrid attention (deepseek-v4 blog, section 1, SWA): for every
 * (b, t, h) one softmax over
 *   compressed keys  idx[b, t, :] entries that are >= 0 and visible (CSA), or
 *                    every visible entry when idx == NULL (HCA), and
 *   raw keys         positions max(0, t-W+1) .. t (rows p - kv_pos0[b]),
 *   o = sum softmax(scale * q . k) v,  lse = log sum exp(scale * q . k).
 * q: [B, Lq, Hq, d]; kc, vc: [B, Nc, Hkv, d]; k_raw, v_raw: [B, Lkv, Hkv, d],
 * all bf16; idx: [B, Lq, topk] int32 (distinct entries) or NULL;
 * o: [B, Lq, Hq, d] bf16; lse: [B, Hq, Lq] fp32 (nullable).  An empty key set
 * gives o = 0 and lse = -inf.  idx entries >= Nc are skipped and flagged as
 * HYB_ERR_DEVICE_BOUNDS. */
hyb_status hyb_attn_fwd(const hyb_problem *p, const void *q, const void *kc, const void *vc,
                        const int32_t *idx, const void *k_raw, const void *v_raw, void *o,
                        float *lse, cudaStream_t stream);

/* The whole forward pass on one stream (deepseek-v4 blog, section 1: CSA
 * compresses every m raw KV rows into one entry and its lightning indexer
 * picks the top-K entries for each query; HCA attends densely to every
 * compressed entry; SWA adds the raw KV of the latest W tokens, and the
 * compressed and raw keys enter one attention):
 *   prefill (wk != NULL): kc = block_merge(k_raw, wk), vc = block_merge(v_raw, wv)
 *     and, for CSA, kic = block_merge(ki_raw, wib); Nc must equal Lkv / m.
 *   decode (wk == NULL): kc, vc, kic are read as ready caches of Nc entries.
 *   CSA (topk > 0): idx = top-K of the indexer scores (stage 2).
 *   then o, lse = hybrid attention (stage 3).
 * ki_raw: [B, Lkv, di] bf16; wk, wv: [m, d] fp32; wib: [m, di] fp32;
 * kc, vc: [B, Nc, Hkv, d]; kic: [B, Nc, di]; idx: [B, Lq, topk] (CSA only).
 * ws must hold hyb_workspace_size(p) bytes. */
hyb_status hyb_fused_fwd(const hyb_problem *p, const void *q, const void *k_raw,
                         const void *v_raw, const float *wk, const float *wv, const void *qi,
                         const float *wi, const void *ki_raw, const float *wib, void *kc,
                         void *vc, void *kic, int32_t *idx, void *o, float *lse, void *ws,
                         size_t ws_bytes, cudaStream_t stream);

/* Decode cache maintenance (deepseek-v4 blog, section 1: the window's raw KV
 * and the compressed KV are separate caches with different lifetimes).  For
 * every sequence b the new token at absolute position t = t_new[b] is
 * appended:
 *   - its K and V rows go to the raw-window ring twice, rows t mod W and
 *     t mod W + W, so that the window max(0, t-W+1) .. t is one contiguous
 *     run of ring rows; kv_pos0[b] (output) is the absolute position of ring
 *     row 0 for that run, i.e. lo - lo mod W with lo = max(0, t-W+1).  Call
 *     hyb_attn_fwd / hyb_fused_fwd next with k_raw = k_ring, v_raw = v_ring,
 *     Lkv = 2W, q_pos = t and this kv_pos0;
 *   - its indexer key (CSA, p->topk > 0) goes to row t mod W of ki_ring;
 *   - when (t + 1) is a multiple of m, block j = (t+1)/m - 1 (positions
 *     j*m .. t) becomes compressed entry j of kc, vc (and kic): the block_merge
 *     of hyb_hca_compress applied to that one block.
 * p: B, Hkv, d, m, W, Nc (cache capacity), topk / di (CSA); requires
 * Lkv == 2*W and m <= W (else HYB_ERR_INVALID_ARG / HYB_ERR_UNSUPPORTED).
 * t_new: [B] int32; k_new, v_new: [B, Hkv, d] bf16; ki_new: [B, di] bf16;
 * wk, wv: [m, d] fp32; wib: [m, di] fp32; k_ring, v_ring: [B, 2W, Hkv, d];
 * ki_ring: [B, W, di]; kc, vc: [B, Nc, Hkv, d]; kic: [B, Nc, di]; kv_pos0:
 * [B] int32 out.  A negative t, or an entry j >= Nc, is skipped and flagged
 * as HYB_ERR_DEVICE_BOUNDS.  The rings start zeroed or filled by earlier
 * calls; rows of positions outside the window are never read. */
hyb_status hyb_decode_append(const hyb_problem *p, const int32_t *t_new, const void *k_new,
                             const void *v_new, const void *ki_new, const float *wk,
                             const float *wv, const float *wib, void *k_ring, void *v_ring,
                             void *ki_ring, void *kc, void *vc, void *kic, int32_t *kv_pos0,
                             cudaStream_t stream);

/* The gated three-branch variant (Tiny-R2 README, "Attention Computation",
 * "branch_gate"): three attentions with separate softmaxes, then
 *   o[b,t,h] = sum_k softmax(gate[b,t,h,:])_k * o_k[b,t,h]
 * with
 *   o_1: every compressed block ending at or before t (all visible with W=0),
 *   o_2: the blocks of idx among those (the selection made with W = 0),
 *   o_3: the raw keys max(0, t-W+1) .. t;
 * a branch with no key gives 0.  Inputs as hyb_attn_fwd (idx required);
 * gate: [B, Lq, Hq, 3] fp32 logits (the output of the page's gate Linear,
 * which is out of scope here); o: [B, Lq, Hq, d] bf16.  ws: device
 * workspace of >= hyb_gated_workspace_size(p) bytes, 256-byte aligned (the
 * three branch outputs, bf16). */
size_t hyb_gated_workspace_size(const hyb_problem *p);
hyb_status hyb_gated_fwd(const hyb_problem *p, const void *q, const void *kc, const void *vc,
                         const int32_t *idx, const void *k_raw, const void *v_raw,
                         const float *gate, void *o, void *ws, size_t ws_bytes,
                         cudaStream_t stream);

/* Backward pass for training (Tiny-R2 README, "Training"), with the top-K
 * selection taken as fixed (the pages define no gradient for it).
 * hyb_attn_bwd: gradients of sum(dout * o) through hyb_attn_fwd for the same
 * problem and inputs; o [B, Lq, Hq, d] bf16 and lse [B, Hq, Lq] fp32 are
 * that call's outputs, dout [B, Lq, Hq, d] bf16.  Per query row with key set
 * S: P_j = exp(scale q.k_j - lse), dS_j = P_j (dout.v_j - dout.o),
 * dq = scale sum_j dS_j k_j, dk_j += scale dS_j q, dv_j += P_j dout.
 * Every pointer 16-byte aligned (else HYB_ERR_INVALID_ARG, nothing launched).
 * Outputs fp32, caller-owned, overwritten: dq [B, Lq, Hq, d]; dkc, dvc
 * [B, Nc, Hkv, d]; dk_raw, dv_raw [B, Lkv, Hkv, d] (the window path only:
 * the path through the compression is hyb_hca_compress_bwd's).  Dense
 * prefill problems (idx NULL, d = 128, q_pos and kv_pos0 NULL, Lq == Lkv) run
 * on the tensor cores: a pass over key tiles for dk / dv and one over query
 * tiles for dq, with P and dS rounded to bf16 as MMA operands (fp32
 * accumulation); dq's memory holds dout.o of each row while the call runs.
 * CSA prefill problems with d = 128 and a window split: those passes take the
 * window keys, an fp32 CUDA-core kernel the selected entries (adding into
 * dq).  Every other problem runs the CUDA-core kernel alone. */
hyb_status hyb_attn_bwd(const hyb_problem *p, const void *q, const void *kc, const void *vc,
                        const int32_t *idx, const void *k_raw, const void *v_raw, const void *o,
                        const float *lse, const void *dout, float *dq, float *dkc, float *dvc,
                        float *dk_raw, float *dv_raw, cudaStream_t stream);
/* hyb_hca_compress_bwd: gradients of sum(dc * c), c = hyb_hca_compress(x, w,
 * m): dx_acc [B, L, H, dx] fp32 += P[i] dc_j at row j m + i (rows of a
 * trailing partial block get nothing), dw [m, dx] fp32 overwritten with
 * P (G - sum_k P_k G_k), G[i] = sum of dc_j x_{jm+i} over blocks, batches and
 * heads (P = softmax over positions of w, per channel).  dc [B, L/m, H, dx]
 * fp32; x bf16 as the forward; dx a multiple of 32, m <= 256.  ws: device
 * workspace of hyb_hca_compress_bwd_workspace_size(dx, m) bytes, 256-byte
 * aligned.  With x, dc and dx_acc 16-byte aligned and the softmax weights,
 * the G partials and one block of dc fitting in shared memory, one pass
 * walks whole compression blocks (contiguous rows of every head); otherwise
 * a pass per 32 channels. */
size_t hyb_hca_compress_bwd_workspace_size(int dx, int m);
hyb_status hyb_hca_compress_bwd(const void *x, int B, int L, int H, int dx, int m, const float *w,
                                const float *dc, float *dx_acc, float *dw, void *ws, size_t ws_bytes,
                                cudaStream_t stream);

/* 4-bit compressed caches (CSDN code page, section 1, compress_to_fp4 /
 * decompress_from_fp4).  Every row of dx channels -- one compressed entry
 * of one head (K, V) or one indexer key -- is stored as dx/2 bytes of codes
 * (element 2i in the low nibble of byte i) and one fp32 pair (min, scale):
 *   scale = (max - min) / 15,  code = clamp(rint((x - min) / scale), 0, 15),
 *   value = code * scale + min, rounded to bf16,
 * each step one IEEE fp32 operation (ties to even; a row with max == min
 * has scale 0 and codes 0).  The page takes min and max over the whole
 * tensor; here they are per row, so a cache grows one entry at a time.
 * codes: [rows, dx/2] uint8, qp: [rows, 2] fp32; all pointers device,
 * 16-byte aligned, caller-owned. */
hyb_status hyb_fp4_quantize(const void *x /*[rows, dx] bf16*/, long long rows, int dx,
                            uint8_t *codes, float *qp, cudaStream_t stream);   /* dx 64/128/256 */
hyb_status hyb_fp4_dequantize(const uint8_t *codes, const float *qp, long long rows, int dx,
                              void *out /*[rows, dx] bf16*/, cudaStream_t stream);
/* Workspace (bytes, 256-aligned use) for hyb_csa_index_topk_fp4 and
 * hyb_attn_fwd_fp4 with this problem. */
size_t hyb_fp4_workspace_size(const hyb_problem *p);
/* hyb_csa_index_topk over a 4-bit indexer-key cache (kic_codes [B, Nc,
 * di/2], kic_qp [B, Nc, 2]); results as hyb_csa_index_topk on the
 * dequantized cache.  Decode shapes (Lq < 64, di = 64, Hi <= 16) dequantize
 * key tiles on chip; others dequantize the cache into ws first. */
hyb_status hyb_csa_index_topk_fp4(const hyb_problem *p, const void *qi, const float *wi,
                                  const uint8_t *kic_codes, const float *kic_qp, int32_t *idx,
                                  float *sel_scores, void *ws, size_t ws_bytes,
                                  cudaStream_t stream);
/* hyb_attn_fwd over 4-bit K / V caches (codes [B, Nc, Hkv, d/2], qp [B, Nc,
 * Hkv, 2]); results as hyb_attn_fwd on the dequantized caches.  When the
 * query batch selects fewer rows than the cache holds (CSA, d = 128, Lq *
 * topk < Nc) only the selected rows are dequantized into ws; otherwise the
 * whole K and V caches are. */
hyb_status hyb_attn_fwd_fp4(const hyb_problem *p, const void *q, const uint8_t *kc_codes,
                            const float *kc_qp, const uint8_t *vc_codes, const float *vc_qp,
                            const int32_t *idx, const void *k_raw, const void *v_raw, void *o,
                            float *lse, void *ws, size_t ws_bytes, cudaStream_t stream);
/* hyb_decode_append with 4-bit caches: a closing block is merged into its
 * bf16 entry as in hyb_decode_append, and each (entry, head) row of it is
 * then quantized as hyb_fp4_quantize does.  Requires d, di <= 256. */
hyb_status hyb_decode_append_fp4(const hyb_problem *p, const int32_t *t_new, const void *k_new,
                                 const void *v_new, const void *ki_new, const float *wk,
                                 const float *wv, const float *wib, void *k_ring, void *v_ring,
                                 void *ki_ring, uint8_t *kc_codes, float *kc_qp,
                                 uint8_t *vc_codes, float *vc_qp, uint8_t *kic_codes,
                                 float *kic_qp, int32_t *kv_pos0, cudaStream_t stream);


/* Synchronises `stream`, then returns and clears the device status word of
 * the current device (HYB_OK, HYB_ERR_DEVICE_TIMEOUT or HYB_ERR_DEVICE_BOUNDS). */
hyb_status hyb_get_device_status(cudaStream_t stream);

/* Static description of a status code. */
const char *hyb_error_string(hyb_status status);

/* Failure detection (the pages have no counterpart): every wait inside a
 * kernel is bounded; when one runs out the kernel records
 * HYB_ERR_DEVICE_TIMEOUT in the status word and every CTA unwinds (waits for
 * its own copies and MMAs in flight, frees its tensor memory, returns).  The
 * bound is 200 ms; this sets it for later launches on the current device
 * (0 restores 200 ms).  A tiny bound makes the first wait that is not already
 * satisfied run out -- the way a test exercises the error path without a
 * fault.  Read the status (hyb_get_device_status) before launching with the
 * normal bound again: a recorded timeout makes later waits give up too. */
hyb_status hyb_set_wait_limit_ns(unsigned long long ns);

/* Debug aid (the pages have no counterpart): a per-role timeline of one CTA.
 * Attaches a caller-owned device buffer of `bytes` bytes (16-byte aligned,
 * >= 96) for the kernels launched afterwards on the current device; NULL
 * detaches.  One thread per role of CTA 0 of a kernel that supports it (the
 * CSA and HCA attention kernels, the fused indexer) then appends a record per event to
 * its role's region.  Layout, in 8-byte words: words 0-3 count the records of
 * roles 0-3 (zero them before the launch); with R = (bytes / 8 - 4) / 8,
 * role r's records start at word 4 + 2 r R, each two words -- the SM clock,
 * then role << 56 | event << 48 | item << 16 | tile.  Records past R are
 * dropped (the count still grows).  Roles and events of the CSA attention
 * kernel: 1 gather (1 K tile issued, 2 V tile issued, 3 item begun, 4 item's
 * selection decoded), 2 MMA (1 QK^T issued, 2 PV issued), 3 softmax
 * warpgroup 0 (1 scores read, 2 P written, 3 item epilogue begun, 4 item
 * done).  The HCA attention kernel: 1 K / V loads (1 K tile, 2 V tile), 2 MMA
 * (1 QK^T of tile A, 2 PV of tile A, 3 QK^T of tile B, 4 PV of tile B), 3 and
 * 0 the softmax of query tiles A and B (1 scores read, 2 P written, 3 item
 * epilogue begun, 4 item done).  A record costs the tracing thread two stores;
 * detach the buffer before timing anything. */
hyb_status hyb_trace_attach(void *buf, size_t bytes);

/* Measurement kernel (the pages have no counterpart): the rate at which the
 * SMs gather random rows held in L2 into shared memory -- the data path of the
 * CSA attention, whose selected compressed rows differ per query token.  One
 * CTA per SM copies rows_per_sm random 256-byte rows of `table` (device, 16-byte
 * aligned, table_bytes bytes; keep it well under the L2 size) into a ring of
 * `stages` (2..6) 32 KB shared-memory stages with 16-byte cp.async, rows
 * chosen by a hash.  sink: device array of 256 uint32 receiving a checksum.
 * Time the call with events on `stream`: bytes moved = SMs * rows_per_sm * 256
 * (rows_per_sm is rounded down to a multiple of 128). */
hyb_status hyb_probe_l2_gather(const void *table, long long table_bytes, long long rows_per_sm,
                               int stages, unsigned int *sink, cudaStream_t stream);

/* The same measurement with the tensor memory accelerator's row gather
 * (cp.async.bulk.tensor tile::gather4, four rows per copy, one warp per CTA):
 * rows land in 128-byte-swizzled stages and each stage's completion is counted
 * in bytes on an mbarrier.  sink: device array of 257 uint32; sink[0..255]
 * receive a checksum and sink[256] the number of 16-byte chunks of each CTA's
 * last stage that are not where the 128-byte swizzle places them (added to
 * what it holds; 0 when the layout is the one the CSA attention reads).  The
 * table must hold fewer than 2^31 rows; other arguments as above. */
hyb_status hyb_probe_l2_gather_tma(const void *table, long long table_bytes, long long rows_per_sm,
                                   int stages, unsigned int *sink, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* HYBATTN_H */

// attn.cu -- stage 3, hybrid attention ("deepseek-v4" blog, section 1, SWA:
// the compressed history and the raw KV of the latest W tokens enter one
// attention; CSA feeds the top-K selected compressed entries, HCA all visible
// ones).  One online softmax in fp32 (flash-style, CS336 notes "Attention
// Alternatives": FlashAttention) runs over the union of both key sets.
//
// tcgen05 design, one CTA = one tile of query rows, 256 threads:
//   warp 0..2   producer.  Dense (HCA) mode: lane 0 of warp 0 issues TMA tile
//               loads (128-byte swizzle).  Sparse (CSA) mode: the 96 threads
//               gather the selected compressed rows and the window rows with
//               16-byte cp.async into the same swizzled layout.
//   warp 3      allocates TMEM (512 columns); lane 0 issues every tcgen05.mma.
//   warp 4..7   softmax + epilogue: thread = one TMEM lane = one query row.
// Rows of a tile:
//   dense  (idx == NULL): BM = 128 consecutive query tokens of one head.
//   sparse (idx != NULL): the g query heads sharing one KV head at one token
//                         (MQA/GQA, CS336 "Attention Heads variants"), padded
//                         to BM = 64 (tcgen05 M = 64, rows in TMEM lanes
//                         0-15 of each 32-lane quadrant).
// Key tiles of BN = 128 keys: first the compressed entries, then raw rows.
// S = Q K^T (TMEM, double-buffered), P = softmax numerators in bf16 written
// to shared memory, O += P V (TMEM).  The running max is only moved (and O
// rescaled) when a new tile max exceeds it by more than 2^8, so the rescale
// of O in TMEM is rare; final o = O / l and lse from the kept max.
#include "common.cuh"

namespace hyb {

constexpr int kAttnThreads = 256;
constexpr int kBN = 128;      // keys per tile
constexpr int kStages = 2;    // K/V pipeline depth
constexpr int kProducerThreads = 96;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnParams {
    int B, Lq, Lkv, Hq, Hkv, g, Nc, m, W, topk;
    float scale_log2;               // softmax scale * log2(e)
    const int32_t *q_pos;           // [B, Lq] or NULL
    const int32_t *kv_pos0;         // [B] or NULL
    const int32_t *idx;             // [B, Lq, topk] or NULL (dense)
    const __nv_bfloat16 *kc, *vc;   // [B, Nc, Hkv, d]
    const __nv_bfloat16 *kr, *vr;   // [B, Lkv, Hkv, d]
    __nv_bfloat16 *o;               // [B, Lq, Hq, d]
    float *lse;                     // [B, Hq, Lq] or NULL
    int n_qtiles;                   // dense: ceil(Lq / 128)
};

template <int D, bool SPARSE>
struct AttnSmem {
    static constexpr int BM = SPARSE ? 64 : 128;
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = kBN * D * 2;
    static constexpr int P_BYTES = BM * kBN * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + kStages * KV_BYTES;
    static constexpr int OFF_P = OFF_V + kStages * KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;          // 16 barriers
    static constexpr int OFF_MISC = OFF_BAR + 16 * 8;        // 32 ints
    static constexpr int OFF_SEL = OFF_MISC + 32 * 4;        // topk ints (sparse)
    static constexpr int BASE_BYTES = OFF_SEL;
};

enum { BAR_Q = 0, BAR_KF = 1, BAR_VF = 3, BAR_KVE = 5, BAR_SF = 7, BAR_PF = 9, BAR_OD = 10,
       BAR_DONE = 11 };
enum { MI_TMEM = 0, MI_ABORT = 1, MI_NCT = 2, MI_NRT = 3, MI_RLO = 4, MI_RHI = 5, MI_NSEL = 6,
       MI_POSMIN = 7, MI_POSMAX = 8, MI_KV0 = 9 };

__device__ __forceinline__ int n_visible(long long t, int m, int W, int Nc)
{
    long long a = t - W + 1;
    if (a <= 0)
        return 0;
    long long n = a / m;
    return n < Nc ? (int)n : Nc;
}

template <int D, bool SPARSE>
__global__ void __launch_bounds__(kAttnThreads, 1)
hybrid_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kr,
                   const __grid_constant__ CUtensorMap tm_vr, const AttnParams p)
{
    using SM = AttnSmem<D, SPARSE>;
    constexpr int BM = SM::BM;
    constexpr int NCB = D / 64;  // 64-element column blocks of a head row

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sQ = smem + SM::OFF_Q;
    uint8_t *sK = smem + SM::OFF_K;
    uint8_t *sV = smem + SM::OFF_V;
    uint8_t *sP = smem + SM::OFF_P;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM::OFF_BAR);
    int *misc = reinterpret_cast<int *>(smem + SM::OFF_MISC);
    int *sel = reinterpret_cast<int *>(smem + SM::OFF_SEL);
    volatile int *abort_flag = misc + MI_ABORT;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- tile coordinates ----
    const int b = blockIdx.z;
    int kvh, h_first, t_tok, t0;
    if (SPARSE) {
        kvh = blockIdx.y;
        h_first = kvh * p.g;
        t_tok = blockIdx.x;
        t0 = t_tok;
    } else {
        h_first = blockIdx.y;
        kvh = h_first / p.g;
        t0 = (p.n_qtiles - 1 - (int)blockIdx.x) * BM;  // long tiles first
        t_tok = t0;
    }
    const long long kv0 = p.kv_pos0 ? p.kv_pos0[b] : 0;

    // ---- setup: barriers, TMEM, tile schedule ----
    if (threadIdx.x == 0) {
        mbar_init(&bar[BAR_Q], 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar[BAR_KF + s], SPARSE ? kProducerThreads : 1);
            mbar_init(&bar[BAR_VF + s], SPARSE ? kProducerThreads : 1);
            mbar_init(&bar[BAR_KVE + s], 1);
            mbar_init(&bar[BAR_SF + s], 1);
        }
        mbar_init(&bar[BAR_PF], 128);
        mbar_init(&bar[BAR_OD], 1);
        mbar_init(&bar[BAR_DONE], 1);
        mbar_fence_init();
        misc[MI_ABORT] = 0;
    }
    if (warp == 3) {
        tmem_alloc(reinterpret_cast<uint32_t *>(&misc[MI_TMEM]), 512);
    }
    if (warp == 0) {
        // positions covered by this tile (min / max over its valid rows)
        long long pmin = LLONG_MAX, pmax = LLONG_MIN;
        const int rows = SPARSE ? 1 : BM;
        for (int r = lane; r < rows; r += 32) {
            int t = t0 + r;
            if (t < p.Lq) {
                long long pos = p.q_pos ? p.q_pos[(size_t)b * p.Lq + t] : t;
                pmin = min(pmin, pos);
                pmax = max(pmax, pos);
            }
        }
        for (int off = 16; off; off >>= 1) {
            pmin = min(pmin, (long long)__shfl_xor_sync(0xffffffffu, pmin, off));
            pmax = max(pmax, (long long)__shfl_xor_sync(0xffffffffu, pmax, off));
        }
        int nsel = 0;
        if (SPARSE) {
            // compact the listed entries that exist and are visible
            const int32_t *row_idx = p.idx + ((size_t)b * p.Lq + t_tok) * p.topk;
            for (int k0 = 0; k0 < p.topk; k0 += 32) {
                int k = k0 + lane;
                int j = k < p.topk ? row_idx[k] : -1;
                if (j >= p.Nc) {
                    set_error(HYB_ERR_DEVICE_BOUNDS);
                    j = -1;
                }
                bool ok = j >= 0 && ((long long)(j + 1) * p.m - 1 < pmax - p.W + 1);
                unsigned bal = __ballot_sync(0xffffffffu, ok);
                if (ok)
                    sel[nsel + __popc(bal & ((1u << lane) - 1))] = j;
                nsel += __popc(bal);
            }
        }
        if (lane == 0) {
            int nct;
            if (SPARSE) {
                nct = (nsel + kBN - 1) / kBN;
            } else {
                int nv = pmax >= pmin ? n_visible(pmax, p.m, p.W, p.Nc) : 0;
                nct = (nv + kBN - 1) / kBN;
            }
            long long lo = pmin - p.W + 1;
            if (lo < 0)
                lo = 0;
            lo -= kv0;
            long long hi = pmax - kv0;
            if (lo < 0)
                lo = 0;
            if (hi > p.Lkv - 1)
                hi = p.Lkv - 1;
            int nrt = (p.W > 0 && pmax >= pmin && hi >= lo) ? (int)((hi - lo + kBN) / kBN) : 0;
            misc[MI_NCT] = nct;
            misc[MI_NRT] = nrt;
            misc[MI_RLO] = (int)lo;
            misc[MI_RHI] = (int)hi;
            misc[MI_NSEL] = nsel;
            misc[MI_POSMIN] = (int)pmin;
            misc[MI_POSMAX] = (int)pmax;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = (uint32_t)misc[MI_TMEM];
    const int nct = misc[MI_NCT];
    const int nrt = misc[MI_NRT];
    const int ntiles = nct + nrt;
    const int rlo = misc[MI_RLO];
    const int rhi = misc[MI_RHI];
    const int nsel = misc[MI_NSEL];

    constexpr uint32_t TM_S0 = 0, TM_O = 2 * kBN;

    if (warp < 3) {
        // =========================== producer ===========================
        if (!SPARSE) {
            if (warp == 0 && lane == 0) {
                tma_prefetch_desc(&tm_q);
                mbar_arrive_expect_tx(&bar[BAR_Q], SM::Q_BYTES);
                for (int cb = 0; cb < NCB; ++cb)
                    tma_load_4d(sQ + cb * BM * 128, &tm_q, &bar[BAR_Q], cb * 64, h_first, t0, b);
                int issued = 0;
                for (int i = 0; i < ntiles; ++i) {
                    const int s = i % kStages;
                    if (i >= kStages && !mbar_wait(&bar[BAR_KVE + s], ((i / kStages) - 1) & 1, abort_flag))
                        break;
                    const bool comp = i < nct;
                    const CUtensorMap *mk = comp ? &tm_kc : &tm_kr;
                    const CUtensorMap *mv = comp ? &tm_vc : &tm_vr;
                    const int row0 = comp ? i * kBN : rlo + (i - nct) * kBN;
                    mbar_arrive_expect_tx(&bar[BAR_KF + s], SM::KV_BYTES);
                    for (int cb = 0; cb < NCB; ++cb)
                        tma_load_4d(sK + s * SM::KV_BYTES + cb * kBN * 128, mk, &bar[BAR_KF + s],
                                    cb * 64, kvh, row0, b);
                    mbar_arrive_expect_tx(&bar[BAR_VF + s], SM::KV_BYTES);
                    for (int cb = 0; cb < NCB; ++cb)
                        tma_load_4d(sV + s * SM::KV_BYTES + cb * kBN * 128, mv, &bar[BAR_VF + s],
                                    cb * 64, kvh, row0, b);
                    ++issued;
                }
                // unwinding: make sure no TMA write is still in flight
                drain_wait(&bar[BAR_Q], 0);
                for (int i = issued - kStages; i < issued; ++i) {
                    if (i < 0)
                        continue;
                    drain_wait(&bar[BAR_KF + i % kStages], (i / kStages) & 1);
                    drain_wait(&bar[BAR_VF + i % kStages], (i / kStages) & 1);
                }
            }
        } else {
            const int pt = threadIdx.x;  // 0..95
            if (pt == 0) {
                mbar_arrive_expect_tx(&bar[BAR_Q], SM::Q_BYTES);
                for (int cb = 0; cb < NCB; ++cb)
                    tma_load_4d(sQ + cb * BM * 128, &tm_q, &bar[BAR_Q], cb * 64, h_first, t_tok, b);
            }
            constexpr int CH = D / 8;  // 16-byte chunks per key row
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % kStages;
                if (i >= kStages && !mbar_wait(&bar[BAR_KVE + s], ((i / kStages) - 1) & 1, abort_flag))
                    break;
                const bool comp = i < nct;
                const uint32_t dk = smem_u32(sK + s * SM::KV_BYTES);
                const uint32_t dv = smem_u32(sV + s * SM::KV_BYTES);
                for (int ch = pt; ch < kBN * CH; ch += kProducerThreads) {
                    const int r = ch / CH, c8 = ch % CH;
                    const int cb = c8 >> 3, cw = c8 & 7;
                    size_t srow = 0;
                    bool ok;
                    const __nv_bfloat16 *bk, *bv;
                    if (comp) {
                        const int k = i * kBN + r;
                        ok = k < nsel;
                        if (ok)
                            srow = ((size_t)b * p.Nc + sel[k]) * p.Hkv + kvh;
                        bk = p.kc;
                        bv = p.vc;
                    } else {
                        const int rr = rlo + (i - nct) * kBN + r;
                        ok = rr <= rhi;
                        if (ok)
                            srow = ((size_t)b * p.Lkv + rr) * p.Hkv + kvh;
                        bk = p.kr;
                        bv = p.vr;
                    }
                    const uint32_t off = cb * kBN * 128 + sw128_offset(r, cw);
                    cp_async_16(dk + off, bk + srow * D + c8 * 8, ok ? 16u : 0u);
                    cp_async_16(dv + off, bv + srow * D + c8 * 8, ok ? 16u : 0u);
                }
                // Signal this tile as soon as its own copies have landed: the
                // MMA issues PV(i-1) only after QK(i), so holding tile i back
                // until tile i+1 is issued would wait on a stage that PV(i-1)
                // has yet to free.
                cp_async_commit();
                cp_async_wait_group<0>();
                fence_proxy_async_smem();
                mbar_arrive(&bar[BAR_KF + s]);
                mbar_arrive(&bar[BAR_VF + s]);
            }
            cp_async_wait_group<0>();
            if (pt == 0)
                drain_wait(&bar[BAR_Q], 0);
        }
    } else if (warp == 3) {
        // ============================ MMA issue ===========================
        if (lane == 0 && ntiles > 0) {
            const uint32_t idesc_qk = idesc_bf16(BM, kBN, false, false);
            const uint32_t idesc_pv = idesc_bf16(BM, D, false, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            bool ok = mbar_wait(&bar[BAR_Q], 0, abort_flag);
            auto issue_pv = [&](int j) -> bool {
                const int sj = j % kStages;
                if (!mbar_wait(&bar[BAR_PF], j & 1, abort_flag))
                    return false;
                if (!mbar_wait(&bar[BAR_VF + sj], (j / kStages) & 1, abort_flag))
                    return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    const uint64_t da = sw128_desc(aP + (kk >> 2) * BM * 128 + (kk & 3) * 32, 16, 1024);
                    const uint64_t db = sw128_desc(aV + sj * SM::KV_BYTES + kk * 16 * 128,
                                                   kBN * 128, 1024);
                    mma_bf16_ss(tmem + TM_O, da, db, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bar[BAR_OD]);
                mma_commit(&bar[BAR_KVE + sj]);
                return true;
            };
            for (int i = 0; ok && i < ntiles; ++i) {
                const int s = i % kStages;
                if (!mbar_wait(&bar[BAR_KF + s], (i / kStages) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dS = tmem + TM_S0 + (i & 1) * kBN;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t da = sw128_desc(aQ + (kk >> 2) * BM * 128 + (kk & 3) * 32, 16, 1024);
                    const uint64_t db = sw128_desc(aK + s * SM::KV_BYTES + (kk >> 2) * kBN * 128 +
                                                       (kk & 3) * 32, 16, 1024);
                    mma_bf16_ss(dS, da, db, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bar[BAR_SF + (i & 1)]);
                if (i > 0 && !issue_pv(i - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok)
                issue_pv(ntiles - 1);
            // every MMA issued above has completed before TMEM is released
            mma_commit(&bar[BAR_DONE]);
            drain_wait(&bar[BAR_DONE], 0);
        }
    } else {
        // ========================= softmax + epilogue =========================
        const int quad = warp & 3;
        const int row = SPARSE ? quad * 16 + lane : quad * 32 + lane;
        const bool lane_row = SPARSE ? (lane < 16) : true;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);  // this warp's TMEM lanes

        // per-row query position and validity
        int t_row, h_row;
        bool valid_row;
        if (SPARSE) {
            t_row = t_tok;
            h_row = h_first + row;
            valid_row = lane_row && row < p.g;
        } else {
            t_row = t0 + row;
            h_row = h_first;
            valid_row = t_row < p.Lq;
        }
        long long pos = 0;
        if (valid_row)
            pos = p.q_pos ? p.q_pos[(size_t)b * p.Lq + t_row] : t_row;
        const int nv = valid_row ? n_visible(pos, p.m, p.W, p.Nc) : 0;
        const long long wlo = pos - p.W + 1;

        float m_ref = -INFINITY;  // kept max (log2 domain)
        float l_sum = 0.f;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bar[BAR_SF + (i & 1)], (i >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kBN];
#pragma unroll
            for (int c = 0; c < kBN / 32; ++c)
                tmem_ld32(tl + TM_S0 + (i & 1) * kBN + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
            tmem_ld_wait();

            // mask + scale into the log2 domain; valid columns are c_lo..c_hi
            int c_lo, c_hi;
            if (i < nct) {
                const int lim = SPARSE ? nsel : nv;
                c_lo = 0;
                c_hi = min(lim - 1 - i * kBN, kBN - 1);
            } else {
                const long long base = (long long)rlo + (long long)(i - nct) * kBN;
                const long long a = wlo - kv0 - base;
                const long long z = min((long long)rhi, pos - kv0) - base;
                c_lo = (int)max(0ll, min(a, (long long)kBN));
                c_hi = (int)max(-1ll, min(z, (long long)kBN - 1));
            }
            if (!valid_row)
                c_hi = -1;
            float tmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < kBN; ++c) {
                s[c] = (c >= c_lo && c <= c_hi) ? s[c] * p.scale_log2 : -INFINITY;
                tmax = fmaxf(tmax, s[c]);
            }
            float alpha = 1.f;
            if (tmax > m_ref + 8.f) {  // also true for the first finite max
                alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - tmax);
                m_ref = tmax;
                l_sum *= alpha;
            }
            // P buffer and O are free once PV of the previous tile completed
            if (i > 0) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bar[BAR_OD], (i - 1) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        float ov[32];
                        tmem_ld32(tl + TM_O + c * 32, ov);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            ov[q] *= alpha;
                        tmem_st32(tl + TM_O + c * 32, ov);
                    }
                    tmem_st_wait();
                }
            }
            const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < kBN; ++c) {
                s[c] = exp2f(s[c] - mu);
                lsum += s[c];
            }
            l_sum += lsum;
            if (lane_row) {
#pragma unroll
                for (int cc = 0; cc < kBN / 8; ++cc) {
                    uint4 v;
                    v.x = pack_bf16x2(s[cc * 8 + 0], s[cc * 8 + 1]);
                    v.y = pack_bf16x2(s[cc * 8 + 2], s[cc * 8 + 3]);
                    v.z = pack_bf16x2(s[cc * 8 + 4], s[cc * 8 + 5]);
                    v.w = pack_bf16x2(s[cc * 8 + 6], s[cc * 8 + 7]);
                    const uint32_t off = (cc >> 3) * BM * 128 + sw128_offset(row, cc & 7);
                    *reinterpret_cast<uint4 *>(sP + off) = v;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[BAR_PF]);
        }
        if (ok && ntiles > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bar[BAR_OD], (ntiles - 1) & 1, abort_flag));
            tc_fence_after();
        }
        // epilogue: o = O / l (0 for an empty key set), lse = ln(sum exp)
        const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
        const size_t obase = (((size_t)b * p.Lq + t_row) * p.Hq + h_row) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            float ov[32];
            if (ok && ntiles > 0) {
                tmem_ld32(tl + TM_O + c * 32, ov);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    ov[q] = 0.f;
            }
            if (valid_row) {
#pragma unroll
                for (int q = 0; q < 32; q += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(ov[q + 0] * inv, ov[q + 1] * inv);
                    v.y = pack_bf16x2(ov[q + 2] * inv, ov[q + 3] * inv);
                    v.z = pack_bf16x2(ov[q + 4] * inv, ov[q + 5] * inv);
                    v.w = pack_bf16x2(ov[q + 6] * inv, ov[q + 7] * inv);
                    *reinterpret_cast<uint4 *>(p.o + obase + c * 32 + q) = v;
                }
            }
        }
        if (valid_row && p.lse) {
            const float lse = l_sum > 0.f ? (m_ref + log2f(l_sum)) / kLog2e : -INFINITY;
            p.lse[((size_t)b * p.Hq + h_row) * p.Lq + t_row] = lse;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[MI_TMEM], 512);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int D, bool SPARSE>
static cudaError_t launch_attn_t(const AttnParams &p, const void *q, cudaStream_t stream)
{
    using SM = AttnSmem<D, SPARSE>;
    CUtensorMap mq, mkc, mvc, mkr, mvr;
    const int Nc1 = p.Nc > 0 ? p.Nc : 1;
    bool ok = true;
    if (SPARSE)
        ok &= make_map(&mq, q, D, p.Hq, p.Lq, p.B, SM::BM, 1);
    else
        ok &= make_map(&mq, q, D, p.Hq, p.Lq, p.B, 1, SM::BM);
    ok &= make_map(&mkc, p.kc ? (const void *)p.kc : q, D, p.Hkv, Nc1, p.B, 1, kBN);
    ok &= make_map(&mvc, p.vc ? (const void *)p.vc : q, D, p.Hkv, Nc1, p.B, 1, kBN);
    ok &= make_map(&mkr, p.kr, D, p.Hkv, p.Lkv, p.B, 1, kBN);
    ok &= make_map(&mvr, p.vr, D, p.Hkv, p.Lkv, p.B, 1, kBN);
    if (!ok)
        return cudaErrorInvalidValue;
    // One CTA per SM: each CTA holds all 512 TMEM columns, so the request is
    // padded above half of the SM's shared memory.
    size_t smem = 1024 + SM::BASE_BYTES + (SPARSE ? (size_t)p.topk * 4 : 0);
    if (smem < 120 * 1024)
        smem = 120 * 1024;
    auto kern = hybrid_attn_kernel<D, SPARSE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid;
    if (SPARSE)
        grid = dim3(p.Lq, p.Hkv, p.B);
    else
        grid = dim3(p.n_qtiles, p.Hq, p.B);
    kern<<<grid, kAttnThreads, smem, stream>>>(mq, mkc, mvc, mkr, mvr, p);
    return cudaGetLastError();
}

cudaError_t launch_hybrid_attn(int B, int Lq, int Lkv, int Hq, int Hkv, int d, int Nc, int m, int W,
                               int topk, float scale, const int32_t *q_pos, const int32_t *kv_pos0,
                               const void *q, const void *kc, const void *vc, const int32_t *idx,
                               const void *kr, const void *vr, void *o, float *lse,
                               cudaStream_t stream)
{
    AttnParams p;
    p.B = B;
    p.Lq = Lq;
    p.Lkv = Lkv;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.g = Hq / Hkv;
    p.Nc = Nc;
    p.m = m;
    p.W = W;
    p.topk = idx ? topk : 0;
    p.scale_log2 = scale * kLog2e;
    p.q_pos = q_pos;
    p.kv_pos0 = kv_pos0;
    p.idx = idx;
    p.kc = static_cast<const __nv_bfloat16 *>(kc);
    p.vc = static_cast<const __nv_bfloat16 *>(vc);
    p.kr = static_cast<const __nv_bfloat16 *>(kr);
    p.vr = static_cast<const __nv_bfloat16 *>(vr);
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.n_qtiles = (Lq + 127) / 128;
    const bool sparse = idx != nullptr;
    if (d == 128)
        return sparse ? launch_attn_t<128, true>(p, q, stream) : launch_attn_t<128, false>(p, q, stream);
    return sparse ? launch_attn_t<64, true>(p, q, stream) : launch_attn_t<64, false>(p, q, stream);
}

}  // namespace hyb

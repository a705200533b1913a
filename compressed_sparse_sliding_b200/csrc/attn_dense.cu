// attn_dense.cu -- stage 3 for HCA (every visible compressed entry, "deepseek-v4"
// blog, section 1, HCA and SWA) in prefill: a persistent, warp-specialised
// tcgen05 kernel that processes two 128-row query tiles per work item
// against one shared stream of key tiles.
//
// Work item = two query tiles that read the same keys:
//   Hq / Hkv >= 2 (GQA / MQA, CS336 "Attention Heads variants"): the same 128
//                tokens for two query heads of one KV group (identical keys);
//   Hq == Hkv (MHA): two consecutive 128-token tiles of one head (their raw
//                windows overlap; a key tile that one of them does not see is
//                skipped for that tile).
// Items are ordered longest first (late tokens see more compressed entries)
// and handed out round-robin to one CTA per SM.
//
// Roles (384 threads, three warpgroups):
//   warps 0-3   softmax + epilogue of tile A, warps 4-7 of tile B: one thread
//               per TMEM lane (= query row).  These two warpgroups raise their
//               register budget to 208 (setmaxnreg) so that a row's 128 scores
//               stay in registers from one TMEM load through max, exp2 and
//               the P write.
//   warp 8      TMA producer: Q_A, Q_B once per item, K and V tiles through
//               separate two-stage rings (128-byte swizzle, no multicast).
//   warp 9      TMEM allocation; lane 0 issues every tcgen05.mma.
//   warps 10-11 idle; the third warpgroup gives registers back (88 each).
// TMEM (512 columns): S_A, S_B (128 fp32 columns each), O_A, O_B (D each).
// After the softmax pass P (bf16 pairs) overwrites the first 64 columns of S
// and feeds O += P V directly from TMEM, so shared memory only holds Q and
// the K / V rings.  The MMA thread alternates [PV_A(i-1), QK_A(i)] and
// [PV_B(i-1), QK_B(i)] so that one softmax warpgroup works while the tensor
// core serves the other.  The running row max moves (and O is rescaled in
// TMEM) only when a tile raises it by more than 2^8.
#include "common.cuh"

namespace hyb {

constexpr int kDnThreads = 384;
constexpr int kDnSoftmaxRegs = 208;   // 2 x 128 x 208 + 128 x 88 = 384 x 168 (the launch budget)
constexpr int kDnOtherRegs = 88;
constexpr int kDnBM = 128;
constexpr int kDnBN = 128;
constexpr int kDnKStages = 2;
constexpr int kDnVStages = 2;
static_assert(kDnKStages == 2 && kDnVStages == 2, "the barrier slots (DB_KF .. DB_VE) hold two stages each");

struct DenseParams {
    int B, L, Lkv, Hq, Hkv, g, Nc, m, W;
    int n_ttiles;      // ceil(L / 128)
    int pair_heads;    // 1: items pair two heads; 0: items pair two token tiles
    int n_pairs;       // head pairs per KV head (pair_heads) or token-tile pairs (else)
    long long n_items;
    float scale_log2;
    __nv_bfloat16 *o;  // [B, L, Hq, D]
    float *lse;        // [B, Hq, L] or NULL
};

template <int D>
struct DenseSmem {
    static constexpr int Q_BYTES = kDnBM * D * 2;
    static constexpr int KV_BYTES = kDnBN * D * 2;
    static constexpr int OFF_QA = 0;
    static constexpr int OFF_QB = Q_BYTES;
    static constexpr int OFF_K = 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + kDnKStages * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + kDnVStages * KV_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + 32 * 8;
    static constexpr int BYTES = OFF_MISC + 16 * 4;
};

// barrier slots
enum {
    DB_QF = 0, DB_QE = 1, DB_KF = 2, DB_KE = 4, DB_VF = 6, DB_VE = 8,
    DB_SF = 10, DB_PF = 12, DB_OF = 14, DB_OE = 16, DB_DONE = 18
};

struct DenseItem {
    int b, hA, hB, tA, tB;   // heads and first tokens of the two query tiles
    bool vA, vB;             // tile has at least one valid row
    int xA1, xB1;            // last valid token of each tile
    int nct, nrt, rlo;       // compressed tiles, raw tiles, first raw row
    int nvA, nvB;            // compressed entries visible to the last row of each tile
};

__device__ __forceinline__ int dn_visible(int t, int m, int W, int Nc)
{
    // positions fit in 32 bits (the launcher checks), so the division is 32-bit
    const int a = t - W + 1;
    if (a <= 0)
        return 0;
    const int n = (int)((unsigned)a / (unsigned)m);
    return n < Nc ? n : Nc;
}

__device__ __forceinline__ DenseItem dense_item(const DenseParams &p, long long w)
{
    // item counts fit in 32 bits (the launcher checks): 32-bit divisions only
    DenseItem it;
    const unsigned wu = (unsigned)w;
    if (p.pair_heads) {
        const unsigned per_b = (unsigned)p.Hkv * (unsigned)p.n_pairs;
        const unsigned per_t = (unsigned)p.B * per_b;
        const int trev = (int)(wu / per_t);
        unsigned r = wu % per_t;
        it.b = (int)(r / per_b);
        r %= per_b;
        const int kvh = (int)(r / (unsigned)p.n_pairs);
        const int hp = (int)(r % (unsigned)p.n_pairs);
        it.hA = kvh * p.g + 2 * hp;
        it.hB = it.hA + 1;
        it.tA = (p.n_ttiles - 1 - trev) * kDnBM;
        it.tB = it.tA;
        it.vA = true;
        it.vB = (2 * hp + 1) < p.g;
    } else {
        const unsigned per_t = (unsigned)p.B * (unsigned)p.Hq;
        const int trev = (int)(wu / per_t);
        const unsigned r = wu % per_t;
        it.b = (int)(r / (unsigned)p.Hq);
        it.hA = (int)(r % (unsigned)p.Hq);
        it.hB = it.hA;
        it.tA = (p.n_pairs - 1 - trev) * 2 * kDnBM;
        it.tB = it.tA + kDnBM;
        it.vA = it.tA < p.L;
        it.vB = it.tB < p.L;
    }
    it.xA1 = min(it.tA + kDnBM - 1, p.L - 1);
    it.xB1 = min(it.tB + kDnBM - 1, p.L - 1);
    const int tmin = it.tA;
    const int tmax = it.vB ? max(it.xA1, it.xB1) : it.xA1;
    const int nv = dn_visible(tmax, p.m, p.W, p.Nc);
    it.nct = (nv + kDnBN - 1) / kDnBN;
    it.nvA = dn_visible(it.xA1, p.m, p.W, p.Nc);
    it.nvB = dn_visible(it.xB1, p.m, p.W, p.Nc);
    int lo = tmin - p.W + 1;
    if (lo < 0)
        lo = 0;
    const int hi = min(tmax, p.Lkv - 1);
    it.rlo = lo;
    it.nrt = (p.W > 0 && hi >= lo) ? (hi - lo + kDnBN) / kDnBN : 0;
    return it;
}

// Does query tile X (tokens x0..x1) need key tile i of the item?
__device__ __forceinline__ bool dn_active(const DenseParams &p, const DenseItem &it, int i, bool B_)
{
    const bool valid = B_ ? it.vB : it.vA;
    if (!valid)
        return false;
    const int x0 = B_ ? it.tB : it.tA;
    const int x1 = B_ ? it.xB1 : it.xA1;
    if (i < it.nct)
        return i * kDnBN < (B_ ? it.nvB : it.nvA);
    const int r0 = it.rlo + (i - it.nct) * kDnBN;
    int need_lo = x0 - p.W + 1;
    if (need_lo < 0)
        need_lo = 0;
    return p.W > 0 && r0 <= x1 && r0 + kDnBN - 1 >= need_lo;
}

template <int D>
__global__ void __launch_bounds__(kDnThreads, 1)
hca_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kr,
                const __grid_constant__ CUtensorMap tm_vr, const DenseParams p)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
    using SM = DenseSmem<D>;
    constexpr int NCB = D / 64;
    extern __shared__ __align__(1024) uint8_t dn_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dn_smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sQ[2] = {smem + SM::OFF_QA, smem + SM::OFF_QB};
    uint8_t *sK = smem + SM::OFF_K;
    uint8_t *sV = smem + SM::OFF_V;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM::OFF_BAR);
    int *misc = reinterpret_cast<int *>(smem + SM::OFF_MISC);
    volatile int *abort_flag = misc + 1;
    unsigned long long *const trb = trace_buffer();   // timeline of CTA 0, when attached
    uint32_t tn = 0;                                  // this thread's trace records

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bar[DB_QF], 1);
        mbar_init(&bar[DB_QE], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[DB_KF + s], 1);
            mbar_init(&bar[DB_KE + s], 1);
            mbar_init(&bar[DB_VF + s], 1);
            mbar_init(&bar[DB_VE + s], 1);
            mbar_init(&bar[DB_SF + s], 1);
            mbar_init(&bar[DB_PF + s], 128);
            mbar_init(&bar[DB_OF + s], 1);
            mbar_init(&bar[DB_OE + s], 128);
        }
        mbar_init(&bar[DB_DONE], 1);
        mbar_fence_init();
        misc[1] = 0;
    }
    if (warp == 9)
        tmem_alloc(reinterpret_cast<uint32_t *>(&misc[0]), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    constexpr uint32_t TM_S[2] = {0, kDnBN};
    constexpr uint32_t TM_O[2] = {2 * kDnBN, 2 * kDnBN + 128};
    if (warp == 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDnOtherRegs));
        // ================================ producer ================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_kr);
            tma_prefetch_desc(&tm_vr);
            uint32_t kc = 0, vc = 0, nq = 0;
            bool ok = true;
            for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
                const DenseItem it = dense_item(p, w);
                const int kvh = it.hA / p.g;
                if (nq > 0 && !mbar_wait(&bar[DB_QE], (nq - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bar[DB_QF], 2 * SM::Q_BYTES);
                for (int cb = 0; cb < NCB; ++cb) {
                    tma_load_4d(sQ[0] + cb * kDnBM * 128, &tm_q, &bar[DB_QF], cb * 64, it.hA, it.tA, it.b);
                    tma_load_4d(sQ[1] + cb * kDnBM * 128, &tm_q, &bar[DB_QF], cb * 64, it.hB, it.tB, it.b);
                }
                ++nq;
                const int nt = it.nct + it.nrt;
                for (int i = 0; i < nt; ++i) {
                    const bool comp = i < it.nct;
                    const int row0 = comp ? i * kDnBN : it.rlo + (i - it.nct) * kDnBN;
                    const uint32_t ks = kc % kDnKStages;
                    if (kc >= kDnKStages &&
                        !mbar_wait(&bar[DB_KE + ks], ((kc / kDnKStages) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar[DB_KF + ks], SM::KV_BYTES);
                    for (int cb = 0; cb < NCB; ++cb)
                        tma_load_4d(sK + ks * SM::KV_BYTES + cb * kDnBN * 128, comp ? &tm_kc : &tm_kr,
                                    &bar[DB_KF + ks], cb * 64, kvh, row0, it.b);
                    trace_ev(trb, tn, 1, 1, w, i);
                    ++kc;
                    const uint32_t vs = vc % kDnVStages;
                    if (vc >= kDnVStages &&
                        !mbar_wait(&bar[DB_VE + vs], ((vc / kDnVStages) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar[DB_VF + vs], SM::KV_BYTES);
                    for (int cb = 0; cb < NCB; ++cb)
                        tma_load_4d(sV + vs * SM::KV_BYTES + cb * kDnBN * 128, comp ? &tm_vc : &tm_vr,
                                    &bar[DB_VF + vs], cb * 64, kvh, row0, it.b);
                    trace_ev(trb, tn, 1, 2, w, i);
                    ++vc;
                }
            }
            // unwinding: wait for the last copies issued into every slot
            if (nq > 0)
                drain_wait(&bar[DB_QF], (nq - 1) & 1);
            for (uint32_t c = (kc > kDnKStages ? kc - kDnKStages : 0); c < kc; ++c)
                drain_wait(&bar[DB_KF + c % kDnKStages], (c / kDnKStages) & 1);
            for (uint32_t c = (vc > kDnVStages ? vc - kDnVStages : 0); c < vc; ++c)
                drain_wait(&bar[DB_VF + c % kDnVStages], (c / kDnVStages) & 1);
        }
    } else if (warp == 9) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDnOtherRegs));
        // ================================ MMA issue ================================
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16(kDnBM, kDnBN, false, false);
            const uint32_t idesc_pv = idesc_bf16(kDnBM, D, false, true);
            const uint32_t aQ[2] = {smem_u32(sQ[0]), smem_u32(sQ[1])};
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
            uint32_t kc = 0, vc = 0, nq = 0;
            uint32_t pcnt[2] = {0, 0};
            bool ok = true;
            for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
                const DenseItem it = dense_item(p, w);
                const int nt = it.nct + it.nrt;
                if (!mbar_wait(&bar[DB_QF], nq & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                bool first_pv[2] = {true, true};
                bool waited_oe = false;
                for (int i = 0; i <= nt && ok; ++i) {
                    bool act_prev[2] = {false, false}, act_cur[2] = {false, false};
                    for (int x = 0; x < 2; ++x) {
                        act_prev[x] = i > 0 && dn_active(p, it, i - 1, x == 1);
                        act_cur[x] = i < nt && dn_active(p, it, i, x == 1);
                    }
                    const uint32_t ks = kc % kDnKStages;
                    if (i < nt && !mbar_wait(&bar[DB_KF + ks], (kc / kDnKStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t vs = vc % kDnVStages;
                    if (i > 0) {
                        if (!mbar_wait(&bar[DB_VF + vs], (vc / kDnVStages) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (!waited_oe && nq > 0) {
                            // both epilogues of the previous item have read O
                            if (!mbar_wait(&bar[DB_OE + 0], (nq - 1) & 1, abort_flag) ||
                                !mbar_wait(&bar[DB_OE + 1], (nq - 1) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            waited_oe = true;
                        }
                    }
                    tc_fence_after();
                    for (int x = 0; x < 2 && ok; ++x) {
                        if (act_prev[x]) {
                            if (!mbar_wait(&bar[DB_PF + x], pcnt[x] & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            ++pcnt[x];
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < kDnBN / 16; ++kk) {
                                const uint64_t db = sw128_desc(aV + vs * SM::KV_BYTES + kk * 16 * 128,
                                                               kDnBN * 128, 1024);
                                mma_bf16_ts(tmem + TM_O[x], tmem + TM_S[x] + kk * 8, db, idesc_pv,
                                            (first_pv[x] && kk == 0) ? 0u : 1u);
                            }
                            first_pv[x] = false;
                            trace_ev(trb, tn, 2, 2 + 2 * x, w, i - 1);
                        }
                        if (act_cur[x]) {
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint64_t da = sw128_desc(aQ[x] + (kk >> 2) * kDnBM * 128 + (kk & 3) * 32,
                                                               16, 1024);
                                const uint64_t db = sw128_desc(aK + ks * SM::KV_BYTES +
                                                                   (kk >> 2) * kDnBN * 128 + (kk & 3) * 32,
                                                               16, 1024);
                                mma_bf16_ss(tmem + TM_S[x], da, db, idesc_qk, kk > 0 ? 1u : 0u);
                            }
                            mma_commit(&bar[DB_SF + x]);
                            trace_ev(trb, tn, 2, 1 + 2 * x, w, i);
                        }
                    }
                    if (!ok)
                        break;
                    if (i > 0) {
                        mma_commit(&bar[DB_VE + vs]);
                        ++vc;
                    }
                    if (i < nt) {
                        mma_commit(&bar[DB_KE + ks]);
                        ++kc;
                        if (i == nt - 1)
                            mma_commit(&bar[DB_QE]);
                    }
                }
                if (!ok)
                    break;
                if (nt == 0)
                    mma_commit(&bar[DB_QE]);
                if (!waited_oe && nq > 0) {
                    // keep one o_empty wait per item even without a PV
                    if (!mbar_wait(&bar[DB_OE + 0], (nq - 1) & 1, abort_flag) ||
                        !mbar_wait(&bar[DB_OE + 1], (nq - 1) & 1, abort_flag))
                        break;
                }
                for (int x = 0; x < 2; ++x)
                    if (!first_pv[x])
                        mma_commit(&bar[DB_OF + x]);
                ++nq;
            }
            mma_commit(&bar[DB_DONE]);
            drain_wait(&bar[DB_DONE], 0);
        }
    } else if (warp >= 10) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDnOtherRegs));
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kDnSoftmaxRegs));
        // ========================== softmax + epilogue ==========================
        const int x = warp >> 2;            // 0: tile A, 1: tile B
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t tS = tl + TM_S[x];
        const uint32_t tO = tl + TM_O[x];
        // the first thread of each softmax warpgroup traces: role 3 (tile A), role 0 (tile B)
        const bool tracer = (threadIdx.x & 127) == 0;
        const int trole = x == 0 ? 3 : 0;
        uint32_t scnt = 0, ocnt = 0;
        bool ok = true;
        for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
            const DenseItem it = dense_item(p, w);
            const int nt = it.nct + it.nrt;
            const int t = (x ? it.tB : it.tA) + row;
            const int h = x ? it.hB : it.hA;
            const bool valid_row = (x ? it.vB : it.vA) && t < p.L;
            const int nv = valid_row ? dn_visible(t, p.m, p.W, p.Nc) : 0;
            const int wlo = t - p.W + 1;
            float m_ref = -INFINITY, l_sum = 0.f;
            bool any = false;
            for (int i = 0; i < nt; ++i) {
                if (!dn_active(p, it, i, x == 1))
                    continue;
                // valid columns c_lo..c_hi of this key tile for this row
                int c_lo, c_hi;
                if (i < it.nct) {
                    c_lo = 0;
                    c_hi = min(nv - 1 - i * kDnBN, kDnBN - 1);
                } else {
                    const int base = it.rlo + (i - it.nct) * kDnBN;
                    c_lo = max(0, min(wlo - base, kDnBN));
                    c_hi = max(-1, min(min(t, p.Lkv - 1) - base, kDnBN - 1));
                }
                if (!valid_row)
                    c_hi = -1;
                const bool full = __all_sync(0xffffffffu, c_lo == 0 && c_hi == kDnBN - 1);
                if (!__all_sync(0xffffffffu, mbar_wait(&bar[DB_SF + x], scnt & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                ++scnt;
                tc_fence_after();
                // all 128 scores in flight (one wait); masked columns become -inf,
                // so they drop out of the max and give exp2 = 0 below
                float sv[kDnBN];
#pragma unroll
                for (int c = 0; c < kDnBN / 32; ++c)
                    tmem_ld32(tS + c * 32, *reinterpret_cast<float(*)[32]>(&sv[c * 32]));
                tmem_ld_wait();
                if (tracer)
                    trace_ev(trb, tn, trole, 1, w, i);
                if (!full) {
#pragma unroll
                    for (int c = 0; c < kDnBN; ++c)
                        sv[c] = (c >= c_lo && c <= c_hi) ? sv[c] : -INFINITY;
                }
                // row max over eight independent 3-input max chains
                float tmax;
                {
                    float mk[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        float a = fmax3f(sv[16 * k], sv[16 * k + 1], sv[16 * k + 2]);
#pragma unroll
                        for (int q = 3; q < 15; q += 2)
                            a = fmax3f(a, sv[16 * k + q], sv[16 * k + q + 1]);
                        mk[k] = fmaxf(a, sv[16 * k + 15]);
                    }
                    tmax = fmax3f(fmax3f(mk[0], mk[1], mk[2]), fmax3f(mk[3], mk[4], mk[5]),
                                  fmaxf(mk[6], mk[7]));
                }
                tmax *= p.scale_log2;  // the scale is positive
                float alpha = 1.f;
                if (tmax > m_ref + 8.f) {
                    alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - tmax);
                    m_ref = tmax;
                    l_sum *= alpha;
                }
                if (any && __any_sync(0xffffffffu, alpha != 1.f)) {
                    // O already holds every earlier PV of this item (S_full
                    // covers all MMAs issued before QK of this tile)
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        float ov[32];
                        tmem_ld32(tO + c * 32, ov);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            ov[q] *= alpha;
                        tmem_st32(tO + c * 32, ov);
                    }
                }
                const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
                // P = exp2(s * scale - mu) from the registers, as bf16 pairs over
                // the first 64 columns of S (the A operand of O += P V; every
                // score was loaded before the first store).  Row sums in four
                // independent packed accumulators.
                const uint64_t sc2 = f2(p.scale_log2, p.scale_log2);
                const uint64_t nmu2 = f2(-mu, -mu);
                uint64_t lacc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int c = 0; c < kDnBN / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 32; q += 2) {
                        float x0, x1;
                        f2_split(fma_f2(f2(sv[c * 32 + q], sv[c * 32 + q + 1]), sc2, nmu2), x0, x1);
                        const float e0 = ex2_approx(x0);
                        const float e1 = ex2_approx(x1);
                        lacc[(q >> 1) & 3] = add_f2(lacc[(q >> 1) & 3], f2(e0, e1));
                        pk[q >> 1] = pack_bf16x2(e0, e1);
                    }
                    tmem_st16(tS + c * 16, pk);
                }
                float lsum;
                {
                    float a0, a1, b0, b1, c0, c1, d0, d1;
                    f2_split(add_f2(lacc[0], lacc[1]), a0, a1);
                    f2_split(add_f2(lacc[2], lacc[3]), b0, b1);
                    lsum = (a0 + a1) + (b0 + b1);
                    (void)c0; (void)c1; (void)d0; (void)d1;
                }
                l_sum += lsum;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bar[DB_PF + x]);
                if (tracer)
                    trace_ev(trb, tn, trole, 2, w, i);
                any = true;
            }
            if (!ok)
                break;
            // epilogue
            if (tracer)
                trace_ev(trb, tn, trole, 3, w, nt);
            if (any) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bar[DB_OF + x], ocnt & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                ++ocnt;
                tc_fence_after();
            }
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            __nv_bfloat16 *orow = p.o + (((size_t)it.b * p.L + t) * p.Hq + h) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; c += 2) {
                float ov[64];
                if (any) {
                    tmem_ld32(tO + c * 32, *reinterpret_cast<float(*)[32]>(&ov[0]));
                    tmem_ld32(tO + c * 32 + 32, *reinterpret_cast<float(*)[32]>(&ov[32]));
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int q = 0; q < 64; ++q)
                        ov[q] = 0.f;
                }
                if (valid_row) {
#pragma unroll
                    for (int q = 0; q < 64; q += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(ov[q + 0] * inv, ov[q + 1] * inv);
                        v.y = pack_bf16x2(ov[q + 2] * inv, ov[q + 3] * inv);
                        v.z = pack_bf16x2(ov[q + 4] * inv, ov[q + 5] * inv);
                        v.w = pack_bf16x2(ov[q + 6] * inv, ov[q + 7] * inv);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + q) = v;
                    }
                }
            }
            if (valid_row && p.lse)
                p.lse[((size_t)it.b * p.Hq + h) * p.L + t] =
                    l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
            tc_fence_before();
            mbar_arrive(&bar[DB_OE + x]);
            if (tracer)
                trace_ev(trb, tn, trole, 4, w, nt);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[0], 512);
    }
}

template <int D>
static cudaError_t launch_hca_t(const DenseParams &p, const void *q, const void *kc, const void *vc,
                                const void *kr, const void *vr, cudaStream_t stream, int num_sms)
{
    using SM = DenseSmem<D>;
    CUtensorMap mq, mkc, mvc, mkr, mvr;
    const int Nc1 = p.Nc > 0 ? p.Nc : 1;
    bool ok = make_map(&mq, q, D, p.Hq, p.L, p.B, 1, kDnBM);
    ok &= make_map(&mkc, kc ? kc : q, D, p.Hkv, Nc1, p.B, 1, kDnBN);
    ok &= make_map(&mvc, vc ? vc : q, D, p.Hkv, Nc1, p.B, 1, kDnBN);
    ok &= make_map(&mkr, kr, D, p.Hkv, p.Lkv, p.B, 1, kDnBN);
    ok &= make_map(&mvr, vr, D, p.Hkv, p.Lkv, p.B, 1, kDnBN);
    if (!ok)
        return cudaErrorInvalidValue;
    size_t smem = 1024 + SM::BYTES;
    if (smem < 120 * 1024)
        smem = 120 * 1024;
    auto kern = hca_attn_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    e = check_reg_split(kern, kDnThreads, 256, kDnSoftmaxRegs, kDnOtherRegs);
    if (e != cudaSuccess)
        return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDnThreads, smem);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        return cudaErrorLaunchOutOfResources;
    long long grid = num_sms;
    if (grid > p.n_items)
        grid = p.n_items;
    if (grid < 1)
        return cudaSuccess;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kDnThreads), smem, stream, mq, mkc, mvc, mkr, mvr, p);
}

// Prefill HCA: idx == NULL, positions 0..L-1, raw rows 0..L-1.
cudaError_t launch_hca_attn(int B, int L, int Lkv, int Hq, int Hkv, int d, int Nc, int m, int W,
                            float scale, const void *q, const void *kc, const void *vc, const void *kr,
                            const void *vr, void *o, float *lse, cudaStream_t stream, int num_sms)
{
    DenseParams p;
    p.B = B;
    p.L = L;
    p.Lkv = Lkv;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.g = Hq / Hkv;
    p.Nc = Nc;
    p.m = m;
    p.W = W;
    p.n_ttiles = (L + kDnBM - 1) / kDnBM;
    p.pair_heads = p.g >= 2 ? 1 : 0;
    if (p.pair_heads) {
        p.n_pairs = (p.g + 1) / 2;
        p.n_items = (long long)p.n_ttiles * B * Hkv * p.n_pairs;
    } else {
        p.n_pairs = (L + 2 * kDnBM - 1) / (2 * kDnBM);
        p.n_items = (long long)p.n_pairs * B * Hq;
    }
    if (p.n_items >= (1LL << 31) || (long long)L + W >= (1LL << 30))
        return cudaErrorInvalidValue;   // item indices and positions use 32-bit arithmetic
    p.scale_log2 = scale * 1.4426950408889634f;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    if (d == 128)
        return launch_hca_t<128>(p, q, kc, vc, kr, vr, stream, num_sms);
    return launch_hca_t<64>(p, q, kc, vc, kr, vr, stream, num_sms);
}

}  // namespace hyb

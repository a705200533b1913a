// index_fused.cu -- stage 2 of CSA for prefill-shaped problems in one kernel:
// the lightning-indexer scores and the exact per-query top-K ("deepseek-v4"
// blog, section 1, CSA: a lightning indexer scores the compressed entries and
// the top-K of them are kept for the current query; score = ReLU-weighted
// head sum, fp32), without ever storing a row of scores.
//
//     I[t, s] = sum_h wi[t, h] * max(0, qi[t, h, :] . kic[s, :])
//
// A CTA owns 128 query rows of one sequence (one TMEM lane each).  Key tiles
// of 64 entries stream through a TMA ring; per tile one tcgen05 MMA per
// indexer head writes D_h [128 rows x 64 keys] into TMEM (double-buffered), and
// the epilogue thread of a row forms the row's 64 scores.  The scores are
// recomputed pass after pass (the GEMM is cheap next to moving the score rows
// through HBM) and only per-row summaries stay on chip:
//   S  (sample)    two tiles spread over the visible range; each row keeps the
//                  order keys of its <= 128 sampled scores and derives a key
//                  window that very likely holds its K-th largest score;
//   H  (histogram) every visible key; each row counts its scores above the
//                  window and histograms those inside it (128 bins, u16
//                  counters in shared memory), then finds the bin holding the
//                  K-th largest.  A row whose window missed (or whose bin is too
//                  full to keep) moves or narrows its window and the CTA runs
//                  H again, so the result never depends on the sample;
//   E  (emit)      every visible key again; scores above the bin are written
//                  straight to the row's index list (ascending, since keys are
//                  visited in order), scores inside the bin are kept in a
//                  per-row buffer of <= 64 entries.  Afterwards the row takes
//                  the largest of them (lower index first on equal scores) and
//                  merges them into its list; when the bin is a single score
//                  value (an exact tie) the first entries in index order are
//                  taken during E itself.
// Order keys are the fp32 scores mapped to uint32 so that larger scores give
// larger keys (-0.0 folded onto +0.0), as in the two-kernel path.
// Roles (320 threads): warp 0 TMA producer, warp 1 TMEM + MMA, and two
// threads per row for the epilogue: warps 2-5 (TMEM lane quadrants 2, 3, 0,
// 1) take the first half of every pass's key tiles, warps 6-9 the second
// half, each half with its own TMEM buffer, so that two warps per SM
// sub-partition hide each other's latencies.  The halves histogram into
// separate arrays and take the row's decisions together from both; for E,
// half 1 starts its list where half 0's keys above the bin end (known from
// half 0's histogram), so that each half writes its part of the ascending
// list on its own.  The epilogue decides after each H pass whether another H
// or the E pass follows; the producer and MMA warps learn it through two
// shared words and stop after E.
#include <type_traits>

#include "common.cuh"

namespace hyb {

constexpr int kFxThreads = 320;
constexpr int kFxBM = 128;          // query rows per CTA
constexpr int kFxBN = 64;           // keys per tile
constexpr int kFxStages = 3;
constexpr int kFxSampleTiles = 2;
constexpr int kFxBins = 128;        // histogram bins per row
constexpr int kFxCap = 64;          // boundary-bin entries kept per row
constexpr int kFxStage = 64;        // list entries staged per row (E pass) before a flush
constexpr int kFxMaxPasses = 16;    // S + H rounds + E, far above what the window moves need
constexpr int kFxMaxNc = 65535;     // index and list position share one 32-bit word

struct FusedIndexParams {
    int B, Lq, Hi, Nc, m, W, K;
    int n_ttiles;
    const int32_t *q_pos;
    const float *wi;          // [B, Lq, Hi]
    int32_t *idx;             // [B, Lq, K]
    float *sel;               // [B, Lq, K] or nullptr
};

template <int HI, int DI>
struct FxSmem {
    static constexpr int Q_BYTES = kFxBM * DI * 2;                   // one head
    static constexpr int K_BYTES = kFxBN * DI * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = HI * Q_BYTES;
    static constexpr int OFF_U = OFF_K + kFxStages * K_BYTES;        // union below
    // pass S: sample keys [slot][row]; later passes: one histogram per half
    // [bin / 2][row] (two u16 counters per word), then the boundary buffer:
    // keys [slot][row], then (index | list position << 16) [slot][row]
    static constexpr int SAMPLE_BYTES = kFxSampleTiles * kFxBN * kFxBM * 4;
    static constexpr int HIST_WORDS = kFxBins / 2 + 1;                // + bin 128: keys above the window
    static constexpr int HIST_BYTES = HIST_WORDS * kFxBM * 4;
    static constexpr int BND_BYTES = 2 * kFxCap * kFxBM * 4;
    static constexpr int U_BYTES = SAMPLE_BYTES > 2 * HIST_BYTES + BND_BYTES ? SAMPLE_BYTES
                                                                             : 2 * HIST_BYTES + BND_BYTES;
    static constexpr int OFF_X = OFF_U + U_BYTES;                    // [4][row] counts exchanged by the halves
    static constexpr int OFF_BAR = OFF_X + 4 * kFxBM * 4;
    static constexpr int OFF_MISC = OFF_BAR + 16 * 8;
    static constexpr int BYTES = OFF_MISC + 16 * 4;
};

// 128-byte swizzle for 64-element bf16 rows, 64-byte swizzle for 32-element rows.
template <int DI>
struct FxLayout {
    static constexpr uint32_t SWZ = DI == 64 ? 2u : 4u;             // descriptor layout field
    static constexpr uint32_t SBO = DI * 2 * 8;                      // bytes per 8-row group
};

__device__ __forceinline__ uint64_t fx_desc(uint32_t saddr, uint32_t sbo, uint32_t layout)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                      // leading byte offset (unused when swizzled)
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)layout << 61;
    return d;
}

// Larger float -> larger key; -0.0 folded onto +0.0.
__device__ __forceinline__ uint32_t fx_key(float f)
{
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float fx_score(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Last key of a window of `n` bins of 2^sh keys starting at lo (saturating).
__device__ __forceinline__ uint32_t fx_last(uint32_t lo, int sh, uint32_t n)
{
    const unsigned long long e = (unsigned long long)lo + ((unsigned long long)n << sh) - 1ull;
    return e > 0xFFFFFFFFull ? 0xFFFFFFFFu : (uint32_t)e;
}

// AND of a predicate over the 256 epilogue threads (named barrier 1).
__device__ __forceinline__ bool fx_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, 256, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Barrier over the 256 epilogue threads (named barrier 1).
__device__ __forceinline__ void fx_sync()
{
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

// Bounded wait until the shared decision word reaches `p` (or the CTA aborts).
__device__ __forceinline__ bool fx_wait_decided(volatile int *decided, int p, volatile int *abort_flag)
{
    const uint64_t t0 = global_ns();
    const uint64_t lim = *reinterpret_cast<volatile uint64_t *>(&g_wait_limit_ns);
    while (*decided < p) {
        if (*abort_flag)
            return false;
        if (global_ns() - t0 > lim) {
            set_error(HYB_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
        __nanosleep(64);
    }
    __threadfence_block();
    return true;
}

// Row modes of the epilogue
enum { FX_ALL = 0, FX_BIN = 1, FX_TIE = 2, FX_OPEN = 3, FX_NONE = 4 };

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void fx_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

template <int HI, int DI>
__global__ void __launch_bounds__(kFxThreads, 1)
index_topk_fused(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const FusedIndexParams p)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
    using SM = FxSmem<HI, DI>;
    using LY = FxLayout<DI>;
    extern __shared__ __align__(1024) uint8_t fx_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(fx_smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sQ = smem + SM::OFF_Q;
    uint8_t *sK = smem + SM::OFF_K;
    uint32_t *sU = reinterpret_cast<uint32_t *>(smem + SM::OFF_U);
    uint32_t *sX = reinterpret_cast<uint32_t *>(smem + SM::OFF_X);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM::OFF_BAR);
    int *misc = reinterpret_cast<int *>(smem + SM::OFF_MISC);
    volatile int *abort_flag = misc + 1;
    volatile int *decided = misc + 2;      // passes 0 .. *decided are known to exist (or not)
    volatile int *last_pass = misc + 3;    // index of the E pass once known
    // bars: 0 Q full, 1.. K full, 1 + S.. K empty, then per half D full, D empty, then done
    constexpr int S = kFxStages;
    constexpr int B_KF = 1, B_KE = 1 + S, B_DF = 1 + 2 * S, B_DE = 3 + 2 * S, B_DONE = 5 + 2 * S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned long long *const trb = trace_buffer();   // timeline of CTA 0, when attached
    uint32_t tn = 0;                                  // this thread's trace records

    // heavy token tiles first, all sequences of one weight class together
    const int ttile = p.n_ttiles - 1 - (int)(blockIdx.x / p.B);
    const int b = (int)(blockIdx.x % p.B);
    const int t0 = ttile * kFxBM;
    const int t_last = min(t0 + kFxBM - 1, p.Lq - 1);
    auto nvis_of = [&](int t) -> int {
        const long long pos = p.q_pos ? p.q_pos[(size_t)b * p.Lq + t] : t;
        const long long a = pos - p.W + 1;
        return a > 0 ? (int)min((long long)p.Nc, a / p.m) : 0;
    };
    int nv_max = 0;
    if (p.q_pos) {
        for (int t = t0; t <= t_last; ++t)
            nv_max = max(nv_max, nvis_of(t));
    } else {
        nv_max = nvis_of(t_last);
    }
    const bool has_sel = nv_max > p.K;
    const int t_vis = (nv_max + kFxBN - 1) / kFxBN;     // key tiles of a full pass
    // sample tiles: disjoint, each starting inside the visible range (a tile
    // that would start past it repeats the first and is ignored: slot_lo)
    int soff[kFxSampleTiles];
    for (int s = 0; s < kFxSampleTiles; ++s) {
        if (nv_max <= kFxSampleTiles * kFxBN) {
            soff[s] = s * kFxBN < nv_max ? s * kFxBN : 0;
        } else {
            const int c = (int)(((2ll * s + 1) * nv_max) / (2 * kFxSampleTiles)) - kFxBN / 2;
            soff[s] = max(0, min(c, nv_max - kFxBN));
        }
    }
    // sampled keys of tile s count only from slot_lo(s) on (no key counted twice)
    auto slot_lo = [&](int s) -> int { return s == 0 ? 0 : soff[s - 1] + kFxBN; };
    // tiles of pass q: the sample pass has its own tiles, every other pass all visible ones
    auto pass_tiles = [&](int q) -> int { return (has_sel && q == 0) ? kFxSampleTiles : t_vis; };
    // The two halves of a pass: half 0 takes its first ceil(nt / 2) tiles, half
    // 1 the rest; tiles go out alternately (u even: half 0, u odd: half 1).
    auto tile_of = [&](int nt, int u) -> int { return (u & 1) ? (nt + 1) / 2 + (u >> 1) : (u >> 1); };
    auto tile_start = [&](int q, int tile) -> int { return (has_sel && q == 0) ? soff[tile] : tile * kFxBN; };

    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar[B_KF + s], 1);
            mbar_init(&bar[B_KE + s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bar[B_DF + h], 1);
            mbar_init(&bar[B_DE + h], 128);
        }
        mbar_init(&bar[B_DONE], 1);
        mbar_fence_init();
        misc[1] = 0;
        // with a selection to make: S, H and one more pass (H or E) always run
        misc[2] = has_sel ? 2 : 0x7fffffff;
        misc[3] = has_sel ? 0x7fffffff : (t_vis > 0 ? 0 : -1);
    }
    if (warp == 1)
        tmem_alloc(reinterpret_cast<uint32_t *>(&misc[0]), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[0], HI * SM::Q_BYTES);
            for (int h = 0; h < HI; ++h)
                tma_load_4d(sQ + h * SM::Q_BYTES, &tm_q, &bar[0], 0, h, t0, b);
            int issued = 0;
            bool ok = true;
            for (int q = 0; ok && q < kFxMaxPasses; ++q) {
                if (q >= 3 && !fx_wait_decided(decided, q, abort_flag))
                    break;
                if (q > *last_pass)
                    break;
                const int nt = pass_tiles(q);
                for (int u = 0; u < nt; ++u) {
                    const int s = issued % S;
                    if (issued >= S && !mbar_wait(&bar[B_KE + s], ((issued / S) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar[B_KF + s], SM::K_BYTES);
                    tma_load_4d(sK + s * SM::K_BYTES, &tm_k, &bar[B_KF + s], 0, 0, tile_start(q, tile_of(nt, u)), b);
                    trace_ev(trb, tn, 1, 1, q, u);
                    ++issued;
                }
            }
            drain_wait(&bar[0], 0);
            for (int i = max(0, issued - S); i < issued; ++i)
                drain_wait(&bar[B_KF + i % S], (i / S) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kFxBM, kFxBN, false, false);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
            bool ok = *last_pass < 0 ? true : mbar_wait(&bar[0], 0, abort_flag);
            int g = 0;
            int nh[2] = {0, 0};     // tiles given to each half so far
            for (int q = 0; ok && q < kFxMaxPasses; ++q) {
                if (q >= 3 && !fx_wait_decided(decided, q, abort_flag))
                    break;
                if (q > *last_pass)
                    break;
                const int nt = pass_tiles(q);
                for (int u = 0; u < nt; ++u, ++g) {
                    const int s = g % S, hx = u & 1;
                    if (!mbar_wait(&bar[B_KF + s], (g / S) & 1, abort_flag) ||
                        (nh[hx] >= 1 && !mbar_wait(&bar[B_DE + hx], (nh[hx] - 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int h = 0; h < HI; ++h) {
#pragma unroll
                        for (int kk = 0; kk < DI / 16; ++kk) {
                            const uint64_t da = fx_desc(aQ + h * SM::Q_BYTES + kk * 32, LY::SBO, LY::SWZ);
                            const uint64_t dbk = fx_desc(aK + s * SM::K_BYTES + kk * 32, LY::SBO, LY::SWZ);
                            mma_bf16_ss(tmem + (hx * HI + h) * kFxBN, da, dbk, idesc, kk > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(&bar[B_DF + hx]);
                    mma_commit(&bar[B_KE + s]);
                    trace_ev(trb, tn, 2, 1, q, u);
                    ++nh[hx];
                }
            }
            mma_commit(&bar[B_DONE]);
            drain_wait(&bar[B_DONE], 0);
        }
    } else if (warp >= 2) {
        // ================================ row epilogue ================================
        // Two threads per row: half 0 (warps 2-5) and half 1 (warps 6-9)
        // take the first and the second half of every pass's tiles.  Both keep
        // the row's window state and take the same decisions from the same
        // shared data; the counts that differ between halves go through sX.
        const int hx = warp >= 6 ? 1 : 0;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int t = t0 + row;
        const bool valid = t < p.Lq;
        const int nv = valid ? nvis_of(t) : 0;
        const int K = p.K;
        float wv[HI];
#pragma unroll
        for (int h = 0; h < HI; ++h)
            wv[h] = valid ? p.wi[((size_t)b * p.Lq + t) * HI + h] : 0.f;
        int32_t *orow = p.idx + ((size_t)b * p.Lq + (valid ? t : 0)) * K;
        float *srow = p.sel ? p.sel + ((size_t)b * p.Lq + (valid ? t : 0)) * K : nullptr;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(hx * HI * kFxBN);
        uint32_t *col = sU + row;                                    // this row's column of the union area
        constexpr int HW = SM::HIST_WORDS;
        uint32_t *hist0 = col;                                       // half 0: [bin / 2] stride kFxBM
        uint32_t *hist1 = col + HW * kFxBM;                          // half 1
        uint32_t *histx = hx ? hist1 : hist0;
        uint32_t *bkey = col + 2 * HW * kFxBM;                       // [slot] stride kFxBM
        uint32_t *bpk = bkey + kFxCap * kFxBM;
        const uint32_t hist_s = smem_u32(histx), bkey_s = smem_u32(bkey), bpk_s = smem_u32(bpk);
        uint32_t *xs = sX + row;                                     // [4][kFxBM]: ns per half, ab per half

        int mode = !valid ? FX_NONE : (nv > K ? FX_OPEN : FX_ALL);
        uint32_t lo = 0, top_m1 = 0xFFFFFFFFu, blo = 0, bhi_m1 = 0;
        int sh = 25, need = 0, a_cnt = 0;
        int ab = 0, ns = 0, pos = 0, taken = 0, quota = 0, nb = 0, nbin = 0;
        // E pass: list entries are staged in this half's histogram area
        // ([slot][row], kFxStage slots) and flushed by the warp, one row at a
        // time with consecutive lanes on consecutive entries; fb is the list
        // position of the row's first staged entry, sc the staged count
        int fb = 0, sc = 0;
        // staging rows of 65 words: a lane's own slots and a row's consecutive
        // slots both fall in distinct banks
        constexpr int SROW = kFxStage + 1;
        static_assert(SROW * kFxBM <= SM::HIST_WORDS * kFxBM, "staging fits a histogram area");
        const uint32_t stage_base = smem_u32(hx ? sU + SM::HIST_WORDS * kFxBM : sU);
        const uint32_t stage_s = stage_base + (uint32_t)(row * SROW * 4);
        auto flush = [&]() {
            __syncwarp();                  // every lane's staged entries are visible
            // eight rows at a time: their shuffles, then their staged-entry
            // loads, then their stores, so that the latencies overlap
#pragma unroll 1
            for (int r0 = 0; r0 < 32; r0 += 8) {
                int n[8], base[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    n[u] = __shfl_sync(0xffffffffu, sc, r0 + u);
                    base[u] = __shfl_sync(0xffffffffu, fb, r0 + u);
                }
                uint32_t v0[8], v1[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t a0 = stage_base + (uint32_t)(((quad * 32 + r0 + u) * SROW + lane) * 4);
                    v0[u] = 0u;
                    v1[u] = 0u;
                    if (lane < n[u])
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v0[u]) : "r"(a0));
                    if (lane + 32 < n[u])
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v1[u]) : "r"(a0 + 128u));
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int rrow = quad * 32 + r0 + u;
                    int32_t *dst = p.idx + ((size_t)b * p.Lq + (size_t)min(t0 + rrow, p.Lq - 1)) * K + base[u];
                    if (lane < n[u])
                        dst[lane] = (int32_t)v0[u];
                    if (lane + 32 < n[u])
                        dst[lane + 32] = (int32_t)v1[u];
                }
            }
            fb += sc;
            sc = 0;
            __syncwarp();                  // read before any lane stages again
        };
        bool ok = true, emitted = false;
        int nd = 0;              // this half's tiles so far (D barrier phases)
        // index of the E pass as this thread knows it (every epilogue thread
        // takes the same decisions from the same barrier votes)
        int lastp = has_sel ? 0x7fffffff : (t_vis > 0 ? 0 : -1);
        const bool tracer = threadIdx.x == 64;
        for (int q = 0; q < kFxMaxPasses; ++q) {
            if (q > lastp)
                break;
            const int ptype = (has_sel && q == 0) ? 0 : (q == lastp ? 2 : 1);   // S / H / E
            const int nt = pass_tiles(q);
            const int ta = (nt + 1) / 2;
            const int nmine = hx ? nt - ta : ta;
            if (ptype == 2 && mode == FX_ALL && hx == 1)
                pos = min(nv, ta * kFxBN);          // every visible key of half 0 comes first
            if (ptype == 2)
                fb = pos;
            for (int i = 0; i < nmine; ++i, ++nd) {
                if (ok)
                    ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_DF + hx], nd & 1, abort_flag));
                if (!ok)
                    continue;
                tc_fence_after();
                const int tile = hx ? ta + i : i;
                const int kbase = tile_start(q, tile);
#pragma unroll 1
                for (int ch = 0; ch < kFxBN / 16; ++ch) {
                    if (ptype == 2 && __any_sync(0xffffffffu, sc > kFxStage - 16))
                        flush();
                    float d[HI][16];
#pragma unroll
                    for (int h = 0; h < HI; ++h)
                        fx_ld16(tl + h * kFxBN + ch * 16, d[h]);
                    tmem_ld_wait();
                    if (ch == kFxBN / 16 - 1) {
                        // the whole tile is read: the MMA may refill this half's buffer
                        tc_fence_before();
                        mbar_arrive(&bar[B_DE + hx]);
                    }
                    const int j0 = kbase + ch * 16;
                    // the chunk's 16 scores and order keys first, in straight-line
                    // code the scheduler can interleave; then the pass's work with
                    // predicated stores (a branch per score serialises the warp)
                    float sv[16];
                    uint32_t kv[16];
#pragma unroll
                    for (int c = 0; c < 16; c += 2) {
                        // two keys at a time: sum_h w_h relu(d_h) in packed pairs
                        uint64_t acc = fma_f2(f2(wv[0], wv[0]), f2(fmaxf(d[0][c], 0.f), fmaxf(d[0][c + 1], 0.f)),
                                              f2(0.f, 0.f));
#pragma unroll
                        for (int h = 1; h < HI; ++h)
                            acc = fma_f2(f2(wv[h], wv[h]), f2(fmaxf(d[h][c], 0.f), fmaxf(d[h][c + 1], 0.f)), acc);
                        f2_split(acc, sv[c], sv[c + 1]);
                        kv[c] = fx_key(sv[c]);
                        kv[c + 1] = fx_key(sv[c + 1]);
                    }
                    const int nvh = max(0, min(16, nv - j0));     // visible: c < nvh
                    // the pass's work, in a variant without per-key visibility
                    // tests for the (common) chunks that are visible throughout
                    auto work = [&](auto full_tag) {
                        constexpr bool FULL = decltype(full_tag)::value;
                        if (ptype == 0) {
                            const int clo = max(0, min(16, slot_lo(tile) - j0));
#pragma unroll
                            for (int c = 0; c < 16; ++c)
                                col[(tile * kFxBN + ch * 16 + c) * kFxBM] = (c < nvh && c >= clo) ? kv[c] : 0u;
                            ns += max(0, nvh - clo);
                        } else if (ptype == 1) {
                            if (mode == FX_OPEN) {
                                // bin 128 collects the keys above the window (when the
                                // window reaches the top key, none are)
#pragma unroll
                                for (int c = 0; c < 16; ++c) {
                                    const uint32_t k = kv[c];
                                    const uint32_t bin = min((k - lo) >> sh, (uint32_t)kFxBins);
                                    if ((FULL || c < nvh) && k >= lo)
                                        asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(hist_s + (bin >> 1) * (kFxBM * 4)),
                                                     "r"(1u << ((bin & 1u) * 16u))
                                                     : "memory");
                                }
                            }
                        } else if (mode != FX_NONE) {
                            // E: this chunk's list entries as a mask, in index order
                            uint32_t pm = 0;
                            if (mode == FX_ALL) {
                                pm = FULL ? 0xFFFFu : ((1u << nvh) - 1u);
                            } else if (mode == FX_TIE) {
                                uint32_t tm = 0;
#pragma unroll
                                for (int c = 0; c < 16; ++c) {
                                    const uint32_t k = kv[c];
                                    const bool v = FULL || c < nvh;
                                    pm |= (uint32_t)(v && k > bhi_m1) << c;
                                    tm |= (uint32_t)(v && k >= blo && k <= bhi_m1) << c;
                                }
                                // the first ties in index order, up to this half's quota
                                while (tm != 0u && taken < quota) {
                                    const uint32_t lowb = tm & (0u - tm);
                                    pm |= lowb;
                                    tm ^= lowb;
                                    ++taken;
                                }
                            } else {   // FX_BIN
#pragma unroll
                                for (int c = 0; c < 16; ++c) {
                                    const uint32_t k = kv[c];
                                    const bool v = FULL || c < nvh;
                                    const bool keep = v && k >= blo && k <= bhi_m1 && nb < kFxCap;
                                    if (keep) {
                                        // with the list position it would take: the row's
                                        // entries so far and this chunk's before it
                                        asm volatile("st.shared.u32 [%0], %1;" ::"r"(bkey_s + nb * (kFxBM * 4)), "r"(k) : "memory");
                                        asm volatile("st.shared.u32 [%0], %1;" ::"r"(bpk_s + nb * (kFxBM * 4)),
                                                     "r"((uint32_t)(j0 + c) | ((uint32_t)(pos + __popc(pm)) << 16))
                                                     : "memory");
                                    }
                                    nb += keep ? 1 : 0;
                                    pm |= (uint32_t)(v && k > bhi_m1) << c;
                                }
                            }
                            if (srow) {
#pragma unroll
                                for (int c = 0; c < 16; ++c)
                                    if ((pm >> c) & 1u)
                                        srow[pos + __popc(pm & ((1u << c) - 1u))] = sv[c];
                            }
                            pos += __popc(pm);
                            uint32_t m = pm;
                            while (m != 0u) {
                                const int c = __ffs(m) - 1;
                                m &= m - 1u;
                                asm volatile("st.shared.u32 [%0], %1;" ::"r"(stage_s + sc * 4), "r"((uint32_t)(j0 + c))
                                             : "memory");
                                ++sc;
                            }
                        }
                    };
                    if (nvh == 16)
                        work(std::true_type{});
                    else
                        work(std::false_type{});
                }
                if (tracer)
                    trace_ev(trb, tn, 3, 1, q, tile);
            }
            // ------------------------------ end of pass q ------------------------------
            if (!fx_all(ok)) {
                if (tracer) {
                    *abort_flag = 1;
                    *last_pass = -1;
                    __threadfence_block();
                    *decided = 0x7fffffff;
                }
                break;
            }
            if (ptype == 2) {
                flush();
                emitted = true;
                break;
            }
            if (ptype == 0) {
                // window from the sample: its lower edge is (a lower bound of) the
                // sample key of rank klo, a rank that the row's K-th largest key
                // reaches with a wide margin; its 96 lower bins span up to the
                // sample maximum, the 32 upper bins leave room above it
                xs[hx * kFxBM] = (uint32_t)ns;
                fx_sync();
                // half 0 derives the window, half 1 takes it from sX
                if (mode == FX_OPEN && hx == 0) {
                    ns = (int)(xs[0] + xs[kFxBM]);
                    uint32_t kmax = 0;
                    for (int u = 0; u < kFxSampleTiles * kFxBN; ++u)
                        kmax = max(kmax, col[u * kFxBM]);
                    if (ns > 0) {
                        const float e = (float)K * (float)ns / (float)nv;
                        int klo = (int)ceilf(e + 3.f * sqrtf(e) + 2.f);
                        klo = max(1, min(klo, ns));
                        // largest 16-bit prefix P with #(key >> 16 >= P) >= klo
                        uint32_t pfx = 0;
                        for (int bit = 15; bit >= 0; --bit) {
                            const uint32_t cand = pfx | (1u << bit);
                            int cnt = 0;
                            for (int u = 0; u < kFxSampleTiles * kFxBN; ++u)
                                cnt += (col[u * kFxBM] >> 16) >= cand;
                            if (cnt >= klo)
                                pfx = cand;
                        }
                        lo = pfx << 16;
                        const uint32_t span = kmax > lo ? kmax - lo : 0u;
                        sh = 0;
                        while (sh < 25 && (span >> sh) >= 96u)
                            ++sh;
                    } else {
                        lo = 0;
                        sh = 25;
                    }
                    xs[2 * kFxBM] = lo;
                    xs[3 * kFxBM] = (uint32_t)sh;
                }
                // every sample read is done: the area becomes the two histograms
                fx_sync();
                if (mode == FX_OPEN) {
                    lo = xs[2 * kFxBM];
                    sh = (int)xs[3 * kFxBM];
                    top_m1 = fx_last(lo, sh, kFxBins);
                }
#pragma unroll 4
                for (int w = 0; w < HW; ++w)
                    histx[w * kFxBM] = 0u;
            } else {
                // after H: find the bin holding the K-th largest key from both
                // halves' histograms (u16 pairs: the sums stay below 2^16)
                fx_sync();
                if (mode == FX_OPEN) {
                    const int ab0 = (int)(hist0[(HW - 1) * kFxBM] & 0xFFFFu);
                    ab = ab0 + (int)(hist1[(HW - 1) * kFxBM] & 0xFFFFu);
                    int cum = ab, cum0 = ab0, bstar = -1, cnt = 0, cnt0 = 0;
                    for (int w = kFxBins / 2 - 1; w >= 0 && bstar < 0; --w) {
                        const uint32_t v0 = hist0[w * kFxBM];
                        const uint32_t v = v0 + hist1[w * kFxBM];
                        const int c_hi = (int)(v >> 16), c_lo = (int)(v & 0xFFFFu);
                        const int c0_hi = (int)(v0 >> 16), c0_lo = (int)(v0 & 0xFFFFu);
                        if (cum + c_hi >= K) {
                            bstar = 2 * w + 1;
                            cnt = c_hi;
                            cnt0 = c0_hi;
                        } else if (cum + c_hi + c_lo >= K) {
                            cum += c_hi;
                            cum0 += c0_hi;
                            bstar = 2 * w;
                            cnt = c_lo;
                            cnt0 = c0_lo;
                        } else {
                            cum += c_hi + c_lo;
                            cum0 += c0_hi + c0_lo;
                        }
                    }
                    if (ab >= K) {
                        // the K-th key lies above the window: move up, wider
                        lo = top_m1 + 1u;
                        sh = min(sh + 7, 25);
                    } else if (bstar < 0) {
                        // below the window: take the whole key range
                        lo = 0;
                        sh = 25;
                    } else {
                        const uint32_t bl = lo + ((uint32_t)bstar << sh);
                        if (sh == 0 || cnt <= kFxCap) {
                            mode = sh == 0 ? FX_TIE : FX_BIN;
                            blo = bl;
                            bhi_m1 = fx_last(bl, sh, 1);
                            a_cnt = cum;
                            need = K - cum;
                            // half 1 writes after half 0's keys above the bin, and
                            // keeps its bin entries after half 0's; of a tie, half 0
                            // takes the first ones
                            const int q0 = min(need, cnt0);
                            pos = hx ? cum0 + (sh == 0 ? q0 : 0) : 0;
                            nb = hx ? cnt0 : 0;
                            nbin = cnt;
                            quota = hx ? need - q0 : q0;
                        } else {
                            // too many keys share the bin: narrow to it
                            lo = bl;
                            sh = max(sh - 7, 0);
                        }
                    }
                    top_m1 = fx_last(lo, sh, kFxBins);
                    ab = 0;
                }
                // every histogram read is done before either half clears its own
                const bool all_set = fx_all(mode != FX_OPEN);
#pragma unroll 4
                for (int w = 0; w < HW; ++w)
                    histx[w * kFxBM] = 0u;
                if (all_set)
                    lastp = q + 1;
                if (tracer) {
                    trace_ev(trb, tn, 3, 2, q, all_set ? 1 : 0);
                    if (all_set) {
                        *last_pass = q + 1;       // the next pass emits
                        __threadfence_block();
                        *decided = 0x7fffffff;
                    } else {
                        __threadfence_block();
                        *decided = q + 2;         // another H pass, then at least one more
                    }
                }
            }
        }
        // ---- boundary bin: take the `need` largest (lower index first), merge ----
        // Once both halves' lists and bin entries are written: half 0 picks the
        // row's threshold T inside the bin and compacts the chosen entries
        // (index order, with their list positions) to the front of the bin
        // buffer; then one warp per row rewrites the row's list with the
        // chosen entries in place, lanes on consecutive positions.
        fx_sync();
        if (tracer)
            trace_ev(trb, tn, 3, 3, lastp, nbin);
        const bool merging = emitted && mode == FX_BIN;
        if (hx == 0) {
            if (merging) {
                // largest key T in [blo, bhi_m1] with #(key >= T) >= need
                uint32_t lo_b = blo, hi_b = bhi_m1;
                while (lo_b < hi_b) {
                    const uint32_t mid = lo_b + ((hi_b - lo_b) >> 1) + 1u;
                    int cnt = 0;
                    for (int e = 0; e < nbin; ++e)
                        cnt += bkey[e * kFxBM] >= mid;
                    if (cnt >= need)
                        lo_b = mid;
                    else
                        hi_b = mid - 1u;
                }
                const uint32_t T = lo_b;
                int gt = 0;
                for (int e = 0; e < nbin; ++e)
                    gt += bkey[e * kFxBM] > T;
                int eq_left = need - gt;          // entries equal to T taken, lower index first
                int w = 0;
                for (int e = 0; e < nbin; ++e) {
                    const uint32_t k = bkey[e * kFxBM];
                    const bool ch = k > T || (k == T && eq_left > 0);
                    eq_left -= (k == T && ch) ? 1 : 0;
                    if (ch) {
                        bpk[w * kFxBM] = bpk[e * kFxBM];
                        bkey[w * kFxBM] = k;
                        ++w;
                    }
                }
            }
            // rows to merge: above count and chosen count
            sX[row] = merging ? (uint32_t)a_cnt : 0xFFFFFFFFu;
            sX[kFxBM + row] = merging ? (uint32_t)need : 0u;
        }
        fx_sync();
        {
            // One warp per row (epilogue warp ew takes rows ew, ew + 8, ...):
            // output position i holds the chosen entry m when i = f_m (its list
            // position plus m), else the above entry i - #(f_m < i).  Every
            // lane gathers its outputs of a block of 512 positions into
            // registers before any lane writes; blocks go from the top, so no
            // write lands on an entry a later block still reads.
            const int et = (warp - 2) * 32 + lane;
            const int ew = et >> 5;                        // epilogue warp 0..7
            for (int list = 0; list < (p.sel ? 2 : 1); ++list) {
#pragma unroll 1
                for (int r = ew; r < kFxBM; r += 8) {
                    const uint32_t ac = sX[r];
                    if (ac == 0xFFFFFFFFu)
                        continue;
                    const int nch = (int)sX[kFxBM + r];
                    // the row's chosen entries in registers: lane l holds numbers
                    // l and l + 32 (f = list position + number; f is strictly
                    // increasing, absent entries have f = ~0)
                    uint32_t f_lo = 0xFFFFFFFFu, f_hi = 0xFFFFFFFFu, j_lo = 0u, j_hi = 0u;
                    auto chosen_of = [&](int m, uint32_t &f, uint32_t &jv) {
                        const uint32_t pk = sU[(2 * HW + kFxCap + m) * kFxBM + r];     // bpk[m] of row r
                        f = (pk >> 16) + (uint32_t)m;
                        jv = list == 0 ? (pk & 0xFFFFu) : __float_as_uint(fx_score(sU[(2 * HW + m) * kFxBM + r]));
                    };
                    if (lane < nch)
                        chosen_of(lane, f_lo, j_lo);
                    if (lane + 32 < nch)
                        chosen_of(lane + 32, f_hi, j_hi);
                    const size_t grow = (size_t)b * p.Lq + (size_t)(t0 + r);
                    uint32_t *L = list == 0 ? reinterpret_cast<uint32_t *>(p.idx + grow * K)
                                            : reinterpret_cast<uint32_t *>(p.sel + grow * K);
#pragma unroll 1
                    for (int i0 = (K - 1) / 512 * 512; i0 >= 0; i0 -= 512) {
                        // chosen entries placed before position i0
                        int c = __popc(__ballot_sync(0xffffffffu, f_lo < (uint32_t)i0)) +
                                __popc(__ballot_sync(0xffffffffu, f_hi < (uint32_t)i0));
                        uint32_t v[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            // the window of 32 positions from w0: which hold chosen entries
                            const uint32_t w0 = (uint32_t)(i0 + 32 * j);
                            const uint32_t bl = f_lo - w0 < 32u ? 1u << (f_lo - w0) : 0u;
                            const uint32_t bh = f_hi - w0 < 32u ? 1u << (f_hi - w0) : 0u;
                            const uint32_t mask = __reduce_or_sync(0xffffffffu, bl | bh);
                            const int i = (int)w0 + lane;
                            const int before = c + __popc(mask & ((1u << lane) - 1u));
                            const uint32_t ca = __shfl_sync(0xffffffffu, j_lo, before & 31);
                            const uint32_t cb = __shfl_sync(0xffffffffu, j_hi, before & 31);
                            if ((mask >> lane) & 1u)
                                v[j] = before < 32 ? ca : cb;
                            else
                                v[j] = i < K ? L[i - before] : 0u;
                            c += __popc(mask);
                        }
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int i = i0 + lane + 32 * j;
                            if (i < K)
                                L[i] = v[j];
                        }
                        __syncwarp();
                    }
                }
            }
        }
        if (hx == 0 && valid && mode == FX_OPEN && !emitted && lastp >= 0 && !*abort_flag)
            set_error(HYB_ERR_DEVICE_BOUNDS);   // the window never settled within the pass limit
        if (tracer)
            trace_ev(trb, tn, 3, 4, lastp, mode);
        // a row with at most K visible keys lists all of them, then -1
        if (hx == 0 && (emitted || lastp < 0) && mode == FX_ALL) {
            for (int u = nv; u < K; ++u) {
                orow[u] = -1;
                if (srow)
                    srow[u] = -INFINITY;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[0], 512);
    }
}

// 4-D map over a [B][rows][heads][DI] bf16 tensor, box (DI, 1, box_rows, 1),
// 128-byte swizzle for DI = 64, 64-byte swizzle for DI = 32.
template <int DI>
static bool fx_map(CUtensorMap *map, const void *base, int n1, int n2, int n3, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[4] = {(cuuint64_t)DI, (cuuint64_t)n1, (cuuint64_t)n2, (cuuint64_t)n3};
    cuuint64_t strides[3] = {(cuuint64_t)DI * 2, (cuuint64_t)DI * 2 * n1, (cuuint64_t)DI * 2 * n1 * n2};
    cuuint32_t box[4] = {(cuuint32_t)DI, 1, (cuuint32_t)box_rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    DI == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int HI, int DI>
static cudaError_t launch_fx_t(const FusedIndexParams &p, const void *qi, const void *kic, cudaStream_t stream)
{
    using SM = FxSmem<HI, DI>;
    CUtensorMap mq, mk;
    // qi [B, Lq, Hi, DI] as (DI, Hi, Lq, B): one head's 128 rows per box
    bool ok = fx_map<DI>(&mq, qi, HI, p.Lq, p.B, kFxBM);
    // kic [B, Nc, DI] as (DI, 1, Nc, B): 64 entries per box (zeros past Nc)
    ok &= fx_map<DI>(&mk, kic, 1, p.Nc, p.B, kFxBN);
    if (!ok)
        return cudaErrorInvalidValue;
    size_t smem = 1024 + SM::BYTES;
    if (smem < 120 * 1024)
        smem = 120 * 1024;   // one CTA per SM: each holds all 512 TMEM columns
    auto kern = index_topk_fused<HI, DI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    const unsigned grid = (unsigned)p.n_ttiles * (unsigned)p.B;
    return launch_pdl(kern, dim3(grid), dim3(kFxThreads), smem, stream, mq, mk, p);
}

// Shapes the fused kernel takes: query tiles of many rows (not the decode
// form), di in {32, 64}, at most 4 indexer heads, entries and K small enough
// for the packed (index, list position) words.
bool index_fused_supported(int Lq, int Hi, int di, int Nc, int K)
{
    return Lq >= 64 && Hi >= 1 && Hi <= 4 && (di == 32 || di == 64) && Nc <= kFxMaxNc && K >= 1 &&
           K <= 2048;
}

cudaError_t launch_index_topk_fused(const void *qi, const float *wi, const void *kic, int32_t *idx,
                                    float *sel, int B, int Lq, int Hi, int di, int Nc, int m, int W, int K,
                                    const int32_t *q_pos, cudaStream_t stream)
{
    if (!index_fused_supported(Lq, Hi, di, Nc, K))
        return cudaErrorNotSupported;
    FusedIndexParams p;
    p.B = B;
    p.Lq = Lq;
    p.Hi = Hi;
    p.Nc = Nc;
    p.m = m;
    p.W = W;
    p.K = K;
    p.n_ttiles = (Lq + kFxBM - 1) / kFxBM;
    p.q_pos = q_pos;
    p.wi = wi;
    p.idx = idx;
    p.sel = sel;
    if (di == 64) {
        switch (Hi) {
        case 1: return launch_fx_t<1, 64>(p, qi, kic, stream);
        case 2: return launch_fx_t<2, 64>(p, qi, kic, stream);
        case 3: return launch_fx_t<3, 64>(p, qi, kic, stream);
        default: return launch_fx_t<4, 64>(p, qi, kic, stream);
        }
    }
    switch (Hi) {
    case 1: return launch_fx_t<1, 32>(p, qi, kic, stream);
    case 2: return launch_fx_t<2, 32>(p, qi, kic, stream);
    case 3: return launch_fx_t<3, 32>(p, qi, kic, stream);
    default: return launch_fx_t<4, 32>(p, qi, kic, stream);
    }
}

}  // namespace hyb

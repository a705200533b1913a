// attn_sparse.cu -- stage 3 for CSA ("deepseek-v4" blog, section 1, CSA and
// SWA): every query token attends to its own top-K compressed entries plus
// the raw window, with all query heads of a KV group (MQA / GQA, CS336
// "Attention Heads variants") sharing those keys.
//
// Because each token has its own key set, query rows of different tokens
// cannot share a key tile.  The kernel therefore computes the transposed
// products with the keys in the MMA's M dimension:
//     S^T [128 keys x NH heads]  = K_tile [128 x d] . Q^T        (tcgen05, TMEM)
//     O^T [d x NH]              += V_tile^T [d x 128] . P^T       (V as MN-major A)
// where NH is the group's head count padded to 16, 32 or 64.  No MMA row is
// padding for the 32- and 64-head groups of the CSA workloads.
//
// Softmax: thread = key (TMEM lane).  For 32- and 64-head groups two
// warpgroups share the keys and split the heads (TMEM columns), each thread
// holding NH / 2 scores of its key; 16-head groups use one warpgroup.  A
// per-head reference max lives in shared memory; it is moved (with a
// block-wide max reduction, and a rescale of O^T and of the partial sums) only
// when some key exceeds it by more than 2^8, i.e. on the first tile of a token
// and rarely after.  Partial row sums stay per thread and are reduced once per
// token.  P^T is written to shared memory in the 32/64/128-byte swizzle
// matching NH.
//
// Gathers: four producer warps copy the selected compressed rows with 16-byte
// cp.async (16 lanes per 256-byte row, so every warp instruction moves two
// whole rows) straight into the 128-byte-swizzled tile layout; each thread
// then arms the stage's mbarrier with an asynchronous arrive that fires when
// its copies land, so the producers never block on a copy.  Window tiles (128
// consecutive raw rows) come by TMA.  (Random 256-byte rows held in L2 move
// through 16-byte cp.async about six times faster than through TMA
// tile::gather4 on B200, 14.1 against 2.3 TB/s in the gather probes, and
// about three times faster than through 256-byte bulk copies.)  K copies run
// one tile ahead of V copies.
// The token's selection is decoded once into one of two shared tables of
// source rows (-1: unselected, invisible or out of range; those slots are
// zero-filled and masked); the softmax reads key validity from the same
// table, published through its own mbarrier.
// Roles: softmax warpgroup(s), then four producer warps (two for 64-head
// groups, whose softmax needs more registers), then one MMA warp; work items
// (b, t, KV head) go round-robin to persistent CTAs.  Every role agrees once
// per item whether to go on, so a failed (bounded) wait never leaves a
// thread waiting at a named barrier.
#include "common.cuh"

namespace hyb {

constexpr int kSpBN = 128;       // keys per tile (the M of S^T)
constexpr int kSpLead = 1;       // tiles by which the K copies run ahead of the V copies
// The next item's prologue runs before this item's K copy of tile
// ntl - kSpPrologueAhead (of ntl tiles).  On the CSA prefill 2 measured best:
// 1.795 ms against 1.870 (0, after the last K tile), 2.18 (1), 1.85 (3),
// 2.10 (4), 2.26 (5), and against forms that ran it at the first ring wait
// that would block (1.95 to 2.3 ms).
constexpr int kSpPrologueAhead = 2;
constexpr int kSpD = 128;        // head dim handled by this kernel

struct SparseParams {
    int B, Lq, Lkv, Hq, Hkv, g, Nc, m, W, topk, NH;
    int pregathered;   // kc / vc hold each token's selected rows in slot order: [B Lq, topk, Hkv, 128]
    int split;         // CTAs (one cluster) sharing each item's key tiles: 1 or 2
    int tsel;          // entries of a decoded selection table: topk rounded up to whole tiles
    int prefetch;      // compressed caches far larger than L2: pull an item's selected rows into L2 first
    long long n_items;
    float scale_log2;
    const int32_t *q_pos, *kv_pos0, *idx;
    const __nv_bfloat16 *kc, *vc, *kr, *vr;   // [B, rows, Hkv, 128]
    __nv_bfloat16 *o;
    float *lse;
};

template <int NH>
struct SparseSmem {
    static constexpr int Q_BYTES = NH * kSpD * 2;
    static constexpr int KV_BYTES = kSpBN * kSpD * 2;
    static constexpr int P_BYTES = kSpBN * NH * 2;
    static constexpr int P_STRIDE = (P_BYTES + 1023) & ~1023;
    // K runs deeper than V: a K stage frees as soon as its scores are taken,
    // a V stage only after the tile's softmax and PV, and the scores of later
    // tiles should not wait on a V stage
    static constexpr int KS = NH == 64 ? 2 : 3;                    // K ring depth
    static constexpr int VS = 2;                                   // V ring depth
    static_assert(KS <= 3 && VS <= 3, "the barrier slots SB_KF .. SB_VE hold three stages each");
    static constexpr int OFF_Q = 0;                                // 2 buffers
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KS * KV_BYTES;
    static constexpr int OFF_P = OFF_V + VS * KV_BYTES;            // 2 buffers
    static constexpr int OFF_RED = OFF_P + 2 * P_STRIDE;           // [2 warpgroups][NH][4] floats
    static constexpr int OFF_MREF = OFF_RED + 2 * 4 * NH * 4;      // [2 warpgroups][2][NH] floats
    static constexpr int OFF_INV = OFF_MREF + 4 * NH * 4;          // [NH] floats
    static constexpr int OFF_BAR = OFF_INV + NH * 4;
    static constexpr int OFF_MISC = OFF_BAR + 32 * 8;
    static constexpr int OFF_PML = OFF_MISC + 16 * 4;               // split: peer's [max, sum] per head
    static constexpr int OFF_CMB = OFF_PML + 2 * NH * 4;            // split / ping-pong: [2][NH] combine factors
    static constexpr int OFF_PPX = OFF_CMB + 2 * NH * 4;            // ping-pong: [2 warpgroups][max, sum][NH]
    static constexpr int OFF_IDX = OFF_PPX + 4 * NH * 4;            // [2][tsel] decoded selections
    static constexpr int BASE_BYTES = OFF_IDX;                      // + 2 tsel * 4, tsel = topk rounded up to 128
};

// mbarriers (two of each per-item or per-buffer kind, three per ring stage)
enum {
    SB_QF = 0, SB_QE = 2, SB_KF = 4, SB_KE = 7, SB_VF = 10, SB_VE = 13, SB_SF = 16, SB_PF = 18,
    SB_OD = 20, SB_OE = 22, SB_IF = 24, SB_DONE = 26,
    SB_GO = 27,      // split, rank 1: rank 0 can take this item's partial (arrived by rank 0)
    SB_PFULL = 28,   // split, rank 0: rank 1's partial has landed (arrived by rank 1's softmax threads)
    SB_SE = 29,      // ping-pong: S^T buffer read into registers (two buffers)
    SB_COUNT = 31
};

struct SparseTok {
    int b, t, kvh;
    long long pos, kv0;
    int nct, nrt, rlo, rhi;
};

__device__ __forceinline__ SparseTok sparse_tok(const SparseParams &p, long long w)
{
    // items number below 2^31 (checked at launch): 32-bit divisions, which
    // cost a fraction of 64-bit ones, and none for the common single KV head
    // or single sequence
    SparseTok k;
    const uint32_t wu = (uint32_t)w, hkv = (uint32_t)p.Hkv, lq = (uint32_t)p.Lq;
    const uint32_t bt = hkv == 1u ? wu : wu / hkv;
    k.kvh = (int)(wu - bt * hkv);
    const uint32_t bb = p.B == 1 ? 0u : bt / lq;
    k.b = (int)bb;
    k.t = (int)(bt - bb * lq);
    k.pos = p.q_pos ? p.q_pos[bt] : k.t;
    k.kv0 = p.kv_pos0 ? p.kv_pos0[k.b] : 0;
    k.nct = (p.topk + kSpBN - 1) / kSpBN;
    long long lo = k.pos - p.W + 1;
    if (lo < 0)
        lo = 0;
    lo -= k.kv0;
    if (lo < 0)
        lo = 0;
    long long hi = k.pos - k.kv0;
    if (hi > p.Lkv - 1)
        hi = p.Lkv - 1;
    k.rlo = (int)lo;
    k.rhi = (int)hi;
    k.nrt = (p.W > 0 && hi >= lo) ? (int)((hi - lo + kSpBN) / kSpBN) : 0;
    return k;
}

// Arrive on `bar` once every cp.async issued so far by this thread has landed
// (the pending count is raised first, so a regular arrive must follow).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// OR-reduction of a predicate over the N softmax threads (named barrier 1).
template <int N>
__device__ __forceinline__ bool sm_any(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(N)
        : "memory");
    return r != 0;
}

// AND of a predicate over the N softmax threads (named barrier 1).
template <int N>
__device__ __forceinline__ bool sm_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(N)
        : "memory");
    return r != 0;
}

template <int N>
__device__ __forceinline__ void sm_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}

// Named barriers with a run-time id (ping-pong softmax: one per warpgroup,
// and one over both warpgroups).
__device__ __forceinline__ void bar_sync_id(uint32_t id, uint32_t n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ bool bar_any_id(uint32_t id, uint32_t n, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ bool bar_all_id(uint32_t id, uint32_t n, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Per-head totals over the 32 lanes of a warp by recursive halving: at each
// step a lane keeps one half of its values (the upper half where its lane
// bit is set), receives the partner's copy of that half and combines.  NH
// values cost NH - 1 shuffles (plus one per remaining lane bit for NH < 32).
// Afterwards lane l holds in v[0 .. SpHeads<NH>::VPL) the warp totals of the
// heads SpHeads<NH>::head(l, e).
template <int NH>
struct SpHeads {
    static constexpr int VPL = NH >= 32 ? NH / 32 : 1;     // values per lane
    static constexpr int LPH = NH >= 32 ? 1 : 32 / NH;     // lanes per head
    __device__ static int head(int lane, int e) { return NH >= 32 ? lane * VPL + e : lane / LPH; }
};

template <bool MAX, int N, int OFF, int NH>
__device__ __forceinline__ void halve_heads(float (&v)[NH], int lane)
{
    if constexpr (OFF >= 1) {
        if constexpr (N > 1) {
            constexpr int H = N / 2;
            const bool up = (lane & OFF) != 0;
#pragma unroll
            for (int j = 0; j < H; ++j) {
                const float send = up ? v[j] : v[j + H];
                const float keep = up ? v[j + H] : v[j];
                const float got = __shfl_xor_sync(0xffffffffu, send, OFF);
                v[j] = MAX ? fmaxf(keep, got) : keep + got;
            }
            halve_heads<MAX, H, OFF / 2>(v, lane);
        } else {
            const float got = __shfl_xor_sync(0xffffffffu, v[0], OFF);
            v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
            halve_heads<MAX, 1, OFF / 2>(v, lane);
        }
    }
}

template <int NH, bool MAX>
__device__ __forceinline__ void warp_reduce_heads(float (&v)[NH], int lane)
{
    halve_heads<MAX, NH, 16>(v, lane);
}

// New reference for one head: moves only when the tile max exceeds the old
// one by more than 2^8.
__device__ __forceinline__ float sp_new_ref(float4 q4, float old)
{
    const float tmx = fmaxf(fmaxf(q4.x, q4.y), fmaxf(q4.z, q4.w));
    return tmx > old + 8.f ? tmx : old;
}

__device__ __forceinline__ float sp_factor(float old, float nw)
{
    return nw == old ? 1.f : (old == -INFINITY ? 0.f : ex2_approx(old - nw));
}

// Shared-memory descriptor with a selectable swizzle (layout 2: 128 B, 4: 64 B, 6: 32 B).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)layout << 61;
    return d;
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[N])
{
    static_assert(N % 16 == 0, "");
#pragma unroll
    for (int c = 0; c < N; c += 16) {
        uint32_t r[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
              "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
              "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr + c));
#pragma unroll
        for (int q = 0; q < 16; ++q)
            v[c + q] = __uint_as_float(r[q]);
    }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float (&v)[N])
{
#pragma unroll
    for (int c = 0; c < N; c += 16) {
        uint32_t r[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
            r[q] = __float_as_uint(v[c + q]);
        tmem_st16(taddr + c, r);
    }
}

// Producer warps: four for up to 32 heads; two for 64 heads, whose softmax
// threads need up to 255 registers (8 warps in all).
// Ping-pong softmax for 32-head groups: the two softmax warpgroups take
// alternate key tiles (all heads of a key each) with their own running maxima,
// sums and O^T accumulators, combined once per item, so that one tile's
// softmax overlaps the next one's instead of both warpgroups splitting every
// tile's heads.
constexpr bool kSpPingPong = false;   // measured slower than the head split on the CSA prefill (2.32 vs 1.87 ms)

template <int NH>
struct SpRoles {
    static constexpr bool PP = kSpPingPong && NH == 32;
    // ping-pong register split (setmaxnreg): 8 softmax warps up, producer and
    // MMA warps down; 256 x 144 + 160 x 96 = 52224 <= 416 x 128, the budget
    // the block launches with (the launcher checks it against the allocated count)
    static constexpr int PP_SOFTMAX_REGS = 144;
    static constexpr int PP_OTHER_REGS = 96;
    static constexpr int HS = NH >= 32 ? 2 : 1;       // softmax warpgroups (head halves, or tile parities)
    static constexpr int NHW = PP ? NH : NH / HS;     // heads per softmax thread
    static constexpr int SMT = 128 * HS;              // softmax threads
    static constexpr int PW = NH == 64 ? 2 : 4;       // producer warps
    static constexpr int PROD_WARP0 = 4 * HS;
    static constexpr int MMA_WARP = PROD_WARP0 + PW;
    static constexpr int THREADS = 32 * (MMA_WARP + 1);
    // selection entries a producer thread loads at once: 4 covers a 512-entry
    // selection over four warps in one batch (CSA prefill: 1.756 ms against
    // 1.793 with 8); 8 for the two-warp decode form (25.6 against 27.6 us)
    static constexpr int SEL_BATCH = NH == 64 ? 8 : 4;
};

template <int NH>
__global__ void __launch_bounds__(SpRoles<NH>::THREADS, 1)
csa_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kr,
                const __grid_constant__ CUtensorMap tm_vr, const SparseParams p)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
    using SM = SparseSmem<NH>;
    constexpr int KS = SM::KS;
    constexpr int VS = SM::VS;
    constexpr int RB = NH * 2;                                  // bytes of one P^T row
    constexpr uint32_t PLAYOUT = RB == 128 ? 2u : (RB == 64 ? 4u : 6u);
    extern __shared__ __align__(1024) uint8_t sp_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sp_smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sQ = smem + SM::OFF_Q;
    uint8_t *sK = smem + SM::OFF_K;
    uint8_t *sV = smem + SM::OFF_V;
    uint8_t *sP = smem + SM::OFF_P;
    float *sRed = reinterpret_cast<float *>(smem + SM::OFF_RED);
    float *sMref = reinterpret_cast<float *>(smem + SM::OFF_MREF);
    float *sInv = reinterpret_cast<float *>(smem + SM::OFF_INV);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM::OFF_BAR);
    int *misc = reinterpret_cast<int *>(smem + SM::OFF_MISC);
    int *sIdx = reinterpret_cast<int *>(smem + SM::OFF_IDX);
    volatile int *abort_flag = misc + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    unsigned long long *const trb = trace_buffer();   // timeline of CTA 0, when attached
    uint32_t tn = 0;                                  // this thread's trace records
    constexpr int PW = SpRoles<NH>::PW;
    constexpr int NPT = 32 * PW;                // producer threads

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[SB_QF + s], 1);
            mbar_init(&bar[SB_QE + s], 1);
            mbar_init(&bar[SB_SF + s], 1);
            mbar_init(&bar[SB_OE + s], SpRoles<NH>::SMT);
            mbar_init(&bar[SB_PF + s], SpRoles<NH>::PP ? 128 : SpRoles<NH>::SMT);
            mbar_init(&bar[SB_SE + s], 128);
            mbar_init(&bar[SB_OD + s], 1);
            mbar_init(&bar[SB_IF + s], NPT);
        }
        for (int s = 0; s < KS; ++s) {
            mbar_init(&bar[SB_KF + s], NPT);
            mbar_init(&bar[SB_KE + s], 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&bar[SB_VF + s], NPT);
            mbar_init(&bar[SB_VE + s], 1);
        }
        mbar_init(&bar[SB_DONE], 1);
        mbar_init(&bar[SB_GO], 1);
        mbar_init(&bar[SB_PFULL], SpRoles<NH>::SMT);
        mbar_fence_init();
        misc[1] = 0;
    }
    if (threadIdx.x < 4 * NH)
        sMref[threadIdx.x] = -INFINITY;
    if (warp == SpRoles<NH>::MMA_WARP)
        tmem_alloc(reinterpret_cast<uint32_t *>(&misc[0]), 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    // Items go round-robin to CTAs, or to clusters of `split` CTAs that share
    // each item's key tiles: CTA rank r takes tiles [nt r / split, nt (r+1) / split).
    const int split = p.split;
    const uint32_t crank = split > 1 ? cluster_ctarank() : 0u;
    const long long w0 = blockIdx.x / split, wstep = gridDim.x / split;
    auto tile_lo = [&](int nt) -> int { return (int)((nt * (int)crank) / split); };
    auto tile_hi = [&](int nt) -> int { return (int)((nt * ((int)crank + 1)) / split); };
    if (split > 1)
        cluster_sync_all();   // the peer's barriers are initialised before any remote arrival
    // TMEM columns: S^T buffers at 0 and NH, O^T buffers at 2NH and 3NH
    const uint32_t TM_S0 = 0, TM_O0 = 2 * NH;

    constexpr int RPI = NPT / 16;               // rows per copy round
    constexpr int CPT = kSpBN / RPI;            // copies per thread per tile and operand
    constexpr int MMA_WARP = SpRoles<NH>::MMA_WARP;
    if (warp >= SpRoles<NH>::PROD_WARP0 && warp < MMA_WARP) {
        if constexpr (SpRoles<NH>::PP)
            asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(SpRoles<NH>::PP_OTHER_REGS));
        // ================================ producer ================================
        // 16 lanes per 256-byte row, two rows per warp instruction.  Each
        // producer warp decodes the selection entries of exactly the rows its
        // own lanes copy, so the warps need no barrier among themselves; the
        // softmax learns that the whole table is written from an mbarrier.
        // Within an item no warp leaves early: a failed wait clears `ok` and
        // the copies go on (every source row stays in range).
        const int pt = threadIdx.x - 32 * SpRoles<NH>::PROD_WARP0;
        const int pw = pt >> 5;                 // producer warp
        const int c8 = pt & 15;                 // 16-byte chunk of the row
        const int rsub = pt >> 4;               // rows rsub, rsub + RPI, ... (2 pw and 2 pw + 1)
        const uint32_t dchunk = (uint32_t)(c8 >> 3) * kSpBN * 128;
        uint32_t kc = 0, vc = 0, nq = 0;
        bool ok = true;
        // slot of this warp's e-th selection entry, tiles counted from t0s:
        // rows u RPI + 2 pw + bit of each tile
        auto slot_of = [&](int t0s, int e) -> int {
            const int tile = e / (2 * CPT), rem = e - tile * (2 * CPT);
            return (t0s + tile) * kSpBN + (rem >> 1) * RPI + 2 * pw + (rem & 1);
        };
        // this CTA's selected tiles of an item: [s0, s1)
        auto sel_tiles = [&](const SparseTok &k, int &s0, int &s1) {
            const int nt = k.nct + k.nrt;
            s0 = min(tile_lo(nt), k.nct);
            s1 = min(tile_hi(nt), k.nct);
        };
        // this warp's entries e0 + lane + 32 j (of ne) of item w's selection,
        // -1 past topk; item w = (b Lq + t) Hkv + KV head, below 2^31
        auto load_sel = [&](long long w, int t0s, int ne, int e0, int (&jv)[SpRoles<NH>::SEL_BATCH]) {
            const int32_t *irow = p.idx + (size_t)((uint32_t)w / (uint32_t)p.Hkv) * p.topk;
#pragma unroll
            for (int j = 0; j < SpRoles<NH>::SEL_BATCH; ++j) {
                const int e = e0 + lane + 32 * j;
                const int q = slot_of(t0s, e);
                // volatile: issued here, not sunk to the first use an item later
                int v = -1;
                if (e < ne && q < p.topk)
                    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(irow + q));
                jv[j] = v;
            }
        };
        auto load_first = [&](long long w, int (&jv)[SpRoles<NH>::SEL_BATCH]) {
            const SparseTok kn = sparse_tok(p, w);
            int s0, s1;
            sel_tiles(kn, s0, s1);
            load_sel(w, s0, (s1 - s0) * 2 * CPT, 0, jv);
        };
        int jnext[SpRoles<NH>::SEL_BATCH];
        uint32_t nql = 0;                       // items whose Q tile was sent for
        // An item's prologue: its Q tile, its selection decoded into buffer
        // nq & 1 (the first batch of entries already in jnext), and the next
        // item's first batch sent for.  It runs during the previous item's
        // copies (before its K tile ntl - kSpPrologueAhead), so that the
        // gather does not pause between items.
        auto prologue = [&](long long w, uint32_t nq) {
            const SparseTok k = sparse_tok(p, w);
            const int qb = nq & 1;
            if (nq >= 2) {
                // Q buffer qb: the last scores of item nq - 2 are done;
                // selection buffer qb: so is that item's softmax
                ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_QE + qb], ((nq >> 1) - 1) & 1, abort_flag));
                ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_OE + qb], ((nq >> 1) - 1) & 1, abort_flag));
            }
            if (pt == 0) {
                trace_ev(trb, tn, 1, 3, w, 0);
                mbar_arrive_expect_tx(&bar[SB_QF + qb], SM::Q_BYTES);
                const int qrow = (int)(((long long)k.b * p.Lq + k.t) * p.Hq) + k.kvh * p.g;
                for (int cb = 0; cb < 2; ++cb)
                    tma_load_2d(sQ + qb * SM::Q_BYTES + cb * NH * 128, &tm_q, &bar[SB_QF + qb], cb * 64,
                                qrow);
            }
            nql = nq + 1;
            // decode this warp's part of the item's selection into buffer qb:
            // source row of every slot, or -1 (unselected, invisible, out of
            // range or past topk).  A batch's loads are all in flight
            // together; the first batch was loaded during the previous item.
            int *sSel = sIdx + qb * p.tsel;
            {
                const long long wstart = k.pos - p.W + 1;
                int s0, s1;
                sel_tiles(k, s0, s1);
                const int ne = (s1 - s0) * 2 * CPT;
#pragma unroll 1
                for (int e0 = 0; e0 < ne; e0 += 32 * SpRoles<NH>::SEL_BATCH) {
                    int jv[SpRoles<NH>::SEL_BATCH];
                    if (e0 == 0) {
#pragma unroll
                        for (int j = 0; j < SpRoles<NH>::SEL_BATCH; ++j)
                            jv[j] = jnext[j];
                    } else {
                        load_sel(w, s0, ne, e0, jv);
                    }
#pragma unroll
                    for (int j = 0; j < SpRoles<NH>::SEL_BATCH; ++j) {
                        const int e = e0 + lane + 32 * j;
                        if (e < ne) {
                            const int q = slot_of(s0, e);
                            int src = -1;
                            if (q < p.topk) {
                                const int jj = jv[j];
                                if (jj >= p.Nc)
                                    set_error(HYB_ERR_DEVICE_BOUNDS);
                                const bool v = jj >= 0 && jj < p.Nc && ((long long)(jj + 1) * p.m - 1 < wstart);
                                const int srow = p.pregathered
                                                     ? ((int)((uint32_t)w / (uint32_t)p.Hkv) * p.topk + q) * p.Hkv +
                                                           k.kvh
                                                     : (k.b * p.Nc + jj) * p.Hkv + k.kvh;
                                src = v ? srow : -1;
                                if (p.prefetch && v) {
                                    // the row's K and V lines into L2 now: the copies
                                    // of the item's tiles then wait on L2, not HBM
                                    const __nv_bfloat16 *kr0 = p.kc + (size_t)srow * kSpD;
                                    const __nv_bfloat16 *vr0 = p.vc + (size_t)srow * kSpD;
                                    asm volatile("prefetch.global.L2 [%0];" ::"l"(kr0));
                                    asm volatile("prefetch.global.L2 [%0];" ::"l"(kr0 + 64));
                                    asm volatile("prefetch.global.L2 [%0];" ::"l"(vr0));
                                    asm volatile("prefetch.global.L2 [%0];" ::"l"(vr0 + 64));
                                }
                            }
                            sSel[q] = src;
                        }
                    }
                }
            }
            mbar_arrive(&bar[SB_IF + qb]);      // the softmax reads key validity from it
            __syncwarp();                       // this warp's lanes read each other's entries
            if (pt == 0)
                trace_ev(trb, tn, 1, 4, w, 0);
            if (w + wstep < p.n_items)
                load_first(w + wstep, jnext);
        };
        if (w0 < p.n_items) {
            load_first(w0, jnext);
            prologue(w0, 0);
        }
        for (long long w = w0; w < p.n_items; w += wstep, ++nq) {
            if (!__all_sync(0xffffffffu, ok && !*abort_flag))
                break;
            const SparseTok k = sparse_tok(p, w);
            const int *sSel = sIdx + (nq & 1) * p.tsel;
            const int nt = k.nct + k.nrt;
            const int tb = tile_lo(nt), ntl = tile_hi(nt) - tb;   // this CTA's tiles
            // source row of copy u of tile i, or -1 (zero-filled)
            // source row of copy u of selected tile i, or -1: an unselected slot
            // is zero-filled without a read (a fixed stand-in row would pile
            // every early token's empty slots onto one L2 line)
            auto src_of = [&](int i, int u) -> int { return sSel[i * kSpBN + u * RPI + rsub]; };
            const __nv_bfloat16 *kc8 = p.kc + c8 * 8, *vc8 = p.vc + c8 * 8;   // this thread's chunk
            // K of tile i goes out kSpLead tiles ahead of V of the same tile, so
            // that the next scores need not queue behind a V stage that a PV
            // still holds.  A tile's source rows are read into registers
            // before its copies (each copy is a compiler barrier), for K and
            // again for V.
            for (int ii = 0; ii < ntl + kSpLead; ++ii) {
                const int i = tb + ii;
                if (ii == max(ntl - kSpPrologueAhead, 0) && w + wstep < p.n_items)
                    prologue(w + wstep, nq + 1);
                if (ii < ntl) {
                    const uint32_t ks = kc % KS;
                    if (kc >= KS)
                        ok &= __all_sync(0xffffffffu,
                                         mbar_wait(&bar[SB_KE + ks], ((kc / KS) - 1) & 1, abort_flag));
                    if (i >= k.nct) {
                        // window tile: 128 consecutive raw rows, two TMA boxes
                        // (rows past the window are masked by the softmax)
                        if (pt == 0) {
                            const int r0 = k.b * p.Lkv + k.rlo + (i - k.nct) * kSpBN;
                            mbar_arrive_expect_tx(&bar[SB_KF + ks], SM::KV_BYTES);
                            tma_load_3d(sK + ks * SM::KV_BYTES, &tm_kr, &bar[SB_KF + ks], 0, k.kvh, r0);
                            tma_load_3d(sK + ks * SM::KV_BYTES + kSpBN * 128, &tm_kr, &bar[SB_KF + ks], 64,
                                        k.kvh, r0);
                        } else {
                            mbar_arrive(&bar[SB_KF + ks]);
                        }
                    } else {
                        int srck[CPT];
#pragma unroll
                        for (int u = 0; u < CPT; ++u)
                            srck[u] = src_of(i, u);
                        const uint32_t dst = smem_u32(sK + ks * SM::KV_BYTES) + dchunk;
#pragma unroll
                        for (int u = 0; u < CPT; ++u) {
                            const int sr = srck[u];
                            cp_async_16(dst + sw128_offset(u * RPI + rsub, c8 & 7), kc8 + (size_t)max(sr, 0) * kSpD,
                                        sr >= 0 ? 16u : 0u);
                        }
                        cp_async_mbar_arrive(&bar[SB_KF + ks]);
                        mbar_arrive(&bar[SB_KF + ks]);
                    }
                    if (pt == 0)
                        trace_ev(trb, tn, 1, 1, w, i);
                    ++kc;
                }
                if (ii >= kSpLead) {
                    const int iv = i - kSpLead;
                    const uint32_t vs = vc % VS;
                    if (vc >= VS)
                        ok &= __all_sync(0xffffffffu,
                                         mbar_wait(&bar[SB_VE + vs], ((vc / VS) - 1) & 1, abort_flag));
                    if (iv >= k.nct) {
                        if (pt == 0) {
                            const int r0 = k.b * p.Lkv + k.rlo + (iv - k.nct) * kSpBN;
                            mbar_arrive_expect_tx(&bar[SB_VF + vs], SM::KV_BYTES);
                            tma_load_3d(sV + vs * SM::KV_BYTES, &tm_vr, &bar[SB_VF + vs], 0, k.kvh, r0);
                            tma_load_3d(sV + vs * SM::KV_BYTES + kSpBN * 128, &tm_vr, &bar[SB_VF + vs], 64,
                                        k.kvh, r0);
                        } else {
                            mbar_arrive(&bar[SB_VF + vs]);
                        }
                    } else {
                        int srcv[CPT];
#pragma unroll
                        for (int u = 0; u < CPT; ++u)
                            srcv[u] = src_of(iv, u);
                        const uint32_t dst = smem_u32(sV + vs * SM::KV_BYTES) + dchunk;
#pragma unroll
                        for (int u = 0; u < CPT; ++u) {
                            const int sr = srcv[u];
                            cp_async_16(dst + sw128_offset(u * RPI + rsub, c8 & 7), vc8 + (size_t)max(sr, 0) * kSpD,
                                        sr >= 0 ? 16u : 0u);
                        }
                        cp_async_mbar_arrive(&bar[SB_VF + vs]);
                        mbar_arrive(&bar[SB_VF + vs]);
                    }
                    if (pt == 0)
                        trace_ev(trb, tn, 1, 2, w, i - kSpLead);
                    ++vc;
                }
            }
        }
        // unwinding: every copy issued by this thread has landed
        cp_async_wait_group<0>();
        if (pt == 0) {
            // the Q tiles of the last two items whose prologue ran (one may be
            // an item the loop did not reach)
            for (uint32_t q = (nql > 2 ? nql - 2 : 0); q < nql; ++q)
                drain_wait(&bar[SB_QF + (q & 1)], (q >> 1) & 1);
        }
    } else if (warp == MMA_WARP) {
        if constexpr (SpRoles<NH>::PP)
            asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(SpRoles<NH>::PP_OTHER_REGS));
        // ================================ MMA issue ================================
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16(kSpBN, NH, false, false);
            const uint32_t idesc_pv = idesc_bf16(kSpD, NH, true, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            uint32_t kc = 0, vc = 0, nq = 0, gt = 0, pcnt = 0;
            bool ok = true;
            for (long long w = w0; ok && w < p.n_items; w += wstep, ++nq) {
                const SparseTok k = sparse_tok(p, w);
                const int nt = k.nct + k.nrt;
                const int tb = tile_lo(nt), ntl = tile_hi(nt) - tb;   // this CTA's tiles
                const int qb = nq & 1, ob = nq & 1;
                if (!mbar_wait(&bar[SB_QF + qb], (nq >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                auto issue_pv = [&](bool first) -> bool {
                    const uint32_t vs = vc % VS;
                    const uint32_t pb = pcnt & 1;
                    if (!mbar_wait(&bar[SB_PF + pb], (pcnt >> 1) & 1, abort_flag) ||
                        !mbar_wait(&bar[SB_VF + vs], (vc / VS) & 1, abort_flag))
                        return false;
                    if (first && nq >= 2 &&
                        !mbar_wait(&bar[SB_OE + ob], ((nq >> 1) - 1) & 1, abort_flag))
                        return false;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kSpBN / 16; ++kk) {
                        const uint64_t da = smem_desc(aV + vs * SM::KV_BYTES + kk * 16 * 128,
                                                      kSpBN * 128, 1024, 2);
                        const uint64_t db = smem_desc(aP + pb * SM::P_STRIDE + kk * 16 * RB, 16, 8 * RB,
                                                      PLAYOUT);
                        mma_bf16_ss(tmem + TM_O0 + ob * NH, da, db, idesc_pv,
                                    (first && kk == 0) ? 0u : 1u);
                    }
                    mma_commit(&bar[SB_OD + pb]);
                    mma_commit(&bar[SB_VE + vs]);
                    trace_ev(trb, tn, 2, 2, w, (int)pcnt);
                    ++vc;
                    ++pcnt;
                    return true;
                };
                if constexpr (SpRoles<NH>::PP) {
                    // ping-pong: QK^T runs two tiles ahead of PV, refilling an S^T
                    // buffer once its warpgroup has read it; PV of tile g goes to
                    // its parity's O^T accumulator
                    const uint32_t gt0 = gt;
                    auto issue_pv_pp = [&](uint32_t g) -> bool {
                        const uint32_t vs = vc % VS, pb = g & 1;
                        if (!mbar_wait(&bar[SB_PF + pb], (g >> 1) & 1, abort_flag) ||
                            !mbar_wait(&bar[SB_VF + vs], (vc / VS) & 1, abort_flag))
                            return false;
                        if (g == gt0 && nq >= 2 && !mbar_wait(&bar[SB_OE + ob], ((nq >> 1) - 1) & 1, abort_flag))
                            return false;
                        tc_fence_after();
                        const bool first = g - gt0 < 2;   // this parity's first tile of the item
#pragma unroll
                        for (int kk = 0; kk < kSpBN / 16; ++kk) {
                            const uint64_t da = smem_desc(aV + vs * SM::KV_BYTES + kk * 16 * 128,
                                                          kSpBN * 128, 1024, 2);
                            const uint64_t db = smem_desc(aP + pb * SM::P_STRIDE + kk * 16 * RB, 16, 8 * RB,
                                                          PLAYOUT);
                            mma_bf16_ss(tmem + TM_O0 + (ob * 2 + pb) * NH, da, db, idesc_pv,
                                        (first && kk == 0) ? 0u : 1u);
                        }
                        mma_commit(&bar[SB_OD + pb]);
                        mma_commit(&bar[SB_VE + vs]);
                        trace_ev(trb, tn, 2, 2, w, (int)(g - gt0));
                        ++vc;
                        return true;
                    };
                    for (int ii = 0; ii < ntl; ++ii, ++gt) {
                        const uint32_t ks = kc % KS;
                        if (!mbar_wait(&bar[SB_KF + ks], (kc / KS) & 1, abort_flag) ||
                            (gt >= 2 && !mbar_wait(&bar[SB_SE + (gt & 1)], ((gt >> 1) - 1) & 1, abort_flag))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < kSpD / 16; ++kk) {
                            const uint64_t da = sw128_desc(aK + ks * SM::KV_BYTES + (kk >> 2) * kSpBN * 128 +
                                                               (kk & 3) * 32, 16, 1024);
                            const uint64_t db = sw128_desc(aQ + qb * SM::Q_BYTES + (kk >> 2) * NH * 128 +
                                                               (kk & 3) * 32, 16, 1024);
                            mma_bf16_ss(tmem + TM_S0 + (gt & 1) * NH, da, db, idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&bar[SB_SF + (gt & 1)]);
                        mma_commit(&bar[SB_KE + ks]);
                        trace_ev(trb, tn, 2, 1, w, ii);
                        ++kc;
                        if (ii == ntl - 1)
                            mma_commit(&bar[SB_QE + qb]);
                        if (ii >= 2 && !issue_pv_pp(gt - 2)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!ok)
                        break;
                    if (ntl == 0)
                        mma_commit(&bar[SB_QE + qb]);
                    for (int jj = ntl >= 2 ? ntl - 2 : 0; ok && jj < ntl; ++jj)
                        ok = issue_pv_pp(gt0 + (uint32_t)jj);
                    if (!ok)
                        break;
                    continue;
                }
                for (int ii = 0; ii < ntl; ++ii, ++gt) {
                    const int i = tb + ii;
                    const uint32_t ks = kc % KS;
                    if (!mbar_wait(&bar[SB_KF + ks], (kc / KS) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kSpD / 16; ++kk) {
                        const uint64_t da = sw128_desc(aK + ks * SM::KV_BYTES + (kk >> 2) * kSpBN * 128 +
                                                           (kk & 3) * 32, 16, 1024);
                        const uint64_t db = sw128_desc(aQ + qb * SM::Q_BYTES + (kk >> 2) * NH * 128 +
                                                           (kk & 3) * 32, 16, 1024);
                        mma_bf16_ss(tmem + TM_S0 + (gt & 1) * NH, da, db, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&bar[SB_SF + (gt & 1)]);
                    mma_commit(&bar[SB_KE + ks]);
                    trace_ev(trb, tn, 2, 1, w, i);
                    ++kc;
                    if (ii == ntl - 1)
                        mma_commit(&bar[SB_QE + qb]);
                    if (ii > 0 && !issue_pv(ii == 1)) {
                        ok = false;
                        break;
                    }
                }
                if (!ok)
                    break;
                if (ntl == 0) {
                    mma_commit(&bar[SB_QE + qb]);
                } else if (!issue_pv(ntl == 1)) {
                    ok = false;
                    break;
                }
            }
            mma_commit(&bar[SB_DONE]);
            drain_wait(&bar[SB_DONE], 0);
        }
    } else if constexpr (SpRoles<NH>::PP) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(SpRoles<NH>::PP_SOFTMAX_REGS));
        // ================= ping-pong softmax + epilogue (32-head groups) =================
        // Warpgroup wg takes the tiles of global parity wg: thread = key lane of
        // the tile, all NH heads, with its own running maxima (sMref[wg][mb]),
        // partial sums and O^T accumulator (TMEM O^T[ob][wg]).  An item ends with
        // the two partial softmaxes combined per head:
        //   M = max(m0, m1), a_w = 2^(m_w - M), o = (a0 O0 + a1 O1) / (a0 l0 + a1 l1).
        using HD = SpHeads<NH>;
        constexpr int SMT = SpRoles<NH>::SMT;
        constexpr int HH = NH / 2;                     // heads each warpgroup writes out
        constexpr uint32_t BAR_ALL = 4;                // named barrier over both warpgroups
        const int wg = warp >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;                // key lane (S^T) / d lane (O^T)
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const bool head_owner = (lane % HD::LPH) == 0;
        const uint32_t barw = 1u + 2u * (uint32_t)wg;  // this warpgroup's named barrier
        float *sRedW = sRed + wg * NH * 4;
        float *sMrefW = sMref + wg * 2 * NH;
        const float4 *red4W = reinterpret_cast<const float4 *>(sRedW);
        float *sXch = reinterpret_cast<float *>(smem + SM::OFF_PPX);   // [wg][max | sum][NH]
        float *sCmb = reinterpret_cast<float *>(smem + SM::OFF_CMB);   // [2][NH]
        const uint32_t prow = smem_u32(sP) + r * RB;
        uint32_t pphys[NH / 8];
#pragma unroll
        for (int cl = 0; cl < NH / 8; ++cl) {
            const uint32_t c = (uint32_t)cl;
            const uint32_t ph = RB == 128 ? (c ^ (r & 7)) : (RB == 64 ? (c ^ ((r >> 1) & 3)) : (c ^ ((r >> 2) & 1)));
            pphys[cl] = ph * 16u;
        }
        const bool trace0 = trb != nullptr && threadIdx.x == 0;
        const float sl = p.scale_log2;
        // x[h] = s[h] scale - m[h] against this warpgroup's current reference
        auto exps_pp = [&](const float (&sr)[NH], float (&x)[NH], const float *mref) {
#pragma unroll
            for (int h = 0; h < NH; h += 4) {
                const float4 m4 = *reinterpret_cast<const float4 *>(mref + h);
                f2_split(fma_f2(f2(sr[h], sr[h + 1]), f2(sl, sl), f2(-m4.x, -m4.y)), x[h], x[h + 1]);
                f2_split(fma_f2(f2(sr[h + 2], sr[h + 3]), f2(sl, sl), f2(-m4.z, -m4.w)), x[h + 2], x[h + 3]);
            }
        };
        uint32_t nq = 0, gt = 0, mb = 0;
        bool ok = true;
        for (long long w = w0; w < p.n_items; w += wstep, ++nq) {
            if (!bar_all_id(BAR_ALL, SMT, ok && !*abort_flag))
                break;
            const SparseTok k = sparse_tok(p, w);
            const int nt = k.nct + k.nrt;
            const int ob = nq & 1;
            const int *sSel = sIdx + ob * p.tsel;
            ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_IF + ob], (nq >> 1) & 1, abort_flag));
            uint64_t lp2[NH / 2];
#pragma unroll
            for (int h = 0; h < NH / 2; ++h)
                lp2[h] = f2(0.f, 0.f);
            bool first = true;
            uint32_t glast = 0;
            for (int i = 0; i < nt; ++i, ++gt) {
                if ((int)(gt & 1) != wg)
                    continue;              // the other warpgroup's tile
                const uint32_t sb = gt & 1;
                ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_SF + sb], (gt >> 1) & 1, abort_flag));
                const bool valid = i < k.nct ? sSel[i * kSpBN + r] >= 0
                                             : k.rlo + (i - k.nct) * kSpBN + r <= k.rhi;
                tc_fence_after();
                float x[NH];
                bool need = first;         // a warpgroup's first tile of an item sets its reference
                {
                    float sr[NH];
                    tmem_ld_cols<NH>(tl + TM_S0 + sb * NH, sr);
                    tmem_ld_wait();
                    if (!need)
                        exps_pp(sr, x, sMrefW + mb * NH);
                }
                if (trace0)
                    trace_ev(trb, tn, 3, 1, w, i);
                if (!need) {
                    bool exceed = false;
#pragma unroll
                    for (int h = 0; h < NH; ++h)
                        exceed |= x[h] > 8.f;
                    need = bar_any_id(barw, 128, valid && exceed);
                }
                if (need) {
                    float sc[NH];
                    tmem_ld_cols<NH>(tl + TM_S0 + sb * NH, sc);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < NH; ++h)
                        sc[h] = valid ? sc[h] * sl : -INFINITY;
                    warp_reduce_heads<NH, true>(sc, lane);
                    if (head_owner) {
#pragma unroll
                        for (int e = 0; e < HD::VPL; ++e)
                            sRedW[HD::head(lane, e) * 4 + quad] = sc[e];
                    }
                    bar_sync_id(barw, 128);
                    const float *mold = sMrefW + mb * NH;
                    bool moved = false;
                    if (!first) {
#pragma unroll
                        for (int h = 0; h < NH; h += 2) {
                            const float o0 = mold[h], o1 = mold[h + 1];
                            const float a0 = sp_factor(o0, sp_new_ref(red4W[h], o0));
                            const float a1 = sp_factor(o1, sp_new_ref(red4W[h + 1], o1));
                            moved |= (a0 != 1.f) | (a1 != 1.f);
                            lp2[h >> 1] = fma_f2(lp2[h >> 1], f2(a0, a1), f2(0.f, 0.f));
                        }
                    }
                    if (moved) {
                        // O^T[ob][wg] holds this warpgroup's earlier PVs of the item;
                        // the last of them is the PV of tile gt - 2
                        ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_OD + sb], ((gt >> 1) - 1) & 1, abort_flag));
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < NH; c += 16) {
                            float ov[16];
                            tmem_ld_cols<16>(tl + TM_O0 + (ob * 2 + wg) * NH + c, ov);
                            tmem_ld_wait();
#pragma unroll
                            for (int q = 0; q < 16; ++q) {
                                const float old = mold[c + q];
                                ov[q] *= sp_factor(old, sp_new_ref(red4W[c + q], old));
                            }
                            tmem_st_cols<16>(tl + TM_O0 + (ob * 2 + wg) * NH + c, ov);
                        }
                        tmem_st_wait();
                    }
                    if (r < NH)
                        sMrefW[(mb ^ 1) * NH + r] = sp_new_ref(red4W[r], mold[r]);
                    bar_sync_id(barw, 128);
                    mb ^= 1;
                    float sr[NH];
                    tmem_ld_cols<NH>(tl + TM_S0 + sb * NH, sr);
                    tmem_ld_wait();
                    exps_pp(sr, x, sMrefW + mb * NH);
                }
                // the scores are in registers: the MMA may refill this S^T buffer
                tc_fence_before();
                mbar_arrive(&bar[SB_SE + sb]);
                uint32_t pk[NH / 2];
                if (valid) {
#pragma unroll
                    for (int h = 0; h < NH; h += 2) {
                        const float e0 = ex2_approx(x[h]), e1 = ex2_approx(x[h + 1]);
                        lp2[h >> 1] = add_f2(lp2[h >> 1], f2(e0, e1));
                        pk[h >> 1] = pack_bf16x2(e0, e1);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < NH / 2; ++h)
                        pk[h] = 0u;
                }
                // P^T buffer sb is free once the PV of tile gt - 2 completed
                if (gt >= 2)
                    ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_OD + sb], ((gt >> 1) - 1) & 1, abort_flag));
                const uint32_t prow_b = prow + sb * SM::P_STRIDE;
#pragma unroll
                for (int cl = 0; cl < NH / 8; ++cl)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow_b + pphys[cl]),
                                 "r"(pk[4 * cl]), "r"(pk[4 * cl + 1]), "r"(pk[4 * cl + 2]), "r"(pk[4 * cl + 3])
                                 : "memory");
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[SB_PF + sb]);
                if (trace0)
                    trace_ev(trb, tn, 3, 2, w, i);
                first = false;
                glast = gt;
            }
            // ---- epilogue: each warpgroup's (max, sum) per head, then the combine ----
            if (trace0)
                trace_ev(trb, tn, 3, 3, w, nt);
            {
                float lpart[NH];
#pragma unroll
                for (int h = 0; h < NH; h += 2)
                    f2_split(lp2[h >> 1], lpart[h], lpart[h + 1]);
                warp_reduce_heads<NH, false>(lpart, lane);
                if (head_owner) {
#pragma unroll
                    for (int e = 0; e < HD::VPL; ++e)
                        sRedW[HD::head(lane, e) * 4 + quad] = lpart[e];
                }
            }
            if (!first) {
                // this warpgroup's last PV of the item has completed
                ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_OD + wg], (glast >> 1) & 1, abort_flag));
                tc_fence_after();
            }
            bar_sync_id(barw, 128);
            if (r < NH) {
                const float4 q4 = red4W[r];
                sXch[(wg * 2 + 0) * NH + r] = sMrefW[mb * NH + r];
                sXch[(wg * 2 + 1) * NH + r] = (q4.x + q4.y) + (q4.z + q4.w);
                sMrefW[(mb ^ 1) * NH + r] = -INFINITY;   // the next item's reference
            }
            bar_sync_id(BAR_ALL, SMT);
            mb ^= 1;
            float lse_v = -INFINITY;
            if (wg == 0 && r < NH) {
                const float m0 = sXch[r], l0 = sXch[NH + r], m1 = sXch[2 * NH + r], l1 = sXch[3 * NH + r];
                const float M = fmaxf(m0, m1);
                const float a0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - M);
                const float a1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - M);
                const float L = a0 * l0 + a1 * l1;
                const float inv = L > 0.f ? 1.f / L : 0.f;
                sCmb[r] = a0 * inv;
                sCmb[NH + r] = a1 * inv;
                lse_v = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
            }
            bar_sync_id(BAR_ALL, SMT);
            tc_fence_after();
            float o0[HH], o1[HH];
            tmem_ld_cols<HH>(tl + TM_O0 + (ob * 2 + 0) * NH + wg * HH, o0);
            tmem_ld_cols<HH>(tl + TM_O0 + (ob * 2 + 1) * NH + wg * HH, o1);
            tmem_ld_wait();
            if (ok) {
                const size_t obase = (((size_t)k.b * p.Lq + k.t) * p.Hq + (size_t)k.kvh * p.g) * kSpD;
#pragma unroll
                for (int h = 0; h < HH; ++h) {
                    const int hh = wg * HH + h;
                    const float f0 = sCmb[hh], f1 = sCmb[NH + hh];
                    // an accumulator a warpgroup did not touch in this item has factor 0
                    const float v = (f0 != 0.f ? o0[h] * f0 : 0.f) + (f1 != 0.f ? o1[h] * f1 : 0.f);
                    if (hh < p.g)
                        p.o[obase + (size_t)hh * kSpD + r] = __float2bfloat16_rn(v);
                }
                if (p.lse && wg == 0 && r < p.g)
                    p.lse[((size_t)k.b * p.Hq + (size_t)k.kvh * p.g + r) * p.Lq + k.t] = lse_v;
            }
            tc_fence_before();
            mbar_arrive(&bar[SB_OE + ob]);
            if (trace0)
                trace_ev(trb, tn, 3, 4, w, nt);
        }
    } else {
        // ========================== softmax + epilogue ==========================
        // HS warpgroups share the tile's keys (TMEM lanes) and split its heads
        // (TMEM columns): warpgroup x owns heads x NHW .. x NHW + NHW - 1.
        // The reference maxima live in shared memory in two buffers, sMref[mb]
        // current; a move writes the other buffer and flips mb after a barrier,
        // so readers of the old values never race the writers.  The softmax
        // threads agree once per item whether to go on; within an item every
        // thread takes the same named barriers (a failed wait clears `ok`).
        constexpr int NHW = SpRoles<NH>::NHW;
        constexpr int SMT = SpRoles<NH>::SMT;
        using HD = SpHeads<NHW>;
        const int hb = (warp >> 2) * NHW;            // first head of this warpgroup
        const int quad = warp & 3;
        const int r = quad * 32 + lane;              // key lane (S^T) / d lane (O^T)
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const bool head_owner = (lane % HD::LPH) == 0;
        uint32_t nq = 0, gt = 0, mb = 0;
        bool ok = true;
        const uint32_t prow = smem_u32(sP) + r * RB;
        // byte offsets of this thread's 16-byte chunks in its P^T row (swizzle matching NH)
        uint32_t pphys[NHW / 8];
#pragma unroll
        for (int cl = 0; cl < NHW / 8; ++cl) {
            const uint32_t c = (uint32_t)(hb / 8 + cl);
            const uint32_t ph = RB == 128 ? (c ^ (r & 7)) : (RB == 64 ? (c ^ ((r >> 1) & 3)) : (c ^ ((r >> 2) & 1)));
            pphys[cl] = ph * 16u;
        }
        const bool trace0 = trb != nullptr && threadIdx.x == 0;
        const float4 *red4 = reinterpret_cast<const float4 *>(sRed);
        float *sPml = reinterpret_cast<float *>(smem + SM::OFF_PML);   // split: peer's [max | sum]
        float *sCmb = reinterpret_cast<float *>(smem + SM::OFF_CMB);   // split: [2][NH]
        for (long long w = w0; w < p.n_items; w += wstep, ++nq) {
            if (!sm_all<SMT>(ok && !*abort_flag))
                break;
            const SparseTok k = sparse_tok(p, w);
            const int nt = k.nct + k.nrt;
            const int tb = tile_lo(nt), ntl = tile_hi(nt) - tb;   // this CTA's tiles
            const int ob = nq & 1;
            // the item's decoded selection (key validity of its compressed tiles)
            const int *sSel = sIdx + ob * p.tsel;
            ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_IF + ob], (nq >> 1) & 1, abort_flag));
            // partial row sums (packed pairs), the warpgroup's reference maxima
            // as -m and as raw-score thresholds (m + 8) / scale, kept in
            // registers and reloaded only when a tile moves them
            uint64_t lp2[NHW / 2];
#pragma unroll
            for (int h = 0; h < NHW / 2; ++h)
                lp2[h] = f2(0.f, 0.f);
            constexpr bool NM_REGS = NHW <= 16;     // -m in registers (else read from shared memory)
            float nm[NM_REGS ? NHW : 1];
            const float sl = p.scale_log2;
            // x[h] = s[h] scale - m[h]: the exponent of this key's P^T entry
            auto exps_of = [&](const float (&sr)[NHW], float (&x)[NHW]) {
#pragma unroll
                for (int h = 0; h < NHW; h += 4) {
                    float n0, n1, n2, n3;
                    if constexpr (NM_REGS) {
                        n0 = nm[h];
                        n1 = nm[h + 1];
                        n2 = nm[h + 2];
                        n3 = nm[h + 3];
                    } else {
                        const float4 m4 = *reinterpret_cast<const float4 *>(sMref + mb * NH + hb + h);
                        n0 = -m4.x;
                        n1 = -m4.y;
                        n2 = -m4.z;
                        n3 = -m4.w;
                    }
                    f2_split(fma_f2(f2(sr[h], sr[h + 1]), f2(sl, sl), f2(n0, n1)), x[h], x[h + 1]);
                    f2_split(fma_f2(f2(sr[h + 2], sr[h + 3]), f2(sl, sl), f2(n2, n3)), x[h + 2], x[h + 3]);
                }
            };
            // No global memory access inside this loop: a CTA barrier (the
            // votes below) waits for every outstanding access of its threads.
            for (int ii = 0; ii < ntl; ++ii, ++gt) {
                const int i = tb + ii;
                const uint32_t sb = gt & 1;
                ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_SF + sb], (gt >> 1) & 1, abort_flag));
                bool valid;
                if (i < k.nct) {
                    valid = sSel[i * kSpBN + r] >= 0;   // the table is padded with -1 to whole tiles
                } else {
                    valid = k.rlo + (i - k.nct) * kSpBN + r <= k.rhi;
                }
                tc_fence_after();
                float x[NHW];
                bool need = ii == 0;   // this CTA's first tile of an item always sets the reference
                {
                    float sr[NHW];                  // raw scores q . k of this key
                    tmem_ld_cols<NHW>(tl + TM_S0 + sb * NH + hb, sr);
                    tmem_ld_wait();
                    if (!need)
                        exps_of(sr, x);
                }
                if (trace0)
                    trace_ev(trb, tn, 3, 1, w, i);
                if (!need) {
                    bool exceed = false;
#pragma unroll
                    for (int h = 0; h < NHW; ++h)
                        exceed |= x[h] > 8.f;
                    need = sm_any<SMT>(valid && exceed);
                }
                if (need) {
                    // per-head max over the tile (scaled, masked keys -inf): warp
                    // halving, then the four quadrants' values through sRed [head][quadrant]
                    float sc[NHW];
                    tmem_ld_cols<NHW>(tl + TM_S0 + sb * NH + hb, sc);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < NHW; ++h)
                        sc[h] = valid ? sc[h] * sl : -INFINITY;
                    warp_reduce_heads<NHW, true>(sc, lane);
                    if (head_owner) {
#pragma unroll
                        for (int e = 0; e < HD::VPL; ++e)
                            sRed[(hb + HD::head(lane, e)) * 4 + quad] = sc[e];
                    }
                    sm_sync<SMT>();
                    const float *mold = sMref + mb * NH;
                    bool moved = false;
                    if (ii > 0) {
#pragma unroll
                        for (int h = 0; h < NHW; h += 2) {
                            const float o0 = mold[hb + h], o1 = mold[hb + h + 1];
                            const float a0 = sp_factor(o0, sp_new_ref(red4[hb + h], o0));
                            const float a1 = sp_factor(o1, sp_new_ref(red4[hb + h + 1], o1));
                            moved |= (a0 != 1.f) | (a1 != 1.f);
                            lp2[h >> 1] = fma_f2(lp2[h >> 1], f2(a0, a1), f2(0.f, 0.f));
                        }
                    }
                    if (moved) {
                        // O^T holds every earlier PV of this item: wait for the
                        // last one, then scale this warpgroup's columns
                        ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_OD + ((gt - 1) & 1)],
                                                                ((gt - 1) >> 1) & 1, abort_flag));
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < NHW; c += 16) {
                            float ov[16];
                            tmem_ld_cols<16>(tl + TM_O0 + ob * NH + hb + c, ov);
                            tmem_ld_wait();
#pragma unroll
                            for (int q = 0; q < 16; ++q) {
                                const float old = mold[hb + c + q];
                                ov[q] *= sp_factor(old, sp_new_ref(red4[hb + c + q], old));
                            }
                            tmem_st_cols<16>(tl + TM_O0 + ob * NH + hb + c, ov);
                        }
                        tmem_st_wait();
                    }
                    if (threadIdx.x < NH)
                        sMref[(mb ^ 1) * NH + threadIdx.x] =
                            sp_new_ref(red4[threadIdx.x], mold[threadIdx.x]);
                    sm_sync<SMT>();
                    mb ^= 1;
                    if constexpr (NM_REGS) {
#pragma unroll
                        for (int h = 0; h < NHW; ++h)
                            nm[h] = -sMref[mb * NH + hb + h];
                    }
                    // the exponents against the new reference
                    float sr[NHW];
                    tmem_ld_cols<NHW>(tl + TM_S0 + sb * NH + hb, sr);
                    tmem_ld_wait();
                    exps_of(sr, x);
                }
                // P^T row of this key: exp2(s scale - m), 0 for masked keys (a
                // visible key never meets m = -inf: it would have moved m)
                uint32_t pk[NHW / 2];
                if (valid) {
#pragma unroll
                    for (int h = 0; h < NHW; h += 2) {
                        const float e0 = ex2_approx(x[h]), e1 = ex2_approx(x[h + 1]);
                        lp2[h >> 1] = add_f2(lp2[h >> 1], f2(e0, e1));
                        pk[h >> 1] = pack_bf16x2(e0, e1);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < NHW / 2; ++h)
                        pk[h] = 0u;
                }
                // P^T buffer sb is free once the PV of tile gt - 2 completed
                if (gt >= 2)
                    ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_OD + sb], ((gt >> 1) - 1) & 1, abort_flag));
                const uint32_t prow_b = prow + sb * SM::P_STRIDE;
#pragma unroll
                for (int cl = 0; cl < NHW / 8; ++cl)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow_b + pphys[cl]),
                                 "r"(pk[4 * cl]), "r"(pk[4 * cl + 1]), "r"(pk[4 * cl + 2]), "r"(pk[4 * cl + 3])
                                 : "memory");
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[SB_PF + sb]);
                if (trace0)
                    trace_ev(trb, tn, 3, 2, w, i);
            }
            float lpart[NHW];
#pragma unroll
            for (int h = 0; h < NHW; h += 2)
                f2_split(lp2[h >> 1], lpart[h], lpart[h + 1]);
            // ---- epilogue: l[h] = sum over keys; o[h][d] = O^T[d][h] / l[h] ----
            if (trace0)
                trace_ev(trb, tn, 3, 3, w, nt);
            warp_reduce_heads<NHW, false>(lpart, lane);
            if (head_owner) {
#pragma unroll
                for (int e = 0; e < HD::VPL; ++e)
                    sRed[(hb + HD::head(lane, e)) * 4 + quad] = lpart[e];
            }
            const bool have_o = ntl > 0;
            if (have_o) {
                ok &= __all_sync(0xffffffffu, mbar_wait(&bar[SB_OD + ((gt - 1) & 1)], ((gt - 1) >> 1) & 1,
                                                        abort_flag));
                tc_fence_after();
            }
            sm_sync<SMT>();
            // thread h < NH (all in the first warpgroup) finishes head h.  With a
            // split item, rank 1 hands its unnormalised O^T and its (max, sum)
            // per head to rank 0 (into rank 0's P buffers, free once rank 0's
            // last PV of the item has completed), and rank 0 combines:
            //   M = max(m0, m1),  a_r = 2^(m_r - M),  L = a0 l0 + a1 l1,
            //   o = (a0 O0 + a1 O1) / L,  lse = (M + log2 L) ln 2.
            const int th = threadIdx.x;
            float lse_v = -INFINITY;
            if (split == 1) {
                if (th < NH) {
                    const float4 q4 = red4[th];
                    const float l = (q4.x + q4.y) + (q4.z + q4.w);
                    sInv[th] = l > 0.f ? 1.f / l : 0.f;
                    lse_v = l > 0.f ? (sMref[mb * NH + th] + log2f(l)) * 0.6931471805599453f : -INFINITY;
                    sMref[(mb ^ 1) * NH + th] = -INFINITY;   // the next item's reference
                }
            } else if (crank == 0) {
                if (th == 0)
                    mbar_arrive_remote(cluster_addr(&bar[SB_GO], 1));
                ok &= __all_sync(0xffffffffu, mbar_wait_cluster(&bar[SB_PFULL], nq & 1, abort_flag));
                if (th < NH) {
                    const float4 q4 = red4[th];
                    const float l0 = (q4.x + q4.y) + (q4.z + q4.w);
                    const float m0 = sMref[mb * NH + th];
                    const float m1 = sPml[th], l1 = sPml[NH + th];
                    const float M = fmaxf(m0, m1);
                    const float a0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - M);
                    const float a1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - M);
                    const float L = a0 * l0 + a1 * l1;
                    const float inv = L > 0.f ? 1.f / L : 0.f;
                    sCmb[th] = a0 * inv;
                    sCmb[NH + th] = a1 * inv;
                    lse_v = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
                    sMref[(mb ^ 1) * NH + th] = -INFINITY;
                }
            } else {
                if (th < NH) {
                    const float4 q4 = red4[th];
                    sCmb[th] = sMref[mb * NH + th];
                    sCmb[NH + th] = (q4.x + q4.y) + (q4.z + q4.w);
                    sMref[(mb ^ 1) * NH + th] = -INFINITY;
                }
            }
            sm_sync<SMT>();  // sRed / sMref read, sInv / sCmb written, next reference cleared
            mb ^= 1;
            float ov[NHW];
            if (have_o) {
                tmem_ld_cols<NHW>(tl + TM_O0 + ob * NH + hb, ov);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int h = 0; h < NHW; ++h)
                    ov[h] = 0.f;
            }
            const size_t obase = (((size_t)k.b * p.Lq + k.t) * p.Hq + (size_t)k.kvh * p.g) * kSpD;
            if (split > 1 && crank != 0) {
                // rank 1: wait until rank 0 takes the partial, then write it there
                ok &= __all_sync(0xffffffffu, mbar_wait_cluster(&bar[SB_GO], nq & 1, abort_flag));
                if (ok) {
                    const uint32_t part0 = cluster_addr(sP, 0);
#pragma unroll
                    for (int h = 0; h < NHW; ++h)
                        cluster_st_f32(part0 + (uint32_t)(((hb + h) * kSpD + r) * 4), ov[h]);
                    if (th < NH) {
                        cluster_st_f32(cluster_addr(sPml + th, 0), sCmb[th]);
                        cluster_st_f32(cluster_addr(sPml + NH + th, 0), sCmb[NH + th]);
                    }
                }
                mbar_arrive_remote(cluster_addr(&bar[SB_PFULL], 0));
            } else if (ok && split > 1) {
                // rank 0: combine with rank 1's partial ([head][d] fp32 in the P buffers)
                const float *part = reinterpret_cast<const float *>(sP);
#pragma unroll
                for (int h = 0; h < NHW; ++h) {
                    const int hh = hb + h;
                    if (hh < p.g)
                        p.o[obase + (size_t)hh * kSpD + r] =
                            __float2bfloat16_rn(ov[h] * sCmb[hh] + part[hh * kSpD + r] * sCmb[NH + hh]);
                }
                if (p.lse && th < p.g)
                    p.lse[((size_t)k.b * p.Hq + (size_t)k.kvh * p.g + th) * p.Lq + k.t] = lse_v;
            } else if (ok) {
                // global stores only after the last barrier of the item
                const float4 *inv4 = reinterpret_cast<const float4 *>(sInv + hb);
#pragma unroll
                for (int h = 0; h < NHW; h += 4) {
                    const float4 iv = inv4[h >> 2];
                    const float ivs[4] = {iv.x, iv.y, iv.z, iv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (hb + h + q < p.g)
                            p.o[obase + (size_t)(hb + h + q) * kSpD + r] = __float2bfloat16_rn(ov[h + q] * ivs[q]);
                }
                if (p.lse && th < p.g)
                    p.lse[((size_t)k.b * p.Hq + (size_t)k.kvh * p.g + th) * p.Lq + k.t] = lse_v;
            }
            tc_fence_before();
            mbar_arrive(&bar[SB_OE + ob]);
            if (trace0)
                trace_ev(trb, tn, 3, 4, w, nt);
        }
    }

    tc_fence_before();
    if (split > 1)
        cluster_sync_all();   // no CTA leaves while its peer may still touch its shared memory
    __syncthreads();
    if (warp == SpRoles<NH>::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[0], 256);
    }
}

// 3-D map over a [rows, heads, 128] bf16 view with a (64, 1, 128) box, 128-byte swizzle.
static bool make_map_3d_rows(CUtensorMap *map, const void *base, int heads, long long rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)kSpD, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)kSpD * 2, (cuuint64_t)kSpD * 2 * heads};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kSpBN};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D map over a [rows, 128] bf16 view with a (64, box_rows) box, 128-byte swizzle.
static bool make_map_2d(CUtensorMap *map, const void *base, long long rows, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)kSpD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kSpD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int NH>
static cudaError_t launch_csa_t(SparseParams p, const void *q, const void *kc, const void *vc,
                                const void *kr, const void *vr, cudaStream_t stream, int num_sms)
{
    using SM = SparseSmem<NH>;
    CUtensorMap mq, mkc, mvc, mkr, mvr;
    bool ok = make_map_2d(&mq, q, (long long)p.B * p.Lq * p.Hq, NH);
    const long long crow = p.pregathered ? (long long)p.B * p.Lq * p.topk * p.Hkv : (long long)p.B * p.Nc * p.Hkv;
    ok &= make_map_2d(&mkc, kc, crow, 1);
    ok &= make_map_2d(&mvc, vc, crow, 1);
    // raw rows [B Lkv, Hkv, 128] as (128, Hkv, B Lkv): one box = 64 channels of
    // 128 consecutive rows of one KV head (a window tile half)
    ok &= make_map_3d_rows(&mkr, kr, p.Hkv, (long long)p.B * p.Lkv);
    ok &= make_map_3d_rows(&mvr, vr, p.Hkv, (long long)p.B * p.Lkv);
    if (!ok)
        return cudaErrorInvalidValue;
    size_t smem = 1024 + SM::BASE_BYTES + (size_t)p.tsel * 8;
    auto kern = csa_attn_kernel<NH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    if constexpr (SpRoles<NH>::PP) {
        e = check_reg_split(kern, SpRoles<NH>::THREADS, SpRoles<NH>::SMT, SpRoles<NH>::PP_SOFTMAX_REGS,
                            SpRoles<NH>::PP_OTHER_REGS);
        if (e != cudaSuccess)
            return e;
    }
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, SpRoles<NH>::THREADS, smem);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        return cudaErrorLaunchOutOfResources;
    const long long slots = (long long)num_sms * per_sm;
    // Few items (decode): two CTAs, one cluster, share each item's key tiles,
    // so that twice as many SMs gather; otherwise one CTA per item.
    p.split = (!SpRoles<NH>::PP && p.n_items * 2 <= slots) ? 2 : 1;
    if (p.split == 1) {
        long long grid = slots < p.n_items ? slots : p.n_items;
        if (grid < 1)
            return cudaSuccess;
        return launch_pdl(kern, dim3((unsigned)grid), dim3(SpRoles<NH>::THREADS), smem, stream, mq, mkc, mvc, mkr,
                          mvr, p);
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_wait
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(SpRoles<NH>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int max_clusters = 0;
    cfg.gridDim = dim3(2 * (unsigned)p.n_items, 1, 1);
    e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
    if (e != cudaSuccess)
        return e;
    if (max_clusters < 1)
        return cudaErrorLaunchOutOfResources;
    const long long clusters = max_clusters < p.n_items ? max_clusters : p.n_items;
    cfg.gridDim = dim3(2 * (unsigned)clusters, 1, 1);
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, mq, mkc, mvc, mkr, mvr, p);
}

// CSA attention with per-token selections, head dim 128, Hq / Hkv <= 64.
cudaError_t launch_csa_attn(int B, int Lq, int Lkv, int Hq, int Hkv, int Nc, int m, int W, int topk,
                            float scale, const int32_t *q_pos, const int32_t *kv_pos0, const void *q,
                            const void *kc, const void *vc, const int32_t *idx, const void *kr,
                            const void *vr, void *o, float *lse, cudaStream_t stream, int num_sms,
                            int pregathered)
{
    SparseParams p;
    p.B = B;
    p.Lq = Lq;
    p.Lkv = Lkv;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.g = Hq / Hkv;
    p.Nc = Nc;
    p.m = m;
    p.W = W;
    p.topk = topk;
    p.NH = p.g <= 16 ? 16 : (p.g <= 32 ? 32 : 64);
    p.n_items = (long long)B * Lq * Hkv;
    if (p.n_items >= (1ll << 31) || (long long)B * Lkv >= (1ll << 31))
        return cudaErrorInvalidValue;
    p.pregathered = pregathered;
    p.split = 1;
    p.tsel = (topk + kSpBN - 1) / kSpBN * kSpBN;
    {
        // the rows a launch selects are spread over the caches: worth pulling
        // into L2 ahead of the copies only when the caches are far larger than L2
        const long long rows = pregathered ? (long long)B * Lq * topk * Hkv : (long long)B * Nc * Hkv;
        p.prefetch = rows * kSpD * 2 * 2 > (64ll << 20) ? 1 : 0;
    }
    if (pregathered && (long long)B * Lq * topk * Hkv >= (1ll << 31))
        return cudaErrorInvalidValue;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.q_pos = q_pos;
    p.kv_pos0 = kv_pos0;
    p.idx = idx;
    p.kc = static_cast<const __nv_bfloat16 *>(kc);
    p.vc = static_cast<const __nv_bfloat16 *>(vc);
    p.kr = static_cast<const __nv_bfloat16 *>(kr);
    p.vr = static_cast<const __nv_bfloat16 *>(vr);
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    if (p.NH == 16)
        return launch_csa_t<16>(p, q, kc, vc, kr, vr, stream, num_sms);
    if (p.NH == 32)
        return launch_csa_t<32>(p, q, kc, vc, kr, vr, stream, num_sms);
    return launch_csa_t<64>(p, q, kc, vc, kr, vr, stream, num_sms);
}

}  // namespace hyb

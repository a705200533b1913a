// backward_tc.cu -- tensor-core backward of the dense hybrid attention (HCA:
// every visible compressed entry, plus the raw window; "deepseek-v4" blog,
// section 1, HCA and SWA; gradients as the Tiny-R2 README's "Training" asks,
// with the forward's lse), for prefill problems with head dim 128.
//
// Per query row t of head h with key set S(t), P_j = exp(scale q.k_j - lse),
// dP_j = dO.v_j, D = dO.o, dS_j = P_j (dP_j - D):
//     dq = scale sum_j dS_j k_j,   dk_j = scale sum dS_j q,   dv_j = sum P_j dO.
// Each key's P only needs the row's lse, so compressed and raw keys are
// handled independently.  Three launches:
//   1. bwd_delta_kernel: D = dO.o per (b, t, h), written to column 0 of dq's
//      own row (b, t, h): launch 3 reads it there before it overwrites that
//      row, in the same thread block, so no other block ever needs it.
//   2. attn_bwd_kv_kernel: one work item per key tile (128 compressed entries
//      or 128 raw rows of one KV head) and a run of (query tile, head) units;
//      per unit S^T = K Q^T and dP^T = V dO^T into TMEM, then dV += P^T dO and
//      dK += dS^T Q with P^T / dS^T read from TMEM.  Raw key tiles take every
//      unit that sees them and store their rows; compressed key tiles are seen
//      by many query tiles, so their units are split over several items whose
//      partial sums are added with vector reductions (dkc / dvc zeroed first).
//   3. attn_bwd_q_kernel: one item per (query tile, head); per key tile S = Q K^T
//      and dP = dO V^T, then dQ += dS K with dS from TMEM; dq stored once per
//      row.
// P and dS enter the MMAs as bf16 (fp32 accumulation), like the forward's P:
// rounding them leaves ~2^-9 relative error per term, which keeps the
// gradients well inside the backward parity bounds (measured: worst case 0.41
// of the max-abs and 0.38 of the mean-abs bound).  kBtLo = true adds a second
// bf16 term lo = bf16(x - hi) per value (twice the P / dS MMAs and
// conversions) for ~16-bit operands.
//
// Timeline (hyb_trace_attach, CTA 0): the dK / dV kernel records roles 1
// (producer: 1 K / V issued, 2 a unit's Q / dO issued and its columns stored),
// 2 (MMA: 1 S^T and dP^T issued, 2 dV issued, 3 dK issued) and 3 (thread 0:
// 1 S^T seen, 2 P written, 3 dS written, 4 epilogue start, 5 epilogue end);
// the dQ kernel records role 0 (thread 0: 1 S seen, 3 dS written, 4 / 5 its
// epilogue), so one attached buffer holds both kernels' timelines.
//
// Gradient rows leave through a 2 KB staging area per softmax warp (16
// columns x 32 rows, 64-byte swizzle), so one store instruction writes eight
// rows' 64-byte segments.
//
// Roles (320 threads): warps 0-3 and 4-7 are two warpgroups that each own
// 64 of the 128 columns of S / dP (thread = TMEM lane = tile row), warp 8 is
// the TMA producer, lane 0 of warp 9 issues every tcgen05.mma.  TMEM: S
// (columns 0-127), dP (128-255), and the accumulators (dV 256-383 and dK
// 384-511, or dQ 256-383).  P (or dS) overwrites the columns it came from in
// 32-column chunks, hi pairs then (with kBtLo) lo pairs:
//     element c (0..127) -> hi column 32 (c / 32) + (c % 32) / 2, lo column + 16,
// so K-step kk of an MMA reads columns 32 (kk / 2) + 8 (kk % 2) (+ 16 for lo),
// and a chunk is written as soon as its 32 values are final.
#include "common.cuh"

namespace hyb {

constexpr int kBtThreads = 320;
constexpr int kBtTile = 128 * 128 * 2;     // one bf16 128 x 128 tile (32 KB)

struct BtParams {
    int B, L, Hq, Hkv, g, Nc, m, W;
    int nqt;            // ceil(L / 128): query tiles (q kernel)
    int nkt_c;          // ceil(Nc / 128): compressed key tiles
    int nkt_r;          // ceil(L / 128) raw key tiles, 0 without a window
    int chunk_qt;       // query tiles per compressed item (chunk c: tiles c chunk_qt ..)
    int max_chunks;     // ceil(nqt / chunk_qt)
    int nqw;            // query tiles per raw key tile
    int win_only;       // 1: raw (window) keys only -- the selected entries of a CSA problem are another pass's
    long long n_comp_items, n_items;
    float scale, scale_log2;
    const float *lse;               // [B, Hq, L], natural log
    const __nv_bfloat16 *o, *dout;  // [B, L, Hq, 128]
    float *dq;          // [B, L, Hq, 128]; launch 1 puts D of row (b, t, h) in its column 0
    float *dkc, *dvc;   // [B, Nc, Hkv, 128], reduced into
    float *dkr, *dvr;   // [B, L, Hkv, 128], stored
};

// smem layout shared by both kernels: six 32 KB tiles (1024-aligned), the
// barriers, the kv kernel's per-stage lse / D columns and a 2 KB staging
// area per softmax warp for coalesced gradient stores.
struct BtSmem {
    static constexpr int OFF_T0 = 0;                 // kv: K     q: Q
    static constexpr int OFF_T1 = kBtTile;           // kv: V     q: dO
    static constexpr int OFF_T2 = 2 * kBtTile;       // kv: Q[0]  q: K[0]
    static constexpr int OFF_T3 = 3 * kBtTile;       // kv: dO[0] q: V[0]
    static constexpr int OFF_T4 = 4 * kBtTile;       // kv: Q[1]  q: K[1]
    static constexpr int OFF_T5 = 5 * kBtTile;       // kv: dO[1] q: V[1]
    static constexpr int OFF_BAR = 6 * kBtTile;
    static constexpr int OFF_MISC = OFF_BAR + 32 * 8;
    static constexpr int OFF_COL = OFF_MISC + 16 * 4;   // kv: lse2[2][128], D[2][128]
    static constexpr int OFF_STAGE = OFF_COL + 4 * 128 * 4;   // 8 warps x 32 rows x 16 fp32
    static constexpr int BYTES = OFF_STAGE + 8 * 32 * 16 * 4;
};

enum {
    BT_KVF = 0, BT_KVE = 2, BT_QF = 4, BT_QE = 6, BT_SF = 8, BT_DPF = 9, BT_PF = 10, BT_DSF = 11,
    BT_OF = 12, BT_OE = 13, BT_DONE = 14
};

__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// Staged store of this warp's 32 rows x 16 consecutive fp32 columns: the
// thread's v[0..15] (times f) go to a 2 KB area of shared memory (16-byte
// chunks swizzled so that neither pass has bank conflicts), then every lane
// moves one 16-byte chunk per pass, so a store instruction covers eight rows'
// 64-byte segments instead of 32 rows' 16 bytes.  dst: the thread's row at
// these columns, or nullptr (row not written); red: add instead of store.
__device__ __forceinline__ void store_rows16(float *stage, const float *v, float *dst, float f, bool red)
{
    const int lane = threadIdx.x & 31;
    float4 *st4 = reinterpret_cast<float4 *>(stage);
#pragma unroll
    for (int c = 0; c < 4; ++c)
        st4[lane * 4 + (c ^ ((lane >> 1) & 3))] =
            make_float4(v[4 * c] * f, v[4 * c + 1] * f, v[4 * c + 2] * f, v[4 * c + 3] * f);
    __syncwarp();
    const unsigned long long mine = reinterpret_cast<unsigned long long>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = 8 * i + (lane >> 2), c = lane & 3;
        const float4 x = st4[r * 4 + (c ^ ((r >> 1) & 3))];
        float *d = reinterpret_cast<float *>(__shfl_sync(0xffffffffu, mine, r));
        if (d) {
            if (red)
                red_add_v4(d + 4 * c, x.x, x.y, x.z, x.w);
            else
                *reinterpret_cast<float4 *>(d + 4 * c) = x;
        }
    }
    __syncwarp();
}

// P and dS enter the MMAs as bf16 hi terms only (kBtLo false) or as hi + lo
// pairs (true): see the header.
constexpr bool kBtLo = false;

// Writes 32 fp32 values x[0..31] as a chunk of hi / lo bf16 pairs at TMEM
// column taddr: hi pairs (x[2i], x[2i+1]) in columns 0-15, lo pairs in 16-31.
__device__ __forceinline__ void tmem_st_hi_lo32(uint32_t taddr, const float *x)
{
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        hi[i] = *reinterpret_cast<const uint32_t *>(&h);
        if (kBtLo) {
            const float2 hf = __bfloat1622float2(h);
            lo[i] = pack_bf16x2(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
        }
    }
    tmem_st16(taddr, hi);
    if (kBtLo)
        tmem_st16(taddr + 16, lo);
}

// 16 consecutive 32-bit TMEM columns of this thread's lane, raw.
__device__ __forceinline__ void tmem_ld16u(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// 64 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64])
{
    tmem_ld32(taddr, *reinterpret_cast<float(*)[32]>(&v[0]));
    tmem_ld32(taddr + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
    tmem_ld_wait();
}

// 2 x 8 MMAs: D (+)= A_hi B + A_lo B, A in TMEM at column a_tmem (hi / lo
// chunks above), B a 128-row tile in shared memory read MN-major (rows = K
// index).  b_desc0: the tile's descriptor (LBO 16 KB, SBO 1 KB); the K steps
// advance its address field by 16 rows (2 KB) each, computed once per call so
// that the issuing thread spends a 64-bit add per MMA.
__device__ __forceinline__ void mma_hi_lo(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc0, uint32_t idesc,
                                          bool first)
{
#pragma unroll
    for (int part = 0; part < (kBtLo ? 2 : 1); ++part) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(d_tmem, a_tmem + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * part, b_desc0 + (uint64_t)(kk * 128),
                        idesc, (first && part == 0 && kk == 0) ? 0u : 1u);
    }
}

// 8 MMAs: D = A B^T over K = 128, both 128-row tiles K-major in shared memory
// (descriptors of the tiles' starts; K step kk moves 32 bytes inside the
// swizzle atom, and the second 64-channel half starts 16 KB on).
__device__ __forceinline__ void mma_nt(uint32_t d_tmem, uint64_t a_desc0, uint64_t b_desc0, uint32_t idesc)
{
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4);
        mma_bf16_ss(d_tmem, a_desc0 + off, b_desc0 + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// Descriptors of a 128-row bf16 tile at shared address a: K-major (A or B of
// mma_nt) and MN-major (B of mma_hi_lo).
__device__ __forceinline__ uint64_t tile_desc_k(uint32_t a) { return sw128_desc(a, 16, 1024); }
__device__ __forceinline__ uint64_t tile_desc_mn(uint32_t a) { return sw128_desc(a, 128 * 128, 1024); }

// ------------------------------------------------------------------ launch 1
// D of row r = (b, t, h): sum_c dO[r, c] o[r, c] (fp32 over the bf16 values),
// stored at dq[r, 0]; one warp per row.
__global__ void __launch_bounds__(256)
bwd_delta_kernel(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ dout, float *dq, int B,
                 int L, int Hq)
{
    const long long rows = (long long)B * L * Hq;
    const int lane = threadIdx.x & 31;
    for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
         r += ((long long)gridDim.x * blockDim.x) >> 5) {
        const uint2 a = *reinterpret_cast<const uint2 *>(o + r * 128 + lane * 4);
        const uint2 c = *reinterpret_cast<const uint2 *>(dout + r * 128 + lane * 4);
        const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&a.x));
        const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&a.y));
        const float2 c0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&c.x));
        const float2 c1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&c.y));
        float s = a0.x * c0.x + a0.y * c0.y + a1.x * c1.x + a1.y * c1.y;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0)
            dq[r * 128] = s;
    }
}

// ------------------------------------------------------------------ launch 2
struct BtKvItem {
    int b, kvh, row0;   // key tile: rows row0 .. row0 + 127 of the compressed or raw cache
    int tq0;            // first query of unit 0's tile; unit u: tq0 + 128 (u / g), head kvh g + u % g
    int u0, u1;         // this item's units [u0, u1)
    bool comp;
};

// Items: first every (b, kvh, chunk, compressed key tile), key tiles
// innermost: a chunk is the same run of 128-aligned query tiles for every key
// tile (the part each one sees), so the key tiles of a chunk run side by side
// and read the same Q / dO tiles through L2; an empty part is an empty item.
// Then every (b, kvh, raw key tile).
__device__ __forceinline__ BtKvItem bt_kv_item(const BtParams &p, long long w)
{
    // item counts and positions fit in 32 bits (the launcher checks)
    BtKvItem it;
    if (w < p.n_comp_items) {
        unsigned wu = (unsigned)w;
        const int kt = (int)(wu % (unsigned)p.nkt_c);
        wu /= (unsigned)p.nkt_c;
        const int chunk = (int)(wu % (unsigned)p.max_chunks);
        wu /= (unsigned)p.max_chunks;
        it.kvh = (int)(wu % (unsigned)p.Hkv);
        it.b = (int)(wu / (unsigned)p.Hkv);
        it.comp = true;
        it.row0 = kt * 128;
        // the first query that sees entry row0: (row0 + 1) m - 1 < t - W + 1
        const int tmin = (it.row0 + 1) * p.m - 1 + p.W;
        const int qt_first = tmin < p.L ? tmin / 128 : p.nqt;
        const int qa = max(qt_first, chunk * p.chunk_qt);
        const int qb = min(p.nqt, (chunk + 1) * p.chunk_qt);
        it.tq0 = qa * 128;
        it.u0 = 0;
        it.u1 = qb > qa ? (qb - qa) * p.g : 0;
    } else {
        unsigned wu = (unsigned)(w - p.n_comp_items);
        const int kt = (int)(wu % (unsigned)p.nkt_r);
        wu /= (unsigned)p.nkt_r;
        it.kvh = (int)(wu % (unsigned)p.Hkv);
        it.b = (int)(wu / (unsigned)p.Hkv);
        it.comp = false;
        it.row0 = kt * 128;
        it.tq0 = it.row0;   // raw row r is seen by queries r .. r + W - 1
        const int nq = min(p.nqw, (p.L - it.tq0 + 127) / 128);
        it.u0 = 0;
        it.u1 = nq * p.g;
    }
    return it;
}

__global__ void __launch_bounds__(kBtThreads, 1)
attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                   const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_vr,
                   const BtParams p)
{
    using SM = BtSmem;
    extern __shared__ __align__(1024) uint8_t bt_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(bt_smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sK = smem + SM::OFF_T0;
    uint8_t *sV = smem + SM::OFF_T1;
    // stage s of the Q / dO ring: T2 / T3 + 2 s tiles
    uint8_t *const sQ0 = smem + SM::OFF_T2;
    uint8_t *const sDO0 = smem + SM::OFF_T3;
    static_assert(SM::OFF_T4 - SM::OFF_T2 == 2 * kBtTile && SM::OFF_T5 - SM::OFF_T3 == 2 * kBtTile, "stage stride");
    float *sLse2 = reinterpret_cast<float *>(smem + SM::OFF_COL);         // [2][128]
    float *sDel = sLse2 + 2 * 128;                                        // [2][128]
    float *const sStage = reinterpret_cast<float *>(smem + SM::OFF_STAGE) + (threadIdx.x >> 5) * 512;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM::OFF_BAR);
    int *misc = reinterpret_cast<int *>(smem + SM::OFF_MISC);
    volatile int *abort_flag = misc + 1;
    unsigned long long *const trb = trace_buffer();   // timeline of CTA 0, when attached
    uint32_t tn = 0;                                  // this thread's trace records
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bar[BT_KVF], 1);
        mbar_init(&bar[BT_KVE], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[BT_QF + s], 33);   // the copies' expect_tx, then every producer lane
            mbar_init(&bar[BT_QE + s], 1);
        }
        mbar_init(&bar[BT_SF], 1);
        mbar_init(&bar[BT_DPF], 1);
        mbar_init(&bar[BT_PF], 256);
        mbar_init(&bar[BT_DSF], 256);
        mbar_init(&bar[BT_OF], 1);
        mbar_init(&bar[BT_OE], 256);
        mbar_init(&bar[BT_DONE], 1);
        mbar_fence_init();
        misc[1] = 0;
    }
    if (warp == 9)
        tmem_alloc(reinterpret_cast<uint32_t *>(&misc[0]), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 384;

    if (warp == 8) {
        // ================================ producer ================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_do);
        }
        uint32_t nk = 0, qc = 0;
        bool ok = true;
        for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
            const BtKvItem it = bt_kv_item(p, w);
            if (it.u0 >= it.u1)
                continue;
            if (nk > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar[BT_KVE], (nk - 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&bar[BT_KVF], 2 * kBtTile);
                for (int cb = 0; cb < 2; ++cb) {
                    tma_load_4d(sK + cb * 128 * 128, it.comp ? &tm_kc : &tm_kr, &bar[BT_KVF], cb * 64, it.kvh,
                                it.row0, it.b);
                    tma_load_4d(sV + cb * 128 * 128, it.comp ? &tm_vc : &tm_vr, &bar[BT_KVF], cb * 64, it.kvh,
                                it.row0, it.b);
                }
            }
            if (lane == 0)
                trace_ev(trb, tn, 1, 1, w, 0);
            ++nk;
            for (int u = it.u0; u < it.u1; ++u) {
                const uint32_t s = qc & 1;
                const int tq = it.tq0 + 128 * (u / p.g);
                const int h = it.kvh * p.g + u % p.g;
                // the unit's 128 columns, four per lane, loaded together before the
                // stage wait: lse in base-2 units (+inf: no keys, or past L) and D
                const size_t rowbase = ((size_t)it.b * p.Hq + h) * p.L;
                float lv[4], dv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int t = min(tq + lane * 4 + k, p.L - 1);
                    lv[k] = p.lse[rowbase + t];
                    dv[k] = p.dq[(((size_t)it.b * p.L + t) * p.Hq + h) * 128];
                }
                if (qc >= 2 &&
                    !__all_sync(0xffffffffu, mbar_wait(&bar[BT_QE + s], ((qc >> 1) - 1) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bar[BT_QF + s], 2 * kBtTile);
                    for (int cb = 0; cb < 2; ++cb) {
                        tma_load_4d(sQ0 + s * 2 * kBtTile + cb * 128 * 128, &tm_q, &bar[BT_QF + s], cb * 64, h, tq, it.b);
                        tma_load_4d(sDO0 + s * 2 * kBtTile + cb * 128 * 128, &tm_do, &bar[BT_QF + s], cb * 64, h, tq, it.b);
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int c = lane * 4 + k;
                    const bool in = tq + c < p.L;
                    sLse2[s * 128 + c] = !in || lv[k] == -INFINITY ? INFINITY : lv[k] * 1.4426950408889634f;
                    sDel[s * 128 + c] = in ? dv[k] : 0.f;
                }
                mbar_arrive(&bar[BT_QF + s]);
                if (lane == 0)
                    trace_ev(trb, tn, 1, 2, w, u);
                ++qc;
            }
        }
        // unwinding: wait for the last copies issued into every slot
        if (lane == 0) {
            if (nk > 0)
                drain_wait(&bar[BT_KVF], (nk - 1) & 1);
            for (uint32_t c = (qc > 2 ? qc - 2 : 0); c < qc; ++c)
                drain_wait(&bar[BT_QF + (c & 1)], (c >> 1) & 1);
        }
    } else if (warp == 9) {
        // ================================ MMA issue ================================
        if (lane == 0) {
            const uint32_t id_nt = idesc_bf16(128, 128, false, false);
            const uint32_t id_mn = idesc_bf16(128, 128, false, true);
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
            const uint32_t aQ0 = smem_u32(sQ0), aDO0 = smem_u32(sDO0);
            uint32_t nk = 0, qc = 0;
            bool ok = true;
            for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
                const BtKvItem it = bt_kv_item(p, w);
                if (it.u0 >= it.u1)
                    continue;
                if (!mbar_wait(&bar[BT_KVF], nk & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                for (int u = it.u0; u < it.u1; ++u) {
                    const uint32_t s = qc & 1;
                    if (!mbar_wait(&bar[BT_QF + s], (qc >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_nt(tmem + TM_S, tile_desc_k(aK), tile_desc_k(aQ0 + s * 2 * kBtTile), id_nt);       // S^T = K Q^T
                    mma_commit(&bar[BT_SF]);
                    mma_nt(tmem + TM_DP, tile_desc_k(aV), tile_desc_k(aDO0 + s * 2 * kBtTile), id_nt);     // dP^T = V dO^T
                    mma_commit(&bar[BT_DPF]);
                    trace_ev(trb, tn, 2, 1, w, u);
                    if (!mbar_wait(&bar[BT_PF], qc & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (u == it.u0 && nk > 0 && !mbar_wait(&bar[BT_OE], (nk - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_hi_lo(tmem + TM_DV, tmem + TM_S, tile_desc_mn(aDO0 + s * 2 * kBtTile), id_mn, u == it.u0);    // dV += P^T dO
                    trace_ev(trb, tn, 2, 2, w, u);
                    if (!mbar_wait(&bar[BT_DSF], qc & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_hi_lo(tmem + TM_DK, tmem + TM_DP, tile_desc_mn(aQ0 + s * 2 * kBtTile), id_mn, u == it.u0);    // dK += dS^T Q
                    mma_commit(&bar[BT_QE + s]);
                    trace_ev(trb, tn, 2, 3, w, u);
                    ++qc;
                }
                if (!ok)
                    break;
                mma_commit(&bar[BT_KVE]);
                mma_commit(&bar[BT_OF]);
                ++nk;
            }
            mma_commit(&bar[BT_DONE]);
            drain_wait(&bar[BT_DONE], 0);
        }
    } else {
        // ==================== P^T, dS^T and the dK / dV epilogue ====================
        const int wg = warp >> 2;            // this warpgroup's query columns: 64 wg .. 64 wg + 63
        const int quad = warp & 3;
        const int row = quad * 32 + lane;    // key row of the tile
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const bool tracer = threadIdx.x == 0;
        uint32_t nk = 0, qc = 0;
        bool ok = true;
        for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
            const BtKvItem it = bt_kv_item(p, w);
            if (it.u0 >= it.u1)
                continue;
            const int kr = it.row0 + row;
            // queries that see this key row: [t_lo, t_hi]
            bool valid;
            int t_lo, t_hi;
            if (it.comp) {
                valid = kr < p.Nc;
                t_lo = valid ? (kr + 1) * p.m - 1 + p.W : p.L;
                t_hi = p.L - 1;
            } else {
                valid = kr < p.L;
                t_lo = kr;
                t_hi = min(kr + p.W - 1, p.L - 1);
            }
            for (int u = it.u0; u < it.u1; ++u) {
                const uint32_t s = qc & 1;
                const int tq = it.tq0 + 128 * (u / p.g);
                const int c_lo = valid ? t_lo - tq - 64 * wg : 64;
                const int c_hi = valid ? t_hi - tq - 64 * wg : -1;
                if (!__all_sync(0xffffffffu, mbar_wait(&bar[BT_QF + s], (qc >> 1) & 1, abort_flag)) ||
                    !__all_sync(0xffffffffu, mbar_wait(&bar[BT_SF], qc & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (tracer)
                    trace_ev(trb, tn, 3, 1, w, u);
                float x[64];
                tmem_ld64(tl + TM_S + 64 * wg, x);
                const float4 *cl = reinterpret_cast<const float4 *>(sLse2 + s * 128 + 64 * wg);
                const float4 *cd = reinterpret_cast<const float4 *>(sDel + s * 128 + 64 * wg);
#pragma unroll
                for (int j = 0; j < 64; j += 4) {
                    const float4 l4 = cl[j >> 2];
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        x[j + e] = (j + e >= c_lo && j + e <= c_hi)
                                       ? ex2_approx(fmaf(x[j + e], p.scale_log2, -lv[e]))
                                       : 0.f;
                }
                tmem_st_hi_lo32(tl + TM_S + 64 * wg, &x[0]);
                tmem_st_hi_lo32(tl + TM_S + 64 * wg + 32, &x[32]);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bar[BT_PF]);
                if (tracer)
                    trace_ev(trb, tn, 3, 2, w, u);
                if (!__all_sync(0xffffffffu, mbar_wait(&bar[BT_DPF], qc & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // dS = P (dP - D) with P read back from TMEM (the bf16 values the
                // dV MMA uses), so P does not stay in registers across the wait
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float y[32];
                    uint32_t pk[16];
                    tmem_ld32(tl + TM_DP + 64 * wg + 32 * c, y);
                    tmem_ld16u(tl + TM_S + 64 * wg + 32 * c, pk);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 d4 = cd[(32 * c + j) >> 2];
                        const float2 p0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pk[j >> 1]));
                        const float2 p1 =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pk[(j >> 1) + 1]));
                        y[j] = p0.x * (y[j] - d4.x);
                        y[j + 1] = p0.y * (y[j + 1] - d4.y);
                        y[j + 2] = p1.x * (y[j + 2] - d4.z);
                        y[j + 3] = p1.y * (y[j + 3] - d4.w);
                    }
                    tmem_st_hi_lo32(tl + TM_DP + 64 * wg + 32 * c, y);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bar[BT_DSF]);
                if (tracer)
                    trace_ev(trb, tn, 3, 3, w, u);
                ++qc;
            }
            if (!ok)
                break;
            // epilogue: this warpgroup's 64 channels of dV and dK for key row kr
            if (!__all_sync(0xffffffffu, mbar_wait(&bar[BT_OF], nk & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (tracer)
                trace_ev(trb, tn, 3, 4, w, 0);
            float *dv_row, *dk_row;
            if (it.comp) {
                const size_t at = (((size_t)it.b * p.Nc + kr) * p.Hkv + it.kvh) * 128 + 64 * wg;
                dv_row = p.dvc + at;
                dk_row = p.dkc + at;
            } else {
                const size_t at = (((size_t)it.b * p.L + kr) * p.Hkv + it.kvh) * 128 + 64 * wg;
                dv_row = p.dvr + at;
                dk_row = p.dkr + at;
            }
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                // this half's 64 columns of dV, then of dK
                float z[64];
                tmem_ld64(tl + (part ? TM_DK : TM_DV) + 64 * wg, z);
                const float f = part ? p.scale : 1.f;
                float *dst = valid ? (part ? dk_row : dv_row) : nullptr;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    store_rows16(sStage, &z[16 * k], dst ? dst + 16 * k : nullptr, f, it.comp);
            }
            tc_fence_before();
            mbar_arrive(&bar[BT_OE]);
            if (tracer)
                trace_ev(trb, tn, 3, 5, w, 0);
            ++nk;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[0], 512);
    }
}

// ------------------------------------------------------------------ launch 3
struct BtQItem {
    int b, h, t0;       // query tile: tokens t0 .. t0 + 127 of head h
    int nct, nrt, rlo;  // compressed key tiles, raw key tiles, first raw row
};

__device__ __forceinline__ int bt_visible(int t, int m, int W, int Nc)
{
    const int a = t - W + 1;
    if (a <= 0)
        return 0;
    const int n = (int)((unsigned)a / (unsigned)m);
    return n < Nc ? n : Nc;
}

// Items longest first: the last query tiles see the most compressed entries.
__device__ __forceinline__ BtQItem bt_q_item(const BtParams &p, long long w)
{
    BtQItem it;
    const unsigned per_t = (unsigned)p.B * (unsigned)p.Hq;
    const unsigned wu = (unsigned)w;
    it.t0 = (p.nqt - 1 - (int)(wu / per_t)) * 128;
    const unsigned r = wu % per_t;
    it.b = (int)(r / (unsigned)p.Hq);
    it.h = (int)(r % (unsigned)p.Hq);
    const int tmax = min(it.t0 + 127, p.L - 1);
    it.nct = p.win_only ? 0 : (bt_visible(tmax, p.m, p.W, p.Nc) + 127) / 128;
    it.rlo = max(0, it.t0 - p.W + 1);
    it.nrt = p.W > 0 ? (tmax - it.rlo + 128) / 128 : 0;
    return it;
}

__global__ void __launch_bounds__(kBtThreads, 1)
attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                  const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_vr,
                  const BtParams p)
{
    using SM = BtSmem;
    extern __shared__ __align__(1024) uint8_t bt_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(bt_smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sQ = smem + SM::OFF_T0;
    uint8_t *sDO = smem + SM::OFF_T1;
    float *const sStage = reinterpret_cast<float *>(smem + SM::OFF_STAGE) + (threadIdx.x >> 5) * 512;
    // stage s of the K / V ring: T2 / T3 + 2 s tiles
    uint8_t *const sK0 = smem + SM::OFF_T2;
    uint8_t *const sV0 = smem + SM::OFF_T3;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM::OFF_BAR);
    int *misc = reinterpret_cast<int *>(smem + SM::OFF_MISC);
    volatile int *abort_flag = misc + 1;
    unsigned long long *const trb = trace_buffer();   // timeline of CTA 0, when attached
    uint32_t tn = 0;                                  // this thread's trace records
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // the barrier slots are reused: KVF / KVE hold the two K / V stages, QF / QE
    // the single Q / dO buffer (slot QF + 0, QE + 0)
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[BT_KVF + s], 1);
            mbar_init(&bar[BT_KVE + s], 1);
        }
        mbar_init(&bar[BT_QF], 1);
        mbar_init(&bar[BT_QE], 1);
        mbar_init(&bar[BT_SF], 1);
        mbar_init(&bar[BT_DPF], 1);
        mbar_init(&bar[BT_DSF], 256);
        mbar_init(&bar[BT_OF], 1);
        mbar_init(&bar[BT_OE], 256);
        mbar_init(&bar[BT_DONE], 1);
        mbar_fence_init();
        misc[1] = 0;
    }
    if (warp == 9)
        tmem_alloc(reinterpret_cast<uint32_t *>(&misc[0]), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256;

    if (warp == 8) {
        // ================================ producer ================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_kr);
            tma_prefetch_desc(&tm_vr);
            uint32_t ni = 0, kc = 0;
            bool ok = true;
            for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
                const BtQItem it = bt_q_item(p, w);
                const int nt = it.nct + it.nrt;
                if (nt == 0)
                    continue;
                const int kvh = it.h / p.g;
                if (ni > 0 && !mbar_wait(&bar[BT_QE], (ni - 1) & 1, abort_flag))
                    break;
                mbar_arrive_expect_tx(&bar[BT_QF], 2 * kBtTile);
                for (int cb = 0; cb < 2; ++cb) {
                    tma_load_4d(sQ + cb * 128 * 128, &tm_q, &bar[BT_QF], cb * 64, it.h, it.t0, it.b);
                    tma_load_4d(sDO + cb * 128 * 128, &tm_do, &bar[BT_QF], cb * 64, it.h, it.t0, it.b);
                }
                ++ni;
                for (int i = 0; i < nt; ++i) {
                    const bool comp = i < it.nct;
                    const int row0 = comp ? i * 128 : it.rlo + (i - it.nct) * 128;
                    const uint32_t s = kc & 1;
                    if (kc >= 2 && !mbar_wait(&bar[BT_KVE + s], ((kc >> 1) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar[BT_KVF + s], 2 * kBtTile);
                    for (int cb = 0; cb < 2; ++cb) {
                        tma_load_4d(sK0 + s * 2 * kBtTile + cb * 128 * 128, comp ? &tm_kc : &tm_kr, &bar[BT_KVF + s], cb * 64, kvh,
                                    row0, it.b);
                        tma_load_4d(sV0 + s * 2 * kBtTile + cb * 128 * 128, comp ? &tm_vc : &tm_vr, &bar[BT_KVF + s], cb * 64, kvh,
                                    row0, it.b);
                    }
                    ++kc;
                }
            }
            if (ni > 0)
                drain_wait(&bar[BT_QF], (ni - 1) & 1);
            for (uint32_t c = (kc > 2 ? kc - 2 : 0); c < kc; ++c)
                drain_wait(&bar[BT_KVF + (c & 1)], (c >> 1) & 1);
        }
    } else if (warp == 9) {
        // ================================ MMA issue ================================
        if (lane == 0) {
            const uint32_t id_nt = idesc_bf16(128, 128, false, false);
            const uint32_t id_mn = idesc_bf16(128, 128, false, true);
            const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO);
            const uint32_t aK0 = smem_u32(sK0), aV0 = smem_u32(sV0);
            uint32_t ni = 0, kc = 0;
            bool ok = true;
            for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
                const BtQItem it = bt_q_item(p, w);
                const int nt = it.nct + it.nrt;
                if (nt == 0)
                    continue;
                if (!mbar_wait(&bar[BT_QF], ni & 1, abort_flag))
                    break;
                for (int i = 0; i < nt; ++i) {
                    const uint32_t s = kc & 1;
                    if (!mbar_wait(&bar[BT_KVF + s], (kc >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_nt(tmem + TM_S, tile_desc_k(aQ), tile_desc_k(aK0 + s * 2 * kBtTile), id_nt);       // S = Q K^T
                    mma_commit(&bar[BT_SF]);
                    mma_nt(tmem + TM_DP, tile_desc_k(aDO), tile_desc_k(aV0 + s * 2 * kBtTile), id_nt);     // dP = dO V^T
                    mma_commit(&bar[BT_DPF]);
                    if (i == nt - 1)
                        mma_commit(&bar[BT_QE]);
                    if (!mbar_wait(&bar[BT_DSF], kc & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (i == 0 && ni > 0 && !mbar_wait(&bar[BT_OE], (ni - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_hi_lo(tmem + TM_DQ, tmem + TM_S, tile_desc_mn(aK0 + s * 2 * kBtTile), id_mn, i == 0);   // dQ += dS K
                    mma_commit(&bar[BT_KVE + s]);
                    ++kc;
                }
                if (!ok)
                    break;
                mma_commit(&bar[BT_OF]);
                ++ni;
            }
            mma_commit(&bar[BT_DONE]);
            drain_wait(&bar[BT_DONE], 0);
        }
    } else {
        // ========================= dS and the dQ epilogue =========================
        const int wg = warp >> 2;            // this warpgroup's key columns: 64 wg .. 64 wg + 63
        const int quad = warp & 3;
        const int row = quad * 32 + lane;    // query row of the tile
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const bool tracer = threadIdx.x == 0;
        uint32_t ni = 0, kc = 0;
        bool ok = true;
        for (long long w = blockIdx.x; ok && w < p.n_items; w += gridDim.x) {
            const BtQItem it = bt_q_item(p, w);
            const int nt = it.nct + it.nrt;
            const int t = it.t0 + row;
            const bool valid_row = t < p.L;
            float *dq_row = p.dq + (((size_t)it.b * p.L + t) * p.Hq + it.h) * 128 + 64 * wg;
            if (nt == 0) {
                if (valid_row)
                    for (int j = 0; j < 64; j += 4)
                        *reinterpret_cast<float4 *>(dq_row + j) = make_float4(0.f, 0.f, 0.f, 0.f);
                continue;
            }
            // the row's lse (base 2) and D = dO . o (launch 1 left it in column 0 of dq's row)
            float lse2 = INFINITY, Drow = 0.f;
            if (valid_row) {
                const float l = p.lse[((size_t)it.b * p.Hq + it.h) * p.L + t];
                lse2 = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
                Drow = dq_row[-64 * wg];
            }
            const int nv = valid_row ? bt_visible(t, p.m, p.W, p.Nc) : 0;
            const int wlo = t - p.W + 1;
            for (int i = 0; i < nt; ++i) {
                // valid key columns c_lo .. c_hi of this tile for this row
                int c_lo, c_hi;
                if (i < it.nct) {
                    c_lo = 0;
                    c_hi = nv - 1 - i * 128;
                } else {
                    const int base = it.rlo + (i - it.nct) * 128;
                    c_lo = wlo - base;
                    c_hi = t - base;
                }
                if (!valid_row) {
                    c_lo = 128;
                    c_hi = -1;
                }
                c_lo -= 64 * wg;
                c_hi -= 64 * wg;
                if (!__all_sync(0xffffffffu, mbar_wait(&bar[BT_SF], kc & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (tracer)
                    trace_ev(trb, tn, 0, 1, w, i);
                float x[64];
                tmem_ld64(tl + TM_S + 64 * wg, x);
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    x[j] = (j >= c_lo && j <= c_hi) ? ex2_approx(fmaf(x[j], p.scale_log2, -lse2)) : 0.f;
                if (!__all_sync(0xffffffffu, mbar_wait(&bar[BT_DPF], kc & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float y[32];
                    tmem_ld32(tl + TM_DP + 64 * wg + 32 * c, y);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        y[j] = x[32 * c + j] * (y[j] - Drow);
                    tmem_st_hi_lo32(tl + TM_S + 64 * wg + 32 * c, y);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bar[BT_DSF]);
                if (tracer)
                    trace_ev(trb, tn, 0, 3, w, i);
                ++kc;
            }
            if (!ok)
                break;
            if (!__all_sync(0xffffffffu, mbar_wait(&bar[BT_OF], ni & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (tracer)
                trace_ev(trb, tn, 0, 4, w, 0);
            float z[64];
            tmem_ld64(tl + TM_DQ + 64 * wg, z);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                store_rows16(sStage, &z[16 * k], valid_row ? dq_row + 16 * k : nullptr, p.scale, false);
            tc_fence_before();
            mbar_arrive(&bar[BT_OE]);
            if (tracer)
                trace_ev(trb, tn, 0, 5, w, 0);
            ++ni;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[0], 512);
    }
}

// Does the tensor-core backward take this problem?  Dense (no selection),
// head dim 128, prefill positions (query t at position t, raw row r at r,
// Lq == Lkv), positions in 32 bits.
static bool attn_bwd_tc_ok(bool has_idx, int d, const int32_t *q_pos, const int32_t *kv_pos0, int Lq, int Lkv,
                           int Nc, int m, int W)
{
    return !has_idx && d == 128 && !q_pos && !kv_pos0 && Lq == Lkv && Lq > 0 && m >= 1 && W >= 0 &&
           (long long)Lq + W < (1LL << 30) && ((long long)Nc + 128) * m + W < (1LL << 30);
}

// CSA prefill problems with d = 128 and a window: the tensor-core passes take
// the window keys (win_only), the CUDA-core pass the selected entries.
static bool attn_bwd_tc_window_ok(int d, const int32_t *q_pos, const int32_t *kv_pos0, int Lq, int Lkv, int W)
{
    return d == 128 && !q_pos && !kv_pos0 && Lq == Lkv && Lq > 0 && W > 0 && (long long)Lq + W < (1LL << 30);
}

// Zeroes dkc / dvc (reduced into), and dk_raw / dv_raw without a window (no
// raw item stores them), then runs the three launches.  win_only: raw keys
// only (no compressed item, no compressed tile in the dq pass).
static cudaError_t launch_attn_bwd_tc(int B, int L, int Hq, int Hkv, int Nc, int m, int W, float scale,
                                      const void *q, const void *kc, const void *vc, const void *kr,
                                      const void *vr, const void *o, const float *lse, const void *dout,
                                      float *dq, float *dkc, float *dvc, float *dkr, float *dvr,
                                      cudaStream_t stream, int num_sms, bool win_only = false)
{
    BtParams p;
    p.B = B;
    p.L = L;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.g = Hq / Hkv;
    p.Nc = Nc;
    p.m = m;
    p.W = W;
    p.nqt = (L + 127) / 128;
    p.win_only = win_only ? 1 : 0;
    p.nkt_c = (Nc > 0 && !win_only) ? (Nc + 127) / 128 : 0;
    p.nkt_r = W > 0 ? (L + 127) / 128 : 0;
    p.nqw = (127 + W + 127) / 128;
    // compressed units (query tile, head) per key tile; key tile 0 has the most
    long long total_cu = 0, units0 = 0;
    for (int kt = 0; kt < p.nkt_c; ++kt) {
        const long long tmin = (long long)(kt * 128 + 1) * m - 1 + W;
        const long long u = tmin < L ? ((L - tmin + 127) / 128) * p.g : 0;
        if (kt == 0)
            units0 = u;
        total_cu += u;
    }
    total_cu *= (long long)B * Hkv;
    // about four compressed items per SM (they are the long ones), at least
    // four units each
    long long chunk = (total_cu + 4LL * num_sms - 1) / (4LL * num_sms);
    if (chunk < 4)
        chunk = 4;
    p.chunk_qt = (int)((chunk + p.g - 1) / p.g);
    p.max_chunks = (p.nqt + p.chunk_qt - 1) / p.chunk_qt;
    p.n_comp_items = units0 > 0 ? (long long)B * Hkv * p.nkt_c * p.max_chunks : 0;
    p.n_items = p.n_comp_items + (long long)B * Hkv * p.nkt_r;
    const long long n_q_items = (long long)p.nqt * B * Hq;
    if (p.n_items >= (1LL << 31) || n_q_items >= (1LL << 31))
        return cudaErrorInvalidValue;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.lse = lse;
    p.o = static_cast<const __nv_bfloat16 *>(o);
    p.dout = static_cast<const __nv_bfloat16 *>(dout);
    p.dq = dq;
    p.dkc = dkc;
    p.dvc = dvc;
    p.dkr = dkr;
    p.dvr = dvr;

    cudaError_t e = cudaSuccess;
    const size_t ck = (size_t)B * Nc * Hkv * 128 * sizeof(float);
    if (ck) {
        e = cudaMemsetAsync(dkc, 0, ck, stream);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(dvc, 0, ck, stream);
    }
    if (e == cudaSuccess && W == 0) {
        const size_t rk = (size_t)B * L * Hkv * 128 * sizeof(float);
        e = cudaMemsetAsync(dkr, 0, rk, stream);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(dvr, 0, rk, stream);
    }
    if (e != cudaSuccess)
        return e;

    CUtensorMap mq, mdo, mkc, mvc, mkr, mvr;
    const int Nc1 = Nc > 0 ? Nc : 1;
    bool ok = make_map(&mq, q, 128, Hq, L, B, 1, 128);
    ok &= make_map(&mdo, dout, 128, Hq, L, B, 1, 128);
    ok &= make_map(&mkc, kc ? kc : q, 128, Hkv, Nc1, B, 1, 128);
    ok &= make_map(&mvc, vc ? vc : q, 128, Hkv, Nc1, B, 1, 128);
    ok &= make_map(&mkr, kr, 128, Hkv, L, B, 1, 128);
    ok &= make_map(&mvr, vr, 128, Hkv, L, B, 1, 128);
    if (!ok)
        return cudaErrorInvalidValue;

    const long long rows = (long long)B * L * Hq;
    long long dgrid = (rows + 7) / 8;
    if (dgrid > 16LL * num_sms)
        dgrid = 16LL * num_sms;
    bwd_delta_kernel<<<(unsigned)dgrid, 256, 0, stream>>>(p.o, p.dout, dq, B, L, Hq);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;

    const size_t smem = 1024 + BtSmem::BYTES;
    e = cudaFuncSetAttribute(attn_bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attn_bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    if (p.n_items > 0) {
        const long long grid = p.n_items < num_sms ? p.n_items : num_sms;
        attn_bwd_kv_kernel<<<(unsigned)grid, kBtThreads, smem, stream>>>(mq, mdo, mkc, mvc, mkr, mvr, p);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    p.n_items = n_q_items;
    const long long grid = n_q_items < num_sms ? n_q_items : num_sms;
    attn_bwd_q_kernel<<<(unsigned)grid, kBtThreads, smem, stream>>>(mq, mdo, mkc, mvc, mkr, mvr, p);
    return cudaGetLastError();
}

}  // namespace hyb

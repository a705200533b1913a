// index_tc.cu -- lightning-indexer scores on tcgen05 for prefill ("deepseek-v4"
// blog, section 1, CSA; score = ReLU-weighted head sum, fp32):
//     I[t, s] = sum_h wi[t, h] * max(0, qi[t, h, :] . kic[s, :])
// A CTA owns 128 query tokens and a run of 64-entry key tiles.  For every key
// tile one MMA per indexer head writes D_h[128 tokens x 64 keys] (fp32) into
// TMEM (two buffers of Hi x 64 columns); the epilogue thread of a token reads
// the Hi accumulators of its row, forms the weighted ReLU sum and stores the
// visible part of the tile into the token's score row.  Queries (one TMA box
// per head) stay in shared memory; key tiles stream through a 4-stage ring.
// Indexer dims 64 (rows of 128 bytes, 128-byte swizzle) and 32 (64-byte rows
// and swizzle): the MMA takes di / 16 steps of K = 16.
// When a score row is a multiple of 16 bytes the epilogue stages each 128 x 32
// block of scores in shared memory (128-byte swizzle) and one thread writes it
// with a TMA tensor store, so the rows leave as whole 128-byte lines instead of
// 32 scattered 16-byte pieces per warp instruction (columns past a row's
// visible prefix are written too; readers only use the prefix).
// Roles (256 threads): warp 0 TMA producer, warp 1 TMEM + MMA, warps 4-7
// epilogue (TMEM lane quadrants 0-3); warps 2-3 idle.
#include <cstring>

#include "common.cuh"

namespace hyb {

constexpr int kIxThreads = 256;
constexpr int kIxBM = 128;        // query tokens per CTA
constexpr int kIxBN = 64;         // keys per tile
constexpr int kIxStages = 4;
static_assert(kIxStages == 4, "the prefill score kernel's barrier map (1-4 K full, 5-8 K empty) is written for four stages");
constexpr int kIxDi = 64;         // indexer dim of the decode form
constexpr int kIxChunkTiles = 32; // key tiles per CTA (2048 entries)

struct IndexParams {
    int B, Lq, Hi, Nc, m, W;
    int n_ttiles, n_chunks;       // token tiles, key chunks per token tile
    int tma_store;                // 1: scores leave through the staged TMA store
    const int32_t *q_pos;
    const float *wi;              // [B, Lq, Hi]
    float *scores;                // [B * Lq, Nc]
};

template <int HI, int DI>
struct IxSmem {
    static constexpr int Q_BYTES = kIxBM * DI * 2;        // one head
    static constexpr int K_BYTES = kIxBN * DI * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = HI * Q_BYTES;
    static constexpr int OFF_BAR = OFF_K + kIxStages * K_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + 16 * 8;
    static constexpr int OFF_ST = (OFF_MISC + 16 * 4 + 1023) & ~1023;  // 2 x [128][32] fp32 staging
    static constexpr int ST_BYTES = kIxBM * 32 * 4;
    static constexpr int BYTES = OFF_ST + 2 * ST_BYTES;
};

// TMA tensor store of one staged box (3-D map), as one bulk async-group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int c0, int c1, int c2)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand whose rows are DI bf16
// (128- or 64-byte swizzle; 8-row groups DI * 16 bytes apart).
template <int DI>
__device__ __forceinline__ uint64_t ix_desc(uint32_t saddr)
{
    static_assert(DI == 64 || DI == 32, "indexer dim 64 or 32");
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                               // leading byte offset (unused when swizzled)
    d |= (uint64_t)(((DI * 16) >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(DI == 64 ? 2u : 4u) << 61;            // 128- or 64-byte swizzle
    return d;
}

template <int HI, int DI>
__global__ void __launch_bounds__(kIxThreads, 1)
index_scores_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_s, const IndexParams p)
{
    using SM = IxSmem<HI, DI>;
    extern __shared__ __align__(1024) uint8_t ix_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(ix_smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sQ = smem + SM::OFF_Q;
    uint8_t *sK = smem + SM::OFF_K;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM::OFF_BAR);
    int *misc = reinterpret_cast<int *>(smem + SM::OFF_MISC);
    volatile int *abort_flag = misc + 1;
    // bars: 0 Q full, 1-4 K full, 5-8 K empty, 9-10 D full, 11-12 D empty, 13 done
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // heavy token tiles first
    const int ttile = p.n_ttiles - 1 - (int)(blockIdx.x / p.n_chunks);
    const int chunk = (int)(blockIdx.x % p.n_chunks);
    const int b = blockIdx.y;
    const int t0 = ttile * kIxBM;
    const int t_last = min(t0 + kIxBM - 1, p.Lq - 1);
    auto pos_of = [&](int t) -> long long { return p.q_pos ? p.q_pos[(size_t)b * p.Lq + t] : t; };
    long long pmax = -1;
    // positions may be arbitrary; the tile covers up to the largest one
    if (p.q_pos) {
        for (int t = t0; t <= t_last; ++t)
            pmax = max(pmax, pos_of(t));
    } else {
        pmax = t_last;
    }
    int nvmax = 0;
    {
        long long a = pmax - p.W + 1;
        if (a > 0)
            nvmax = (int)min((long long)p.Nc, a / p.m);
    }
    const int ntiles_all = (nvmax + kIxBN - 1) / kIxBN;
    const int j0 = chunk * kIxChunkTiles;
    const int j1 = min(ntiles_all, j0 + kIxChunkTiles);
    const int nt = j1 - j0;
    if (nt <= 0)
        return;  // uniform across the CTA: nothing to score here

    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        for (int s = 0; s < kIxStages; ++s) {
            mbar_init(&bar[1 + s], 1);
            mbar_init(&bar[5 + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[9 + s], 1);
            mbar_init(&bar[11 + s], 128);
        }
        mbar_init(&bar[13], 1);
        mbar_fence_init();
        misc[1] = 0;
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
            for (int i = 0; i < nt; ++i) {
                const int s = i % kIxStages;
                if (i >= kIxStages && !mbar_wait(&bar[5 + s], ((i / kIxStages) - 1) & 1, abort_flag))
                    break;
                mbar_arrive_expect_tx(&bar[1 + s], SM::K_BYTES);
                tma_load_4d(sK + s * SM::K_BYTES, &tm_k, &bar[1 + s], 0, 0, (j0 + i) * kIxBN, b);
                ++issued;
            }
            drain_wait(&bar[0], 0);
            for (int i = max(0, issued - kIxStages); i < issued; ++i)
                drain_wait(&bar[1 + i % kIxStages], (i / kIxStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kIxBM, kIxBN, false, false);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
            bool ok = mbar_wait(&bar[0], 0, abort_flag);
            for (int i = 0; ok && i < nt; ++i) {
                const int s = i % kIxStages, db = i & 1;
                if (!mbar_wait(&bar[1 + s], (i / kIxStages) & 1, abort_flag))
                    break;
                if (i >= 2 && !mbar_wait(&bar[11 + db], ((i >> 1) - 1) & 1, abort_flag))
                    break;
                tc_fence_after();
                for (int h = 0; h < HI; ++h) {
#pragma unroll
                    for (int kk = 0; kk < DI / 16; ++kk) {
                        const uint64_t da = ix_desc<DI>(aQ + h * SM::Q_BYTES + kk * 32);
                        const uint64_t dbk = ix_desc<DI>(aK + s * SM::K_BYTES + kk * 32);
                        mma_bf16_ss(tmem + (db * HI + h) * kIxBN, da, dbk, idesc, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(&bar[9 + db]);
                mma_commit(&bar[5 + s]);
            }
            mma_commit(&bar[13]);
            drain_wait(&bar[13], 0);
        }
    } else if (warp >= 4) {
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int t = t0 + row;
        const bool valid = t < p.Lq;
        int nv = 0;
        float wv[HI];
        if (valid) {
            const long long a = pos_of(t) - p.W + 1;
            nv = a > 0 ? (int)min((long long)p.Nc, a / p.m) : 0;
#pragma unroll
            for (int h = 0; h < HI; ++h)
                wv[h] = p.wi[((size_t)b * p.Lq + t) * HI + h];
        } else {
#pragma unroll
            for (int h = 0; h < HI; ++h)
                wv[h] = 0.f;
        }
        float *srow = p.scores + ((size_t)b * p.Lq + (valid ? t : 0)) * p.Nc;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t stage0 = smem_u32(smem + SM::OFF_ST);
        uint32_t u = 0;                                  // staged blocks written
        // Every epilogue thread runs every iteration (the staged store meets a
        // named barrier); after a failed wait it only skips the TMEM work.
        bool ok = true;
        for (int i = 0; i < nt; ++i) {
            const int db = i & 1;
            if (ok)
                ok = __all_sync(0xffffffffu, mbar_wait(&bar[9 + db], (i >> 1) & 1, abort_flag));
            if (!ok && !p.tma_store)
                break;
            tc_fence_after();
            const int s0 = (j0 + i) * kIxBN;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float acc[32];
                if (ok) {
                    // the Hi accumulators of this row's 32 keys, one wait
                    float d[HI][32];
#pragma unroll
                    for (int h = 0; h < HI; ++h)
                        tmem_ld32(tl + (db * HI + h) * kIxBN + half * 32, d[h]);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        float a = wv[0] * fmaxf(d[0][q], 0.f);
#pragma unroll
                        for (int h = 1; h < HI; ++h)
                            a = fmaf(wv[h], fmaxf(d[h][q], 0.f), a);
                        acc[q] = a;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        acc[q] = 0.f;
                }
                const int sb = s0 + half * 32;
                if (p.tma_store) {
                    // this row's 32 scores into the staging block (128-byte swizzle:
                    // 16-byte chunk c of row r at chunk c ^ (r & 7))
                    const uint32_t buf = stage0 + (u & 1) * SM::ST_BYTES + row * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                                         buf + ((c ^ (row & 7)) << 4)),
                                     "f"(acc[4 * c]), "f"(acc[4 * c + 1]), "f"(acc[4 * c + 2]),
                                     "f"(acc[4 * c + 3])
                                     : "memory");
                    fence_proxy_async_smem();
                    // the other buffer's copy has read its rows before anyone
                    // rewrites them (one copy in flight at most)
                    if (row == 0)
                        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (row == 0)
                        tma_store_3d(&tm_s, stage0 + (u & 1) * SM::ST_BYTES, sb, t0, b);
                    ++u;
                } else if (valid && sb < nv) {
                    if (sb + 32 <= nv && (p.Nc & 3) == 0) {
#pragma unroll
                        for (int q = 0; q < 32; q += 4)
                            *reinterpret_cast<float4 *>(srow + sb + q) =
                                make_float4(acc[q], acc[q + 1], acc[q + 2], acc[q + 3]);
                    } else {
                        for (int q = 0; q < 32 && sb + q < nv; ++q)
                            srow[sb + q] = acc[q];
                    }
                }
            }
            if (ok) {
                tc_fence_before();
                mbar_arrive(&bar[11 + db]);
            }
        }
        if (row == 0)
            asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[0], 512);
    }
}

// 4-D map over a [n3][n2][n1][DI] bf16 tensor with a (DI, 1, box_rows, 1) box,
// 128-byte swizzle for DI = 64 and 64-byte swizzle for DI = 32.
template <int DI>
static bool ix_map(CUtensorMap *map, const void *base, int n1, int n2, int n3, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[4] = {(cuuint64_t)DI, (cuuint64_t)n1, (cuuint64_t)n2, (cuuint64_t)n3};
    cuuint64_t strides[3] = {(cuuint64_t)DI * 2, (cuuint64_t)DI * 2 * n1, (cuuint64_t)DI * 2 * n1 * n2};
    cuuint32_t box[4] = {(cuuint32_t)DI, 1, (cuuint32_t)box_rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, DI == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HI, int DI>
static cudaError_t launch_index_tc_t(const IndexParams &p, const void *qi, const void *kic,
                                     cudaStream_t stream)
{
    using SM = IxSmem<HI, DI>;
    CUtensorMap mq, mk;
    // qi [B, Lq, Hi, DI] as (DI, Hi, Lq, B) with a (DI, 1, 128, 1) box
    bool ok = ix_map<DI>(&mq, qi, HI, p.Lq, p.B, kIxBM);
    // kic [B, Nc, DI] as (DI, 1, Nc, B) with a (DI, 1, 64, 1) box
    ok &= ix_map<DI>(&mk, kic, 1, p.Nc, p.B, kIxBN);
    if (!ok)
        return cudaErrorInvalidValue;
    // scores [B, Lq, Nc] fp32 as (Nc, Lq, B) with a (32, 128, 1) box, 128-byte
    // swizzle; rows past Lq and columns past Nc are clipped by the copy
    CUtensorMap ms;
    std::memset(&ms, 0, sizeof(ms));
    if (p.tma_store) {
        EncodeTiledFn fn = encode_fn();
        cuuint64_t dims[3] = {(cuuint64_t)p.Nc, (cuuint64_t)p.Lq, (cuuint64_t)p.B};
        cuuint64_t strides[2] = {(cuuint64_t)p.Nc * 4, (cuuint64_t)p.Nc * 4 * p.Lq};
        cuuint32_t box[3] = {32, (cuuint32_t)kIxBM, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (!fn || fn(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.scores, dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    size_t smem = 1024 + SM::BYTES;
    if (smem < 120 * 1024)
        smem = 120 * 1024;  // one CTA per SM: each holds all 512 TMEM columns
    auto kern = index_scores_tc<HI, DI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.n_ttiles * p.n_chunks, p.B);
    kern<<<grid, kIxThreads, smem, stream>>>(mq, mk, ms, p);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------
// Decode form: few query rows per sequence.  Keys go in the MMA's M
// dimension (128 per tile) and the query row's indexer heads, padded to 16,
// in N: D[128 keys x 16] = K_tile . Q^T.  The epilogue thread of a key forms
// sum_h w[h] relu(D[key][h]) and stores one fp32 score; the kernel streams the
// indexer-key cache once (HBM bound).  One CTA per (query row, run of tiles).
// Roles (192 threads): warp 0 TMA producer, warp 1 TMEM + MMA, warps 2-5
// epilogue (warp w reads TMEM lane quadrant w % 4).
// With a 4-bit key cache (codes and per-row (min, scale), see fp4.cu) four
// converter warps replace the TMA producer (288 threads): thread r copies
// key r's codes of tiles kDcAhead ahead into a staging ring with cp.async,
// and, when they have landed, writes the row's bf16 values into the K stage
// in the 128-byte swizzle; the MMA warp is then warp 4, the epilogue warps
// 5-8.
// ------------------------------------------------------------------------
constexpr int kDcThreads = 192;
constexpr int kDcAhead = 8;      // 4-bit form: tiles of codes in flight per converter thread
constexpr int kDcBM = 128;       // keys per tile
constexpr int kDcN = 16;         // padded indexer heads
constexpr int kDcStages = 4;
static_assert(kDcStages == 4, "the decode score kernel's barrier map (1-4 K full, 5-8 K empty) is written for four stages");
constexpr int kDcChunk = 16;     // key tiles per CTA

struct DecIndexParams {
    int B, Lq, Hi, Nc, m, W, n_chunks;
    const int32_t *q_pos;
    const float *wi;
    float *scores;
    const uint8_t *kcodes;   // 4-bit form: [B Nc, 32] codes, [B Nc] (min, scale)
    const float2 *kqp;
};

template <bool Q4>
struct DecRoles {
    static constexpr int PW = Q4 ? 4 : 1;            // producer (converter) warps
    static constexpr int MMA_WARP = PW;
    static constexpr int THREADS = 32 * (PW + 5);
    static constexpr int Q_BYTES = kDcN * kIxDi * 2;       // 2 KB
    static constexpr int K_BYTES = kDcBM * kIxDi * 2;      // 16 KB
    static constexpr int ST_CODES = kDcBM * kIxDi / 2;     // 4 KB of codes per staged tile
    static constexpr int ST_BYTES = Q4 ? kDcAhead * (ST_CODES + kDcBM * 8) : 0;
    static constexpr int SMEM = 1024 + kDcStages * K_BYTES + Q_BYTES + 16 * 8 + 16 * 4 + ST_BYTES;
};

template <bool Q4>
__global__ void __launch_bounds__(DecRoles<Q4>::THREADS, 1)
index_scores_dec(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const DecIndexParams p)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
    using RL = DecRoles<Q4>;
    constexpr int Q_BYTES = RL::Q_BYTES;
    constexpr int K_BYTES = RL::K_BYTES;
    extern __shared__ __align__(1024) uint8_t dc_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dc_smem_raw) + 1023) &
                                                ~(uintptr_t)1023);
    uint8_t *sK = smem;                              // stages, 1024-aligned
    uint8_t *sQ = smem + kDcStages * K_BYTES;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sQ + Q_BYTES);
    int *misc = reinterpret_cast<int *>(bar + 16);
    volatile int *abort_flag = misc + 1;
    uint8_t *sSt = reinterpret_cast<uint8_t *>(misc + 16);   // 4-bit staging: codes, then (min, scale)
    // bars: 0 Q, 1-4 K full, 5-8 K empty, 9-10 D full, 11-12 D empty, 13 done
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int row = blockIdx.x / p.n_chunks;          // b * Lq + t
    const int chunk = blockIdx.x % p.n_chunks;
    const int b = row / p.Lq, t = row % p.Lq;
    const long long pos = p.q_pos ? p.q_pos[row] : t;
    int nv = 0;
    {
        const long long a = pos - p.W + 1;
        if (a > 0)
            nv = (int)min((long long)p.Nc, a / p.m);
    }
    const int j0 = chunk * kDcChunk;
    const int j1 = min((nv + kDcBM - 1) / kDcBM, j0 + kDcChunk);
    const int nt = j1 - j0;
    if (nt <= 0)
        return;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 16; ++i)
            mbar_init(&bar[i], (i == 11 || i == 12 || (Q4 && i >= 1 && i <= 4)) ? 128 : 1);
        mbar_fence_init();
        misc[1] = 0;
    }
    if (warp == RL::MMA_WARP)
        tmem_alloc(reinterpret_cast<uint32_t *>(&misc[0]), 32);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];

    if (Q4 && warp < RL::PW) {
        // converters: thread r owns key row r of every tile
        const int r = threadIdx.x;
        if (r == 0) {
            mbar_arrive_expect_tx(&bar[0], Q_BYTES);
            tma_load_2d_box(sQ, &tm_q, &bar[0], 0, row * p.Hi);
        }
        const uint32_t st_codes = smem_u32(sSt), st_qp = st_codes + kDcAhead * RL::ST_CODES;
        // copies of tile i's row r into staging slot i % kDcAhead (zero past the cache)
        auto stage = [&](int i) {
            const int s = i % kDcAhead;
            const long long kr = (long long)(j0 + i) * kDcBM + r;
            const bool in = kr < p.Nc;
            const long long src = (long long)b * p.Nc + (in ? kr : 0);
            const uint32_t n = in ? 16u : 0u;
            const uint8_t *cs = p.kcodes + src * (kIxDi / 2);
            cp_async_16(st_codes + s * RL::ST_CODES + r * 32, cs, n);
            cp_async_16(st_codes + s * RL::ST_CODES + r * 32 + 16, cs + 16, n);
            asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(st_qp + s * kDcBM * 8 + r * 8),
                         "l"(p.kqp + src), "r"(in ? 8u : 0u)
                         : "memory");
        };
#pragma unroll 1
        for (int i = 0; i < kDcAhead - 1; ++i) {
            if (i < nt)
                stage(i);
            cp_async_commit();
        }
        bool ok = true;
        for (int i = 0; i < nt; ++i) {
            const int s = i % kDcStages;
            if (i + kDcAhead - 1 < nt)
                stage(i + kDcAhead - 1);
            cp_async_commit();
            cp_async_wait_group<kDcAhead - 1>();     // tile i's copies of this thread have landed
            if (i >= kDcStages)
                ok &= mbar_wait(&bar[5 + s], ((i / kDcStages) - 1) & 1, abort_flag);
            const int ss = i % kDcAhead;
            const uint8_t *cr = sSt + ss * RL::ST_CODES + r * 32;
            const float2 qv = *reinterpret_cast<const float2 *>(sSt + kDcAhead * RL::ST_CODES +
                                                                ss * kDcBM * 8 + r * 8);
            const uint4 c0 = *reinterpret_cast<const uint4 *>(cr);
            const uint4 c1 = *reinterpret_cast<const uint4 *>(cr + 16);
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            const uint32_t dst = smem_u32(sK + s * K_BYTES);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = fp4_dequant8(cw[c], qv.x, qv.y);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + sw128_offset(r, c)),
                             "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                             : "memory");
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[1 + s]);
        }
        (void)ok;
        cp_async_wait_group<0>();
        if (r == 0)
            drain_wait(&bar[0], 0);
    } else if (!Q4 && warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[0], Q_BYTES);
            // rows row*Hi .. row*Hi+15 of the [B*Lq*Hi, 64] view; rows past this
            // query's heads only feed unused columns
            tma_load_2d_box(sQ, &tm_q, &bar[0], 0, row * p.Hi);
            int issued = 0;
            for (int i = 0; i < nt; ++i) {
                const int s = i % kDcStages;
                if (i >= kDcStages && !mbar_wait(&bar[5 + s], ((i / kDcStages) - 1) & 1, abort_flag))
                    break;
                mbar_arrive_expect_tx(&bar[1 + s], K_BYTES);
                tma_load_4d(sK + s * K_BYTES, &tm_k, &bar[1 + s], 0, 0, (j0 + i) * kDcBM, b);
                ++issued;
            }
            drain_wait(&bar[0], 0);
            for (int i = max(0, issued - kDcStages); i < issued; ++i)
                drain_wait(&bar[1 + i % kDcStages], (i / kDcStages) & 1);
        }
    } else if (warp == RL::MMA_WARP) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kDcBM, kDcN, false, false);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
            bool ok = mbar_wait(&bar[0], 0, abort_flag);
            for (int i = 0; ok && i < nt; ++i) {
                const int s = i % kDcStages, db = i & 1;
                if (!mbar_wait(&bar[1 + s], (i / kDcStages) & 1, abort_flag))
                    break;
                if (i >= 2 && !mbar_wait(&bar[11 + db], ((i >> 1) - 1) & 1, abort_flag))
                    break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kIxDi / 16; ++kk)
                    mma_bf16_ss(tmem + db * kDcN, sw128_desc(aK + s * K_BYTES + kk * 32, 16, 1024),
                                sw128_desc(aQ + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                mma_commit(&bar[9 + db]);
                mma_commit(&bar[5 + s]);
            }
            mma_commit(&bar[13]);
            drain_wait(&bar[13], 0);
        }
    } else {
        const int quad = warp & 3;
        const int key = quad * 32 + lane;
        float wv[kDcN];
#pragma unroll
        for (int h = 0; h < kDcN; ++h)
            wv[h] = h < p.Hi ? p.wi[(size_t)row * p.Hi + h] : 0.f;
        float *srow = p.scores + (size_t)row * p.Nc;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        for (int i = 0; i < nt; ++i) {
            const int db = i & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&bar[9 + db], (i >> 1) & 1, abort_flag)))
                break;
            tc_fence_after();
            uint32_t d[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]),
                  "=r"(d[6]), "=r"(d[7]), "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]),
                  "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
                : "r"(tl + db * kDcN));
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&bar[11 + db]);
            float I = 0.f;
#pragma unroll
            for (int h = 0; h < kDcN; ++h)
                if (h < p.Hi)
                    I = fmaf(wv[h], fmaxf(__uint_as_float(d[h]), 0.f), I);
            const int sidx = (j0 + i) * kDcBM + key;
            if (sidx < nv)
                srow[sidx] = I;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == RL::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc((uint32_t)misc[0], 32);
    }
}

// kic: bf16 cache (TMA tiles), or nullptr with kcodes / kqp set (4-bit form).
static cudaError_t launch_index_dec(const void *qi, const float *wi, const void *kic,
                                    const uint8_t *kcodes, const float *kqp, float *scores, int B, int Lq,
                                    int Hi, int Nc, int m, int W, const int32_t *q_pos, cudaStream_t stream)
{
    CUtensorMap mq, mk;
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return cudaErrorInvalidValue;
    {
        cuuint64_t dims[2] = {(cuuint64_t)kIxDi, (cuuint64_t)B * Lq * Hi};
        cuuint64_t strides[1] = {(cuuint64_t)kIxDi * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)kDcN};
        cuuint32_t es[2] = {1, 1};
        if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(qi), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const bool q4 = kic == nullptr;
    if (q4)
        mk = mq;   // unused by the 4-bit form
    else if (!make_map(&mk, kic, kIxDi, 1, Nc, B, 1, kDcBM))
        return cudaErrorInvalidValue;
    DecIndexParams p;
    p.B = B;
    p.Lq = Lq;
    p.Hi = Hi;
    p.Nc = Nc;
    p.m = m;
    p.W = W;
    p.n_chunks = (Nc + kDcBM * kDcChunk - 1) / (kDcBM * kDcChunk);
    if (p.n_chunks < 1)
        p.n_chunks = 1;
    p.q_pos = q_pos;
    p.wi = wi;
    p.scores = scores;
    p.kcodes = kcodes;
    p.kqp = reinterpret_cast<const float2 *>(kqp);
    const unsigned grid = (unsigned)(B * Lq * p.n_chunks);
    if (q4) {
        const size_t smem = DecRoles<true>::SMEM;
        cudaError_t e = cudaFuncSetAttribute(index_scores_dec<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        e = launch_pdl(index_scores_dec<true>, dim3(grid), dim3(DecRoles<true>::THREADS), smem, stream, mq, mk, p);
        if (e != cudaSuccess)
            return e;
    } else {
        const size_t smem = DecRoles<false>::SMEM;
        cudaError_t e = cudaFuncSetAttribute(index_scores_dec<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        e = launch_pdl(index_scores_dec<false>, dim3(grid), dim3(DecRoles<false>::THREADS), smem, stream, mq, mk,
                       p);
        if (e != cudaSuccess)
            return e;
    }
    return cudaGetLastError();
}

// Decode indexer scores over a 4-bit indexer-key cache (di = 64, Hi <= 16).
cudaError_t launch_index_dec_fp4(const void *qi, const float *wi, const uint8_t *kic_codes,
                                 const float *kic_qp, float *scores, int B, int Lq, int Hi, int di, int Nc,
                                 int m, int W, const int32_t *q_pos, cudaStream_t stream)
{
    if (di != kIxDi || Hi < 1 || Hi > kDcN)
        return cudaErrorNotSupported;
    return launch_index_dec(qi, wi, nullptr, kic_codes, kic_qp, scores, B, Lq, Hi, Nc, m, W, q_pos,
                            stream);
}

// Indexer scores on tensor cores: prefill (di 64 or 32, Hi <= 4) and decode
// (di 64).  Returns cudaErrorNotSupported for other shapes (the caller uses
// the CUDA-core path).
cudaError_t launch_index_scores_tc(const void *qi, const float *wi, const void *kic, float *scores,
                                   int B, int Lq, int Hi, int di, int Nc, int m, int W,
                                   const int32_t *q_pos, cudaStream_t stream)
{
    if ((di != 64 && di != 32) || Hi < 1)
        return cudaErrorNotSupported;
    if (Lq < 64) {
        if (di != kIxDi)
            return cudaErrorNotSupported;
        // decode: one tile of keys per MMA, the query's heads in N
        if (Hi > kDcN)
            return cudaErrorNotSupported;
        return launch_index_dec(qi, wi, kic, nullptr, nullptr, scores, B, Lq, Hi, Nc, m, W, q_pos, stream);
    }
    if (Hi > 4)
        return cudaErrorNotSupported;
    IndexParams p;
    p.B = B;
    p.Lq = Lq;
    p.Hi = Hi;
    p.Nc = Nc;
    p.m = m;
    p.W = W;
    p.n_ttiles = (Lq + kIxBM - 1) / kIxBM;
    p.n_chunks = (Nc + kIxBN * kIxChunkTiles - 1) / (kIxBN * kIxChunkTiles);
    if (p.n_chunks < 1)
        p.n_chunks = 1;
    p.q_pos = q_pos;
    p.wi = wi;
    p.scores = scores;
    // the tensor store needs 16-byte row strides and a 16-byte aligned base
    p.tma_store = (Nc % 4 == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0) ? 1 : 0;
    if (di == 32) {
        switch (Hi) {
        case 1: return launch_index_tc_t<1, 32>(p, qi, kic, stream);
        case 2: return launch_index_tc_t<2, 32>(p, qi, kic, stream);
        case 3: return launch_index_tc_t<3, 32>(p, qi, kic, stream);
        default: return launch_index_tc_t<4, 32>(p, qi, kic, stream);
        }
    }
    switch (Hi) {
    case 1: return launch_index_tc_t<1, 64>(p, qi, kic, stream);
    case 2: return launch_index_tc_t<2, 64>(p, qi, kic, stream);
    case 3: return launch_index_tc_t<3, 64>(p, qi, kic, stream);
    default: return launch_index_tc_t<4, 64>(p, qi, kic, stream);
    }
}

}  // namespace hyb

// probe.cu -- measurement kernel for the roofline denominators: the rate at
// which an SM can gather random rows that live in L2 into shared memory, the
// data path of the CSA attention (every query token attends to its own
// selected compressed rows, "deepseek-v4" blog, section 1, CSA).
//
// One persistent CTA per SM copies random 256-byte rows of an L2-resident
// table into a ring of 32 KB shared-memory stages with 16-byte cp.async
// (16 lanes per row, 128 rows per stage), keeping `stages - 1` stages in
// flight.  Row numbers come from a hash of (CTA, row), so no index load sits
// on the path.  A checksum of the copied words goes to `sink` so that the
// copies cannot be removed.
#include "common.cuh"

namespace hyb {

constexpr int kPgThreads = 256;
constexpr int kPgRowBytes = 256;
constexpr int kPgStageRows = 128;
constexpr int kPgStageBytes = kPgStageRows * kPgRowBytes;   // 32 KB
constexpr int kPgMaxStages = 6;

__device__ __forceinline__ uint32_t pg_hash(uint32_t x)
{
    x ^= x >> 16;
    x *= 0x7feb352dU;
    x ^= x >> 15;
    x *= 0x846ca68bU;
    x ^= x >> 16;
    return x;
}

__global__ void __launch_bounds__(kPgThreads, 1)
l2_gather_probe(const uint8_t *__restrict__ table, uint32_t table_rows, int n_stage_rounds, int stages,
                uint32_t *__restrict__ sink)
{
    extern __shared__ __align__(16) uint8_t pg_ring[];
    const int c16 = threadIdx.x & 15;        // 16-byte chunk of the row
    const int rsub = threadIdx.x >> 4;       // rows rsub, rsub + 16, ...
    const uint32_t base = smem_u32(pg_ring);
    for (int r = 0; r < n_stage_rounds; ++r) {
        const uint32_t st = base + (uint32_t)(r % stages) * kPgStageBytes;
#pragma unroll
        for (int u = 0; u < kPgStageRows / 16; ++u) {
            const int row = u * 16 + rsub;
            const uint32_t src = pg_hash((uint32_t)blockIdx.x * 0x9E3779B9u + (uint32_t)(r * kPgStageRows + row)) %
                                 table_rows;
            cp_async_16(st + row * kPgRowBytes + c16 * 16, table + (size_t)src * kPgRowBytes + c16 * 16, 16u);
        }
        cp_async_commit();
        // keep stages - 1 rounds in flight: wait for the oldest beyond that
        switch (stages) {
        case 2: cp_async_wait_group<1>(); break;
        case 3: cp_async_wait_group<2>(); break;
        case 4: cp_async_wait_group<3>(); break;
        case 5: cp_async_wait_group<4>(); break;
        default: cp_async_wait_group<5>(); break;
        }
    }
    cp_async_wait_group<0>();
    __syncthreads();
    const uint32_t *w = reinterpret_cast<const uint32_t *>(pg_ring);
    uint32_t acc = 0;
    for (int i = threadIdx.x; i < stages * kPgStageBytes / 4; i += kPgThreads)
        acc ^= w[i];
    atomicXor(sink + (blockIdx.x & 255), acc);
}


// The same gather by the tensor memory accelerator: one warp per CTA, lane l
// loading rows 4l..4l+3 of every stage with two tile::gather4 copies (channels
// 0-63 and 64-127, one-row boxes of a 128-byte-swizzled map, so each copy
// writes four 128-byte rows at a 512-byte offset of the stage half).  Stage
// completion is counted in bytes on one mbarrier per stage.  After the last
// round the warp checks every 16-byte chunk of the last stage against the
// table at the place the 128-byte swizzle assigns it and adds the number of
// misplaced chunks to sink[256].
constexpr int kPtThreads = 32;

__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int c0,
                                            int r0, int r1, int r2, int r3)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
        : "memory");
}

__global__ void __launch_bounds__(kPtThreads, 1)
l2_gather_probe_tma(const __grid_constant__ CUtensorMap tm, const uint8_t *__restrict__ table,
                    uint32_t table_rows, int n_stage_rounds, int stages, uint32_t *__restrict__ sink)
{
    extern __shared__ __align__(16) uint8_t pt_ring_raw[];
    __shared__ __align__(8) uint64_t bars[kPgMaxStages];
    __shared__ int abort_s;
    const int lane = threadIdx.x;
    // stages start on 1024-byte boundaries (the swizzle repeat)
    const uint32_t raw = smem_u32(pt_ring_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint8_t *ring = pt_ring_raw + (base - raw);
    if (lane == 0) {
        for (int s = 0; s < stages; ++s)
            mbar_init(&bars[s], 1);
        abort_s = 0;
        mbar_fence_init();
    }
    __syncwarp();
    auto rows_of = [&](int r, int (&rw)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            rw[k] = (int)(pg_hash((uint32_t)blockIdx.x * 0x9E3779B9u + (uint32_t)(r * kPgStageRows + 4 * lane + k)) %
                          table_rows);
    };
    int issued = 0;
    for (int r = 0; r < n_stage_rounds; ++r) {
        const int s = r % stages;
        if (r >= stages - 1) {
            // keep stages - 1 rounds in flight
            const int rr = r - (stages - 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[rr % stages], (uint32_t)(rr / stages) & 1u, &abort_s)))
                break;
        }
        if (lane == 0)
            mbar_arrive_expect_tx(&bars[s], kPgStageBytes);
        __syncwarp();
        int rw[4];
        rows_of(r, rw);
        const uint32_t dst = base + (uint32_t)s * kPgStageBytes + (uint32_t)lane * 512u;
        tma_gather4(dst, &tm, &bars[s], 0, rw[0], rw[1], rw[2], rw[3]);
        tma_gather4(dst + kPgStageBytes / 2, &tm, &bars[s], 64, rw[0], rw[1], rw[2], rw[3]);
        issued = r + 1;
    }
    // every issued round has landed before the CTA leaves
    for (int rr = issued > stages - 1 ? issued - (stages - 1) : 0; rr < issued; ++rr)
        drain_wait(&bars[rr % stages], (uint32_t)(rr / stages) & 1u);
    __syncwarp();
    uint32_t acc = 0, bad = 0;
    if (issued == n_stage_rounds && issued > 0) {
        const int r = issued - 1;
        const uint8_t *st = ring + (size_t)(r % stages) * kPgStageBytes;
        int rw[4];
        rows_of(r, rw);
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
            const uint32_t row = 4u * lane + k;
            const uint4 *src = reinterpret_cast<const uint4 *>(table + (size_t)rw[k] * kPgRowBytes);
#pragma unroll 1
            for (int c = 0; c < 16; ++c) {
                const uint4 want = src[c];
                const uint4 got = *reinterpret_cast<const uint4 *>(st + (c >> 3) * (kPgStageBytes / 2) +
                                                                    sw128_offset(row, (uint32_t)(c & 7)));
                bad += (want.x != got.x) | (want.y != got.y) | (want.z != got.z) | (want.w != got.w);
                acc ^= got.x ^ got.y ^ got.z ^ got.w;
            }
        }
    }
    atomicXor(sink + (blockIdx.x & 255), acc);
    if (bad)
        atomicAdd(sink + 256, bad);
}

}  // namespace hyb

using namespace hyb;

extern "C" hyb_status hyb_probe_l2_gather(const void *table, long long table_bytes, long long rows_per_sm,
                                          int stages, unsigned int *sink, cudaStream_t stream)
{
    if (!table || !sink || table_bytes < kPgRowBytes || rows_per_sm < kPgStageRows || stages < 2 ||
        stages > kPgMaxStages || (reinterpret_cast<uintptr_t>(table) & 15u))
        return HYB_ERR_INVALID_ARG;
    const long long rows = table_bytes / kPgRowBytes;
    if (rows > 0xFFFFFFFFll || rows_per_sm / kPgStageRows > 0x7FFFFFFFll)
        return HYB_ERR_UNSUPPORTED;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = (size_t)stages * kPgStageBytes;
    if (cudaFuncSetAttribute(l2_gather_probe, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return HYB_ERR_CUDA;
    l2_gather_probe<<<sms, kPgThreads, smem, stream>>>(static_cast<const uint8_t *>(table), (uint32_t)rows,
                                                       (int)(rows_per_sm / kPgStageRows), stages, sink);
    return cudaGetLastError() == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

extern "C" hyb_status hyb_probe_l2_gather_tma(const void *table, long long table_bytes, long long rows_per_sm,
                                              int stages, unsigned int *sink, cudaStream_t stream)
{
    if (!table || !sink || table_bytes < kPgRowBytes || rows_per_sm < kPgStageRows || stages < 2 ||
        stages > kPgMaxStages || (reinterpret_cast<uintptr_t>(table) & 15u))
        return HYB_ERR_INVALID_ARG;
    const long long rows = table_bytes / kPgRowBytes;
    if (rows > 0x7FFFFFFFll || rows_per_sm / kPgStageRows > 0x7FFFFFFFll)
        return HYB_ERR_UNSUPPORTED;
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return HYB_ERR_CUDA;
    // [rows][128] bf16 view, (64, 1) boxes, 128-byte swizzle
    CUtensorMap tm;
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {kPgRowBytes};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t es[2] = {1, 1};
    if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(table), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return HYB_ERR_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = (size_t)stages * kPgStageBytes + 1024;
    if (cudaFuncSetAttribute(l2_gather_probe_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return HYB_ERR_CUDA;
    l2_gather_probe_tma<<<sms, kPtThreads, smem, stream>>>(tm, static_cast<const uint8_t *>(table), (uint32_t)rows,
                                                           (int)(rows_per_sm / kPgStageRows), stages, sink);
    return cudaGetLastError() == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

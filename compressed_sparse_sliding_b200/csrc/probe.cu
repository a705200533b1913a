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

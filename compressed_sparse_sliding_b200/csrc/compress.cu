// compress.cu -- stage 1, block_merge (CSDN DeepSeek-V4 CSA/HCA code page,
// section 1): one compressed entry per block of m tokens, the weighted sum of
// the block's tokens with per-channel softmax weights over the m positions.
//
// Memory-bound streaming kernel.  Every thread owns 8 consecutive channels of
// one (b, j) block row and reads 16-byte vectors; a warp covers 512
// contiguous bytes of a token row, so each load instruction is fully
// coalesced.  When there are too few (b, j, channel-octet) items to fill the
// GPU (few, long blocks such as m = 128), the m positions are split over S
// thread groups of the CTA and their partial sums are reduced in shared
// memory.  CTAs are persistent: the [m, dx] weights arrive in shared memory
// by one bulk copy and are turned into softmax weights once per CTA, then
// reused for every block the CTA processes.
#include "common.cuh"

namespace hyb {

constexpr int kMergeThreads = 256;
constexpr int kMergeStages = 3;   // cp.async ring depth of the register-weight kernel

__global__ void __launch_bounds__(kMergeThreads)
block_merge_kernel(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ w,
                   __nv_bfloat16 *__restrict__ out, int B, int L, int H, int dx, int m, int S)
{
    extern __shared__ __align__(16) float sm_merge[];
    float *P = sm_merge;                        // [m][dx]
    float *part = sm_merge + (size_t)m * dx;    // [S-1][items_per_cta][8]
    __shared__ __align__(8) uint64_t wbar;
    __shared__ int wabort;
    const int tid = threadIdx.x;

    // ---- stage the [m, dx] weights with one bulk copy, then softmax over the
    //      m positions separately for every channel, in place ----
    if (tid == 0) {
        wabort = 0;
        mbar_init(&wbar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0) {
        const uint32_t bytes = (uint32_t)(m * dx) * 4u;
        mbar_arrive_expect_tx(&wbar, bytes);
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_u32(P)),
            "l"(w), "r"(bytes), "r"(smem_u32(&wbar))
            : "memory");
    }
    if (!mbar_wait(&wbar, 0, &wabort))
        return;  // recorded as a device timeout; the copy was issued by thread 0 only
    __syncthreads();
    {
        int G = 1;  // threads per channel (power of two)
        while (G * 2 * dx <= kMergeThreads && G * 2 <= m)
            G *= 2;
        const int cpr = kMergeThreads / G;  // channels per round
        const int g = tid % G;
        for (int c = tid / G; c < dx + (cpr - (dx % cpr)) % cpr; c += cpr) {
            const bool live = c < dx;
            float mx = -INFINITY;
            if (live)
                for (int i = g; i < m; i += G)
                    mx = fmaxf(mx, P[(size_t)i * dx + c]);
            for (int off = 1; off < G; off <<= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            float den = 0.f;
            if (live)
                for (int i = g; i < m; i += G) {
                    float e = expf(P[(size_t)i * dx + c] - mx);
                    P[(size_t)i * dx + c] = e;
                    den += e;
                }
            for (int off = 1; off < G; off <<= 1)
                den += __shfl_xor_sync(0xffffffffu, den, off);
            if (live) {
                float inv = 1.f / den;
                for (int i = g; i < m; i += G)
                    P[(size_t)i * dx + c] *= inv;
            }
        }
    }
    __syncthreads();

    const int Nc = L / m;
    const int E8 = H * dx / 8;                 // 16-byte octets per token row
    const long long items = (long long)B * Nc * E8;
    const int ipc = kMergeThreads / S;         // items per CTA tile
    const int s = tid / ipc;                   // position split owned by this thread
    const int li = tid % ipc;
    const long long ntiles = (items + ipc - 1) / ipc;
    const size_t row_elems = (size_t)H * dx;

    for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const long long item = tile * ipc + li;
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            acc[k] = 0.f;
        const bool live = item < items;
        if (live) {
            const long long unit = item / E8;
            const int e8 = (int)(item % E8);
            const int b = (int)(unit / Nc);
            const int j = (int)(unit % Nc);
            const int c0 = (e8 * 8) % dx;
            const __nv_bfloat16 *src =
                x + ((size_t)b * L + (size_t)j * m) * row_elems + (size_t)e8 * 8;
            int i = s;
            // eight independent 16-byte loads in flight per thread
            for (; i + 7 * S < m; i += 8 * S) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    v[u] = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)(i + u * S) * row_elems));
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float *pw = P + (size_t)(i + u * S) * dx + c0;
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&v[u]);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float2 f = __bfloat1622float2(h2[k]);
                        acc[2 * k] = fmaf(pw[2 * k], f.x, acc[2 * k]);
                        acc[2 * k + 1] = fmaf(pw[2 * k + 1], f.y, acc[2 * k + 1]);
                    }
                }
            }
            for (; i < m; i += S) {
                uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)i * row_elems));
                const float *pw = P + (size_t)i * dx + c0;
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float2 f = __bfloat1622float2(h2[k]);
                    acc[2 * k] = fmaf(pw[2 * k], f.x, acc[2 * k]);
                    acc[2 * k + 1] = fmaf(pw[2 * k + 1], f.y, acc[2 * k + 1]);
                }
            }
        }
        if (S > 1) {
            if (s > 0) {
                float4 *dst = reinterpret_cast<float4 *>(part + ((size_t)(s - 1) * ipc + li) * 8);
                dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
            __syncthreads();
            if (s == 0) {
                for (int q = 1; q < S; ++q) {
                    const float4 *srcp =
                        reinterpret_cast<const float4 *>(part + ((size_t)(q - 1) * ipc + li) * 8);
                    float4 a = srcp[0], bq = srcp[1];
                    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
                    acc[4] += bq.x; acc[5] += bq.y; acc[6] += bq.z; acc[7] += bq.w;
                }
            }
            __syncthreads();
        }
        if (s == 0 && live) {
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            *reinterpret_cast<uint4 *>(out + (size_t)item * 8) = o;
        }
    }
}

// ---------------------------------------------------------------------------
// Register-weight form.  With S chosen so that each thread owns at most 8
// positions (NPOS = m / S) and a fixed octet of channels (items per tile times
// 8 is a multiple of dx), the thread's NPOS x 8 softmax weights live in
// registers: the main loop is only 16-byte global loads and FMAs.  The
// per-channel max and sum over the m positions are combined across the S
// position groups through a small shared table (2 x S x dx floats).
// ---------------------------------------------------------------------------
template <int NPOS>
__global__ void __launch_bounds__(kMergeThreads)
block_merge_regs(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ w,
                 __nv_bfloat16 *__restrict__ out, int B, int L, int H, int dx, int m, int S)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
    extern __shared__ __align__(16) float sm_rg[];
    const int tid = threadIdx.x;
    const int ipc = kMergeThreads / S;
    const int gw = ipc < 32 ? 32 / ipc : 1;     // position groups per warp
    const int np = S / gw;                      // partial sets after the warp fold
    float *part = sm_rg;                        // [2][np][ipc][8] partial sums (S > 1)
    float *ring_f = sm_rg + (S > 1 ? (size_t)2 * np * ipc * 8 : 0);
    float *red = ring_f;                        // [S][dx] partial max, then sums, and [dx]
    float *fin = ring_f + (size_t)S * dx;       // combined values (prologue only, before the
                                                // ring is filled)
    const int s = tid / ipc;
    const int li = tid % ipc;
    const int c0 = (li * 8) % dx;               // fixed channel octet of this thread
    const bool owner = li < dx / 8;             // one thread per (s, channel octet) writes

    // ---- the block stream ----
    // Every thread copies its own NPOS 16-byte pieces of a tile into private
    // slots of a kMergeStages-deep shared ring with cp.async, kMergeStages - 1
    // tiles ahead of the one it reduces; a thread only ever reads the slots it
    // filled, so the ring needs no barrier (cp.async.wait_group orders it).
    // Tile k uses stage (k + 1) mod kMergeStages: the first tiles go to stages
    // 1, 2, ... before the weight prologue, whose scratch lives in stage 0.
    const int Nc = L / m;
    const int E8 = H * dx / 8;
    const long long items = (long long)B * Nc * E8;
    const long long ntiles = (items + ipc - 1) / ipc;
    const size_t row_elems = (size_t)H * dx;
    const uint32_t ring = smem_u32(ring_f);
    auto slot = [&](int stage, int k) -> uint32_t {
        return ring + (uint32_t)(((stage * NPOS + k) * kMergeThreads + tid) * 16);
    };
    auto issue = [&](long long tile, int stage) {
        const long long item = tile * ipc + li;
        if (tile < ntiles && item < items) {
            const long long unit = item / E8;
            const int e8 = (int)(item % E8);
            const int b = (int)(unit / Nc);
            const int j = (int)(unit % Nc);
            const __nv_bfloat16 *src =
                x + ((size_t)b * L + (size_t)j * m + s) * row_elems + (size_t)e8 * 8;
#pragma unroll
            for (int k = 0; k < NPOS; ++k)
                cp_async_16(slot(stage, k), src + (size_t)k * S * row_elems, 16u);
        }
        cp_async_commit();   // one group per tile, empty past the end
    };
#pragma unroll
    for (int d = 0; d < kMergeStages - 1; ++d)
        issue((long long)blockIdx.x + (long long)d * gridDim.x, d + 1);

    // ---- this thread's weights: positions s, s + S, ... (NPOS of them) ----
    float P[NPOS][8];
#pragma unroll
    for (int k = 0; k < NPOS; ++k) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(w + (size_t)(s + k * S) * dx + c0));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(w + (size_t)(s + k * S) * dx + c0 + 4));
        P[k][0] = a.x; P[k][1] = a.y; P[k][2] = a.z; P[k][3] = a.w;
        P[k][4] = b.x; P[k][5] = b.y; P[k][6] = b.z; P[k][7] = b.w;
    }
    float mx[8], den[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float v = P[0][q];
#pragma unroll
        for (int k = 1; k < NPOS; ++k)
            v = fmaxf(v, P[k][q]);
        mx[q] = v;
    }
    // Per-channel max and sum over the S position groups: the groups' values go
    // to red [S][dx]; thread c < dx combines channel c (consecutive threads,
    // consecutive addresses) into fin [dx]; every thread reads its 8 channels
    // back as two 16-byte loads.
    if (owner) {
        reinterpret_cast<float4 *>(red + s * dx + c0)[0] = make_float4(mx[0], mx[1], mx[2], mx[3]);
        reinterpret_cast<float4 *>(red + s * dx + c0)[1] = make_float4(mx[4], mx[5], mx[6], mx[7]);
    }
    __syncthreads();
    if (tid < dx) {
        float v = red[tid];
        for (int g = 1; g < S; ++g)
            v = fmaxf(v, red[g * dx + tid]);
        fin[tid] = v;
    }
    __syncthreads();
    {
        const float4 a = reinterpret_cast<const float4 *>(fin + c0)[0];
        const float4 b = reinterpret_cast<const float4 *>(fin + c0)[1];
        mx[0] = a.x; mx[1] = a.y; mx[2] = a.z; mx[3] = a.w;
        mx[4] = b.x; mx[5] = b.y; mx[6] = b.z; mx[7] = b.w;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < NPOS; ++k) {
            P[k][q] = expf(P[k][q] - mx[q]);
            acc += P[k][q];
        }
        den[q] = acc;
    }
    if (owner) {
        reinterpret_cast<float4 *>(red + s * dx + c0)[0] = make_float4(den[0], den[1], den[2], den[3]);
        reinterpret_cast<float4 *>(red + s * dx + c0)[1] = make_float4(den[4], den[5], den[6], den[7]);
    }
    __syncthreads();   // (every thread has read fin's maxima)
    if (tid < dx) {
        float v = 0.f;
        for (int g = 0; g < S; ++g)
            v += red[g * dx + tid];
        fin[tid] = v;
    }
    __syncthreads();
    {
        const float4 a = reinterpret_cast<const float4 *>(fin + c0)[0];
        const float4 b = reinterpret_cast<const float4 *>(fin + c0)[1];
        den[0] = a.x; den[1] = a.y; den[2] = a.z; den[3] = a.w;
        den[4] = b.x; den[5] = b.y; den[6] = b.z; den[7] = b.w;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float inv = 1.f / den[q];
#pragma unroll
        for (int k = 0; k < NPOS; ++k)
            P[k][q] *= inv;
    }

    __syncthreads();   // every thread is done with `red` / `fin` (ring stage 0)
    int parity = 0, stage = 1;
    for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        issue(tile + (long long)(kMergeStages - 1) * gridDim.x, (stage + kMergeStages - 1) % kMergeStages);
        cp_async_wait_group<kMergeStages - 1>();   // this tile's copies have landed
        const long long item = tile * ipc + li;
        const bool live = item < items;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            acc[q] = 0.f;
        if (live) {
            uint4 v[NPOS];
#pragma unroll
            for (int k = 0; k < NPOS; ++k)
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v[k].x), "=r"(v[k].y), "=r"(v[k].z), "=r"(v[k].w)
                             : "r"(slot(stage, k)));
#pragma unroll
            for (int k = 0; k < NPOS; ++k) {
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&v[k]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __bfloat1622float2(h2[q]);
                    acc[2 * q] = fmaf(P[k][2 * q], f.x, acc[2 * q]);
                    acc[2 * q + 1] = fmaf(P[k][2 * q + 1], f.y, acc[2 * q + 1]);
                }
            }
        }
        if (S > 1) {
            // fold the position groups that share a warp, then the per-warp
            // partial sets through the table (double-buffered: one barrier)
            for (int off = ipc; off < 32; off <<= 1)
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], off);
            float *pt = part + (size_t)(parity & 1) * np * ipc * 8;
            if ((tid & 31) < ipc) {
                float4 *dst = reinterpret_cast<float4 *>(pt + ((size_t)(s / gw) * ipc + li) * 8);
                dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
            __syncthreads();
            for (int e = tid; e < ipc * 8; e += kMergeThreads) {
                float v = 0.f;
                for (int g = 0; g < np; ++g)
                    v += pt[(size_t)g * ipc * 8 + e];
                const long long item2 = tile * ipc + (e >> 3);
                if (item2 < items)
                    out[(size_t)item2 * 8 + (e & 7)] = __float2bfloat16_rn(v);
            }
            ++parity;
        } else if (live) {
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            *reinterpret_cast<uint4 *>(out + (size_t)item * 8) = o;
        }
        stage = stage + 1 == kMergeStages ? 0 : stage + 1;
    }
    cp_async_wait_group<0>();
}

template <int NPOS>
static cudaError_t launch_merge_regs(const void *x, int B, int L, int H, int dx, int m, const float *w,
                                     void *out, int S, long long items, cudaStream_t stream,
                                     int num_sms)
{
    const int ipc = kMergeThreads / S;
    const int gw = ipc < 32 ? 32 / ipc : 1;
    const int np = S / gw;
    const size_t ring = (size_t)kMergeStages * NPOS * kMergeThreads * 16;
    const size_t red = sizeof(float) * (size_t)(S + 1) * dx;
    const size_t smem = (S > 1 ? sizeof(float) * (size_t)2 * np * ipc * 8 : 0) + (ring > red ? ring : red);
    cudaError_t e = cudaFuncSetAttribute(block_merge_regs<NPOS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, block_merge_regs<NPOS>, kMergeThreads,
                                                      smem);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        per_sm = 1;
    const long long ntiles = (items + ipc - 1) / ipc;
    long long grid = (long long)num_sms * per_sm;
    if (grid > ntiles)
        grid = ntiles;
    return launch_pdl(block_merge_regs<NPOS>, dim3((unsigned)grid), dim3(kMergeThreads), smem, stream,
                      static_cast<const __nv_bfloat16 *>(x), w, static_cast<__nv_bfloat16 *>(out), B, L, H, dx,
                      m, S);
}

// Launch helper: picks the position split S and a persistent grid.
cudaError_t launch_block_merge(const void *x, int B, int L, int H, int dx, int m, const float *w,
                               void *out, cudaStream_t stream, int num_sms)
{
    const int Nc = L / m;
    const long long items = (long long)B * Nc * (H * dx / 8);
    if (items == 0)
        return cudaSuccess;
    {
        // register-weight form: at most 8 positions per thread, fixed channel octet
        int Sr = 1;
        while (Sr * 8 < m && Sr < 32)
            Sr *= 2;
        while (Sr < 32 && m % (Sr * 2) == 0 && m / (Sr * 2) >= 4 &&
               ((kMergeThreads / (Sr * 2)) * 8) % dx == 0 && items * Sr < (long long)num_sms * 2048)
            Sr *= 2;  // more position groups while the grid is short of work
        const int ipc = kMergeThreads / Sr;
        if (m % Sr == 0 && m / Sr <= 8 && (ipc * 8) % dx == 0 && dx <= 256) {
            switch (m / Sr) {
            case 1: return launch_merge_regs<1>(x, B, L, H, dx, m, w, out, Sr, items, stream, num_sms);
            case 2: return launch_merge_regs<2>(x, B, L, H, dx, m, w, out, Sr, items, stream, num_sms);
            case 4: return launch_merge_regs<4>(x, B, L, H, dx, m, w, out, Sr, items, stream, num_sms);
            case 8: return launch_merge_regs<8>(x, B, L, H, dx, m, w, out, Sr, items, stream, num_sms);
            default: break;
            }
        }
    }
    // split the m positions over S thread groups only while every thread keeps
    // at least 8 loads and the grid is short of ~1024 threads per SM
    int S = 1;
    const long long target = (long long)num_sms * 1024;
    while (S * 2 <= m / 8 && S * 2 <= 32 && items * S < target)
        S *= 2;
    const size_t smem = sizeof(float) * ((size_t)m * dx + (size_t)(S - 1) * (kMergeThreads / S) * 8);
    cudaError_t e = cudaFuncSetAttribute(block_merge_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, block_merge_kernel, kMergeThreads,
                                                      smem);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        per_sm = 1;
    const int ipc = kMergeThreads / S;
    const long long ntiles = (items + ipc - 1) / ipc;
    long long grid = (long long)num_sms * per_sm;
    if (grid > ntiles)
        grid = ntiles;
    block_merge_kernel<<<(unsigned)grid, kMergeThreads, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(x), w, static_cast<__nv_bfloat16 *>(out), B, L, H, dx,
        m, S);
    return cudaGetLastError();
}

}  // namespace hyb

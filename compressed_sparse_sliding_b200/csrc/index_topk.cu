// index_topk.cu -- stage 2 of CSA ("deepseek-v4" blog, section 1, CSA: a
// lightning indexer picks the top-K compressed entries for the current
// query).  Score: I[t, s] = sum_h wi[t, h] * relu(qi[t, h, :] . kic[s, :]),
// kept in fp32, over the entries visible to t; then an exact top-K with ties
// resolved toward the lower entry index, written in ascending index order.
//
// Kernels here (the tensor-core score kernels are in index_tc.cu):
//   index_scores_simt  CUDA-core scores for a tile of query rows x keys into a
//                      workspace row per query (only the visible prefix);
//                      the fallback for shapes the tensor-core kernels do not
//                      take (di != 64, more than 4 heads in prefill).
//   topk_hist          one CTA per query row (rows of up to 16384 entries),
//                      the row's keys in registers; histogram select of the
//                      K-th largest order key by a narrowing key interval.
//   topk_radix         rows longer than that: keys in shared memory, a
//                      12 + 10 + 10-bit radix select.
//   Both emit in index order: every key above the threshold and the
//   lowest-index keys equal to it.
#include "common.cuh"

namespace hyb {

// Number of compressed entries visible to a query at absolute position t:
// j is visible iff (j + 1) * m - 1 < t - W + 1.
__device__ __forceinline__ int visible_entries(long long t, int m, int W, int Nc)
{
    long long a = t - W + 1;
    if (a <= 0)
        return 0;
    long long n = a / m;
    return n < Nc ? (int)n : Nc;
}

// ------------------------------------------------------------------------
// Scores on CUDA cores.  CTA tile: kRows query rows x kKeys entries.  The
// key tile and the query tile are staged in shared memory as fp32 (rows of
// the key tile padded by one float so that 16 different keys read by a warp
// fall in distinct banks).
// ------------------------------------------------------------------------
constexpr int kScRows = 16;
constexpr int kScKeys = 128;
constexpr int kScThreads = 256;

__global__ void __launch_bounds__(kScThreads)
index_scores_simt(const __nv_bfloat16 *__restrict__ qi, const float *__restrict__ wi,
                  const __nv_bfloat16 *__restrict__ kic, float *__restrict__ scores, int B, int Lq,
                  int Hi, int di, int Nc, int m, int W, const int32_t *__restrict__ q_pos)
{
    extern __shared__ __align__(16) float sm_sc[];
    const int ldk = di + 1;
    float *sk = sm_sc;                                 // [kScKeys][di + 1]
    float *sq = sk + kScKeys * ldk;                    // [kScRows][Hi][di]
    float *sw = sq + kScRows * Hi * di;                // [kScRows][Hi]
    int *snv = reinterpret_cast<int *>(sw + kScRows * Hi);  // [kScRows]

    const int b = blockIdx.z;
    const int r0 = blockIdx.y * kScRows;
    const int k0 = blockIdx.x * kScKeys;
    const int tid = threadIdx.x;

    if (tid < kScRows) {
        int t = r0 + tid;
        int nv = 0;
        if (t < Lq) {
            long long pos = q_pos ? q_pos[(size_t)b * Lq + t] : t;
            nv = visible_entries(pos, m, W, Nc);
        }
        snv[tid] = nv;
    }
    __syncthreads();
    int nv_max = 0;
#pragma unroll 1
    for (int r = 0; r < kScRows; ++r)
        nv_max = max(nv_max, snv[r]);
    if (k0 >= nv_max)
        return;  // no row of this tile sees any entry of this key tile

    // stage keys (bf16 -> fp32), 8 channels per thread step
    const int kd8 = di / 8;
    for (int e = tid; e < kScKeys * kd8; e += kScThreads) {
        int kk = e / kd8, c8 = e % kd8;
        int s = k0 + kk;
        float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (s < Nc) {
            uint4 u = __ldg(reinterpret_cast<const uint4 *>(kic + ((size_t)b * Nc + s) * di + c8 * 8));
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 f = __bfloat1622float2(h2[q]);
                v[2 * q] = f.x;
                v[2 * q + 1] = f.y;
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
            sk[kk * ldk + c8 * 8 + q] = v[q];
    }
    const int qd8 = Hi * di / 8;
    for (int e = tid; e < kScRows * qd8; e += kScThreads) {
        int r = e / qd8, c8 = e % qd8;
        int t = r0 + r;
        float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (t < Lq) {
            uint4 u = __ldg(reinterpret_cast<const uint4 *>(qi + ((size_t)b * Lq + t) * Hi * di + c8 * 8));
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 f = __bfloat1622float2(h2[q]);
                v[2 * q] = f.x;
                v[2 * q + 1] = f.y;
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
            sq[r * Hi * di + c8 * 8 + q] = v[q];
    }
    for (int e = tid; e < kScRows * Hi; e += kScThreads) {
        int r = e / Hi, h = e % Hi;
        int t = r0 + r;
        sw[e] = t < Lq ? wi[((size_t)b * Lq + t) * Hi + h] : 0.f;
    }
    __syncthreads();

    // thread -> (row, key lane); each thread scores kScKeys / 16 keys of one row
    const int r = tid / 16;
    const int kl = tid % 16;
    const int t = r0 + r;
    if (t >= Lq)
        return;
    const int nv = snv[r];
    float *out = scores + ((size_t)b * Lq + t) * Nc;
    for (int kk = kl; kk < kScKeys; kk += 16) {
        const int s = k0 + kk;
        if (s >= nv)
            break;
        float I = 0.f;
        for (int h = 0; h < Hi; ++h) {
            const float *qv = sq + (r * Hi + h) * di;
            const float *kv = sk + kk * ldk;
            float dot = 0.f;
            for (int c = 0; c < di; ++c)
                dot = fmaf(qv[c], kv[c], dot);
            I = fmaf(sw[r * Hi + h], fmaxf(dot, 0.f), I);
        }
        out[s] = I;
    }
}

cudaError_t launch_index_scores_simt(const void *qi, const float *wi, const void *kic, float *scores,
                                     int B, int Lq, int Hi, int di, int Nc, int m, int W,
                                     const int32_t *q_pos, cudaStream_t stream)
{
    const size_t smem = sizeof(float) * ((size_t)kScKeys * (di + 1) + (size_t)kScRows * Hi * di +
                                         (size_t)kScRows * Hi) +
                        sizeof(int) * kScRows;
    cudaError_t e = cudaFuncSetAttribute(index_scores_simt,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid((Nc + kScKeys - 1) / kScKeys, (Lq + kScRows - 1) / kScRows, B);
    index_scores_simt<<<grid, kScThreads, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(qi), wi, static_cast<const __nv_bfloat16 *>(kic), scores,
        B, Lq, Hi, di, Nc, m, W, q_pos);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------
// Exact top-K by radix select.
// ------------------------------------------------------------------------
constexpr int kTkThreads = 512;
constexpr int kTkWarps = kTkThreads / 32;

// Larger float -> larger unsigned key; -0.0 is folded onto +0.0 first so that
// equal scores give equal keys.
__device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum (in thread order) of one value per thread.
__device__ __forceinline__ int block_excl_scan(int v, int *warp_tot, int *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off)
            x += y;
    }
    if (lane == 31)
        warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = lane < kTkWarps ? warp_tot[lane] : 0;
        int inc = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off)
                inc += y;
        }
        if (lane < kTkWarps)
            warp_tot[lane] = inc - w;  // exclusive warp offsets
        if (lane == kTkWarps - 1)
            *total = inc;
    }
    __syncthreads();
    int r = warp_tot[wid] + x - v;
    __syncthreads();
    return r;
}

// Histogram the digit (key >> shift) & (NB - 1) of the keys whose bits under
// `pmask` equal `prefix`; then find the digit holding the `need`-th largest
// such key.  Returns that digit; *above receives the number of matching keys
// with a larger digit.
template <int BITS>
__device__ int radix_pass(const uint32_t *keys, int n, uint32_t prefix, uint32_t pmask, int shift,
                          int need, int *hist, int *warp_tot, int *scratch, int *above)
{
    constexpr int NB = 1 << BITS;
    for (int i = threadIdx.x; i < NB; i += kTkThreads)
        hist[i] = 0;
    __syncthreads();
    const int n_round = (n + kTkThreads - 1) / kTkThreads * kTkThreads;
    for (int i = threadIdx.x; i < n_round; i += kTkThreads) {
        uint32_t k = i < n ? keys[i] : 0u;
        bool match = i < n && (k & pmask) == prefix;
        unsigned active = __ballot_sync(0xffffffffu, match);
        if (match) {
            int dg = (int)((k >> shift) & (NB - 1));
            unsigned peers = __match_any_sync(active, dg);
            if ((__ffs(peers) - 1) == (int)(threadIdx.x & 31))
                atomicAdd(&hist[dg], __popc(peers));
        }
    }
    __syncthreads();
    // thread t owns PER consecutive bins counted down from the top digit
    constexpr int PER = (NB + kTkThreads - 1) / kTkThreads;
    int mine = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        int bin = NB - 1 - ((int)threadIdx.x * PER + q);
        if (bin >= 0)
            mine += hist[bin];
    }
    const int ex = block_excl_scan(mine, warp_tot, scratch);  // keys in higher runs
    if (ex < need && ex + mine >= need) {
        int acc = ex;
        for (int q = 0; q < PER; ++q) {
            int bin = NB - 1 - ((int)threadIdx.x * PER + q);
            int c = hist[bin];
            if (acc + c >= need) {
                scratch[1] = bin;
                scratch[2] = acc;
                break;
            }
            acc += c;
        }
    }
    __syncthreads();
    const int dg = scratch[1];
    *above = scratch[2];
    __syncthreads();
    return dg;
}

__global__ void __launch_bounds__(kTkThreads)
topk_radix(const float *__restrict__ scores, int B, int Lq, int Nc, int m, int W, int K,
           const int32_t *__restrict__ q_pos, int32_t *__restrict__ idx_out,
           float *__restrict__ sel_scores)
{
    extern __shared__ __align__(16) uint32_t sm_tk[];
    __shared__ int hist[4096];
    __shared__ int warp_tot[32];
    __shared__ int scratch[4];

    const int row = blockIdx.x;  // b * Lq + t
    const int b = row / Lq;
    const int t = row % Lq;
    const long long pos = q_pos ? q_pos[row] : t;
    const int n = visible_entries(pos, m, W, Nc);
    const int keff = n < K ? n : K;
    const float *src = scores + (size_t)row * Nc;
    int32_t *dst = idx_out + (size_t)row * K;
    float *dsc = sel_scores ? sel_scores + (size_t)row * K : nullptr;
    (void)b;

    if (keff == n) {  // every visible entry is selected
        for (int i = threadIdx.x; i < K; i += kTkThreads) {
            dst[i] = i < n ? i : -1;
            if (dsc)
                dsc[i] = i < n ? src[i] : -INFINITY;
        }
        return;
    }

    uint32_t *keys = sm_tk;
    for (int i = threadIdx.x; i < n; i += kTkThreads)
        keys[i] = order_key(src[i]);
    __syncthreads();

    int need = keff, above;
    uint32_t prefix = 0, pmask = 0;
    int dg = radix_pass<12>(keys, n, prefix, pmask, 20, need, hist, warp_tot, scratch, &above);
    need -= above;
    prefix |= (uint32_t)dg << 20;
    pmask |= 0xFFFu << 20;
    dg = radix_pass<10>(keys, n, prefix, pmask, 10, need, hist, warp_tot, scratch, &above);
    need -= above;
    prefix |= (uint32_t)dg << 10;
    pmask |= 0x3FFu << 10;
    dg = radix_pass<10>(keys, n, prefix, pmask, 0, need, hist, warp_tot, scratch, &above);
    need -= above;
    const uint32_t T = prefix | (uint32_t)dg;  // key of the K-th largest score
    // select: every key > T, plus the `need` lowest-index keys == T

    // contiguous chunk per thread (odd length: conflict-free shared reads)
    int C = (n + kTkThreads - 1) / kTkThreads;
    C |= 1;
    const int i0 = threadIdx.x * C;
    const int i1 = min(n, i0 + C);
    int gt = 0, eq = 0;
    for (int i = i0; i < i1; ++i) {
        uint32_t k = keys[i];
        gt += k > T;
        eq += k == T;
    }
    int eq_before = block_excl_scan(eq, warp_tot, scratch);
    int take_eq = min(eq, max(0, need - eq_before));
    int sel = gt + take_eq;
    int out_base = block_excl_scan(sel, warp_tot, scratch);
    int e_seen = 0;
    for (int i = i0; i < i1; ++i) {
        uint32_t k = keys[i];
        bool pick = k > T;
        if (k == T) {
            pick = e_seen < take_eq;
            ++e_seen;
        }
        if (pick) {
            dst[out_base] = i;
            if (dsc)
                dsc[out_base] = src[i];
            ++out_base;
        }
    }
    for (int i = keff + threadIdx.x; i < K; i += kTkThreads) {
        dst[i] = -1;
        if (dsc)
            dsc[i] = -INFINITY;
    }
}

// Block-wide exclusive prefix sum (thread order) for NT threads.

template <int NT>
__device__ __forceinline__ int blk_excl_scan(int v, int *warp_tot)
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off)
            x += y;
    }
    if (lane == 31)
        warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = lane < NW ? warp_tot[lane] : 0;
        int inc = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off)
                inc += y;
        }
        if (lane < NW)
            warp_tot[lane] = inc - w;
    }
    __syncthreads();
    const int r = warp_tot[wid] + x - v;
    __syncthreads();
    return r;
}

// Block-wide max / sum over NT threads (every thread gets the result).
template <int NT>
__device__ __forceinline__ uint32_t blk_max_u32(uint32_t v, int *tmp)
{
    constexpr int NW = NT / 32;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
    if ((threadIdx.x & 31) == 0)
        tmp[threadIdx.x >> 5] = (int)v;
    __syncthreads();
    uint32_t r = 0u;
#pragma unroll
    for (int w = 0; w < NW; ++w)
        r = max(r, (uint32_t)tmp[w]);
    __syncthreads();
    return r;
}

template <int NT>
__device__ __forceinline__ int blk_sum_i32(int v, int *tmp)
{
    constexpr int NW = NT / 32;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0)
        tmp[threadIdx.x >> 5] = v;
    __syncthreads();
    int r = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w)
        r += tmp[w];
    __syncthreads();
    return r;
}

// ------------------------------------------------------------------------
// Exact top-K, row in registers, histogram select.  Thread t owns entries
// [t * KPT, (t + 1) * KPT) of its row.  The K-th largest order key is found
// by narrowing a key interval [lo, hi] that holds it, starting from the whole
// key range: each round histograms the candidates (keys inside the interval)
// on the offset (key - lo) >> sh, sh chosen so that the interval spans at
// most 2048 shared bins, and a descending scan of the bins finds the one that
// holds the K-th key; that bin becomes the next interval.  From the full
// range the digits are the key's bits 21-31, 10-20 and 0-9, so three rounds
// reach a single key; the search stops early when the bin is taken whole.
// One block scan of the packed (greater, equal) counts then places each
// selected entry in index order; ties at the threshold go to the lowest
// indices.
// ------------------------------------------------------------------------
constexpr int kHbBins = 2048;

__device__ __forceinline__ float key_to_score(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <int NT, int KPT>
__global__ void __launch_bounds__(NT)
topk_hist(const float *__restrict__ scores, int Lq, int Nc, int m, int W, int K,
          const int32_t *__restrict__ q_pos, int32_t *__restrict__ idx_out,
          float *__restrict__ sel_scores)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
    constexpr int PER = kHbBins / NT;          // bins per thread in the descending scan
    static_assert(PER >= 1 && kHbBins % NT == 0, "");
    __shared__ int hist[2][kHbBins];
    __shared__ int s_scan[32];
    __shared__ int s_sel[3];

    const int row = blockIdx.x;
    const int t = row % Lq;
    const long long pos = q_pos ? q_pos[row] : t;
    const int n = visible_entries(pos, m, W, Nc);
    const int keff = n < K ? n : K;
    const float *src = scores + (size_t)row * Nc;
    int32_t *dst = idx_out + (size_t)row * K;
    float *dsc = sel_scores ? sel_scores + (size_t)row * K : nullptr;

    if (keff == n) {  // every visible entry is selected
        for (int i = threadIdx.x; i < K; i += NT) {
            dst[i] = i < n ? i : -1;
            if (dsc)
                dsc[i] = i < n ? src[i] : -INFINITY;
        }
        return;
    }

    const int i0 = threadIdx.x * KPT;
    uint32_t key[KPT];
    if ((Nc & 3) == 0 && i0 + KPT <= n) {
#pragma unroll
        for (int u = 0; u < KPT; u += 4) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(src + i0 + u));
            key[u] = order_key(v.x);
            key[u + 1] = order_key(v.y);
            key[u + 2] = order_key(v.z);
            key[u + 3] = order_key(v.w);
        }
    } else {
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            key[u] = (i0 + u < n) ? order_key(__ldg(src + i0 + u)) : 0u;
    }
    const int nv = min(KPT, max(0, n - i0));   // this thread's visible entries
    for (int i = threadIdx.x; i < kHbBins; i += NT)
        hist[0][i] = 0;
    __syncthreads();   // hist[0] cleared
    uint32_t lo = 0u, hi = 0xFFFFFFFFu;

    int need = keff;
    // Start from the keys within a factor 16 of the row's largest score (the
    // 2^25 order keys up to the top key): the K-th largest nearly always lies
    // there, and bins over that window spread the keys, where over the whole
    // key range a row's scores share a few exponents and pile into a handful
    // of bins (their atomics serialise).  Otherwise the rest of the range.
    {
        uint32_t kmax = 0u;
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            if (u < nv)
                kmax = max(kmax, key[u]);
        kmax = blk_max_u32<NT>(kmax, s_scan);
        const uint32_t wlo = kmax >= (1u << 25) ? kmax - ((1u << 25) - 1u) : 0u;
        int cnt = 0;
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            cnt += (u < nv && key[u] >= wlo) ? 1 : 0;
        cnt = blk_sum_i32<NT>(cnt, s_scan);
        if (cnt >= need) {
            lo = wlo;
            hi = kmax;
        } else {              // wlo > 0: some visible keys lie below it
            need -= cnt;
            hi = wlo - 1u;
        }
    }
    bool whole = false;
    uint32_t T = lo;   // the K-th key (or, when whole, the lowest selected key)
#pragma unroll 1
    for (int rnd = 0; lo < hi; ++rnd) {
        const uint32_t span = hi - lo;                       // >= 1
        const int bits = 32 - __clz(span);                   // bits of the largest offset
        const int sh = bits > 11 ? bits - 11 : 0;
        int *h = hist[rnd & 1];
        int *hn = hist[(rnd + 1) & 1];
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            if (u < nv && key[u] >= lo && key[u] <= hi)
                atomicAdd(&h[(key[u] - lo) >> sh], 1);
        for (int i = threadIdx.x; i < kHbBins; i += NT)
            hn[i] = 0;         // the next round's histogram (last read a round ago)
        __syncthreads();
        int mine = 0;
#pragma unroll
        for (int q = 0; q < PER; ++q)
            mine += h[kHbBins - 1 - ((int)threadIdx.x * PER + q)];
        const int ex = blk_excl_scan<NT>(mine, s_scan);   // candidates in higher bins
        if (ex < need && ex + mine >= need) {
            int acc = ex;
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int bin = kHbBins - 1 - ((int)threadIdx.x * PER + q);
                const int c = h[bin];
                if (acc + c >= need) {
                    s_sel[0] = bin;
                    s_sel[1] = acc;
                    s_sel[2] = c;
                    break;
                }
                acc += c;
            }
        }
        __syncthreads();
        const uint32_t bin = (uint32_t)s_sel[0];
        need -= s_sel[1];
        const int cnt = s_sel[2];
        const uint32_t nlo = lo + (bin << sh);
        const uint32_t nhi = (uint32_t)min((unsigned long long)hi,
                                           (unsigned long long)nlo + ((1ull << sh) - 1ull));
        lo = nlo;
        hi = nhi;
        T = lo;
        if (cnt == need) {     // the whole bin is selected: every key >= lo
            whole = true;
            break;
        }
    }
    // whole: every key >= T; else every key > T and the `need` lowest-index
    // keys equal to T (lo == hi == T)
    int gt = 0, eq = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        if (u < nv) {
            gt += whole ? key[u] >= T : key[u] > T;
            eq += !whole && key[u] == T;
        }
    }
    const int exs = blk_excl_scan<NT>((gt << 16) | eq, s_scan);
    const int eq_before = exs & 0xffff;
    const int take_eq = min(eq, max(0, need - eq_before));
    int out = (exs >> 16) + min(eq_before, need);
    int e_seen = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        if (u < nv) {
            bool pick = whole ? key[u] >= T : key[u] > T;
            if (!whole && key[u] == T) {
                pick = e_seen < take_eq;
                ++e_seen;
            }
            if (pick) {
                dst[out] = i0 + u;
                if (dsc)
                    dsc[out] = key_to_score(key[u]);
                ++out;
            }
        }
    }
    for (int i = keff + threadIdx.x; i < K; i += NT) {
        dst[i] = -1;
        if (dsc)
            dsc[i] = -INFINITY;
    }
}

cudaError_t launch_topk_radix(const float *scores, int B, int Lq, int Nc, int m, int W, int K,
                              const int32_t *q_pos, int32_t *idx, float *sel_scores,
                              cudaStream_t stream)
{
    // Rows of up to 16384 entries: keys in registers, histogram select
    // (512 threads per row measured faster than 128 or 256 on 8192-entry
    // rows); longer rows: the shared-memory radix select.
    const unsigned rows = (unsigned)B * (unsigned)Lq;
#define HYB_TOPK_HIST(NT, KPT)                                                                     \
    do {                                                                                        \
        return launch_pdl(topk_hist<NT, KPT>, dim3(rows), dim3(NT), 0, stream, scores, Lq, Nc, m, W, K,  \
                          q_pos, idx, sel_scores);                                              \
    } while (0)
    if (Nc <= 512 * 8)
        HYB_TOPK_HIST(512, 8);
    if (Nc <= 512 * 16)
        HYB_TOPK_HIST(512, 16);
    // One wave of long rows (decode: 64 rows of 16384 entries): 1024 threads
    // per row, 16 keys each (decode indexer + top-K 0.052 against 0.056 ms
    // with 512 threads x 32)
    if (Nc <= 1024 * 16 && rows <= 148u)
        HYB_TOPK_HIST(1024, 16);
    if (Nc <= 512 * 32)
        HYB_TOPK_HIST(512, 32);
#undef HYB_TOPK_HIST
    const size_t smem = sizeof(uint32_t) * (size_t)Nc;
    cudaError_t e = cudaFuncSetAttribute(topk_radix, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    topk_radix<<<B * Lq, kTkThreads, smem, stream>>>(scores, B, Lq, Nc, m, W, K, q_pos, idx,
                                                     sel_scores);
    return cudaGetLastError();
}

}  // namespace hyb

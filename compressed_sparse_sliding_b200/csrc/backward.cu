// backward.cu -- gradients for training (Tiny-R2 README, "Training"): the
// hybrid attention step and block_merge.  The top-K selection is taken as
// fixed (the pages define no gradient for it).
//
// Attention, per query row with key set S (the forward's: selected or all
// visible compressed entries, and the raw window), with the forward's lse:
//     P_j = exp(scale q.k_j - lse),  dP_j = dO.v_j,  D = dO.o = sum_j P_j dP_j
//     dS_j = P_j (dP_j - D)
//     dq = scale sum_j dS_j k_j,  dk_j += scale dS_j q,  dv_j += P_j dO
// One CTA per (token, KV head): warp w holds heads w, w + 8, ... of the group
// (q, dO and the dq accumulators in registers; lane = d/32 channels); warps
// without a head (groups of fewer than eight) only take part in the sums.  Keys go
// four or eight at a time (NK): each warp adds its heads' dk / dv parts into
// shared memory, then the CTA adds the keys' sums to the fp32 gradients with one
// vector reduction per four channels (the form for problems the tensor-core
// passes do not take: CSA selections, d = 64, decode positions).
//
// block_merge, c_j = sum_i P[i] x_{jm+i} with P = softmax over i of w (per
// channel):  dx_{jm+i} += P[i] dc_j  (each raw row belongs to one block, so
// plain read-modify-write), dw[i] = P[i] (G[i] - sum_k P[k] G[k]) with
// G[i] = sum over blocks, batches, heads of dc_j x_{jm+i}; a CTA owns 32
// channels and eight rows (more when the grid would be too tall), reduces its
// share of G in shared memory and
// adds it to a global G with one atomic per (i, channel); a last small
// kernel forms dw from G.
#include "common.cuh"

namespace hyb {

constexpr int kBwWarps = 8;
// Keys per shared-memory round: NK (4 or 8), partials 2 x NK x 4 KB in dynamic shared memory.

struct BwdParams {
    int B, Lq, Lkv, Hq, Hkv, g, d, Nc, m, W, topk;
    int comp_only;     // 1: the window keys are another pass's (the tensor-core one): skip them
                       // here and add this pass's part to dq instead of storing it
    float scale;
    const int32_t *q_pos, *kv_pos0, *idx;
    const __nv_bfloat16 *q, *kc, *vc, *kr, *vr, *o, *dout;
    const float *lse;
    float *dq, *dkc, *dvc, *dkr, *dvr;
};

__device__ __forceinline__ float bw_warp_sum(float v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}


// The 2 HPW per-lane partial dot products of a key (q_e . k and dO_e . v over
// this lane's CPL channels, e < HPW) summed over the warp: a halving butterfly
// (each step a lane keeps the half of its values named by its lane bit and adds
// the partner's copy of it: 2 HPW - 1 shuffles) leaves each lane one value's
// partial over its group, plain steps finish the sums, and 2 HPW shuffles hand
// every total to every lane -- against 5 shuffles per value one by one.
template <int HPW, int CPL>
__device__ __forceinline__ void bw_multi_sum_impl(const float (&qv)[HPW][CPL], const float (&dov)[HPW][CPL],
                                                  const float (&kv)[CPL], const float (&vv)[CPL],
                                                  float (&out)[2 * HPW])
{
    constexpr int NV = 2 * HPW;
    const int lane = threadIdx.x & 31;
    float v[NV];
#pragma unroll
    for (int e = 0; e < HPW; ++e) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            a = fmaf(qv[e][c], kv[c], a);
            b = fmaf(dov[e][c], vv[c], b);
        }
        v[e] = a;
        v[HPW + e] = b;
    }
    // halving steps over lane bits 4, 3, ...: after them v[0] holds value
    // idx(lane) = the lane's top log2(NV) bits read as a binary number
    int off = 16;
#pragma unroll
    for (int n = NV; n > 1; n >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float t = v[0];
#pragma unroll
    for (; off > 0; off >>= 1)
        t += __shfl_xor_sync(0xffffffffu, t, off);
    // value j sits in the lanes whose top bits spell j
    constexpr int LOGNV = NV == 2 ? 1 : NV == 4 ? 2 : NV == 8 ? 3 : 4;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        int src = 0;
#pragma unroll
        for (int bit = 0; bit < LOGNV; ++bit)
            if (j & (1 << (LOGNV - 1 - bit)))
                src |= 16 >> bit;
        out[j] = __shfl_sync(0xffffffffu, t, src);
    }
}

template <int CPL, int HPW, int NK>
// Four heads per warp (32-head groups): capped for three blocks per SM, which
// measured faster than two blocks with no spill
__global__ void __launch_bounds__(32 * kBwWarps, HPW == 4 ? 3 : 1)
attn_bwd_kernel(const BwdParams p)
{
    // item = (b, t, KV head)
    const long long item = blockIdx.x;
    const int kvh = (int)(item % p.Hkv);
    const long long bt = item / p.Hkv;
    const int b = (int)(bt / p.Lq), t = (int)(bt % p.Lq);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = 32 * CPL;
    const long long pos = p.q_pos ? p.q_pos[bt] : t;
    const long long kv0 = p.kv_pos0 ? p.kv_pos0[b] : 0;
    long long lo = pos - p.W + 1;
    if (lo < 0)
        lo = 0;
    lo -= kv0;
    if (lo < 0)
        lo = 0;
    long long hi = pos - kv0;
    if (hi > p.Lkv - 1)
        hi = p.Lkv - 1;
    const int nwin = (!p.comp_only && p.W > 0 && hi >= lo) ? (int)(hi - lo + 1) : 0;
    const long long wstart = pos - p.W + 1;
    int nvis = 0;
    if (wstart > 0)
        nvis = (int)min((long long)p.Nc, wstart / p.m);
    const int ncomp = p.idx ? p.topk : nvis;

    // this warp's heads: h = warp + kBwWarps * e
    const float scale_log2 = p.scale * 1.4426950408889634f;
    float qv[HPW][CPL], dov[HPW][CPL], dqv[HPW][CPL], lse[HPW], Dh[HPW];
#pragma unroll
    for (int e = 0; e < HPW; ++e) {
        const int h = warp + kBwWarps * e;
        const bool on = h < p.g;
        const size_t row = ((size_t)bt * p.Hq + (size_t)kvh * p.g + (on ? h : 0)) * d + lane * CPL;
        float od = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            qv[e][c] = on ? __bfloat162float(p.q[row + c]) : 0.f;
            dov[e][c] = on ? __bfloat162float(p.dout[row + c]) : 0.f;
            od += on ? dov[e][c] * __bfloat162float(p.o[row + c]) : 0.f;
            dqv[e][c] = 0.f;
        }
        Dh[e] = bw_warp_sum(od);
        // the row's lse in base-2 units (+inf for a row without keys: P = 0)
        const float l = on ? p.lse[((size_t)b * p.Hq + (size_t)kvh * p.g + h) * p.Lq + t] : -INFINITY;
        lse[e] = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
    }

    extern __shared__ __align__(16) float bw_partials[];
    float(*sdk)[kBwWarps][128] = reinterpret_cast<float(*)[kBwWarps][128]>(bw_partials);   // [NK][warps][128]
    float(*sdv)[kBwWarps][128] = reinterpret_cast<float(*)[kBwWarps][128]>(bw_partials + NK * kBwWarps * 128);
    __shared__ long long srow[NK];     // source row of each key (-1: none)
    __shared__ int scomp[NK];          // compressed (1) or raw (0)
    const int total = ncomp + nwin;
    const int nw = p.g < kBwWarps ? p.g : kBwWarps;   // warps holding a head
    for (int k0 = 0; k0 < total; k0 += NK) {
        if (threadIdx.x < NK) {
            const int kk = k0 + threadIdx.x;
            long long r = -1;
            int comp = 0;
            if (kk < ncomp) {
                comp = 1;
                int j = p.idx ? p.idx[(size_t)bt * p.topk + kk] : kk;
                if (p.idx && j >= p.Nc)
                    set_error(HYB_ERR_DEVICE_BOUNDS);
                const bool v = j >= 0 && j < p.Nc && ((long long)(j + 1) * p.m - 1 < wstart);
                r = v ? ((long long)b * p.Nc + j) * p.Hkv + kvh : -1;
            } else if (kk < total) {
                r = ((long long)b * p.Lkv + lo + (kk - ncomp)) * p.Hkv + kvh;
            }
            srow[threadIdx.x] = r;
            scomp[threadIdx.x] = comp;
        }
        __syncthreads();
#pragma unroll 1
        for (int u = 0; u < NK && warp < nw; ++u) {
            const long long r = srow[u];
            float dkp[CPL], dvp[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                dkp[c] = 0.f;
                dvp[c] = 0.f;
            }
            if (r >= 0) {
                const __nv_bfloat16 *kp = (scomp[u] ? p.kc : p.kr) + r * d + lane * CPL;
                const __nv_bfloat16 *vp = (scomp[u] ? p.vc : p.vr) + r * d + lane * CPL;
                // this lane's CPL channels of the key and value rows in one load each
                // (rows are 256-byte aligned; CPL = 4 or 2 bf16 = 8 or 4 bytes)
                float kv[CPL], vv[CPL];
                static_assert(CPL == 2 || CPL == 4, "lane channel counts of d = 64 and 128");
                if constexpr (CPL == 4) {
                    const uint2 ka = *reinterpret_cast<const uint2 *>(kp);
                    const uint2 va = *reinterpret_cast<const uint2 *>(vp);
                    const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ka.x));
                    const float2 k1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ka.y));
                    const float2 v0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&va.x));
                    const float2 v1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&va.y));
                    kv[0] = k0.x; kv[1] = k0.y; kv[2] = k1.x; kv[3] = k1.y;
                    vv[0] = v0.x; vv[1] = v0.y; vv[2] = v1.x; vv[3] = v1.y;
                } else {
                    const uint32_t ka = *reinterpret_cast<const uint32_t *>(kp);
                    const uint32_t va = *reinterpret_cast<const uint32_t *>(vp);
                    const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ka));
                    const float2 v0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&va));
                    kv[0] = k0.x; kv[1] = k0.y;
                    vv[0] = v0.x; vv[1] = v0.y;
                }
                // the warp's 2 HPW dot products (scores, then dP) reduced together
                float sums[2 * HPW];
                bw_multi_sum_impl<HPW, CPL>(qv, dov, kv, vv, sums);
#pragma unroll
                for (int e = 0; e < HPW; ++e) {
                    if (warp + kBwWarps * e >= p.g)
                        continue;
                    const float s = sums[e], dp = sums[HPW + e];
                    const float pr = ex2_approx(fmaf(s, scale_log2, -lse[e]));
                    const float ds = pr * (dp - Dh[e]);
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        dqv[e][c] = fmaf(ds, kv[c], dqv[e][c]);
                        dkp[c] = fmaf(ds, qv[e][c], dkp[c]);
                        dvp[c] = fmaf(pr, dov[e][c], dvp[c]);
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                sdk[u][warp][lane * CPL + c] = dkp[c];
                sdv[u][warp][lane * CPL + c] = dvp[c];
            }
        }
        __syncthreads();
        // thread -> (key, four channels) sums over the warps, one vector
        // reduction each for dk and dv
        for (int e = threadIdx.x; e < NK * d / 4; e += 32 * kBwWarps) {
            const int u = e / (d / 4), c = (e % (d / 4)) * 4;
            const long long r = srow[u];
            if (r < 0)
                continue;
            float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
            for (int w = 0; w < nw; ++w) {
                const float4 a = *reinterpret_cast<const float4 *>(&sdk[u][w][c]);
                const float4 b = *reinterpret_cast<const float4 *>(&sdv[u][w][c]);
                sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
                sv.x += b.x; sv.y += b.y; sv.z += b.z; sv.w += b.w;
            }
            float *dk = (scomp[u] ? p.dkc : p.dkr) + r * d + c;
            float *dv = (scomp[u] ? p.dvc : p.dvr) + r * d + c;
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dk), "f"(sk.x * p.scale),
                         "f"(sk.y * p.scale), "f"(sk.z * p.scale), "f"(sk.w * p.scale)
                         : "memory");
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dv), "f"(sv.x), "f"(sv.y),
                         "f"(sv.z), "f"(sv.w)
                         : "memory");
        }
        __syncthreads();
    }
#pragma unroll
    for (int e = 0; e < HPW; ++e) {
        const int h = warp + kBwWarps * e;
        if (h >= p.g)
            continue;
        const size_t row = ((size_t)bt * p.Hq + (size_t)kvh * p.g + h) * d + lane * CPL;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
            p.dq[row + c] = p.comp_only ? p.dq[row + c] + dqv[e][c] * p.scale : dqv[e][c] * p.scale;
    }
}

// One launch with NK keys per round (dynamic shared memory for the partials).
template <int CPL, int HPW, int NK>
static cudaError_t launch_attn_bwd_k(const BwdParams &p, long long items, cudaStream_t stream)
{
    const size_t smem = (size_t)2 * NK * kBwWarps * 128 * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<CPL, HPW, NK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    attn_bwd_kernel<CPL, HPW, NK><<<(unsigned)items, 32 * kBwWarps, smem, stream>>>(p);
    return cudaGetLastError();
}

// Heads per warp by group width; groups wider than 16 take eight keys per
// round (half the block barriers, and every thread busy in the reduction),
// the narrower ones four (more blocks per SM).
template <int CPL>
static cudaError_t launch_attn_bwd_c(const BwdParams &p, long long items, cudaStream_t stream)
{
    const int hpw = (p.g + kBwWarps - 1) / kBwWarps;
    if (hpw <= 1)
        return launch_attn_bwd_k<CPL, 1, 4>(p, items, stream);
    if (hpw <= 2)
        return launch_attn_bwd_k<CPL, 2, 4>(p, items, stream);
    if (hpw <= 4)
        return launch_attn_bwd_k<CPL, 4, 8>(p, items, stream);
    return launch_attn_bwd_k<CPL, 8, 8>(p, items, stream);
}

cudaError_t launch_attn_bwd(const BwdParams &p, cudaStream_t stream)
{
    const long long items = (long long)p.B * p.Lq * p.Hkv;
    if (items <= 0)
        return cudaSuccess;
    if (items >= (1ll << 31) || p.g > 64)
        return cudaErrorInvalidValue;
    return p.d == 128 ? launch_attn_bwd_c<4>(p, items, stream) : launch_attn_bwd_c<2>(p, items, stream);
}

// ---------------------------------------------------------------- block_merge
// sP[i][lane] = softmax over positions i of w[i, c] for the CTA's channel
// c = 32 blockIdx.x + lane, computed by all eight warps (warp w takes
// positions w, w + 8, ...); sRed: 8 x 32 floats of scratch.
__device__ __forceinline__ void bm_softmax_weights(const float *__restrict__ w, int D, int m, float *sP,
                                                   float *sRed)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = blockIdx.x * 32 + lane;
    float mx = -INFINITY;
    for (int i = warp; i < m; i += 8)
        mx = fmaxf(mx, w[(size_t)i * D + c]);
    sRed[warp * 32 + lane] = mx;
    __syncthreads();
    mx = sRed[lane];
    for (int k = 1; k < 8; ++k)
        mx = fmaxf(mx, sRed[k * 32 + lane]);
    __syncthreads();
    float den = 0.f;
    for (int i = warp; i < m; i += 8) {
        const float e = expf(w[(size_t)i * D + c] - mx);
        sP[i * 32 + lane] = e;
        den += e;
    }
    sRed[warp * 32 + lane] = den;
    __syncthreads();
    den = 0.f;
    for (int k = 0; k < 8; ++k)
        den += sRed[k * 32 + lane];
    const float inv = 1.f / den;
    for (int i = warp; i < m; i += 8)
        sP[i * 32 + lane] *= inv;
    __syncthreads();
}

// grid (dx / 32, row groups of rpc rows, about two CTAs per SM in all); warp
// w of the CTA takes rows w, w + 8, ... of its group; lane = channel.
// Positions go 16 at a time and rows two at a time: the two rows' 32 x and
// dx values are loaded together, dx written back, and the G terms kept in
// registers over the warp's rows, then added to the CTA's G partials in
// shared memory [m][32] (one atomic per position and lane).
__device__ __forceinline__ void bm_rows16(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ dc,
                                          float *__restrict__ dx, const float *sP, int L, int H, int D, int m,
                                          int Nc, long long r, int i0, int c, float (&gacc)[16], bool two)
{
    const int lane = threadIdx.x & 31;
    const size_t istride = (size_t)H * D;
    size_t x0[2];
    float g[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const long long rr = r + 8 * q;
        const int h = (int)(rr % H);
        const long long bj = rr / H;
        const int b = (int)(bj / Nc), j = (int)(bj % Nc);
        const bool on = q == 0 || two;
        g[q] = on ? dc[((size_t)bj * H + h) * D + c] : 0.f;
        x0[q] = (((size_t)b * L + (size_t)j * m + i0) * H + h) * D + c;
    }
    float xv[2][16], dv[2][16];
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int k = 0; k < 16; ++k)
            if ((q == 0 || two) && i0 + k < m) {
                xv[q][k] = __bfloat162float(x[x0[q] + k * istride]);
                dv[q][k] = dx[x0[q] + k * istride];
            }
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int k = 0; k < 16; ++k)
            if ((q == 0 || two) && i0 + k < m) {
                dx[x0[q] + k * istride] = dv[q][k] + sP[(i0 + k) * 32 + lane] * g[q];
                gacc[k] += g[q] * xv[q][k];
            }
}

__global__ void __launch_bounds__(256, 2)
block_merge_bwd_kernel(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ w,
                       const float *__restrict__ dc, float *__restrict__ dx, float *__restrict__ G,
                       int B, int L, int H, int D, int m, int rpc)
{
    extern __shared__ float bm_smem[];
    float *sP = bm_smem;                  // [m][32] softmax weights of the CTA's channels
    float *sG = bm_smem + m * 32;         // [m][32] G partials
    float *sRed = sG + m * 32;            // [8][32]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = blockIdx.x * 32 + lane;
    const int Nc = L / m;
    const long long rows = (long long)B * Nc * H;
    for (int e = threadIdx.x; e < m * 32; e += 256)
        sG[e] = 0.f;
    bm_softmax_weights(w, D, m, sP, sRed);
    const long long r0 = (long long)blockIdx.y * rpc;
    const long long rend = min(r0 + rpc, rows);
    for (int i0 = 0; i0 < m; i0 += 16) {
        float gacc[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
            gacc[k] = 0.f;
        for (long long r = r0 + warp; r < rend; r += 16)
            bm_rows16(x, dc, dx, sP, L, H, D, m, Nc, r, i0, c, gacc, r + 8 < rend);
#pragma unroll
        for (int k = 0; k < 16; ++k)
            if (i0 + k < m)
                atomicAdd(&sG[(i0 + k) * 32 + lane], gacc[k]);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < m * 32; e += 256)
        atomicAdd(&G[(size_t)(e / 32) * D + blockIdx.x * 32 + (e % 32)], sG[e]);
}

constexpr int kBmHeads = 8;   // heads of one position in flight per thread

// Whole-block form (dx / 8 dividing 256, P, G and one block's dc in shared
// memory): a work unit is one compression block (b, j) and a share of its m
// positions; thread t takes channels 8 (t % CG) .. + 7 (CG = dx / 8) and
// positions t / CG, + 256 / CG, ...; for each position it runs over the H
// heads, so CG consecutive threads read 16 contiguous bytes each of x and 32
// of dx (one 256- / 512-byte run at dx = 128).  Each thread owns its
// (position, channel) G partials in shared memory; the CTA adds them to G
// with vector reductions at the end.  Persistent: one CTA per SM.
__global__ void __launch_bounds__(256, 1)
block_merge_bwd_blocks_kernel(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ w,
                              const float *__restrict__ dc, float *__restrict__ dx, float *__restrict__ G,
                              int B, int L, int H, int D, int m, int splits)
{
    extern __shared__ float bm_smem[];
    float *sP = bm_smem;            // [m][D]
    float *sG = sP + m * D;         // [m][D]
    float *sDc = sG + m * D;        // [H][D]
    const int CG = D / 8, PL = 256 / CG;
    const int cg = threadIdx.x % CG, il = threadIdx.x / CG;
    const int c0 = cg * 8;
    const int Nc = L / m;
    for (int c = threadIdx.x; c < D; c += 256) {
        float mx = -INFINITY;
        for (int i = 0; i < m; ++i)
            mx = fmaxf(mx, w[(size_t)i * D + c]);
        float den = 0.f;
        for (int i = 0; i < m; ++i) {
            const float e = expf(w[(size_t)i * D + c] - mx);
            sP[i * D + c] = e;
            den += e;
        }
        const float inv = 1.f / den;
        for (int i = 0; i < m; ++i)
            sP[i * D + c] *= inv;
    }
    for (int e = threadIdx.x; e < m * D; e += 256)
        sG[e] = 0.f;
    const int kpos = (m + PL - 1) / PL;               // positions per thread and block
    const int kper = (kpos + splits - 1) / splits;    // of them per work unit
    const long long units = (long long)B * Nc * splits;
    for (long long u = blockIdx.x; u < units; u += gridDim.x) {
        const long long bj = u / splits;
        const int part = (int)(u % splits);
        __syncthreads();   // the previous unit's sDc reads are done (and sP / sG are set)
        for (int e = threadIdx.x * 4; e < H * D; e += 1024)
            *reinterpret_cast<float4 *>(&sDc[e]) = *reinterpret_cast<const float4 *>(&dc[(size_t)bj * H * D + e]);
        __syncthreads();
        const int b = (int)(bj / Nc), j = (int)(bj % Nc);
        for (int k = part * kper; k < min(kpos, (part + 1) * kper); ++k) {
            const int i = il + PL * k;
            if (i >= m)
                break;
            float pv[8], ga[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                pv[e] = sP[i * D + c0 + e];
                ga[e] = 0.f;
            }
            const size_t base = ((size_t)b * L + (size_t)j * m + i) * H * D + c0;
            for (int h0 = 0; h0 < H; h0 += kBmHeads) {
                uint4 xr[kBmHeads];
                float4 d0[kBmHeads], d1[kBmHeads];
#pragma unroll
                for (int q = 0; q < kBmHeads; ++q) {
                    if (h0 + q < H) {
                        const size_t at = base + (size_t)(h0 + q) * D;
                        xr[q] = *reinterpret_cast<const uint4 *>(x + at);
                        d0[q] = *reinterpret_cast<const float4 *>(dx + at);
                        d1[q] = *reinterpret_cast<const float4 *>(dx + at + 4);
                    }
                }
#pragma unroll
                for (int q = 0; q < kBmHeads; ++q) {
                    if (h0 + q < H) {
                        const size_t at = base + (size_t)(h0 + q) * D;
                        const float *g = &sDc[(h0 + q) * D + c0];
                        const uint32_t xw[4] = {xr[q].x, xr[q].y, xr[q].z, xr[q].w};
                        float xv[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xw[e]));
                            xv[2 * e] = f.x;
                            xv[2 * e + 1] = f.y;
                        }
                        float gv[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            gv[e] = g[e];
                            ga[e] += gv[e] * xv[e];
                        }
                        *reinterpret_cast<float4 *>(dx + at) =
                            make_float4(d0[q].x + pv[0] * gv[0], d0[q].y + pv[1] * gv[1], d0[q].z + pv[2] * gv[2],
                                        d0[q].w + pv[3] * gv[3]);
                        *reinterpret_cast<float4 *>(dx + at + 4) =
                            make_float4(d1[q].x + pv[4] * gv[4], d1[q].y + pv[5] * gv[5], d1[q].z + pv[6] * gv[6],
                                        d1[q].w + pv[7] * gv[7]);
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e)
                sG[i * D + c0 + e] += ga[e];
        }
    }
    __syncthreads();
    for (int e = threadIdx.x * 4; e < m * D; e += 1024)
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(G + e), "f"(sG[e]), "f"(sG[e + 1]),
                     "f"(sG[e + 2]), "f"(sG[e + 3])
                     : "memory");
}

// dw[i, c] = P[i, c] (G[i, c] - sum_k P[k, c] G[k, c]); a CTA per 32 channels,
// warp w takes positions w, w + 8, ...
__global__ void __launch_bounds__(256)
block_merge_dw_kernel(const float *__restrict__ w, const float *__restrict__ G, float *__restrict__ dw, int D,
                      int m)
{
    extern __shared__ float bm_smem[];
    float *sP = bm_smem;          // [m][32]
    float *sRed = sP + m * 32;    // [8][32]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = blockIdx.x * 32 + lane;
    bm_softmax_weights(w, D, m, sP, sRed);
    float pg = 0.f;
    for (int i = warp; i < m; i += 8)
        pg += sP[i * 32 + lane] * G[(size_t)i * D + c];
    sRed[warp * 32 + lane] = pg;
    __syncthreads();
    pg = 0.f;
    for (int k = 0; k < 8; ++k)
        pg += sRed[k * 32 + lane];
    for (int i = warp; i < m; i += 8)
        dw[(size_t)i * D + c] = sP[i * 32 + lane] * (G[(size_t)i * D + c] - pg);
}

// G: m * D floats of workspace, zeroed by the caller.
cudaError_t launch_block_merge_bwd(const void *x, int B, int L, int H, int D, int m, const float *w,
                                   const float *dc, float *dx, float *dw, float *G, cudaStream_t stream,
                                   int num_sms)
{
    const long long rows = (long long)B * (L / m) * H;
    const size_t bsmem = ((size_t)2 * m * D + (size_t)H * D) * sizeof(float);
    const bool al16 = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dx) |
                        reinterpret_cast<uintptr_t>(dc)) & 15u) == 0;
    if (rows > 0 && al16 && D % 8 == 0 && 256 % (D / 8) == 0 && bsmem <= 200 * 1024) {
        // whole-block form: about two work units per SM
        const long long blocks = (long long)B * (L / m);
        const int PL = 256 / (D / 8);
        const int kpos = (m + PL - 1) / PL;
        int splits = (int)((2LL * num_sms + blocks - 1) / blocks);
        if (splits > kpos)
            splits = kpos;
        if (splits < 1)
            splits = 1;
        cudaError_t e = cudaFuncSetAttribute(block_merge_bwd_blocks_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bsmem);
        if (e != cudaSuccess)
            return e;
        const long long units = blocks * splits;
        const int grid = (int)(units < num_sms ? units : num_sms);
        block_merge_bwd_blocks_kernel<<<grid, 256, bsmem, stream>>>(static_cast<const __nv_bfloat16 *>(x), w, dc,
                                                                    dx, G, B, L, H, D, m, splits);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    } else if (rows > 0) {
        // rows per CTA: a multiple of 16 (two per warp and pass) giving about two
        // CTAs per SM over all channel blocks, within the grid's y limit
        const long long cblocks = D / 32;
        long long rpc = (rows * cblocks + 2LL * num_sms - 1) / (2LL * num_sms);
        rpc = (rpc + 15) / 16 * 16;
        while ((rows + rpc - 1) / rpc > 65535)
            rpc += 16;
        const long long groups = (rows + rpc - 1) / rpc;
        const size_t smem = ((size_t)2 * m * 32 + 8 * 32) * sizeof(float);   // 66 KB at m = 256
        cudaError_t e = cudaFuncSetAttribute(block_merge_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess)
            return e;
        dim3 grid(D / 32, (unsigned)groups);
        block_merge_bwd_kernel<<<grid, 256, smem, stream>>>(static_cast<const __nv_bfloat16 *>(x), w, dc, dx,
                                                            G, B, L, H, D, m, (int)rpc);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    block_merge_dw_kernel<<<D / 32, 256, ((size_t)m * 32 + 8 * 32) * sizeof(float), stream>>>(w, G, dw, D, m);
    return cudaGetLastError();
}

}  // namespace hyb

// decode_append.cu -- decode cache maintenance ("deepseek-v4" blog, section 1:
// the window's raw KV and the compressed KV are separate caches with
// different lifetimes; raw rows age out of the window, compressed entries
// live as long as the sequence).  One launch per decode step, one CTA per
// sequence b, with t = t_new[b] the new token's absolute position:
//
//   * the new K and V rows are written twice into a 2W-row ring, at rows
//     t mod W and t mod W + W, so the live window [lo, t], lo = max(0,
//     t - W + 1), is one contiguous run of ring rows starting at lo mod W;
//     kv_pos0[b] = lo - (lo mod W) is the absolute position of ring row 0
//     for that run, which is what the attention kernels take;
//   * the new indexer key (CSA) goes to a W-row ring at row t mod W;
//   * when t + 1 is a multiple of m, block j = (t + 1) / m - 1 (positions
//     j m .. t, all still in the rings because m <= W) becomes compressed
//     entry j of kc / vc (and kic): per channel, a softmax over the block's
//     positions of the block weights, times the rows, summed in fp32 and
//     rounded to bf16 -- the same arithmetic as block_merge.
//
// Work unit = 8 channels (16 bytes) of one of the three rows; units loop over
// the CTA's threads.  Reads of the block come from the ring rows written by
// earlier steps (kernel boundaries order them) and from registers for t.
#include "common.cuh"

namespace hyb {

constexpr int kApThreads = 128;

struct AppendParams {
    int B, Hkv, d, di, m, W, Nc;
    const int32_t *t_new;
    const __nv_bfloat16 *k_new, *v_new, *ki_new;    // [B, Hkv, d], [B, Hkv, d], [B, di]
    const float *wk, *wv, *wib;                      // [m, d], [m, d], [m, di]
    __nv_bfloat16 *k_ring, *v_ring, *ki_ring;        // [B, 2W, Hkv, d], [B, 2W, Hkv, d], [B, W, di]
    __nv_bfloat16 *kc, *vc, *kic;                    // [B, Nc, Hkv, d], [B, Nc, Hkv, d], [B, Nc, di]
    int32_t *kv_pos0;                                // [B] out
};

__global__ void __launch_bounds__(kApThreads)
decode_append_kernel(const AppendParams p)
{
    const int b = blockIdx.x;
    const long long t = p.t_new[b];
    if (t < 0) {
        if (threadIdx.x == 0)
            set_error(HYB_ERR_DEVICE_BOUNDS);
        return;
    }
    const long long lo = t - p.W + 1 > 0 ? t - p.W + 1 : 0;
    if (threadIdx.x == 0)
        p.kv_pos0[b] = (int32_t)(lo - lo % p.W);
    const int slot = (int)(t % p.W);
    const bool close = (t + 1) % p.m == 0;
    const long long j = (t + 1) / p.m - 1;
    if (close && threadIdx.x == 0 && j >= p.Nc)
        set_error(HYB_ERR_DEVICE_BOUNDS);
    const bool emit = close && j < p.Nc;

    const int kv_row = p.Hkv * p.d;                  // elements of one K or V row
    const int nkv = kv_row / 8;
    const int ni = p.ki_new ? p.di / 8 : 0;
    for (int u = threadIdx.x; u < 2 * nkv + ni; u += kApThreads) {
        const int which = u < nkv ? 0 : (u < 2 * nkv ? 1 : 2);   // K, V, indexer key
        const int e = which == 2 ? u - 2 * nkv : u - which * nkv;
        const int dx = which == 2 ? p.di : p.d;
        const int row = which == 2 ? p.di : kv_row;
        const int c0 = (e * 8) % dx;
        const __nv_bfloat16 *src = which == 0 ? p.k_new : (which == 1 ? p.v_new : p.ki_new);
        __nv_bfloat16 *ring = which == 0 ? p.k_ring : (which == 1 ? p.v_ring : p.ki_ring);
        const int rrows = which == 2 ? p.W : 2 * p.W;
        const uint4 nv = *reinterpret_cast<const uint4 *>(src + (size_t)b * row + (size_t)e * 8);
        __nv_bfloat16 *rb = ring + (size_t)b * rrows * row + (size_t)e * 8;
        *reinterpret_cast<uint4 *>(rb + (size_t)slot * row) = nv;
        if (which != 2)
            *reinterpret_cast<uint4 *>(rb + (size_t)(slot + p.W) * row) = nv;
        if (!emit)
            continue;
        // block j: per-channel softmax of the weights over the m positions
        const float *w = which == 0 ? p.wk : (which == 1 ? p.wv : p.wib);
        float mx[8], den[8], acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            mx[q] = -INFINITY;
            den[q] = 0.f;
            acc[q] = 0.f;
        }
        for (int i = 0; i < p.m; ++i)
#pragma unroll
            for (int q = 0; q < 8; ++q)
                mx[q] = fmaxf(mx[q], w[(size_t)i * dx + c0 + q]);
        for (int i = 0; i < p.m; ++i) {
            const long long pos = j * p.m + i;
            const uint4 xv = pos == t ? nv
                                      : *reinterpret_cast<const uint4 *>(rb + (size_t)(pos % p.W) * row);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&xv);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __bfloat1622float2(h2[q]);
                const float e0 = expf(w[(size_t)i * dx + c0 + 2 * q] - mx[2 * q]);
                const float e1 = expf(w[(size_t)i * dx + c0 + 2 * q + 1] - mx[2 * q + 1]);
                den[2 * q] += e0;
                den[2 * q + 1] += e1;
                acc[2 * q] = fmaf(e0, f.x, acc[2 * q]);
                acc[2 * q + 1] = fmaf(e1, f.y, acc[2 * q + 1]);
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0] / den[0], acc[1] / den[1]);
        o.y = pack_bf16x2(acc[2] / den[2], acc[3] / den[3]);
        o.z = pack_bf16x2(acc[4] / den[4], acc[5] / den[5]);
        o.w = pack_bf16x2(acc[6] / den[6], acc[7] / den[7]);
        __nv_bfloat16 *cache = which == 0 ? p.kc : (which == 1 ? p.vc : p.kic);
        *reinterpret_cast<uint4 *>(cache + ((size_t)b * p.Nc + j) * row + (size_t)e * 8) = o;
    }
}

cudaError_t launch_decode_append(const AppendParams &p, cudaStream_t stream)
{
    if (p.B <= 0)
        return cudaSuccess;
    decode_append_kernel<<<p.B, kApThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace hyb

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
    // 4-bit caches instead of kc / vc / kic: codes [rows, dx / 2], (min, scale) [rows]
    uint8_t *kcq, *vcq, *kicq;
    float2 *kqp, *vqp, *kiqp;
};

// 4-bit form of the three caches (codes and per-row (min, scale) as in
// fp4.cu): the ring writes as above; a closing block is merged into the
// bf16 entry exactly as above, then each (entry, head) row is quantized by
// one warp (min / max over the row, then the codes).
__device__ __forceinline__ uint32_t ap_fp4_code(float x, float mn, float sc)
{
    if (!(sc > 0.f))
        return 0u;
    const float r = rintf(__fdiv_rn(__fsub_rn(x, mn), sc));
    return (uint32_t)fminf(fmaxf(r, 0.f), 15.f);
}

__global__ void __launch_bounds__(kApThreads)
decode_append_fp4_kernel(const AppendParams p)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
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

    const int kv_row = p.Hkv * p.d;
    const int nkv = kv_row / 8;
    const int ni = p.ki_new ? p.di / 8 : 0;
    for (int u = threadIdx.x; u < 2 * nkv + ni; u += kApThreads) {
        const int which = u < nkv ? 0 : (u < 2 * nkv ? 1 : 2);
        const int e = which == 2 ? u - 2 * nkv : u - which * nkv;
        const int row = which == 2 ? p.di : kv_row;
        const __nv_bfloat16 *src = which == 0 ? p.k_new : (which == 1 ? p.v_new : p.ki_new);
        __nv_bfloat16 *ring = which == 0 ? p.k_ring : (which == 1 ? p.v_ring : p.ki_ring);
        const int rrows = which == 2 ? p.W : 2 * p.W;
        const uint4 nv = *reinterpret_cast<const uint4 *>(src + (size_t)b * row + (size_t)e * 8);
        __nv_bfloat16 *rb = ring + (size_t)b * rrows * row + (size_t)e * 8;
        *reinterpret_cast<uint4 *>(rb + (size_t)slot * row) = nv;
        if (which != 2)
            *reinterpret_cast<uint4 *>(rb + (size_t)(slot + p.W) * row) = nv;
    }
    if (!emit)
        return;
    // rows to emit: Hkv of K, Hkv of V, one indexer key; warp per row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nrows = 2 * p.Hkv + (p.ki_new ? 1 : 0);
    for (int rw = warp; rw < nrows; rw += kApThreads / 32) {
        const int which = rw < p.Hkv ? 0 : (rw < 2 * p.Hkv ? 1 : 2);
        const int h = which == 2 ? 0 : rw - which * p.Hkv;
        const int dx = which == 2 ? p.di : p.d;
        const int row = which == 2 ? p.di : kv_row;          // elements per position
        const int rrows = which == 2 ? p.W : 2 * p.W;
        const __nv_bfloat16 *src = which == 0 ? p.k_new : (which == 1 ? p.v_new : p.ki_new);
        const __nv_bfloat16 *ring = which == 0 ? p.k_ring : (which == 1 ? p.v_ring : p.ki_ring);
        const float *w = which == 0 ? p.wk : (which == 1 ? p.wv : p.wib);
        const bool active = lane * 8 < dx;
        const int c0 = active ? lane * 8 : 0;
        const size_t coff = (size_t)(which == 2 ? 0 : h * p.d) + c0;   // channel offset in a position
        float val[8];
        {
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
                const uint4 xv = pos == t
                                     ? *reinterpret_cast<const uint4 *>(src + (size_t)b * row + coff)
                                     : *reinterpret_cast<const uint4 *>(ring + (size_t)b * rrows * row +
                                                                        (size_t)(pos % p.W) * row + coff);
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
            // the bf16 entry block_merge would store, then its 4-bit codes
#pragma unroll
            for (int q = 0; q < 8; ++q)
                val[q] = __bfloat162float(__float2bfloat16_rn(acc[q] / den[q]));
        }
        float mn = INFINITY, mxv = -INFINITY;
        if (active) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                mn = fminf(mn, val[q]);
                mxv = fmaxf(mxv, val[q]);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mxv = fmaxf(mxv, __shfl_xor_sync(0xffffffffu, mxv, off));
        }
        const float sc = __fdiv_rn(__fsub_rn(mxv, mn), 15.f);
        const size_t crow = ((size_t)b * p.Nc + j) * (which == 2 ? 1 : p.Hkv) + h;
        if (active) {
            uint32_t packed = 0;
#pragma unroll
            for (int q = 0; q < 8; q += 2)
                packed |= (ap_fp4_code(val[q], mn, sc) | (ap_fp4_code(val[q + 1], mn, sc) << 4)) << (4 * q);
            uint8_t *codes = which == 0 ? p.kcq : (which == 1 ? p.vcq : p.kicq);
            *reinterpret_cast<uint32_t *>(codes + crow * (dx / 2) + lane * 4) = packed;
        }
        if (lane == 0) {
            float2 *qp = which == 0 ? p.kqp : (which == 1 ? p.vqp : p.kiqp);
            qp[crow] = make_float2(mn, sc);
        }
    }
}

__global__ void __launch_bounds__(kApThreads)
decode_append_kernel(const AppendParams p)
{
    pdl_wait();      // launched as a programmatic dependent: the previous kernel's writes
    pdl_trigger();   // are visible from here on; the next kernel may start its launch
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
    if (p.kcq)
        return launch_pdl(decode_append_fp4_kernel, dim3(p.B), dim3(kApThreads), 0, stream, p);
    return launch_pdl(decode_append_kernel, dim3(p.B), dim3(kApThreads), 0, stream, p);
}

}  // namespace hyb

// fp4.cu -- 4-bit storage for the compressed caches (DeepSeek-V4 CSDN
// article, "compress_to_fp4" / "decompress_from_fp4"): every row of dx
// channels (one compressed entry of one head) keeps dx / 2 bytes of codes,
// element 2i in the low nibble of byte i, and one fp32 pair (min, scale):
//     scale = (max - min) / 15,  code = clamp(rint((x - min) / scale), 0, 15)
// (scale 0 and codes 0 for a constant row), read back as code * scale + min.
// Every step is one IEEE fp32 operation (the __f*_rn intrinsics keep the
// compiler from contracting them), so a code and a dequantized bf16 value
// are the same on any implementation that follows these steps.
//
// Kernels here: quantize, dequantize, and the gather-dequantize of the rows
// a token selected (decode attention reads those from an L2-resident buffer
// instead of dequantizing while it gathers).
#include "common.cuh"

namespace hyb {

// A code as an exact float without an int-to-float conversion: with the code
// in the low mantissa bits of 2^23 the float is 2^23 + code, and subtracting
// 2^23 is exact.
__device__ __forceinline__ float fp4_level(uint32_t code)
{
    return __fsub_rn(__uint_as_float(0x4B000000u | code), 8388608.f);
}

// Eight codes (four bytes) -> eight bf16 values.
__device__ __forceinline__ uint4 fp4_dequant8(uint32_t c, float mn, float sc)
{
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float lo = fp4_level((c >> (8 * q)) & 15u);
        const float hi = fp4_level((c >> (8 * q + 4)) & 15u);
        out[q] = pack_bf16x2(__fadd_rn(__fmul_rn(lo, sc), mn), __fadd_rn(__fmul_rn(hi, sc), mn));
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// Code of one value given its row's min and scale.
__device__ __forceinline__ uint32_t fp4_code(float x, float mn, float sc)
{
    if (!(sc > 0.f))
        return 0u;
    const float r = rintf(__fdiv_rn(__fsub_rn(x, mn), sc));
    return (uint32_t)fminf(fmaxf(r, 0.f), 15.f);
}

// One warp per row of dx = 32 V channels; lane l owns channels [l V, l V + V).
template <int V>
__global__ void __launch_bounds__(256)
fp4_quantize_kernel(const __nv_bfloat16 *__restrict__ x, uint8_t *__restrict__ codes,
                    float2 *__restrict__ qp, long long rows)
{
    constexpr int DX = 32 * V;
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        float v[V];
        const __nv_bfloat16 *src = x + r * DX + lane * V;
#pragma unroll
        for (int e = 0; e < V; e += 2) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(src + e));
            v[e] = f.x;
            v[e + 1] = f.y;
        }
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int e = 1; e < V; ++e) {
            mn = fminf(mn, v[e]);
            mx = fmaxf(mx, v[e]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        const float sc = __fdiv_rn(__fsub_rn(mx, mn), 15.f);
        uint32_t packed = 0;   // V / 2 bytes
#pragma unroll
        for (int e = 0; e < V; e += 2)
            packed |= (fp4_code(v[e], mn, sc) | (fp4_code(v[e + 1], mn, sc) << 4)) << (4 * e);
        uint8_t *dst = codes + r * (DX / 2) + lane * (V / 2);
        if (V == 2)
            *dst = (uint8_t)packed;
        else if (V == 4)
            *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
        else
            *reinterpret_cast<uint32_t *>(dst) = packed;
        if (lane == 0)
            qp[r] = make_float2(mn, sc);
    }
}

// Thread per eight channels.
__global__ void __launch_bounds__(256)
fp4_dequantize_kernel(const uint8_t *__restrict__ codes, const float2 *__restrict__ qp,
                      __nv_bfloat16 *__restrict__ out, long long rows, int dx)
{
    const int per_row = dx / 8;
    const long long units = rows * per_row;
    for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units;
         u += (long long)gridDim.x * blockDim.x) {
        const long long r = u / per_row;
        const float2 p = qp[r];
        const uint32_t c = *reinterpret_cast<const uint32_t *>(codes + u * 4);
        *reinterpret_cast<uint4 *>(out + u * 8) = fp4_dequant8(c, p.x, p.y);
    }
}

// Selected rows of a 4-bit K / V cache, dequantized in selection order:
// out[(row q) Hkv + h] for row = b Lq + t, slot q < topk, head h, from cache
// row (b Nc + idx[row][q]) Hkv + h; slots with an index outside [0, Nc) are
// zero (the attention masks them).  One warp per kGaSlots consecutive slots:
// lanes 0-15 take K, lanes 16-31 V, each lane eight channels of a head row,
// so that a row's codes are one coalesced load and its values one store; the
// loads of all the warp's slots are issued before any value is formed.
constexpr int kGaWarps = 8;
constexpr int kGaSlots = 8;

__global__ void __launch_bounds__(32 * kGaWarps)
fp4_gather_kernel(const uint8_t *__restrict__ kcodes, const float2 *__restrict__ kqp,
                  const uint8_t *__restrict__ vcodes, const float2 *__restrict__ vqp,
                  const int32_t *__restrict__ idx, __nv_bfloat16 *__restrict__ kout,
                  __nv_bfloat16 *__restrict__ vout, int Lq, int topk, int Hkv, int Nc, int d,
                  long long nsel)
{
    const long long sel0 = ((long long)blockIdx.x * kGaWarps + (threadIdx.x >> 5)) * kGaSlots;
    if (sel0 >= nsel)
        return;
    const int lane = threadIdx.x & 31;
    const bool isv = lane >= 16;
    const int c = lane & 15;                   // eight-channel chunk of a head row
    const int per_row = d / 8;
    const uint8_t *codes = isv ? vcodes : kcodes;
    const float2 *qp = isv ? vqp : kqp;
    __nv_bfloat16 *out = isv ? vout : kout;
    int j[kGaSlots];
#pragma unroll
    for (int s = 0; s < kGaSlots; ++s)
        j[s] = sel0 + s < nsel ? __ldg(idx + sel0 + s) : -1;
    for (int h = 0; h < Hkv; ++h) {
        float2 p[kGaSlots];
        uint32_t cw[kGaSlots];
#pragma unroll
        for (int s = 0; s < kGaSlots; ++s) {
            const long long sel = sel0 + s;
            const bool in = j[s] >= 0 && j[s] < Nc && c < per_row;
            const long long b = sel / topk / Lq;
            const long long src = (b * Nc + (in ? j[s] : 0)) * Hkv + h;
            p[s] = in ? __ldg(qp + src) : make_float2(0.f, 0.f);
            cw[s] = in ? __ldg(reinterpret_cast<const uint32_t *>(codes + src * (d / 2)) + c) : 0u;
        }
#pragma unroll
        for (int s = 0; s < kGaSlots; ++s) {
            const long long sel = sel0 + s;
            if (sel >= nsel || c >= per_row)
                continue;
            const bool in = j[s] >= 0 && j[s] < Nc;
            const uint4 val = in ? fp4_dequant8(cw[s], p[s].x, p[s].y) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(out + (sel * Hkv + h) * d + c * 8) = val;
        }
    }
}

static unsigned grid_for(long long work, int threads, int num_sms)
{
    long long g = (work + threads - 1) / threads;
    const long long cap = (long long)num_sms * 16;
    if (g > cap)
        g = cap;
    return (unsigned)(g < 1 ? 1 : g);
}

cudaError_t launch_fp4_quantize(const void *x, long long rows, int dx, uint8_t *codes, float *qp,
                                cudaStream_t stream, int num_sms)
{
    if (rows <= 0)
        return cudaSuccess;
    const unsigned grid = grid_for(rows * 32, 256, num_sms);
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
    float2 *q2 = reinterpret_cast<float2 *>(qp);
    switch (dx) {
    case 64: fp4_quantize_kernel<2><<<grid, 256, 0, stream>>>(xb, codes, q2, rows); break;
    case 128: fp4_quantize_kernel<4><<<grid, 256, 0, stream>>>(xb, codes, q2, rows); break;
    case 256: fp4_quantize_kernel<8><<<grid, 256, 0, stream>>>(xb, codes, q2, rows); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_fp4_dequantize(const uint8_t *codes, const float *qp, long long rows, int dx,
                                  void *out, cudaStream_t stream, int num_sms)
{
    if (rows <= 0)
        return cudaSuccess;
    const long long units = rows * (dx / 8);
    fp4_dequantize_kernel<<<grid_for(units, 256, num_sms), 256, 0, stream>>>(
        codes, reinterpret_cast<const float2 *>(qp), static_cast<__nv_bfloat16 *>(out), rows, dx);
    return cudaGetLastError();
}

cudaError_t launch_fp4_gather(const uint8_t *kcodes, const float *kqp, const uint8_t *vcodes,
                              const float *vqp, const int32_t *idx, void *kout, void *vout, int B, int Lq,
                              int topk, int Hkv, int Nc, int d, cudaStream_t stream, int num_sms)
{
    const long long nsel = (long long)B * Lq * topk;
    if (nsel <= 0)
        return cudaSuccess;
    const long long blocks = (nsel + (long long)kGaWarps * kGaSlots - 1) / ((long long)kGaWarps * kGaSlots);
    if (blocks >= (1ll << 31))
        return cudaErrorInvalidValue;
    fp4_gather_kernel<<<(unsigned)blocks, 32 * kGaWarps, 0, stream>>>(
        kcodes, reinterpret_cast<const float2 *>(kqp), vcodes, reinterpret_cast<const float2 *>(vqp),
        idx, static_cast<__nv_bfloat16 *>(kout), static_cast<__nv_bfloat16 *>(vout), Lq, topk, Hkv, Nc,
        d, nsel);
    return cudaGetLastError();
}

}  // namespace hyb

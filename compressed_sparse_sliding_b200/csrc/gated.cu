// gated.cu -- the gated three-branch variant (Tiny-R2 README, "Attention
// Computation" and "branch_gate"): three attentions with separate softmaxes,
// weighted per (token, head) by a softmax over three gate logits.  The
// branches are runs of the hybrid attention kernels with a smaller key set
// (see hyb_gated_fwd); this file holds their combination:
//     g = softmax(gate[b, t, h, 0..2]),   o = g0 o1 + g1 o2 + g2 o3.
// Thread = 8 channels (16 bytes) of one (token, head) row.
#include "common.cuh"

namespace hyb {

constexpr int kGtThreads = 256;

__global__ void __launch_bounds__(kGtThreads)
gated_combine(const __nv_bfloat16 *__restrict__ o1, const __nv_bfloat16 *__restrict__ o2,
              const __nv_bfloat16 *__restrict__ o3, const float *__restrict__ gate,
              __nv_bfloat16 *__restrict__ o, long long rows, int d)
{
    const int per_row = d / 8;
    const long long units = rows * per_row;
    for (long long u = (long long)blockIdx.x * kGtThreads + threadIdx.x; u < units;
         u += (long long)gridDim.x * kGtThreads) {
        const long long r = u / per_row;
        const float l0 = gate[r * 3], l1 = gate[r * 3 + 1], l2 = gate[r * 3 + 2];
        const float mx = fmaxf(l0, fmaxf(l1, l2));
        const float e0 = expf(l0 - mx), e1 = expf(l1 - mx), e2 = expf(l2 - mx);
        const float inv = 1.f / (e0 + e1 + e2);
        const float g0 = e0 * inv, g1 = e1 * inv, g2 = e2 * inv;
        const size_t off = (size_t)u * 8;
        const uint4 a = *reinterpret_cast<const uint4 *>(o1 + off);
        const uint4 b = *reinterpret_cast<const uint4 *>(o2 + off);
        const uint4 c = *reinterpret_cast<const uint4 *>(o3 + off);
        const __nv_bfloat162 *pa = reinterpret_cast<const __nv_bfloat162 *>(&a);
        const __nv_bfloat162 *pb = reinterpret_cast<const __nv_bfloat162 *>(&b);
        const __nv_bfloat162 *pc = reinterpret_cast<const __nv_bfloat162 *>(&c);
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 fa = __bfloat1622float2(pa[q]);
            const float2 fb = __bfloat1622float2(pb[q]);
            const float2 fc = __bfloat1622float2(pc[q]);
            out[q] = pack_bf16x2(g0 * fa.x + g1 * fb.x + g2 * fc.x, g0 * fa.y + g1 * fb.y + g2 * fc.y);
        }
        *reinterpret_cast<uint4 *>(o + off) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

cudaError_t launch_gated_combine(const void *o1, const void *o2, const void *o3, const float *gate,
                                 void *o, long long rows, int d, cudaStream_t stream, int num_sms)
{
    const long long units = rows * (d / 8);
    if (units <= 0)
        return cudaSuccess;
    long long grid = (units + kGtThreads - 1) / kGtThreads;
    const long long cap = (long long)num_sms * 8;
    if (grid > cap)
        grid = cap;
    gated_combine<<<(unsigned)grid, kGtThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o1), static_cast<const __nv_bfloat16 *>(o2),
        static_cast<const __nv_bfloat16 *>(o3), gate, static_cast<__nv_bfloat16 *>(o), rows, d);
    return cudaGetLastError();
}

}  // namespace hyb

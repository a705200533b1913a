// noalloc.cu -- hyb_csa_index_topk_noalloc: the indexer + top-K stage with
// its score scratch held in a fixed device array inside this library instead
// of a caller-provided workspace.
//
// Who needs it: callers that cannot hand the library a workspace because
// they are not allowed to allocate device memory on their own schedule --
// for example an inference engine whose memory planner owns every device
// buffer and forbids allocations outside it, or a latency-critical decode loop
// in which cudaMalloc / cudaFree would synchronise the whole device.
//
// The scratch is a file-scope array of kNoallocScratchBytes.  Every GPU that
// loads the library keeps it resident until the process exits.  The host
// cannot use the array's name as a device address, so the first call on each
// device looks the address up with cudaGetSymbolAddress (with that device
// current) and caches it; make that first call before any stream capture.
// All calls share the one array and it keeps the previous call's contents:
// the score kernel writes every score the top-K kernel later reads, so nothing
// needs clearing, but calls whose kernels overlap on the GPU (for example on
// two streams) race on the array and must be serialised by the caller.
#include <mutex>

#include "common.cuh"

namespace hyb {

constexpr size_t kNoallocScratchBytes = HYB_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) float g_noalloc_scores[kNoallocScratchBytes / sizeof(float)];

static std::mutex g_noalloc_mu;
static float *g_noalloc_ptr[256] = {};

// Device address of the scratch array on the current device (looked up once).
static hyb_status noalloc_scratch(float **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256)
        return HYB_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scores) != cudaSuccess || !p)
            return HYB_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return HYB_OK;
}

}  // namespace hyb

extern "C" hyb_status hyb_csa_index_topk_noalloc(const hyb_problem *p, const void *qi,
                                                 const float *wi, const void *kic, int32_t *idx,
                                                 float *sel_scores, cudaStream_t stream)
{
    using namespace hyb;
    hyb_status st = check_problem(p, true);
    if (st != HYB_OK)
        return st;
    if (!qi || !wi || !kic || !idx || !aligned16(qi) || !aligned16(kic))
        return HYB_ERR_INVALID_ARG;
    // the two-kernel path on the fixed scratch where it is the faster one and
    // the rows fit; otherwise the one kernel, which needs no scratch at all
    if (index_topk_fused_path(p, kNoallocScratchBytes))
        return cuda_status(launch_index_topk_fused(qi, wi, kic, idx, sel_scores, p->B, p->Lq, p->Hi, p->di,
                                                   p->Nc, p->m, p->W, p->topk, p->q_pos, stream));
    const size_t need = (size_t)p->B * p->Lq * p->Nc * sizeof(float);
    if (need > kNoallocScratchBytes)
        return HYB_ERR_UNSUPPORTED;  // the problem's score rows do not fit the fixed scratch
    float *scores = nullptr;
    st = noalloc_scratch(&scores);
    if (st != HYB_OK)
        return st;
    // the same kernels as hyb_csa_index_topk, on the fixed scratch
    return cuda_status(index_topk_into(p, qi, wi, kic, idx, sel_scores, scores, stream));
}

// runtime.cu -- status strings, device queries, tensor-map encoding and the
// programmatic-dependent-launch helper.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "bq_internal.h"

namespace bq {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::once_flag g_encode_once;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

void load_encode()
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}
}  // namespace

int device_sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return -1;
    if (dev < kMaxDevices) {
        int v = g_sm_count[dev].load(std::memory_order_relaxed);
        if (v > 0)
            return v;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    if (dev < kMaxDevices)
        g_sm_count[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base,
                       const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                       CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promotion)
{
    std::call_once(g_encode_once, load_encode);
    if (!g_encode)
        return false;
    cuuint64_t gdim[3], gstride[2];
    cuuint32_t bdim[3], estride[3] = {1, 1, 1};
    for (int i = 0; i < rank; i++) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
    }
    for (int i = 0; i < rank - 1; i++)
        gstride[i] = strides_bytes[i];
    CUresult r = g_encode(map, dtype, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstride,
                          bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promotion,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_pdl(const void *kernel, dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, void **args, int cluster)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (cluster > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelExC(&cfg, kernel, args);
}

int32_t check_qmat(const bq_qmat *W)
{
    if (!W || !W->codes || !W->scales)
        return BQ_ERR_NULL;
    if (W->N < 1 || W->K < 32 || W->K % 32 != 0 || W->N > (1 << 30) || W->K > (1 << 30))
        return BQ_ERR_SHAPE;
    if (!aligned16(W->codes) || !aligned16(W->scales))
        return BQ_ERR_ALIGN;
    return BQ_OK;
}

}  // namespace bq

extern "C" const char *bq_status_string(int32_t s)
{
    switch (s) {
    case BQ_OK: return "ok";
    case BQ_ERR_NULL: return "null pointer";
    case BQ_ERR_SHAPE: return "bad shape";
    case BQ_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case BQ_ERR_BATCH: return "batch out of range";
    case BQ_ERR_EXPERT_INDEX: return "expert index out of range";
    case BQ_ERR_CUDA: return "CUDA error";
    case BQ_ERR_TIMEOUT: return "bounded wait timed out";
    case BQ_ERR_WORKSPACE: return "workspace missing or too small";
    case BQ_ERR_RANGE: return "value out of range";
    default: return "unknown status";
    }
}

extern "C" int32_t bq_scales_ld(int32_t K)
{
    if (K < 32 || K % 32 != 0)
        return 0;
    return (K / 32 + 7) / 8 * 8;
}

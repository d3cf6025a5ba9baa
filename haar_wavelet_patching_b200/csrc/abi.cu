// Library-wide entry points of tok.h (version, status names, errors) and host
// helpers shared by the kernels' launchers.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "tma.cuh"
#include "umma.cuh"
#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {

static thread_local int g_last_cuda_error = 0;

void record_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }

tok_status launch_status()
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return TOK_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base, const uint64_t *dims,
                       const uint64_t *strides_bytes, const uint32_t *box)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encoder();
    if (!fn)
        return false;
    cuuint64_t gdim[5], gstr[4];
    cuuint32_t bdim[5], estr[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estr[i] = 1;
        if (i + 1 < rank)
            gstr[i] = strides_bytes[i];
    }
    return fn(map, dtype, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstr, bdim, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tensor_map_sw128(CUtensorMap *map, int rank, const void *base, const uint64_t *dims,
                             const uint64_t *strides_bytes, const uint32_t *box)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encoder();
    if (!fn)
        return false;
    cuuint64_t gdim[5], gstr[4];
    cuuint32_t bdim[5], estr[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estr[i] = 1;
        if (i + 1 < rank)
            gstr[i] = strides_bytes[i];
    }
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstr, bdim,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count()
{
    static int counts[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return 0;
    if (dev >= 64 || counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        if (dev >= 64)
            return n;
        counts[dev] = n;
    }
    return counts[dev];
}

} // namespace tok

extern "C" int tok_abi_version(void) { return TOK_ABI_VERSION; }

extern "C" int tok_last_cuda_error(void) { return tok::g_last_cuda_error; }

extern "C" tok_status tok_check_device(cudaStream_t stream)
{
    unsigned int nh = 0, nf = 0, nb = 0, nc = 0;
    tok_status st = tok::read_and_clear_haar_timeouts(stream, &nh);
    if (st == TOK_OK)
        st = tok::read_and_clear_fsq_timeouts(stream, &nf);
    if (st == TOK_OK)
        st = tok::read_and_clear_fsq_bwd_timeouts(stream, &nb);
    if (st == TOK_OK)
        st = tok::read_and_clear_conv_timeouts(stream, &nc);
    if (st != TOK_OK)
        return st;
    return (nh || nf || nb || nc) ? TOK_ERR_TIMEOUT : TOK_OK;
}

extern "C" const char *tok_status_str(tok_status status)
{
    switch (status) {
    case TOK_OK:
        return "TOK_OK";
    case TOK_ERR_NULL:
        return "TOK_ERR_NULL: a required pointer is NULL";
    case TOK_ERR_SHAPE:
        return "TOK_ERR_SHAPE: extents violate the shape rule or overflow";
    case TOK_ERR_ALIGN:
        return "TOK_ERR_ALIGN: a pointer is not aligned to its element size";
    case TOK_ERR_DTYPE:
        return "TOK_ERR_DTYPE: unknown dtype";
    case TOK_ERR_ALIAS:
        return "TOK_ERR_ALIAS: an input overlaps an output";
    case TOK_ERR_CUDA:
        return "TOK_ERR_CUDA: a CUDA call or kernel launch failed";
    case TOK_ERR_TIMEOUT:
        return "TOK_ERR_TIMEOUT: a kernel stopped after a barrier wait ran out; its output is incomplete";
    case TOK_ERR_TOO_LARGE:
        return "TOK_ERR_TOO_LARGE: the call needs more than the 3 MB fixed scratch of the allocation-free call "
               "(at most 8388608 tokens at C = 16), or runs on a device ordinal above 63";
    }
    return "unknown tok_status";
}

// Library-wide entry points of tok.h: version, status names, launch errors.
#include "tok_common.cuh"

namespace tok {

static thread_local int g_last_cuda_error = 0;

tok_status launch_status()
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        g_last_cuda_error = (int)e;
        return TOK_ERR_CUDA;
    }
    return TOK_OK;
}

} // namespace tok

extern "C" int tok_abi_version(void) { return TOK_ABI_VERSION; }

extern "C" int tok_last_cuda_error(void) { return tok::g_last_cuda_error; }

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
        return "TOK_ERR_CUDA: kernel launch failed";
    }
    return "unknown tok_status";
}

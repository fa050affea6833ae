// rb_gemm.cu -- batched application on the tcgen05 tensor cores (in progress).
#include "rbw_internal.cuh"

extern "C" size_t rb_gemm_workspace_bytes(int n_out, int k_in, int k_planes, int M)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 8 || M < 1) return 0;
    return ((size_t)M * (size_t)k_in * 2 + 255) / 256 * 256;
}

extern "C" rb_status rb_gemm(const rb_layer_t* layer, const uint16_t* X, int M, void* Y, rb_dtype y_dtype,
                             void*, size_t, int32_t*, unsigned flags, cudaStream_t)
{
    rb_status st = rbw::check_apply_args(layer, X, M, Y, y_dtype, flags);
    if (st != RB_OK) return st;
    return RB_ERR_UNSUPPORTED;
}

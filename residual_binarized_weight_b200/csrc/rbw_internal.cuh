// rbw_internal.cuh -- shared device/host helpers of the CUDA library (not part
// of the C ABI).  Storage layout of the sign planes, launch helpers, status
// plumbing.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/rbw.h"

namespace rbw {

// ---------------------------------------------------------------- layout
// Plane i, column slice s (256 columns), row tile t (32 rows): a block of 256
// words.  Logical word w (columns 32w..32w+31 of the slice) of row
// rho = r % 32 sits in slot w ^ (rho / 4) of the block: index slot*32 + rho.
// A warp whose lane l owns row l therefore reads slot `sl` with one coalesced
// 128-byte load and obtains logical word sl ^ (l / 4).
__host__ __device__ inline int64_t num_slices(int K) { return (K + 255) / 256; }
__host__ __device__ inline int64_t num_row_tiles(int N) { return (N + 31) / 32; }
__host__ __device__ inline int64_t block_index(int i, int64_t s, int64_t t, int64_t S, int64_t Nt) {
    return ((int64_t)i * S + s) * Nt + t;
}
__host__ __device__ inline int64_t word_offset(int i, int64_t s, int64_t r, int w, int64_t S, int64_t Nt) {
    int rho = (int)(r & 31);
    return block_index(i, s, r >> 5, S, Nt) * 256 + (int64_t)((w ^ (rho >> 2)) * 32 + rho);
}

// ---------------------------------------------------------------- device helpers
// Thread-block cluster: rank, a full barrier (release / acquire), and stores
// into another CTA's shared memory at the same offset as a local address.
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_dsmem_f32(uint32_t local_saddr, uint32_t rank, float v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_saddr), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(remote), "f"(v) : "memory");
}
__device__ __forceinline__ void st_dsmem_v4(uint32_t local_saddr, uint32_t rank, float a, float b, float c, float d) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_saddr), "r"(rank));
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" :: "r"(remote), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ float lds_f32(uint32_t saddr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(saddr));
    return v;
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}
__device__ __forceinline__ void set_dev_status(int32_t* st, int bits) {
    if (st && bits) atomicOr(st, bits);
}
__device__ __forceinline__ void store_y(void* Y, int ydt, int64_t idx, float v) {
    if (ydt == RB_BF16)
        reinterpret_cast<__nv_bfloat16*>(Y)[idx] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(Y)[idx] = v;
}

// ---------------------------------------------------------------- host helpers
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch `kern` with optional programmatic dependent launch.
template <typename... KArgs, typename... Args>
inline rb_status launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t stream, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
    return e == cudaSuccess ? RB_OK : RB_ERR_CUDA;
}

// Common argument checks of rb_gemv / rb_gemm.
inline rb_status check_apply_args(const rb_layer_t* L, const void* X, int M, const void* Y,
                                  rb_dtype y_dtype, unsigned flags)
{
    if (!L || !L->planes || !L->g16 || !L->h16 || L->reserved != 0) return RB_ERR_ARG;
    if (L->k_planes < 1 || L->k_planes > 8) return RB_ERR_ARG;
    if (!X || !Y || (y_dtype != RB_F32 && y_dtype != RB_BF16) || (flags & ~RB_LAUNCH_PDL)) return RB_ERR_ARG;
    if (L->n_out < 1 || L->k_in < 32 || L->k_in % 32 != 0 || M < 1) return RB_ERR_SHAPE;
    if (!aligned16(L->planes) || !aligned16(L->g16) || !aligned16(L->h16) || !aligned16(X) || !aligned16(Y))
        return RB_ERR_ALIGN;
    return RB_OK;
}

int num_sms();                 // of the current device (cached per device)

// The tcgen05 kernel (rb_gemm.cu); decode = small-M tiles with a K split.
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;    // bound on each device-side wait (1 s)
rb_status gemm_with_timeout(const rb_layer_t* layer, const uint16_t* X, int M, void* Y, rb_dtype y_dtype,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status, unsigned flags,
                            cudaStream_t stream, uint64_t timeout_ns, bool decode);
// rb_pack's sign-plane kernel alone (no fp16 scale copies); arguments already checked
rb_status pack_planes(const float* W, const float* g, const float* h, int N, int K, int kp, uint32_t* planes,
                      int32_t* dev_status, cudaStream_t stream);
size_t gemm_workspace(int k_in, int k_planes, int M);  // bytes of its workspace (X in fp16, h pairs)
bool device_is_sm100();        // current device is compute capability 10.x

}  // namespace rbw

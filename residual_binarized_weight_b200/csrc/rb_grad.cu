// rb_grad.cu -- gradients of the coupled-training layer (RaBiT, Algorithm 2
// backward pass).  The signs B_i are derived from the latent weight W by the
// forward recurrence (rb_pack) and held constant; the latent weight takes the
// gradient of the effective weight What = sum_i diag(g_i) B_i diag(h_i), and
// the scales follow by the chain rule:
//
//   G        = dY^T X                       (N x K; dL/dWhat = dL/dW)
//   dg_i[n]  = sum_c G[n][c] B_i[n][c] h_i[c]
//   dh_i[c]  = sum_n G[n][c] g_i[n] B_i[n][c]
//
// G is a dense contraction over the tokens, so it runs on the tcgen05 tensor
// cores: bf16 operands (exact products), fp32 accumulation in tensor memory.
// dY [M][N] and X [M][K] are both contiguous along the output dimensions and
// strided along the contraction, so TMA brings 64-token x 64-column boxes in
// with the 128-byte swizzle and the MMA reads them MN-major, with no transpose
// pass.  The scale gradients are one HBM-bound pass over G and the planes,
// written as per-block partial sums and added in a fixed order (no atomics),
// so every result is deterministic.
#include <atomic>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "rbw_internal.cuh"
#include "rb_tcgen05.cuh"

namespace rbw {
namespace {

constexpr int kGN = 128;                       // rows n of G per CTA (MMA M, tensor-memory lanes)
constexpr int kGC = 256;                       // columns c per CTA (MMA N)
constexpr int kGM = 64;                        // tokens per pipeline stage (four MMAs of K = 16)
constexpr int kGStages = 4;
constexpr int kGThreads = 192;
constexpr uint32_t kGStageA = kGM * kGN * 2;   // two 64-column boxes of dY: 16 KB
constexpr uint32_t kGStageB = kGM * kGC * 2;   // four 64-column boxes of X: 32 KB
constexpr uint32_t kGBox = kGM * 128;          // one box: 64 tokens x 128 bytes
constexpr int kGSmem = kGStages * (kGStageA + kGStageB) + 1024 + 256;

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// each 8-token group of 128-byte rows is one swizzle atom (1024 B apart, SBO),
// consecutive 64-element blocks along the output dimension are `lbo` apart.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// kind::f16 instruction descriptor: fp32 D, bf16 A and B, both MN-major, N = 256, M = 128.
constexpr uint32_t kGIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                             ((uint32_t)(kGC >> 3) << 17) | ((uint32_t)(kGN >> 4) << 24);

__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// G tile [n0, n0 + 128) x [c0, c0 + 256): warp 0 = TMA producer (+ tensor
// memory allocation), warp 1 = MMA issuer, warps 2..5 = epilogue (tensor
// memory -> registers -> G).  Waits are bounded as in the prefill GEMM.
__global__ void __launch_bounds__(kGThreads, 1)
grad_gemm_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x,
                 int N, int K, int M, float* __restrict__ G, int32_t* dev_status, uint64_t timeout_ns)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (sbase - smem_u32(smem_raw));
    auto stage_a = [&](int s) { return sbase + (uint32_t)s * (kGStageA + kGStageB); };
    auto stage_b = [&](int s) { return stage_a(s) + kGStageA; };
    uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + kGStages * (kGStageA + kGStageB));
    const uint32_t bar0 = smem_u32(bars);
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kGStages + s); };
    const uint32_t acc_full = bar0 + 8u * (2 * kGStages);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kGStages + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kGN, c0 = blockIdx.y * kGC;
    const int nkb = (M + kGM - 1) / kGM;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(&tm_dy) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(&tm_x) : "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"((uint32_t)kGC) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {                                  // ---------------- TMA producer
            int issued = 0, s = 0, j = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                if (j > 0 && !mbar_wait(empty(s), (j - 1) & 1, abort_flag, dev_status, timeout_ns)) break;
                mbar_arrive_expect_tx(full(s), kGStageA + kGStageB);
#pragma unroll
                for (int q = 0; q < kGN / 64; ++q) tma_load_2d(stage_a(s) + q * kGBox, &tm_dy, full(s), n0 + 64 * q, kb * kGM);
#pragma unroll
                for (int q = 0; q < kGC / 64; ++q) tma_load_2d(stage_b(s) + q * kGBox, &tm_x, full(s), c0 + 64 * q, kb * kGM);
                ++issued;
                if (++s == kGStages) { s = 0; ++j; }
            }
            if (*abort_flag) {                            // drain the loads this thread issued: they always land
                const uint64_t t0 = globaltimer_ns();
                for (int kb = issued - kGStages < 0 ? 0 : issued - kGStages; kb < issued; ++kb)
                    mbar_drain(full(kb % kGStages), (kb / kGStages) & 1, t0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {                                  // ---------------- MMA issuer
            int s = 0;
            uint32_t ph = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(full(s), ph, abort_flag, dev_status, timeout_ns)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kGM / 16; ++kk) {   // 16 tokens = two 8-row atoms = 2048 B
                    const uint64_t ad = smem_desc_mn_sw128(stage_a(s) + kk * 2048, kGBox);
                    const uint64_t bd = smem_desc_mn_sw128(stage_b(s) + kk * 2048, kGBox);
                    tc_mma_ss(tmem, ad, bd, kGIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(empty(s));
                if (++s == kGStages) { s = 0; ph ^= 1u; }
            }
            tc_commit(acc_full);                          // arrives once every MMA issued above is done
        }
    } else {                                              // ---------------- epilogue
        const int q = warp & 3;
        const int64_t n = (int64_t)n0 + q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        if (mbar_wait_warp(acc_full, 0, abort_flag, dev_status, timeout_ns)) {
            tc_fence_after();
#pragma unroll 1
            for (int j = 0; j < kGC / 32; ++j) {
                uint32_t v[32];
                tc_ld_32x32b_x32(tmem + lane_base + (uint32_t)(32 * j), v);
                tc_wait_ld();
                const int64_t c = (int64_t)c0 + 32 * j;
                if (n < N && c < K) {                     // K % 32 == 0: a chunk is all in or all out
                    float4* dst = reinterpret_cast<float4*>(G + n * K + c);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                             __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
                }
            }
        }
    }

    if (warp == 1 && lane == 0 && *abort_flag) mbar_drain(acc_full, 0, globaltimer_ns());
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) set_dev_status(dev_status, RB_DEV_TIMEOUT);
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"((uint32_t)kGC) : "memory");
    }
}

// ---------------------------------------------------------------- scale gradients
// CTA = 256 rows x one 256-column slice; warp w takes rows 32 w .. 32 w + 31 of
// the block one at a time, lane l columns 8 l .. 8 l + 7 of the slice (two
// 16-byte loads of G per row, the byte of the row's sign word that holds them).
// dg partial of a row: butterfly sum over the lanes -> dg_part[s][i][n].  dh
// partial of a column: this lane's running sum over the warp's rows, then the
// eight warps in order -> dh_part[row block][i][c].
constexpr int kSgThreads = 256;
constexpr int kSgRows = 256;

template <int KP>
__global__ void __launch_bounds__(kSgThreads)
scale_grad_partial_kernel(const float* __restrict__ G, const uint32_t* __restrict__ planes,
                          const float* __restrict__ g, const float* __restrict__ h, int N, int K,
                          float* __restrict__ dg_part, float* __restrict__ dh_part)
{
    __shared__ float red[kSgThreads / 32][256];
    pdl_launch_dependents();
    pdl_wait();                                           // G comes from the GEMM launched before
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int s = blockIdx.y, rb = blockIdx.x;
    const int64_t c = (int64_t)s * 256 + lane * 8;
    const bool col_ok = c < K;
    float hv[KP][8];
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f), b = a;
        if (col_ok) {
            a = *reinterpret_cast<const float4*>(h + (int64_t)i * K + c);
            b = *reinterpret_cast<const float4*>(h + (int64_t)i * K + c + 4);
        }
        hv[i][0] = a.x; hv[i][1] = a.y; hv[i][2] = a.z; hv[i][3] = a.w;
        hv[i][4] = b.x; hv[i][5] = b.y; hv[i][6] = b.z; hv[i][7] = b.w;
    }
    float dh_acc[KP][8];
#pragma unroll
    for (int i = 0; i < KP; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) dh_acc[i][e] = 0.0f;

    // U rows per step: their G, sign words and g are all in flight before any is used
    // (four for k <= 2, fewer as the per-plane registers grow)
    constexpr int U = KP <= 2 ? 4 : KP <= 4 ? 2 : 1;
    for (int j0 = 0; j0 < 32; j0 += U) {
        const int64_t r0 = (int64_t)rb * kSgRows + warp * 32 + j0;
        if (r0 >= N) break;                               // warp-uniform
        float gv[U][8];
        uint32_t wd[U][KP];
        float gi[U][KP];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = r0 + u;
            const bool rok = r < N;
            float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f), b = a;
            if (rok && col_ok) {
                a = *reinterpret_cast<const float4*>(G + r * K + c);
                b = *reinterpret_cast<const float4*>(G + r * K + c + 4);
            }
            gv[u][0] = a.x; gv[u][1] = a.y; gv[u][2] = a.z; gv[u][3] = a.w;
            gv[u][4] = b.x; gv[u][5] = b.y; gv[u][6] = b.z; gv[u][7] = b.w;
#pragma unroll
            for (int i = 0; i < KP; ++i) {
                wd[u][i] = rok ? planes[word_offset(i, s, r, lane >> 2, S, Nt)] : 0u;
                gi[u][i] = rok ? g[(int64_t)i * N + r] : 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = r0 + u;
            if (r >= N) break;                            // warp-uniform
#pragma unroll
            for (int i = 0; i < KP; ++i) {
                const uint32_t byte = (wd[u][i] >> ((lane & 3) * 8)) & 0xffu;
                float dgp = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float v = ((byte >> e) & 1u) ? gv[u][e] : -gv[u][e];
                    dgp = fmaf(v, hv[i][e], dgp);
                    dh_acc[i][e] = fmaf(v, gi[u][i], dh_acc[i][e]);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dgp += __shfl_xor_sync(0xffffffffu, dgp, o);
                if (lane == 0) dg_part[((int64_t)s * KP + i) * N + r] = dgp;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < KP; ++i) {                        // one plane at a time through shared memory
        if (i > 0) __syncthreads();
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = dh_acc[i][e];
        __syncthreads();
        const int cc = threadIdx.x;                       // kSgThreads == 256 columns
        if ((int64_t)s * 256 + cc < K) {
            float v = 0.0f;
            for (int w = 0; w < kSgThreads / 32; ++w) v += red[w][cc];
            dh_part[((int64_t)rb * KP + i) * K + (int64_t)s * 256 + cc] = v;
        }
    }
}

// dg[i][n] = sum over slices of dg_part (slice order); dh[i][c] = sum over row
// blocks of dh_part (block order).
__global__ void scale_grad_reduce_kernel(const float* __restrict__ dg_part, const float* __restrict__ dh_part,
                                         int N, int K, int kp, int S, int RB, float* __restrict__ dg,
                                         float* __restrict__ dh)
{
    pdl_launch_dependents();
    pdl_wait();
    const int64_t ng = (int64_t)kp * N, nh = (int64_t)kp * K;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < ng + nh;
         x += (int64_t)gridDim.x * blockDim.x) {
        float v = 0.0f;
        if (x < ng) {
            for (int s = 0; s < S; ++s) v += dg_part[(int64_t)s * ng + x];
            dg[x] = v;
        } else {
            const int64_t y = x - ng;
            for (int b = 0; b < RB; ++b) v += dh_part[(int64_t)b * nh + y];
            dh[y] = v;
        }
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> cache{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 fn = cache.load(std::memory_order_acquire);
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
            cache.store(fn, std::memory_order_release);
        }
    }
    return fn;
}

// bf16 [rows][cols] row-major, 64 x 64 boxes with the 128-byte swizzle.
bool encode_bf16_map(CUtensorMap* map, const void* base, int64_t cols, int64_t rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kGM};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct GradWs {
    float* dg_part;      // [S][k][N]
    float* dh_part;      // [RB][k][K]
    size_t bytes;
};

GradWs grad_ws_layout(int N, int K, int kp, void* base)
{
    const int64_t S = num_slices(K), RB = (N + kSgRows - 1) / kSgRows;
    const size_t a = ((size_t)S * kp * N * 4 + 255) / 256 * 256;
    const size_t b = ((size_t)RB * kp * K * 4 + 255) / 256 * 256;
    GradWs w;
    w.dg_part = reinterpret_cast<float*>(base);
    w.dh_part = reinterpret_cast<float*>(reinterpret_cast<char*>(base) + a);
    w.bytes = a + b;
    return w;
}

template <int KP>
rb_status launch_scale_grad(const float* G, const uint32_t* planes, const float* g, const float* h, int N, int K,
                            const GradWs& ws, cudaStream_t stream)
{
    const int64_t S = num_slices(K), RB = (N + kSgRows - 1) / kSgRows;
    return launch(scale_grad_partial_kernel<KP>, dim3((unsigned)RB, (unsigned)S), dim3(kSgThreads), 0, stream, true,
                  G, planes, g, h, N, K, ws.dg_part, ws.dh_part);
}

}  // namespace
}  // namespace rbw

using namespace rbw;

extern "C" size_t rb_qat_backward_workspace_bytes(int n_out, int k_in, int k_planes)
{
    if (n_out < 32 || n_out % 32 != 0 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 8) return 0;
    return grad_ws_layout(n_out, k_in, k_planes, nullptr).bytes;
}

extern "C" rb_status rb_qat_backward(const uint32_t* planes, const float* g, const float* h, int n_out, int k_in,
                                     int k_planes, const uint16_t* X, const uint16_t* dY, int M, float* dW,
                                     float* dg, float* dh, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, cudaStream_t stream)
{
    if (!planes || !g || !h || !X || !dY || !dW || !dg || !dh) return RB_ERR_ARG;
    if (k_planes < 1 || k_planes > 8) return RB_ERR_ARG;
    if (n_out < 32 || n_out % 32 != 0 || k_in < 32 || k_in % 32 != 0 || M < 1) return RB_ERR_SHAPE;
    const void* ptrs[] = {planes, g, h, X, dY, dW, dg, dh};
    for (const void* p : ptrs)
        if (!aligned16(p)) return RB_ERR_ALIGN;
    if (dev_status && !aligned16(dev_status)) return RB_ERR_ALIGN;
    const GradWs ws = grad_ws_layout(n_out, k_in, k_planes, workspace);
    if (!workspace || workspace_bytes < ws.bytes) return RB_ERR_WORKSPACE;
    if (!aligned16(workspace)) return RB_ERR_ALIGN;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;

    CUtensorMap tm_dy, tm_x;
    if (!encode_bf16_map(&tm_dy, dY, n_out, M) || !encode_bf16_map(&tm_x, X, k_in, M)) return RB_ERR_CUDA;
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RB_ERR_CUDA;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(grad_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem) != cudaSuccess)
            return RB_ERR_CUDA;
        attr_set[dev].store(true, std::memory_order_release);
    }
    const dim3 grid((unsigned)((n_out + kGN - 1) / kGN), (unsigned)((k_in + kGC - 1) / kGC));
    rb_status st = launch(grad_gemm_kernel, grid, dim3(kGThreads), (size_t)kGSmem, stream, false, tm_dy, tm_x,
                          n_out, k_in, M, dW, dev_status, kTimeoutNs);
    if (st != RB_OK) return st;
    switch (k_planes) {
        case 1: st = launch_scale_grad<1>(dW, planes, g, h, n_out, k_in, ws, stream); break;
        case 2: st = launch_scale_grad<2>(dW, planes, g, h, n_out, k_in, ws, stream); break;
        case 3: st = launch_scale_grad<3>(dW, planes, g, h, n_out, k_in, ws, stream); break;
        case 4: st = launch_scale_grad<4>(dW, planes, g, h, n_out, k_in, ws, stream); break;
        case 5: st = launch_scale_grad<5>(dW, planes, g, h, n_out, k_in, ws, stream); break;
        case 6: st = launch_scale_grad<6>(dW, planes, g, h, n_out, k_in, ws, stream); break;
        case 7: st = launch_scale_grad<7>(dW, planes, g, h, n_out, k_in, ws, stream); break;
        default: st = launch_scale_grad<8>(dW, planes, g, h, n_out, k_in, ws, stream); break;
    }
    if (st != RB_OK) return st;
    const int64_t S = num_slices(k_in), RB = (n_out + kSgRows - 1) / kSgRows;
    const int64_t items = (int64_t)k_planes * (n_out + k_in);
    int64_t ctas = (items + 255) / 256;
    if (ctas > 4 * num_sms()) ctas = 4 * num_sms();
    return launch(scale_grad_reduce_kernel, dim3((unsigned)ctas), dim3(256), 0, stream, true, ws.dg_part, ws.dh_part,
                  n_out, k_in, k_planes, (int)S, (int)RB, dg, dh);
}

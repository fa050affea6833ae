// rb_svid.cu -- greedy SVID scales on the device (RaBiT names Greedy SVID as
// the traditional initialiser it improves on; the greedy form takes, plane by
// plane, the rank-1 approximation of |R_{i-1}|).
//
// For plane i the matrix A = |R_{i-1}| is never stored: every pass recomputes
// R_{i-1} from W and the scales of the earlier planes with the fp32
// recurrence of rb_pack (t = fl(g*h); R = fl(R -/+ t)).  Power iteration runs
// in float64 with fixed summation orders (warp tree per row, row chunks in
// order per column), so the result is deterministic.
#include <math.h>

#include "rbw_internal.cuh"

namespace rbw {
namespace {

constexpr int kRowChunks = 64;

struct SvidWs {
    double* u;        // [N]
    double* v;        // [K]
    double* av;       // [N]
    double* vpart;    // [kRowChunks][K]
    double* scal;     // [8]
    size_t bytes;
};

SvidWs svid_ws_layout(int N, int K, void* base)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    SvidWs w;
    char* p = reinterpret_cast<char*>(base);
    size_t off = 0;
    w.u = reinterpret_cast<double*>(p + off);     off += up((size_t)N * 8);
    w.v = reinterpret_cast<double*>(p + off);     off += up((size_t)K * 8);
    w.av = reinterpret_cast<double*>(p + off);    off += up((size_t)N * 8);
    w.vpart = reinterpret_cast<double*>(p + off); off += up((size_t)kRowChunks * K * 8);
    w.scal = reinterpret_cast<double*>(p + off);  off += 256;
    w.bytes = off;
    return w;
}

// |R_{i-1}[r][c]| for plane i (0-based) from W and the scales of planes < i.
__device__ __forceinline__ double abs_residual(const float* W, const float* g, const float* h,
                                               int N, int K, int plane, int64_t r, int64_t c)
{
    float R = W[r * K + c];
    for (int p = 0; p < plane; ++p) {
        const bool b = R >= 0.0f;
        const float tt = __fmul_rn(g[(int64_t)p * N + r], h[(int64_t)p * K + c]);
        R = b ? __fsub_rn(R, tt) : __fadd_rn(R, tt);
    }
    return fabs((double)R);
}

// out[r] = sum_c A[r][c] * x[c]   (one warp per row)
__global__ void svid_av_kernel(const float* __restrict__ W, const float* __restrict__ g,
                               const float* __restrict__ h, int N, int K, int plane,
                               const double* __restrict__ x, double* __restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= N) return;
    double acc = 0.0;
    for (int64_t c = lane; c < K; c += 32) acc += abs_residual(W, g, h, N, K, plane, r, c) * x[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[r] = acc;
}

// vpart[chunk][c] = sum_{r in chunk} A[r][c] * u[r]   (rows in order)
__global__ void svid_atu_partial_kernel(const float* __restrict__ W, const float* __restrict__ g,
                                        const float* __restrict__ h, int N, int K, int plane,
                                        const double* __restrict__ u, double* __restrict__ vpart)
{
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int chunk = blockIdx.y;
    if (c >= K) return;
    const int64_t r0 = (int64_t)N * chunk / kRowChunks, r1 = (int64_t)N * (chunk + 1) / kRowChunks;
    double acc = 0.0;
    for (int64_t r = r0; r < r1; ++r) acc += abs_residual(W, g, h, N, K, plane, r, c) * u[r];
    vpart[(int64_t)chunk * K + c] = acc;
}

__global__ void svid_atu_reduce_kernel(const double* __restrict__ vpart, int K, double* __restrict__ v)
{
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= K) return;
    double acc = 0.0;
    for (int ch = 0; ch < kRowChunks; ++ch) acc += vpart[(int64_t)ch * K + c];
    v[c] = acc;
}

// Fixed-order block reduction of sum(a[j] * b[j]) by one CTA of 1024 threads.
__device__ double block_dot(const double* a, const double* b, int64_t n)
{
    __shared__ double red[1024];
    double acc = 0.0;
    for (int64_t j = threadIdx.x; j < n; j += blockDim.x) acc += a[j] * b[j];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int st = blockDim.x / 2; st > 0; st >>= 1) {
        if ((int)threadIdx.x < st) red[threadIdx.x] += red[threadIdx.x + st];
        __syncthreads();
    }
    const double r = red[0];
    __syncthreads();
    return r;
}

__global__ void svid_normalize_kernel(double* __restrict__ x, int64_t n)
{
    const double nrm = sqrt(block_dot(x, x, n));
    for (int64_t j = threadIdx.x; j < n; j += blockDim.x) x[j] = nrm > 0.0 ? x[j] / nrm : 0.0;
}

__global__ void svid_init_kernel(double* __restrict__ v, int K)
{
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < K; j += (int64_t)gridDim.x * blockDim.x)
        v[j] = 1.0 / sqrt((double)K);
}

// sigma = u^T (A v); g_i = fp32(sqrt(sigma) u); h_i = fp32(sqrt(sigma) v)
__global__ void svid_finish_kernel(const double* __restrict__ u, const double* __restrict__ v,
                                   const double* __restrict__ av, int N, int K, int plane,
                                   float* __restrict__ g, float* __restrict__ h)
{
    const double sigma = block_dot(u, av, N);
    const double rs = sigma > 0.0 ? sqrt(sigma) : 0.0;
    for (int64_t r = threadIdx.x; r < N; r += blockDim.x) g[(int64_t)plane * N + r] = (float)(rs * u[r]);
    for (int64_t c = threadIdx.x; c < K; c += blockDim.x) h[(int64_t)plane * K + c] = (float)(rs * v[c]);
}

}  // namespace
}  // namespace rbw

using namespace rbw;

extern "C" size_t rb_svid_workspace_bytes(int n_out, int k_in)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0) return 0;
    return svid_ws_layout(n_out, k_in, nullptr).bytes;
}

extern "C" rb_status rb_svid_greedy(const float* W, int n_out, int k_in, int k_planes, int iters,
                                    float* g, float* h, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream)
{
    if (!W || !g || !h || !workspace) return RB_ERR_ARG;
    if (k_planes < 1 || k_planes > 8 || iters < 1 || iters > 10000) return RB_ERR_ARG;
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0) return RB_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(g) || !aligned16(h) || !aligned16(workspace)) return RB_ERR_ALIGN;
    SvidWs ws = svid_ws_layout(n_out, k_in, workspace);
    if (workspace_bytes < ws.bytes) return RB_ERR_WORKSPACE;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    const int N = n_out, K = k_in;
    const dim3 av_grid((unsigned)((N + 7) / 8)), av_blk(256);
    const dim3 atu_grid((unsigned)((K + 255) / 256), kRowChunks), atu_blk(256);
    const dim3 red_grid((unsigned)((K + 255) / 256)), red_blk(256);
    for (int i = 0; i < k_planes; ++i) {
        rb_status st = launch(svid_init_kernel, dim3(8), dim3(256), 0, stream, false, ws.v, K);
        for (int it = 0; it < iters && st == RB_OK; ++it) {
            st = launch(svid_av_kernel, av_grid, av_blk, 0, stream, false, W, (const float*)g,
                        (const float*)h, N, K, i, (const double*)ws.v, ws.u);
            if (st == RB_OK) st = launch(svid_normalize_kernel, dim3(1), dim3(1024), 0, stream, false, ws.u, (int64_t)N);
            if (st == RB_OK)
                st = launch(svid_atu_partial_kernel, atu_grid, atu_blk, 0, stream, false, W, (const float*)g,
                            (const float*)h, N, K, i, (const double*)ws.u, ws.vpart);
            if (st == RB_OK) st = launch(svid_atu_reduce_kernel, red_grid, red_blk, 0, stream, false,
                                         (const double*)ws.vpart, K, ws.v);
            if (st == RB_OK) st = launch(svid_normalize_kernel, dim3(1), dim3(1024), 0, stream, false, ws.v, (int64_t)K);
        }
        if (st == RB_OK)
            st = launch(svid_av_kernel, av_grid, av_blk, 0, stream, false, W, (const float*)g,
                        (const float*)h, N, K, i, (const double*)ws.v, ws.av);
        if (st == RB_OK)
            st = launch(svid_finish_kernel, dim3(1), dim3(1024), 0, stream, false, (const double*)ws.u,
                        (const double*)ws.v, (const double*)ws.av, N, K, i, g, h);
        if (st != RB_OK) return st;
    }
    return RB_OK;
}

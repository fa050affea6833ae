// rb_svid.cu -- greedy SVID scales on the device (RaBiT names Greedy SVID as
// the traditional initialiser it improves on; the greedy form takes, plane by
// plane, the rank-1 approximation of |R_{i-1}|), and the iterative residual
// SVID of RaBiT's Algorithm 1 without the I/O channel preprocessing
// (Gauss-Seidel sweeps: plane i is refitted to T_i = W - sum_{j != i}
// diag(g_j) B_j diag(h_j) with the latest values of the other planes,
// B_i = sign(T_i), (g_i, h_i) = rank-1 of |T_i|).
//
// For plane i the matrix A = |R_{i-1}| is never stored: every pass recomputes
// R_{i-1} from W and the scales of the earlier planes with the fp32
// recurrence of rb_pack (t = fl(g*h); R = fl(R -/+ t)).  Power iteration runs
// in float64 with fixed summation orders (warp tree per row, row chunks in
// order per column), so the result is deterministic.  One iteration is three
// launches (A v, A^T u in row chunks, the chunk sum).  The vectors stay
// unnormalised: the kernel that produces one also produces 1 / its norm --
// every CTA writes the sum of squares of its part, the last CTA to finish
// (a counter, no waiting) adds the parts in index order -- and the consumer
// scales on the fly, so no single-CTA normalisation pass sits between them.
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
    double* scal;     // [8]: 1/|u|, 1/|v|
    double* part;     // per-CTA sums of squares of the vector being produced
    unsigned* cnt;    // finished-CTA counters (zeroed by svid_init_kernel, reset by their last CTA)
    size_t bytes;
};
constexpr int kAvRows = 8;           // rows per CTA of svid_av_kernel (one warp each)

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
    const size_t nparts = (size_t)((N + kAvRows - 1) / kAvRows) > (size_t)((K + 255) / 256)
                        ? (size_t)((N + kAvRows - 1) / kAvRows) : (size_t)((K + 255) / 256);
    w.part = reinterpret_cast<double*>(p + off);  off += up(nparts * 8);
    w.cnt = reinterpret_cast<unsigned*>(p + off); off += 256;
    w.bytes = off;
    return w;
}

// Iterative form: the signs B_j of every plane, [k][N][K/32] words, bit c % 32
// of word c / 32 set for +1, after the power-iteration scratch.
size_t svid_sign_bytes(int N, int K, int k) { return ((size_t)k * N * (K / 32) * 4 + 255) / 256 * 256; }

// T_i[r][c] = W - sum_{j != i} g_j[r] h_j[c] B_j[r][c] in float64: each product
// of two fp32 values is exact, subtracted in plane order.
__device__ __forceinline__ double target_value(const float* W, const float* g, const float* h, const uint32_t* S,
                                               int N, int K, int k, int plane, int64_t r, int64_t c)
{
    double x = (double)W[r * K + c];
    const int64_t words = K / 32;
    for (int j = 0; j < k; ++j) {
        if (j == plane) continue;
        const double p = __dmul_rn((double)g[(int64_t)j * N + r], (double)h[(int64_t)j * K + c]);
        const bool pos = (S[((int64_t)j * N + r) * words + (c >> 5)] >> (c & 31)) & 1u;
        x = pos ? __dsub_rn(x, p) : __dadd_rn(x, p);
    }
    return x;
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

// A[r][c] for plane `plane`: |R_{plane-1}| (greedy) or |T_plane| (iterative, S != nullptr).
template <bool ITER>
__device__ __forceinline__ double abs_target(const float* W, const float* g, const float* h, const uint32_t* S,
                                             int N, int K, int k, int plane, int64_t r, int64_t c)
{
    if constexpr (ITER) return fabs(target_value(W, g, h, S, N, K, k, plane, r, c));
    else return abs_residual(W, g, h, N, K, plane, r, c);
}

// Called by every thread of every CTA after the CTA's sum of squares `mine`
// (valid in thread 0) is final: stores it as part[blockIdx.x]; the last CTA
// to arrive adds all parts in index order and writes 1 / sqrt(sum) (0 for a
// zero vector) to *inv, then re-arms the counter.
__device__ void finish_norm(double mine, double* part, unsigned* cnt, double* inv)
{
    __shared__ bool last;
    if (threadIdx.x == 0) {
        part[blockIdx.x] = mine;
        __threadfence();
        last = atomicAdd(cnt, 1u) == gridDim.x * gridDim.y - 1;
    }
    __syncthreads();
    if (last && threadIdx.x == 0) {
        __threadfence();
        double sum = 0.0;
        for (unsigned b = 0; b < gridDim.x * gridDim.y; ++b) sum += reinterpret_cast<volatile double*>(part)[b];
        *inv = sum > 0.0 ? 1.0 / sqrt(sum) : 0.0;
        *cnt = 0u;
    }
}

// out[r] = sum_c A[r][c] * (x[c] * sx)   (one warp per row; sx = 1/|x|, x unnormalised);
// with inv_out, also 1 / |out|.
template <bool ITER>
__global__ void __launch_bounds__(kAvRows * 32)
svid_av_kernel(const float* __restrict__ W, const float* __restrict__ g,
               const float* __restrict__ h, const uint32_t* __restrict__ S, int N, int K, int k,
               int plane, const double* __restrict__ x, const double* __restrict__ sxp, double* __restrict__ out,
               double* part, unsigned* cnt, double* inv_out)
{
    __shared__ double sq[kAvRows];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double sx = *sxp;
    const int64_t r = (int64_t)blockIdx.x * kAvRows + warp;
    double acc = 0.0;
    if (r < N) {
        for (int64_t c = lane; c < K; c += 32) acc += abs_target<ITER>(W, g, h, S, N, K, k, plane, r, c) * (x[c] * sx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) out[r] = acc;
    }
    if (!inv_out) return;
    if (lane == 0) sq[warp] = acc * acc;              // 0 for rows past N
    __syncthreads();
    double mine = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < kAvRows; ++w) mine += sq[w];
    finish_norm(mine, part, cnt, inv_out);
}

// vpart[chunk][c] = sum_{r in chunk} A[r][c] * (u[r] * su)   (rows in order; su = 1/|u|)
template <bool ITER>
__global__ void svid_atu_partial_kernel(const float* __restrict__ W, const float* __restrict__ g,
                                        const float* __restrict__ h, const uint32_t* __restrict__ S, int N, int K,
                                        int k, int plane, const double* __restrict__ u, const double* __restrict__ sup,
                                        double* __restrict__ vpart)
{
    const double su = *sup;
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int chunk = blockIdx.y;
    if (c >= K) return;
    const int64_t r0 = (int64_t)N * chunk / kRowChunks, r1 = (int64_t)N * (chunk + 1) / kRowChunks;
    double acc = 0.0;
    for (int64_t r = r0; r < r1; ++r) acc += abs_target<ITER>(W, g, h, S, N, K, k, plane, r, c) * (u[r] * su);
    vpart[(int64_t)chunk * K + c] = acc;
}

// v[c] = sum of the chunks in order; 1 / |v| through the CTAs' sums of squares.
__global__ void __launch_bounds__(256)
svid_atu_reduce_kernel(const double* __restrict__ vpart, int K, double* __restrict__ v, double* part,
                       unsigned* cnt, double* inv_v)
{
    __shared__ double sq[256];
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    double acc = 0.0;
    if (c < K) {
        for (int ch = 0; ch < kRowChunks; ++ch) acc += vpart[(int64_t)ch * K + c];
        v[c] = acc;
    }
    sq[threadIdx.x] = acc * acc;
    __syncthreads();
    for (int st = 128; st > 0; st >>= 1) {
        if ((int)threadIdx.x < st) sq[threadIdx.x] += sq[threadIdx.x + st];
        __syncthreads();
    }
    finish_norm(sq[0], part, cnt, inv_v);
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

// v0 = 1/sqrt(K) (already unit: 1/|v0| = 1); counters armed.
__global__ void svid_init_kernel(double* __restrict__ v, int K, double* scal, unsigned* cnt)
{
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < K; j += (int64_t)gridDim.x * blockDim.x)
        v[j] = 1.0 / sqrt((double)K);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        scal[1] = 1.0;
        cnt[0] = 0u;
    }
}

// With u = u_raw * su, v = v_raw * sv and av = A v:
// sigma = u^T av; g_i = fp32(sqrt(sigma) u); h_i = fp32(sqrt(sigma) v)
__global__ void svid_finish_kernel(const double* __restrict__ u, const double* __restrict__ v,
                                   const double* __restrict__ av, const double* __restrict__ scal, int N, int K,
                                   int plane, float* __restrict__ g, float* __restrict__ h)
{
    const double su = scal[0], sv = scal[1];
    const double sigma = block_dot(u, av, N) * su;
    const double rs = sigma > 0.0 ? sqrt(sigma) : 0.0;
    for (int64_t r = threadIdx.x; r < N; r += blockDim.x) g[(int64_t)plane * N + r] = (float)(rs * (u[r] * su));
    for (int64_t c = threadIdx.x; c < K; c += blockDim.x) h[(int64_t)plane * K + c] = (float)(rs * (v[c] * sv));
}

// Signs of the greedy pass (the fp32 recurrence of rb_pack): one warp per
// (row, word); the ballot of the 32 columns is the word of each plane.
__global__ void svid_signs_greedy_kernel(const float* __restrict__ W, const float* __restrict__ g,
                                         const float* __restrict__ h, int N, int K, int k, uint32_t* __restrict__ S)
{
    const int lane = threadIdx.x & 31;
    const int64_t words = K / 32, items = (int64_t)N * words;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items;
         it += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int64_t r = it / words, w = it % words, c = w * 32 + lane;
        float R = W[r * K + c];
        for (int p = 0; p < k; ++p) {
            const bool b = R >= 0.0f;
            const uint32_t word = __ballot_sync(0xffffffffu, b);
            if (lane == 0) S[((int64_t)p * N + r) * words + w] = word;
            const float tt = __fmul_rn(g[(int64_t)p * N + r], h[(int64_t)p * K + c]);
            R = b ? __fsub_rn(R, tt) : __fadd_rn(R, tt);
        }
    }
}

// B_plane = sign(T_plane) with the other planes' current scales and signs.
__global__ void svid_signs_update_kernel(const float* __restrict__ W, const float* __restrict__ g,
                                         const float* __restrict__ h, uint32_t* __restrict__ S, int N, int K, int k,
                                         int plane)
{
    const int lane = threadIdx.x & 31;
    const int64_t words = K / 32, items = (int64_t)N * words;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items;
         it += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int64_t r = it / words, w = it % words, c = w * 32 + lane;
        const bool b = target_value(W, g, h, S, N, K, k, plane, r, c) >= 0.0;
        const uint32_t word = __ballot_sync(0xffffffffu, b);
        if (lane == 0) S[((int64_t)plane * N + r) * words + w] = word;
    }
}

// Power iteration on A (greedy or iterative form) for one plane, then
// (g_plane, h_plane) = fp32(sqrt(sigma) u), fp32(sqrt(sigma) v).
template <bool ITER>
rb_status svid_plane(const float* W, float* g, float* h, const uint32_t* S, int N, int K, int k, int plane,
                     int iters, const SvidWs& ws, cudaStream_t stream)
{
    const dim3 av_grid((unsigned)((N + kAvRows - 1) / kAvRows)), av_blk(kAvRows * 32);
    const dim3 atu_grid((unsigned)((K + 255) / 256), kRowChunks), atu_blk(256);
    const dim3 red_grid((unsigned)((K + 255) / 256)), red_blk(256);
    double* inv_u = ws.scal;
    double* inv_v = ws.scal + 1;
    rb_status st = launch(svid_init_kernel, dim3(8), dim3(256), 0, stream, false, ws.v, K, ws.scal, ws.cnt);
    for (int it = 0; it < iters && st == RB_OK; ++it) {
        st = launch(svid_av_kernel<ITER>, av_grid, av_blk, 0, stream, false, W, (const float*)g, (const float*)h, S,
                    N, K, k, plane, (const double*)ws.v, (const double*)inv_v, ws.u, ws.part, ws.cnt, inv_u);
        if (st == RB_OK)
            st = launch(svid_atu_partial_kernel<ITER>, atu_grid, atu_blk, 0, stream, false, W, (const float*)g,
                        (const float*)h, S, N, K, k, plane, (const double*)ws.u, (const double*)inv_u, ws.vpart);
        if (st == RB_OK) st = launch(svid_atu_reduce_kernel, red_grid, red_blk, 0, stream, false,
                                     (const double*)ws.vpart, K, ws.v, ws.part, ws.cnt, inv_v);
    }
    if (st == RB_OK)                              // A v with the final v, no norm needed
        st = launch(svid_av_kernel<ITER>, av_grid, av_blk, 0, stream, false, W, (const float*)g, (const float*)h, S,
                    N, K, k, plane, (const double*)ws.v, (const double*)inv_v, ws.av, ws.part, ws.cnt,
                    (double*)nullptr);
    if (st == RB_OK)
        st = launch(svid_finish_kernel, dim3(1), dim3(1024), 0, stream, false, (const double*)ws.u,
                    (const double*)ws.v, (const double*)ws.av, (const double*)ws.scal, N, K, plane, g, h);
    return st;
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
    for (int i = 0; i < k_planes; ++i) {
        rb_status st = svid_plane<false>(W, g, h, nullptr, n_out, k_in, k_planes, i, iters, ws, stream);
        if (st != RB_OK) return st;
    }
    return RB_OK;
}

extern "C" size_t rb_svid_iterative_workspace_bytes(int n_out, int k_in, int k_planes)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 8) return 0;
    return svid_ws_layout(n_out, k_in, nullptr).bytes + svid_sign_bytes(n_out, k_in, k_planes);
}

extern "C" rb_status rb_svid_iterative(const float* W, int n_out, int k_in, int k_planes, int sweeps, int iters,
                                       float* g, float* h, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream)
{
    if (!W || !g || !h || !workspace) return RB_ERR_ARG;
    if (k_planes < 1 || k_planes > 8 || iters < 1 || iters > 10000 || sweeps < 0 || sweeps > 1000) return RB_ERR_ARG;
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0) return RB_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(g) || !aligned16(h) || !aligned16(workspace)) return RB_ERR_ALIGN;
    SvidWs ws = svid_ws_layout(n_out, k_in, workspace);
    if (workspace_bytes < ws.bytes + svid_sign_bytes(n_out, k_in, k_planes)) return RB_ERR_WORKSPACE;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    uint32_t* S = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + ws.bytes);
    for (int i = 0; i < k_planes; ++i) {                  // sweep 0: the greedy pass
        rb_status st = svid_plane<false>(W, g, h, nullptr, n_out, k_in, k_planes, i, iters, ws, stream);
        if (st != RB_OK) return st;
    }
    if (sweeps == 0) return RB_OK;
    const int64_t items = (int64_t)n_out * (k_in / 32);
    int64_t ctas = (items + 7) / 8;
    if (ctas > 16 * num_sms()) ctas = 16 * num_sms();
    rb_status st = launch(svid_signs_greedy_kernel, dim3((unsigned)ctas), dim3(256), 0, stream, false, W,
                          (const float*)g, (const float*)h, n_out, k_in, k_planes, S);
    for (int t = 0; t < sweeps && st == RB_OK; ++t) {
        for (int i = 0; i < k_planes && st == RB_OK; ++i) {
            st = launch(svid_signs_update_kernel, dim3((unsigned)ctas), dim3(256), 0, stream, false, W,
                        (const float*)g, (const float*)h, S, n_out, k_in, k_planes, i);
            if (st == RB_OK) st = svid_plane<true>(W, g, h, S, n_out, k_in, k_planes, i, iters, ws, stream);
        }
    }
    return st;
}

extern "C" size_t rb_svid_pack_workspace_bytes(int n_out, int k_in, int k_planes)
{
    return rb_svid_iterative_workspace_bytes(n_out, k_in, k_planes);
}

extern "C" rb_status rb_svid_pack(const float* W, int n_out, int k_in, int k_planes, int sweeps, int iters,
                                  float* g, float* h, uint32_t* planes, uint16_t* g16, uint16_t* h16,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream)
{
    if (!planes || !g16 || !h16) return RB_ERR_ARG;
    if (!aligned16(planes) || !aligned16(g16) || !aligned16(h16) || (dev_status && !aligned16(dev_status)))
        return RB_ERR_ALIGN;
    rb_status st = rb_svid_iterative(W, n_out, k_in, k_planes, sweeps, iters, g, h, workspace, workspace_bytes, stream);
    if (st != RB_OK) return st;
    return rb_pack(W, g, h, n_out, k_in, k_planes, planes, g16, h16, dev_status, stream);
}

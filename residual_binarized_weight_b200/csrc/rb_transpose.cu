// rb_transpose.cu -- sign planes of the transposed layer, for the gradient
// that reaches the layer input (RaBiT, Algorithm 2 backward pass:
// dX = dY What with What = sum_i diag(g_i) B_i diag(h_i)).
//
// What^T = sum_i diag(h_i) B_i^T diag(g_i) is again a residual binarized
// layer, K x N, with the scales exchanged.  Its planes are the bit-matrix
// transposes of the forward planes, so dX is the forward product of that
// layer applied to dY, by the same rb_gemv / rb_gemm kernels.
//
// One CTA moves 8 consecutive source blocks (8 row tiles of one column slice,
// 8 KB contiguous) to 8 consecutive destination blocks (8 KB contiguous):
// both sides are 16-byte coalesced streams, staged in shared memory.  Warp w
// owns source word w of the slice = destination row tile 8 s + w; for each of
// the 8 source row tiles it reads one 32 x 32 bit block (one word per lane,
// conflict-free thanks to the slot swizzle) and transposes it across the warp
// with five shuffle stages.  HBM-bound: 2 k N K / 8 bytes per call.
#include "rbw_internal.cuh"

namespace rbw {
namespace {

constexpr int kTrThreads = 256;

// 32 x 32 bit matrix held one row per lane (bit c = column c); returns column
// `lane`.  The stage of width j swaps bit j of the row index with bit j of the
// column index (the two off-diagonal j x j blocks of every 2j x 2j block
// change places); the five stages together swap row and column.
__device__ __forceinline__ uint32_t transpose32(uint32_t v, int lane)
{
    const uint32_t low_half[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int st = 0; st < 5; ++st) {
        const int j = 16 >> st;
        const uint32_t m = low_half[st];
        const uint32_t p = __shfl_xor_sync(0xffffffffu, v, j);
        v = (lane & j) ? ((v & ~m) | ((p >> j) & m)) : ((v & m) | ((p << j) & ~m));
    }
    return v;
}

// CTA (q, s, i): source row tiles 8q .. 8q+7 of column slice s of plane i
// -> destination row tiles 8s .. 8s+7 of column slice q of plane i.
__global__ void __launch_bounds__(kTrThreads)
transpose_kernel(const uint32_t* __restrict__ src, int N, int K, uint32_t* __restrict__ dst)
{
    __shared__ __align__(16) uint32_t in_s[8 * 256];
    __shared__ __align__(16) uint32_t out_s[8 * 256];
    const int q = blockIdx.x, s = blockIdx.y, i = blockIdx.z;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);     // source layer, N x K
    const int64_t St = num_slices(N), Ntt = num_row_tiles(K);   // transposed layer, K x N
    const int ntile = (int)(Nt - 8 * q < 8 ? Nt - 8 * q : 8);    // source tiles present (>= 1)
    const int nout = (int)(Ntt - 8 * s < 8 ? Ntt - 8 * s : 8);   // destination tiles present (>= 1)

    // absent source tiles (columns >= N of the transposed layer) read as zero
    const uint4* in = reinterpret_cast<const uint4*>(src + block_index(i, s, 8 * q, S, Nt) * 256);
    for (int x = threadIdx.x; x < 8 * 64; x += kTrThreads)
        reinterpret_cast<uint4*>(in_s)[x] = x < ntile * 64 ? __ldcs(in + x) : make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();

    // source words w >= nout of a ragged last slice are padding: no destination row
    if (warp < nout) {
        const int sw = (warp ^ (lane >> 2)) * 32 + lane;         // slot of logical word `warp`, row `lane`
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint32_t col = transpose32(in_s[t * 256 + sw], lane);
            out_s[warp * 256 + (t ^ (lane >> 2)) * 32 + lane] = col;
        }
    }
    __syncthreads();

    uint4* out = reinterpret_cast<uint4*>(dst + block_index(i, q, 8 * s, St, Ntt) * 256);
    for (int x = threadIdx.x; x < nout * 64; x += kTrThreads)
        __stcs(out + x, reinterpret_cast<const uint4*>(out_s)[x]);
}

}  // namespace
}  // namespace rbw

using namespace rbw;

extern "C" rb_status rb_transpose_planes(const rb_layer_t* layer, uint32_t* planes_t, cudaStream_t stream)
{
    if (!layer || !layer->planes || layer->reserved != 0 || !planes_t) return RB_ERR_ARG;
    const int N = layer->n_out, K = layer->k_in, k = layer->k_planes;
    if (k < 1 || k > 8) return RB_ERR_ARG;
    if (N < 32 || N % 32 != 0 || K < 32 || K % 32 != 0) return RB_ERR_SHAPE;
    if (!aligned16(layer->planes) || !aligned16(planes_t)) return RB_ERR_ALIGN;
    const size_t src_bytes = (size_t)k * num_slices(K) * num_row_tiles(N) * 1024;
    const size_t dst_bytes = (size_t)k * num_slices(N) * num_row_tiles(K) * 1024;
    const uintptr_t a = reinterpret_cast<uintptr_t>(layer->planes), b = reinterpret_cast<uintptr_t>(planes_t);
    if (a < b + dst_bytes && b < a + src_bytes) return RB_ERR_ARG;              // buffers must not overlap
    if (num_slices(K) > 65535) return RB_ERR_SHAPE;                              // grid y
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)num_slices(N), (unsigned)num_slices(K), (unsigned)k);
    return launch(transpose_kernel, grid, dim3(kTrThreads), 0, stream, false,
                  layer->planes, N, K, planes_t);
}

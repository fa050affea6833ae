// rb_pack.cu -- derive the residual sign planes and bit-pack them in one pass
// over W (RaBiT, Algorithm 2 forward pass: R_0 = W, B_i = sign(R_{i-1}),
// R_i = R_{i-1} - g_i h_i^T .* B_i; deployment keeps the planes and drops W).
//
// One warp owns a 32-row x 32-column item (one sign word per row and plane).
// Lane l holds column c = 256 s + 32 w + l and walks the 32 rows of the tile:
// each W row segment is one coalesced 128-byte load, the residual stays in a
// register across the k planes, and a warp ballot turns the 32 sign decisions
// of a row into its packed word, which the lane owning that row keeps.  After
// the tile, lane l stores its row's word to slot w ^ (l/4) of the tile block.
//
// The fp32 residual update is written with explicitly rounded intrinsics
// (__fmul_rn, __fadd_rn, __fsub_rn), so no fused multiply-add can be formed:
// t = fl(g*h), then R = fl(R -/+ t).  This makes the planes bit-exact with
// any IEEE fp32 evaluation of the same recurrence.
#include <float.h>

#include "rbw_internal.cuh"

namespace rbw {
namespace {

constexpr int kPackThreads = 256;

template <int KP, bool FULL>
__device__ __forceinline__ void pack_item(const float* __restrict__ W, const float* __restrict__ g,
                                          const float* __restrict__ h, int N, int K, int t, int c,
                                          int lane, uint32_t (&mine)[KP], int& bad)
{
    float hv[KP], gv[KP];
    const int my_row = t * 32 + lane;
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        hv[i] = h[(int64_t)i * K + c];
        gv[i] = (FULL || my_row < N) ? g[(int64_t)i * N + my_row] : 0.0f;
    }
    // all 32 row segments in flight at once (4 KB per warp) before any arithmetic
    const float* p = W + (int64_t)t * 32 * K + c;
    float wv[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) wv[j] = (FULL || t * 32 + j < N) ? __ldcs(p + (int64_t)j * K) : 0.0f;
    float nonfinite = 0.0f;                   // stays 0 unless some W is NaN or +-inf
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        float R = wv[j];
        nonfinite = fmaf(R, 0.0f, nonfinite);
#pragma unroll
        for (int i = 0; i < KP; ++i) {
            const float gi = __shfl_sync(0xffffffffu, gv[i], j);
            const float tt = __fmul_rn(gi, hv[i]);
            const bool b = R >= 0.0f;                   // sign(0) = +1, -0.0 too
            R = __fadd_rn(R, b ? -tt : tt);             // R - t or R + t, one rounding
            const uint32_t word = __ballot_sync(0xffffffffu, b);
            mine[i] = lane == j ? word : mine[i];
        }
    }
    bad |= nonfinite != 0.0f;
}

// Items are (row tile t, slice s, word w), numbered t-major so that the warps
// of a CTA stream neighbouring columns of the same rows; 32-bit index math.
// The recurrence is a chain of dependent shuffles, multiplies, adds and
// ballots, so latency is hidden by warps, not by ILP: four CTAs per SM (32
// warps) for k <= 4 (measured 19.7 against 23.0 us at 4096 x 4096, k = 2,
// with two; 224 against 261 us at 28672 x 8192).
template <int KP>
__global__ void __launch_bounds__(kPackThreads, KP <= 4 ? 4 : 2)
pack_kernel(const float* __restrict__ W, const float* __restrict__ g,
            const float* __restrict__ h, int N, int K,
            uint32_t* __restrict__ planes, int32_t* dev_status)
{
    const int lane = threadIdx.x & 31;
    const int S = (int)num_slices(K), Nt = (int)num_row_tiles(N);
    const int words = K / 32;                     // valid words per row
    const int items = Nt * words;
    const int gwarp = (int)((blockIdx.x * (unsigned)blockDim.x + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * (unsigned)blockDim.x) >> 5);
    const int full_tiles = N / 32;
    int bad = 0;

    for (int it = gwarp; it < items; it += nwarps) {
        const int t = it / words, wg = it - t * words;      // word wg of the row = slice wg/8, word wg%8
        const int c = wg * 32 + lane;
        uint32_t mine[KP];
#pragma unroll
        for (int i = 0; i < KP; ++i) mine[i] = 0u;
        if (t < full_tiles) {
            pack_item<KP, true>(W, g, h, N, K, t, c, lane, mine, bad);
        } else {
            pack_item<KP, false>(W, g, h, N, K, t, c, lane, mine, bad);
            if (t * 32 + lane >= N) {
#pragma unroll
                for (int i = 0; i < KP; ++i) mine[i] = 0u;   // padding rows of the last tile
            }
        }
        const int s = wg >> 3, w = wg & 7;
#pragma unroll
        for (int i = 0; i < KP; ++i)
            planes[word_offset(i, s, t * 32 + lane, w, S, Nt)] = mine[i];
    }
    // padding words of a ragged last slice (K % 256 != 0) stay zero
    const int pad_words = S * 8 - words;
    if (pad_words > 0) {
        for (int it = gwarp; it < Nt * pad_words; it += nwarps) {
            const int t = it / pad_words, wg = words + (it - t * pad_words);
#pragma unroll
            for (int i = 0; i < KP; ++i)
                planes[word_offset(i, wg >> 3, t * 32 + lane, wg & 7, S, Nt)] = 0u;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_dev_status(dev_status, RB_DEV_NONFINITE);
}

// fp16 copies of the scales (round to nearest even) with range checks.
__global__ void cast_scales_kernel(const float* __restrict__ g, const float* __restrict__ h,
                                   int64_t ng, int64_t nh, uint16_t* __restrict__ g16,
                                   uint16_t* __restrict__ h16, int32_t* dev_status)
{
    int flags = 0;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < ng + nh;
         x += (int64_t)gridDim.x * blockDim.x) {
        const float v = x < ng ? g[x] : h[x - ng];
        const __half q = __float2half_rn(v);
        if (!(fabsf(v) <= FLT_MAX)) flags |= RB_DEV_NONFINITE;
        else if (__hisinf(q)) flags |= RB_DEV_RANGE;
        const uint16_t bits = __half_as_ushort(q);
        if (x < ng) g16[x] = bits;
        else h16[x - ng] = bits;
    }
    if (flags) set_dev_status(dev_status, flags);
}

template <int KP>
rb_status launch_pack(const float* W, const float* g, const float* h, int N, int K,
                      uint32_t* planes, int32_t* dev_status, cudaStream_t stream)
{
    const int64_t items = num_row_tiles(N) * num_slices(K) * 8;
    if (items > INT32_MAX / 2) return RB_ERR_UNSUPPORTED;          // 32-bit item numbering
    const int64_t warps_per_cta = kPackThreads / 32;
    int64_t ctas = (items + warps_per_cta - 1) / warps_per_cta;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (ctas > cap) ctas = cap;
    return launch(pack_kernel<KP>, dim3((unsigned)ctas), dim3(kPackThreads), 0, stream, false,
                  W, g, h, N, K, planes, dev_status);
}

}  // namespace

rb_status pack_planes(const float* W, const float* g, const float* h, int N, int K, int kp, uint32_t* planes,
                      int32_t* dev_status, cudaStream_t stream)
{
    switch (kp) {
        case 1: return launch_pack<1>(W, g, h, N, K, planes, dev_status, stream);
        case 2: return launch_pack<2>(W, g, h, N, K, planes, dev_status, stream);
        case 3: return launch_pack<3>(W, g, h, N, K, planes, dev_status, stream);
        case 4: return launch_pack<4>(W, g, h, N, K, planes, dev_status, stream);
        case 5: return launch_pack<5>(W, g, h, N, K, planes, dev_status, stream);
        case 6: return launch_pack<6>(W, g, h, N, K, planes, dev_status, stream);
        case 7: return launch_pack<7>(W, g, h, N, K, planes, dev_status, stream);
        default: return launch_pack<8>(W, g, h, N, K, planes, dev_status, stream);
    }
}

}  // namespace rbw

using namespace rbw;

extern "C" rb_status rb_pack(const float* W, const float* g, const float* h,
                             int n_out, int k_in, int k_planes,
                             uint32_t* planes, uint16_t* g16, uint16_t* h16,
                             int32_t* dev_status, cudaStream_t stream)
{
    if (!W || !g || !h || !planes || !g16 || !h16) return RB_ERR_ARG;
    if (k_planes < 1 || k_planes > 8) return RB_ERR_ARG;
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0) return RB_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(g) || !aligned16(h) || !aligned16(planes) ||
        !aligned16(g16) || !aligned16(h16) || (dev_status && !aligned16(dev_status)))
        return RB_ERR_ALIGN;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;

    const int64_t ng = (int64_t)k_planes * n_out, nh = (int64_t)k_planes * k_in;
    int64_t cast_ctas = (ng + nh + 255) / 256;
    if (cast_ctas > 4 * num_sms()) cast_ctas = 4 * num_sms();
    rb_status st = launch(cast_scales_kernel, dim3((unsigned)cast_ctas), dim3(256), 0, stream,
                          false, g, h, ng, nh, g16, h16, dev_status);
    if (st != RB_OK) return st;
    return pack_planes(W, g, h, n_out, k_in, k_planes, planes, dev_status, stream);
}

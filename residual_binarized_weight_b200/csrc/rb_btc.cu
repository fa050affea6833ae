// rb_btc.cu -- binary codebook of a sign plane (BTC-LLM, "Binary codebook":
// binary k-means over the 16-column sign vectors, majority-vote centroids with
// sign(0) = +1, Hamming assignment by XOR + popcount, dynamic codebook size;
// index width ceil(log2 c), "Memory layout").
//
// The vectors are the v = 16 column groups of plane i; a vector is its 16-bit
// pattern (bit q = column 16j + q is +1), so the whole set is summarised by a
// 65536-bin histogram and every step works on distinct patterns weighted by
// their counts:
//   1. histogram (one pass over the plane, integer atomics);
//   2. the c = min(c_max, distinct patterns) most frequent patterns, count
//      descending then pattern ascending, are the initial centroids: the keys
//      count << 16 | (65535 - pattern) are sorted by one CTA (bitonic network);
//   3. `iters` rounds of assignment (each distinct pattern to the centroid at
//      the least Hamming distance, ties to the smaller index; the codebook sits
//      in shared memory) and majority update (per-bit signed count sums,
//      integer atomics, so the result does not depend on their order;
//      a centroid without members is kept), then a final assignment;
//   4. the per-row index streams: index j of row r at bits [j w, j w + w).
// Every step is integer arithmetic, so the codebook and the streams are
// bit-exact with any other evaluation of the same steps.
#include "rbw_internal.cuh"

namespace rbw {
namespace {

constexpr int kPatterns = 65536;

struct BtcWs {
    uint32_t* hist;       // [65536]
    uint64_t* keys;       // [65536]
    int32_t* assign;      // [65536]
    int32_t* sums;        // [c_max][16]
    uint32_t* members;    // [c_max]
    int32_t* scal;        // [0] = c
    size_t bytes;
};

BtcWs btc_ws_layout(int c_max, void* base)
{
    BtcWs w;
    size_t off = 0;
    auto take = [&](size_t b) { size_t o = off; off += (b + 255) / 256 * 256; return o; };
    const size_t o_hist = take(kPatterns * 4), o_keys = take(kPatterns * 8), o_assign = take(kPatterns * 4);
    const size_t o_sums = take((size_t)c_max * 16 * 4), o_mem = take((size_t)c_max * 4), o_scal = take(16);
    char* b = static_cast<char*>(base);
    w.hist = reinterpret_cast<uint32_t*>(b + o_hist);
    w.keys = reinterpret_cast<uint64_t*>(b + o_keys);
    w.assign = reinterpret_cast<int32_t*>(b + o_assign);
    w.sums = reinterpret_cast<int32_t*>(b + o_sums);
    w.members = reinterpret_cast<uint32_t*>(b + o_mem);
    w.scal = reinterpret_cast<int32_t*>(b + o_scal);
    w.bytes = off;
    return w;
}

__global__ void btc_clear_kernel(uint32_t* __restrict__ p, int64_t words)
{
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < words; x += (int64_t)gridDim.x * blockDim.x)
        p[x] = 0u;
}

// the 16-bit patterns of one plane word: columns 32 w .. 32 w + 15 and + 16 .. + 31
__device__ __forceinline__ uint32_t plane_word(const uint32_t* __restrict__ planes, int i, int64_t r, int64_t wg,
                                               int64_t S, int64_t Nt)
{
    return planes[word_offset(i, wg >> 3, r, (int)(wg & 7), S, Nt)];
}

__global__ void btc_hist_kernel(const uint32_t* __restrict__ planes, int N, int K, int i, uint32_t* __restrict__ hist)
{
    const int64_t S = num_slices(K), Nt = num_row_tiles(N), kw = K / 32;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < (int64_t)N * kw;
         x += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t word = plane_word(planes, i, x / kw, x % kw, S, Nt);
        atomicAdd(hist + (word & 0xFFFFu), 1u);
        atomicAdd(hist + (word >> 16), 1u);
    }
}

__global__ void btc_keys_kernel(const uint32_t* __restrict__ hist, uint64_t* __restrict__ keys)
{
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u < kPatterns) keys[u] = hist[u] ? ((uint64_t)hist[u] << 16) | (uint64_t)(0xFFFF - u) : 0ull;
}

// Bitonic sort of the 65536 keys into descending order by one CTA (the keys
// are distinct where non-zero, so the order is unique).
__global__ void __launch_bounds__(1024) btc_sort_kernel(uint64_t* __restrict__ keys)
{
    for (int k = 2; k <= kPatterns; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int x = threadIdx.x; x < kPatterns; x += 1024) {
                const int l = x ^ j;
                if (l > x) {
                    const uint64_t a = keys[x], b = keys[l];
                    const bool desc = (x & k) == 0;
                    if (desc ? a < b : a > b) { keys[x] = b; keys[l] = a; }
                }
            }
            __syncthreads();
        }
    }
}

// c = min(c_max, distinct patterns); centroid p = the p-th key's pattern
__global__ void btc_init_kernel(const uint64_t* __restrict__ keys, int c_max, uint16_t* __restrict__ codebook,
                                int32_t* __restrict__ scal, int32_t* __restrict__ c_out)
{
    __shared__ int s_u;
    if (threadIdx.x == 0) s_u = 0;
    __syncthreads();
    for (int x = threadIdx.x; x < kPatterns; x += blockDim.x)
        if (keys[x] != 0ull && (x == kPatterns - 1 || keys[x + 1] == 0ull)) s_u = x + 1;   // one writer
    __syncthreads();
    const int c = s_u < c_max ? s_u : c_max;
    for (int p = threadIdx.x; p < c_max; p += blockDim.x)
        codebook[p] = p < c ? (uint16_t)(0xFFFF - (int)(keys[p] & 0xFFFFull)) : (uint16_t)0;
    if (threadIdx.x == 0) {
        scal[0] = c;
        if (c_out) *c_out = c;
    }
}

// Every distinct pattern to its nearest centroid (ties to the smaller index).
__global__ void __launch_bounds__(256) btc_assign_kernel(const uint32_t* __restrict__ hist,
                                                         const uint16_t* __restrict__ codebook,
                                                         const int32_t* __restrict__ scal, int32_t* __restrict__ assign)
{
    extern __shared__ uint16_t cb[];
    const int c = scal[0];
    for (int p = threadIdx.x; p < c; p += blockDim.x) cb[p] = codebook[p];
    __syncthreads();
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= kPatterns) return;
    if (hist[u] == 0) { assign[u] = -1; return; }
    int best = 0, bd = 17;
    for (int p = 0; p < c && bd > 0; ++p) {
        const int d = __popc((uint32_t)u ^ (uint32_t)cb[p]);
        if (d < bd) { bd = d; best = p; }
    }
    assign[u] = best;
}

__global__ void btc_msum_kernel(const uint32_t* __restrict__ hist, const int32_t* __restrict__ assign,
                                int32_t* __restrict__ sums, uint32_t* __restrict__ members)
{
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= kPatterns || hist[u] == 0) return;
    const int p = assign[u];
    const int32_t n = (int32_t)hist[u];
    atomicAdd(members + p, (uint32_t)n);
#pragma unroll
    for (int q = 0; q < 16; ++q) atomicAdd(sums + p * 16 + q, ((u >> q) & 1) ? n : -n);
}

// majority per bit, +1 on a tie; a centroid without members is kept; the sums
// are cleared for the next round
__global__ void btc_update_kernel(int32_t* __restrict__ sums, uint32_t* __restrict__ members,
                                  const int32_t* __restrict__ scal, uint16_t* __restrict__ codebook)
{
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= scal[0]) return;
    if (members[p] > 0) {
        uint32_t cw = 0;
#pragma unroll
        for (int q = 0; q < 16; ++q) cw |= (sums[p * 16 + q] >= 0 ? 1u : 0u) << q;
        codebook[p] = (uint16_t)cw;
    }
    members[p] = 0;
#pragma unroll
    for (int q = 0; q < 16; ++q) sums[p * 16 + q] = 0;
}

// One thread per stream word: bit b of word q of row r is bit (32 q + b) % w
// of index (32 q + b) / w.
__global__ void btc_streams_kernel(const uint32_t* __restrict__ planes, int N, int K, int i, int w, int64_t rw,
                                   const int32_t* __restrict__ assign, uint32_t* __restrict__ streams)
{
    const int64_t S = num_slices(K), Nt = num_row_tiles(N), J = K / 16;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < (int64_t)N * rw;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = x / rw, q = x % rw;
        uint32_t out = 0u;
        int64_t jprev = -1;
        uint32_t v = 0u;
        for (int b = 0; b < 32; ++b) {
            const int64_t bit = 32 * q + b, j = bit / w;
            if (j >= J) break;
            if (j != jprev) {
                const uint32_t word = plane_word(planes, i, r, (16 * j) / 32, S, Nt);
                const uint32_t pat = (word >> (16 * (j & 1))) & 0xFFFFu;
                v = (uint32_t)assign[pat];
                jprev = j;
            }
            out |= ((v >> (bit % w)) & 1u) << b;
        }
        streams[x] = out;
    }
}

unsigned grid_for(int64_t items, int threads, int per_sm)
{
    int64_t ctas = (items + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms() * per_sm;
    return (unsigned)(ctas < 1 ? 1 : ctas > cap ? cap : ctas);
}

}  // namespace
}  // namespace rbw

using namespace rbw;

extern "C" int rb_btc_index_bits(int c_max)
{
    if (c_max < 1 || c_max > 65536) return 0;
    int w = 1;
    while ((1 << w) < c_max) ++w;
    return w;
}

extern "C" size_t rb_btc_row_words(int k_in, int index_bits)
{
    if (k_in < 32 || k_in % 32 != 0 || index_bits < 1 || index_bits > 16) return 0;
    return ((size_t)(k_in / 16) * (size_t)index_bits + 31) / 32;
}

extern "C" size_t rb_btc_encode_workspace_bytes(int c_max)
{
    if (c_max < 1 || c_max > 65536) return 0;
    return btc_ws_layout(c_max, nullptr).bytes;
}

extern "C" rb_status rb_btc_encode(const rb_layer_t* layer, int plane, int c_max, int iters, uint16_t* codebook,
                                   int32_t* c_out, uint32_t* indices, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream)
{
    if (!layer || !layer->planes || !codebook || !indices || layer->reserved != 0) return RB_ERR_ARG;
    if (layer->k_planes < 1 || layer->k_planes > 8 || plane < 0 || plane >= layer->k_planes) return RB_ERR_ARG;
    if (c_max < 1 || c_max > 65536 || iters < 0 || iters > 1000) return RB_ERR_ARG;
    const int N = layer->n_out, K = layer->k_in;
    if (N < 1 || K < 32 || K % 32 != 0) return RB_ERR_SHAPE;
    if ((int64_t)N * (K / 16) > INT32_MAX) return RB_ERR_UNSUPPORTED;       // counts held in int32
    // the planes as everywhere; the outputs only at their element size (one plane of
    // a [k][c_max] codebook array or a [k][N][row words] stream array is passed)
    const auto al = [](const void* q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; };
    if (!aligned16(layer->planes) || !al(codebook, 2) || !al(indices, 4) || (c_out && !al(c_out, 4)))
        return RB_ERR_ALIGN;
    const BtcWs ws = btc_ws_layout(c_max, workspace);
    if (!workspace || workspace_bytes < ws.bytes) return RB_ERR_WORKSPACE;
    if (!aligned16(workspace)) return RB_ERR_ALIGN;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    const int w = rb_btc_index_bits(c_max);
    const int64_t rw = (int64_t)rb_btc_row_words(K, w);
    const int cb_smem = (c_max * 2 + 15) / 16 * 16;
    if (cb_smem > 48 * 1024 &&
        cudaFuncSetAttribute(btc_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cb_smem) != cudaSuccess)
        return RB_ERR_CUDA;
    rb_status st = launch(btc_clear_kernel, dim3(grid_for(ws.bytes / 4, 256, 8)), dim3(256), 0, stream, false,
                          reinterpret_cast<uint32_t*>(ws.hist), (int64_t)(ws.bytes / 4));
    if (st != RB_OK) return st;
    st = launch(btc_hist_kernel, dim3(grid_for((int64_t)N * (K / 32), 256, 8)), dim3(256), 0, stream, false,
                layer->planes, N, K, plane, ws.hist);
    if (st != RB_OK) return st;
    st = launch(btc_keys_kernel, dim3(kPatterns / 256), dim3(256), 0, stream, false, (const uint32_t*)ws.hist,
                ws.keys);
    if (st != RB_OK) return st;
    st = launch(btc_sort_kernel, dim3(1), dim3(1024), 0, stream, false, ws.keys);
    if (st != RB_OK) return st;
    st = launch(btc_init_kernel, dim3(1), dim3(1024), 0, stream, false, (const uint64_t*)ws.keys, c_max, codebook,
                ws.scal, c_out);
    if (st != RB_OK) return st;
    for (int round = 0; round <= iters; ++round) {
        st = launch(btc_assign_kernel, dim3(kPatterns / 256), dim3(256), (size_t)cb_smem, stream, false,
                    (const uint32_t*)ws.hist, (const uint16_t*)codebook, (const int32_t*)ws.scal, ws.assign);
        if (st != RB_OK || round == iters) break;
        st = launch(btc_msum_kernel, dim3(kPatterns / 256), dim3(256), 0, stream, false, (const uint32_t*)ws.hist,
                    (const int32_t*)ws.assign, ws.sums, ws.members);
        if (st != RB_OK) break;
        st = launch(btc_update_kernel, dim3((c_max + 255) / 256), dim3(256), 0, stream, false, ws.sums, ws.members,
                    (const int32_t*)ws.scal, codebook);
        if (st != RB_OK) break;
    }
    if (st != RB_OK) return st;
    return launch(btc_streams_kernel, dim3(grid_for((int64_t)N * rw, 256, 8)), dim3(256), 0, stream, false,
                  layer->planes, N, K, plane, w, rw, (const int32_t*)ws.assign, indices);
}

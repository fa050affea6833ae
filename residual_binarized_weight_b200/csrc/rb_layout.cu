// rb_layout.cu -- conversions between the plain row-major packing of the sign
// planes and this library's tiled storage layout.
//
// The plain form is the one RaBiT's kernel paragraph names ("32 columns packed
// into one uint32_t"): words [k][N][K/32], column c of row r at bit c % 32 of
// word c / 32, bit = 1 meaning B = +1.  The storage layout groups the same
// words into (plane, 256-column slice, 32-row tile) blocks with XOR-swizzled
// slots (rbw.h).  Both directions are pure word permutations (bits never move
// inside a word), so planes packed by another tool can be handed to the
// decode and prefill kernels, and planes derived here can be exported.
//
// One thread per destination word.  from_rowmajor writes the storage layout
// in order (coalesced stores); a warp's 32 reads fall in 32 rows of one block,
// each the 32-byte sector holding that row's 8 words of the slice, so every
// sector is fetched once.  to_rowmajor is the mirror image.  HBM-bound:
// k N K / 8 bytes read and written.
#include "rbw_internal.cuh"

namespace rbw {
namespace {

constexpr int kLayoutThreads = 256;

__global__ void __launch_bounds__(kLayoutThreads)
from_rowmajor_kernel(const uint32_t* __restrict__ rm, int N, int K, int kp, uint32_t* __restrict__ planes)
{
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int64_t kw = K / 32;                                   // words per row in the plain form
    const int64_t total = (int64_t)kp * S * Nt * 256;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = x >> 8;
        const int slot = (int)((x >> 5) & 7), rho = (int)(x & 31);
        const int64_t t = blk % Nt, s = (blk / Nt) % S, i = blk / (Nt * S);
        const int64_t r = t * 32 + rho, cw = s * 8 + (slot ^ (rho >> 2));
        planes[x] = (r < N && cw < kw) ? __ldg(rm + (i * N + r) * kw + cw) : 0u;
    }
}

__global__ void __launch_bounds__(kLayoutThreads)
to_rowmajor_kernel(const uint32_t* __restrict__ planes, int N, int K, int kp, uint32_t* __restrict__ rm)
{
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int64_t kw = K / 32;
    const int64_t total = (int64_t)kp * N * kw;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t cw = x % kw, r = (x / kw) % N, i = x / (kw * N);
        rm[x] = __ldg(planes + word_offset((int)i, cw >> 3, r, (int)(cw & 7), S, Nt));
    }
}

rb_status check_layout_args(const void* src, int n_out, int k_in, int k_planes, const void* dst)
{
    if (!src || !dst) return RB_ERR_ARG;
    if (k_planes < 1 || k_planes > 8) return RB_ERR_ARG;
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0) return RB_ERR_SHAPE;
    if (!aligned16(src) || !aligned16(dst)) return RB_ERR_ALIGN;
    return RB_OK;
}

// The two buffers may not overlap: [a, a + na) and [b, b + nb) in bytes.
bool overlaps(const void* a, size_t na, const void* b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

unsigned layout_grid(int64_t words)
{
    int64_t ctas = (words + kLayoutThreads - 1) / kLayoutThreads;
    const int64_t cap = (int64_t)num_sms() * 16;
    return (unsigned)(ctas < cap ? (ctas < 1 ? 1 : ctas) : cap);
}

}  // namespace
}  // namespace rbw

using namespace rbw;

extern "C" size_t rb_rowmajor_words(int n_out, int k_in, int k_planes)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 8) return 0;
    return (size_t)k_planes * (size_t)n_out * (size_t)(k_in / 32);
}

extern "C" rb_status rb_planes_from_rowmajor(const uint32_t* rowmajor, int n_out, int k_in, int k_planes,
                                             uint32_t* planes, cudaStream_t stream)
{
    rb_status st = check_layout_args(rowmajor, n_out, k_in, k_planes, planes);
    if (st != RB_OK) return st;
    const size_t nw = rb_packed_words(n_out, k_in, k_planes);
    if (overlaps(rowmajor, rb_rowmajor_words(n_out, k_in, k_planes) * 4, planes, nw * 4)) return RB_ERR_ARG;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    return launch(from_rowmajor_kernel, dim3(layout_grid((int64_t)nw)), dim3(kLayoutThreads), 0, stream, false,
                  rowmajor, n_out, k_in, k_planes, planes);
}

extern "C" rb_status rb_planes_to_rowmajor(const uint32_t* planes, int n_out, int k_in, int k_planes,
                                           uint32_t* rowmajor, cudaStream_t stream)
{
    rb_status st = check_layout_args(planes, n_out, k_in, k_planes, rowmajor);
    if (st != RB_OK) return st;
    const size_t nr = rb_rowmajor_words(n_out, k_in, k_planes);
    if (overlaps(planes, rb_packed_words(n_out, k_in, k_planes) * 4, rowmajor, nr * 4)) return RB_ERR_ARG;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    return launch(to_rowmajor_kernel, dim3(layout_grid((int64_t)nr)), dim3(kLayoutThreads), 0, stream, false,
                  planes, n_out, k_in, k_planes, rowmajor);
}

// ---------------------------------------------------------------- row shards
// Rows [row0, row0 + rows) of a layer as a layer of their own (row0 a multiple
// of 32): every (plane, slice, row tile) block of the shard is the source
// block of tile row0/32 + t, with the rows past `rows` of a ragged last tile
// cleared; g16 rows are copied, h16 is the same array for every shard.  This
// is the per-GPU part of a row-parallel split (each GPU applies its shard to
// the full X and the outputs are concatenated along N).
namespace rbw {
namespace {

__global__ void __launch_bounds__(kLayoutThreads)
shard_rows_kernel(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ g16, int N, int K, int kp,
                  int row0, int rows, uint32_t* __restrict__ out, uint16_t* __restrict__ g_out)
{
    const int64_t S = num_slices(K), Nt = num_row_tiles(N), Ntd = num_row_tiles(rows);
    const int64_t t0 = row0 / 32;
    const int64_t total = (int64_t)kp * S * Ntd * 256, ng = (int64_t)kp * rows;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total + ng;
         x += (int64_t)gridDim.x * blockDim.x) {
        if (x < total) {
            const int64_t blk = x >> 8, t = blk % Ntd, s = (blk / Ntd) % S, i = blk / (Ntd * S);
            const int rho = (int)(x & 31);
            out[x] = t * 32 + rho < rows ? __ldg(planes + block_index((int)i, s, t0 + t, S, Nt) * 256 + (x & 255))
                                         : 0u;
        } else {
            const int64_t y = x - total, i = y / rows, r = y % rows;
            g_out[y] = g16[i * N + row0 + r];
        }
    }
}

}  // namespace
}  // namespace rbw

extern "C" rb_status rb_shard_rows(const rb_layer_t* layer, int row0, int rows, uint32_t* planes_out,
                                   uint16_t* g16_out, cudaStream_t stream)
{
    if (!layer || !layer->planes || !layer->g16 || !planes_out || !g16_out || layer->reserved != 0) return RB_ERR_ARG;
    if (layer->k_planes < 1 || layer->k_planes > 8) return RB_ERR_ARG;
    if (layer->n_out < 1 || layer->k_in < 32 || layer->k_in % 32 != 0) return RB_ERR_SHAPE;
    if (row0 < 0 || row0 % 32 != 0 || rows < 1 || (int64_t)row0 + rows > layer->n_out) return RB_ERR_SHAPE;
    if (!aligned16(layer->planes) || !aligned16(planes_out) || !aligned16(g16_out)) return RB_ERR_ALIGN;
    const size_t nw = rb_packed_words(rows, layer->k_in, layer->k_planes);
    const size_t nsrc = rb_packed_words(layer->n_out, layer->k_in, layer->k_planes);
    if (overlaps(layer->planes, nsrc * 4, planes_out, nw * 4)) return RB_ERR_ARG;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    return launch(shard_rows_kernel, dim3(layout_grid((int64_t)nw + (int64_t)layer->k_planes * rows)),
                  dim3(kLayoutThreads), 0, stream, false, layer->planes, layer->g16, layer->n_out, layer->k_in,
                  layer->k_planes, row0, rows, planes_out, g16_out);
}

// rb_gemv.cu -- decode-time application Y = sum_i g_i .* (B_i (h_i .* x))
// (RaBiT, "Residual binarization": matmul-free inference with additions and
// element-wise scaling; the k paths run side by side).
//
// M = 1, k <= 4: byte-table kernel.  For each 256-column slice a CTA builds,
// per plane, T_i[byte][group] = sum_{q<8} (bit q of byte ? +1 : -1) * hx_i[8*group + q]
// with hx_i = h_i .* x formed exactly in fp32 (a bf16 x fp16 product has at
// most 19 significant bits).  One table lookup then stands for eight signed
// additions.  Lane l of a warp owns row l of a 32-row tile; the XOR-swizzled
// storage layout hands it logical word (slot ^ l/4), so at every step the 32
// lanes read 32 different groups: group (4*slot + b) ^ l lives in smem bank
// ((4*slot + b) ^ l) and the lookups are conflict-free.  One PRMT forms the
// byte offset (byte << 8 | group << 2), one LDS fetches the entry, one FADD
// accumulates: three instructions per eight weights.  The CTAs that share a
// row chunk form a thread-block cluster, one CTA per group of slices; their
// per-row sums are pushed over distributed shared memory to the CTA that owns
// the row, and after one cluster barrier added in rank order, so the result is
// deterministic and no global workspace is needed.  Weights, g and h are
// fetched before the programmatic-dependent-launch wait; only X after it.
//
// M >= 2 (up to 64), and M = 1 with k > 4: tensor-core kernel (mma.sync,
// fp16 operands, fp32 accumulation) with the sign words expanded to +-h in
// registers; see gemv_mma_kernel.
#include "rbw_internal.cuh"

#include <atomic>

#include <mutex>

namespace rbw {
namespace {

// Threads per CTA: 256 (two CTAs per SM) while the tables of a plane pair fit
// 64 KB; 512 for k >= 3, whose 128 KB of tables leave room for one CTA per SM,
// so that an SM still runs 16 warps.
template <int KP> struct LutCfg {
    static constexpr int threads = KP >= 3 ? 512 : 256;
    static constexpr int warps = threads / 32;
    static constexpr int min_blocks = KP >= 3 ? 1 : 2;
};
constexpr int kLutPF = 2;              // row tiles per warp held in registers ahead of use

__host__ __device__ constexpr int lut_table_bytes(int kp) { return ((kp + 1) / 2) * 65536; }

template <int KP>
__device__ __forceinline__ void lut_load_tile(uint32_t (&wd)[KP][8], const uint32_t* __restrict__ planes,
                                              int64_t s, int64_t t, int64_t S, int64_t Nt, int lane)
{
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        const uint32_t* blk = planes + block_index(i, s, t, S, Nt) * 256 + lane;
#pragma unroll
        for (int sl = 0; sl < 8; ++sl) wd[i][sl] = __ldcs(blk + sl * 32);
    }
}

// g as raw fp16 bits: converting here would stall on the load before the wait.
template <int KP>
__device__ __forceinline__ void lut_load_g(uint16_t (&gv)[KP], const uint16_t* __restrict__ g16, int64_t r, int N)
{
#pragma unroll
    for (int i = 0; i < KP; ++i) gv[i] = r < N ? g16[(int64_t)i * N + r] : (uint16_t)0;
}

// The byte tables start at the dynamic shared memory base.  That base is the
// same for every thread of a CTA, so the compiler keeps it in a uniform
// register and folds it, with the plane's constant offset, into the LDS
// address: a lookup stays PRMT + LDS + FADD.  (The base is not a compile-time
// constant: in a cluster launch the shared window of CTA rank r starts at
// r << 24.)

template <int I>
__device__ __forceinline__ float lut_entry(uint32_t tbase, uint32_t off) {
    constexpr uint32_t C = (uint32_t)((I >> 1) * 65536 + (I & 1) * 128);
    return lds_f32(tbase + C + off);
}


// Per-row sums (red) plus, with a cluster, the receive area of the rows this CTA
// sums: CS slots of at most ceil(rows/CS) rows, which never exceeds rows + CS;
// rounded up to 16 bytes.
__host__ __device__ inline int lut_row_bytes(int64_t Nt, int R, int CS)
{
    const int64_t rows = ((Nt + R - 1) / R) * 32;
    return (int)(((CS > 1 ? 2 * rows + CS : rows) + 3) / 4 * 16);
}

// Byte tables of slice s for all KP planes (thread (group gg, part) writes
// the part's 256 / (threads / 32) consecutive bytes of group gg).  Plane i's entry
// (byte, group) sits at region(i/2) + byte*256 + (i%2)*128 + group*4.
template <int KP>
__device__ __forceinline__ void lut_load_h(uint4 (&hr)[KP], const uint16_t* __restrict__ h16, int64_t s, int K)
{
    const int64_t c0 = s * 256 + (threadIdx.x & 31) * 8;
#pragma unroll
    for (int i = 0; i < KP; ++i)
        hr[i] = c0 < K ? *reinterpret_cast<const uint4*>(h16 + (int64_t)i * K + c0) : make_uint4(0, 0, 0, 0);
}

template <int KP, int PARTS>
__device__ __forceinline__ void lut_build_part(float* lut, const uint4 (&hrr)[KP], const uint16_t* __restrict__ X,
                                               int64_t s, int K, int gg, int part)
{
    const int64_t c0 = s * 256 + gg * 8;
    const bool col_ok = c0 < K;                   // K % 32 == 0: a group is all in or all out
    float xv[8];
    const uint4 xr = col_ok ? *reinterpret_cast<const uint4*>(X + c0) : make_uint4(0, 0, 0, 0);
    const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        xv[2 * q] = bf16_bits_to_f32(xw[q] & 0xffffu);
        xv[2 * q + 1] = bf16_bits_to_f32(xw[q] >> 16);
    }
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        const uint32_t hw[4] = {hrr[i].x, hrr[i].y, hrr[i].z, hrr[i].w};
        float v[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            v[2 * q] = __half2float(__ushort_as_half((unsigned short)(hw[q] & 0xffffu))) * xv[2 * q];
            v[2 * q + 1] = __half2float(__ushort_as_half((unsigned short)(hw[q] >> 16))) * xv[2 * q + 1];
        }
        float L[16];                              // signed sums of columns 0..3 of the group
        L[0] = -((v[0] + v[1]) + (v[2] + v[3]));
#pragma unroll
        for (int n = 1; n < 16; ++n) {
            const int low = n & -n;
            const int q = low == 1 ? 0 : low == 2 ? 1 : low == 4 ? 2 : 3;
            L[n] = L[n & (n - 1)] + 2.0f * v[q];
        }
        constexpr int kBPP = 256 / PARTS;                       // table bytes per part (thread of a group)
        constexpr int kHN = kBPP >= 16 ? kBPP / 16 : 1;         // high nibbles per part
        float Hh[kHN];                            // signed sums of columns 4..7 for this part's high nibbles
#pragma unroll
        for (int e = 0; e < kHN; ++e) {
            const int n = kHN * part + e;
            float acc = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) acc += ((n >> q) & 1) ? v[4 + q] : -v[4 + q];
            Hh[e] = acc;
        }
        char* base = reinterpret_cast<char*>(lut) + (i >> 1) * 65536 + (i & 1) * 128 + gg * 4;
#pragma unroll
        for (int j = 0; j < kBPP; ++j) {
            const int b = kBPP * part + j;
            *reinterpret_cast<float*>(base + b * 256) = L[b & 15] + Hh[(b >> 4) - kHN * part];
        }
    }
}

template <int KP>
__device__ __forceinline__ void lut_build(float* lut, const uint4 (&hrr)[KP], const uint16_t* __restrict__ X,
                                          int64_t s, int K)
{
    lut_build_part<KP, LutCfg<KP>::warps>(lut, hrr, X, s, K, threadIdx.x & 31, threadIdx.x >> 5);
}

// All lookups of the kLutPF register-held tiles: for each word slot, the PRMT
// offsets of 4 bytes x kLutPF tiles x KP planes are formed first, then all the
// LDS are issued, then the FADDs, so each warp keeps 4*kLutPF*KP independent
// table reads in flight.
template <int KP>
__device__ __forceinline__ void lut_lookups(float (&acc)[kLutPF][KP][2], const uint32_t (&wd)[kLutPF][KP][8],
                                            const uint32_t (&G)[8], const uint32_t (&SEL)[4], uint32_t tbase)
{
#pragma unroll
    for (int sl = 0; sl < 8; ++sl) {
        uint32_t off[4][kLutPF][KP];
        float e[4][kLutPF][KP];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int p = 0; p < kLutPF; ++p)
#pragma unroll
                for (int i = 0; i < KP; ++i) off[b][p][i] = prmt(wd[p][i][sl], G[sl], SEL[b]);
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int p = 0; p < kLutPF; ++p) {
                e[b][p][0] = lut_entry<0>(tbase, off[b][p][0]);
                if constexpr (KP > 1) e[b][p][1] = lut_entry<1>(tbase, off[b][p][1]);
                if constexpr (KP > 2) e[b][p][2] = lut_entry<2>(tbase, off[b][p][2]);
                if constexpr (KP > 3) e[b][p][3] = lut_entry<3>(tbase, off[b][p][3]);
            }
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int p = 0; p < kLutPF; ++p)
#pragma unroll
                for (int i = 0; i < KP; ++i) acc[p][i][b & 1] += e[b][p][i];
    }
}

// The row tiles of one slice for this warp: t = tb + warp + 8 j, j < nw, kLutPF
// at a time from registers.  Each slot is refilled right after its lookups:
// with the tile kLutPF further on, clamped to the warp's last tile when that
// runs past the end (the slot is then not used), and after the last group with
// tile j = slot of the CTA's next slice, so a slice starts on loaded registers.
// Tile validity only gates the red[] update, so no load is guarded by a branch.
// (Software L2 prefetches further ahead, per line or as bulk copies of whole
// tiles, measured 1-10 % slower: the loads two tiles ahead already keep up.)
template <int KP>
__device__ __forceinline__ void lut_tiles(uint32_t (&wd)[kLutPF][KP][8], uint16_t (&gv)[kLutPF][KP],
                                          const uint32_t (&G)[8], const uint32_t (&SEL)[4], uint32_t tbase,
                                          float* red, const uint32_t* __restrict__ planes,
                                          const uint16_t* __restrict__ g16, int64_t s, int64_t s_next,
                                          int64_t S, int64_t Nt, int N, int tb, int te, int warp, int lane)
{
    const int nw = te - tb > warp ? (te - tb - warp + LutCfg<KP>::warps - 1) / LutCfg<KP>::warps : 0;
    const int iters = (nw + kLutPF - 1) / kLutPF;
    const bool has_next = s_next < S;
    const uint32_t* cur[KP];
    const uint32_t* nxt[KP];
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        cur[i] = planes + block_index(i, s, 0, S, Nt) * 256 + lane;
        nxt[i] = has_next ? planes + block_index(i, s_next, 0, S, Nt) * 256 + lane : cur[i];
    }
    const int t_w = tb + warp;                    // the warp's first tile
    for (int it = 0; it < iters; ++it) {
        float acc[kLutPF][KP][2];
#pragma unroll
        for (int p = 0; p < kLutPF; ++p)
#pragma unroll
            for (int i = 0; i < KP; ++i) acc[p][i][0] = acc[p][i][1] = 0.0f;
        lut_lookups<KP>(acc, wd, G, SEL, tbase);
        const bool last = it + 1 == iters;
#pragma unroll
        for (int p = 0; p < kLutPF; ++p) {
            const int j = it * kLutPF + p;
            float pr = 0.0f;
#pragma unroll
            for (int i = 0; i < KP; ++i)
                pr += __half2float(__ushort_as_half(gv[p][i])) * (acc[p][i][0] + acc[p][i][1]);
            if (j < nw) red[(j * LutCfg<KP>::warps + warp) * 32 + lane] += pr;
            if (!last || (has_next && p < nw)) {
                const int jn = last ? p : min(j + kLutPF, nw - 1);
                const size_t tn = (size_t)(t_w + jn * LutCfg<KP>::warps);
#pragma unroll
                for (int i = 0; i < KP; ++i) {
                    const uint32_t* q = (last ? nxt[i] : cur[i]) + tn * 256;
#pragma unroll
                    for (int sl = 0; sl < 8; ++sl) wd[p][i][sl] = __ldcs(q + sl * 32);
                }
                const int64_t r = min((int64_t)tn * 32 + lane, (int64_t)N - 1);
#pragma unroll
                for (int i = 0; i < KP; ++i) gv[p][i] = g16[(int64_t)i * N + r];
            }
        }
    }
}

// Grid: R clusters of CS CTAs.  Cluster c owns row tiles [Nt*c/R, Nt*(c+1)/R);
// its CTA of rank j handles slices j, j+CS, j+2CS, ... < S.  Per-row slice sums
// stay in shared memory until each is stored into the receive area of the CTA
// that sums that row; after one cluster barrier that CTA adds the CS partial
// sums in rank order and writes Y.  With CS = 1 the CTA owns every slice.
constexpr int kMaxBatch = 128;         // layers per launch of the byte-table kernel

// Independent layers of one shape handled by one launch (pointers per layer).
struct LutBatch {
    const uint32_t* planes[kMaxBatch];
    const uint16_t* g16[kMaxBatch];
    const uint16_t* h16[kMaxBatch];
    const uint16_t* X[kMaxBatch];
    void* Y[kMaxBatch];
};

template <int KP>
__global__ void __launch_bounds__(LutCfg<KP>::threads, LutCfg<KP>::min_blocks)
gemv_lut_kernel(const __grid_constant__ LutBatch batch, int N, int K, int CS, int R, int ydt)
{
    extern __shared__ __align__(1024) float lut[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int rank = CS > 1 ? (int)cluster_rank() : 0;
    const int layer = blockIdx.x / (CS * R);
    const uint32_t* __restrict__ planes = batch.planes[layer];
    const uint16_t* __restrict__ g16 = batch.g16[layer];
    const uint16_t* __restrict__ h16 = batch.h16[layer];
    const uint16_t* __restrict__ X = batch.X[layer];
    void* __restrict__ Y = batch.Y[layer];
    const int chunk = (blockIdx.x / CS) % R;
    const int64_t t_begin = Nt * chunk / R, t_end = Nt * (chunk + 1) / R;
    const int64_t chunk_rows = (t_end - t_begin) * 32;
    float* red = lut + lut_table_bytes(KP) / 4;   // per-row sums of this CTA's slices

    // ---- before the dependency wait: everything that does not depend on X --
    // the weights of the first slice's first tiles, their g values, h.
    uint32_t wd[kLutPF][KP][8];
    uint16_t gv[kLutPF][KP];
    uint4 hr[KP];
    const int64_t s_first = rank;
#pragma unroll
    for (int p = 0; p < kLutPF; ++p) {
        const int64_t t = t_begin + warp + (int64_t)p * LutCfg<KP>::warps;
        if (t < t_end && s_first < S) {
            lut_load_tile<KP>(wd[p], planes, s_first, t, S, Nt, lane);
            lut_load_g<KP>(gv[p], g16, t * 32 + lane, N);
        } else {                                  // an unused slot: defined values for its lookups
#pragma unroll
            for (int i = 0; i < KP; ++i) {
#pragma unroll
                for (int sl = 0; sl < 8; ++sl) wd[p][i][sl] = 0u;
                gv[p][i] = 0;
            }
        }
    }
    if (s_first < S) lut_load_h<KP>(hr, h16, s_first, K);
    for (int64_t x = threadIdx.x; x < chunk_rows; x += LutCfg<KP>::threads) red[x] = 0.0f;

    // Per-lane lookup constants: G[sl] byte b' = group offset ((4 sl + b') ^ lane) * 4;
    // SEL[b'] = PRMT selector giving (word byte (b' ^ lane%4)) << 8 | G byte b', zeros above.
    uint32_t G[8], SEL[4];
#pragma unroll
    for (int sl = 0; sl < 8; ++sl) {
        uint32_t gw = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) gw |= (uint32_t)((((4 * sl + b) ^ lane) * 4) & 0xff) << (8 * b);
        G[sl] = gw;
    }
#pragma unroll
    for (int b = 0; b < 4; ++b)
        SEL[b] = (uint32_t)(4 + b) | ((uint32_t)(b ^ (lane & 3)) << 4) |
                 ((uint32_t)(12 + b) << 8) | ((uint32_t)(12 + b) << 12);

    const uint32_t tbase = smem_u32(lut);
    pdl_launch_dependents();
    pdl_wait();

    for (int64_t s = s_first; s < S; s += CS) {
        if (s != s_first) {
            __syncthreads();                      // the previous slice's lookups are done with the tables
            lut_load_h<KP>(hr, h16, s, K);        // (its tiles are in registers already)
        }
        lut_build<KP>(lut, hr, X, s, K);
        __syncthreads();

        lut_tiles<KP>(wd, gv, G, SEL, tbase, red, planes, g16, s, s + CS, S, Nt, N, (int)t_begin,
                            (int)t_end, warp, lane);
    }

    // ---- cross-slice sum
    if (CS == 1) {
        __syncthreads();
        for (int64_t x = threadIdx.x; x < chunk_rows; x += LutCfg<KP>::threads) {
            const int64_t r = t_begin * 32 + x;
            if (r < N) store_y(Y, ydt, r, red[x]);
        }
        return;
    }
    // Rows [x0(j), x1(j)) of the chunk are summed by rank j.  Every CTA stores its
    // partial of such a row into rank j's receive area, slot (own rank, row);
    // one cluster barrier (release / acquire) later each CTA adds its rows'
    // CS partials from local shared memory, in rank order.
    float* recv = red + chunk_rows;
    const uint32_t recv_s = smem_u32(recv);
    const int rows = (int)chunk_rows;             // <= 32 * Nt, fits 32 bits
    __syncthreads();                              // red[] complete within the CTA
    {                                             // rows [x0(j), x1(j)) go to rank j
        const int tpo = LutCfg<KP>::threads / CS;         // threads per destination rank
        const int j = threadIdx.x / tpo;
        if (j < CS) {
            const int jx0 = rows * j / CS, span = rows * (j + 1) / CS - jx0;
            const uint32_t dst = recv_s + (uint32_t)(rank * span) * 4u;
            for (int xo = threadIdx.x - j * tpo; xo < span; xo += tpo)
                st_dsmem_f32(dst + (uint32_t)xo * 4u, (uint32_t)j, red[jx0 + xo]);
        }
    }
    cluster_sync_all();
    const int x0 = rows * rank / CS, my_span = rows * (rank + 1) / CS - x0;
    for (int xo = threadIdx.x; xo < my_span; xo += LutCfg<KP>::threads) {
        float y = 0.0f;
        for (int j = 0; j < CS; ++j) y += recv[j * my_span + xo];
        const int64_t r = t_begin * 32 + x0 + xo;
        if (r < N) store_y(Y, ydt, r, y);
    }
}

// ---------------------------------------------------------------- binary-codebook LUT kernel
// rb_btc_gemv (BTC-LLM, "LUT-GEMM").  CTA = (block of 8 row tiles, slice s):
// it builds the byte tables of slice s, then warp w takes tile 8 b + w with
// lane l on byte group l of the slice (16-column group l / 2, its low or high
// byte), so the 32 lanes read 32 different groups of the table (conflict-free)
// and every lane walks the tile's 32 rows: index from the row's stream
// (funnel shift of two words), pattern from the codebook (read-only cache),
// one table entry.  Each lane then holds 32 partial row sums; a transposing
// warp reduction (16 + 8 + 4 + 2 + 1 shuffles) leaves row r's sum in lane r,
// which applies g and writes the slice's partial.
constexpr int kBtcWarps = 8;

// a[32] per lane -> the sum over the warp's lanes of a[lane], in lane `lane`
__device__ __forceinline__ float warp_transpose_sum(const float (&a)[32], int lane)
{
    float b16[16], b8[8], b4[4], b2[2];
#pragma unroll
    for (int v = 0; v < 16; ++v) {
        const bool up = lane & 16;
        b16[v] = (up ? a[v + 16] : a[v]) + __shfl_xor_sync(0xffffffffu, up ? a[v] : a[v + 16], 16);
    }
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const bool up = lane & 8;
        b8[v] = (up ? b16[v + 8] : b16[v]) + __shfl_xor_sync(0xffffffffu, up ? b16[v] : b16[v + 8], 8);
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const bool up = lane & 4;
        b4[v] = (up ? b8[v + 4] : b8[v]) + __shfl_xor_sync(0xffffffffu, up ? b8[v] : b8[v + 4], 4);
    }
#pragma unroll
    for (int v = 0; v < 2; ++v) {
        const bool up = lane & 2;
        b2[v] = (up ? b4[v + 2] : b4[v]) + __shfl_xor_sync(0xffffffffu, up ? b4[v] : b4[v + 2], 2);
    }
    const bool up = lane & 1;
    return (up ? b2[1] : b2[0]) + __shfl_xor_sync(0xffffffffu, up ? b2[0] : b2[1], 1);
}

// Independent codebook layers of one shape handled by one launch (pointers per layer).
constexpr int kBtcMaxBatch = 64;
struct BtcBatch {
    const uint32_t* indices[kBtcMaxBatch];
    const uint16_t* codebooks[kBtcMaxBatch];
    const uint16_t* g16[kBtcMaxBatch];
    const uint16_t* h16[kBtcMaxBatch];
    const uint16_t* X[kBtcMaxBatch];
    void* Y[kBtcMaxBatch];
};

// grid: layers x row blocks x slices; part [layer][S][N]
template <int KP>
__global__ void __launch_bounds__(kBtcWarps * 32)
btc_gemv_kernel(const __grid_constant__ BtcBatch B, int N, int K, int c_max, int w, float* __restrict__ part)
{
    static_assert(KP <= 2, "one 64 KB table region holds k <= 2");
    extern __shared__ __align__(1024) float lut[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int64_t per_layer = (Nt + kBtcWarps - 1) / kBtcWarps * S;
    const int layer = (int)(blockIdx.x / per_layer);
    const int64_t bx = blockIdx.x % per_layer;
    const int64_t s = bx % S, t = (bx / S) * kBtcWarps + warp;
    const int64_t rw = ((int64_t)(K / 16) * w + 31) / 32;
    const uint32_t* __restrict__ indices = B.indices[layer];
    const uint16_t* __restrict__ codebooks = B.codebooks[layer];
    const uint16_t* __restrict__ g16 = B.g16[layer];
    const uint16_t* __restrict__ X = B.X[layer];
    part += (int64_t)layer * S * N;
    uint4 hr[KP];
    lut_load_h<KP>(hr, B.h16[layer], s, K);
    pdl_launch_dependents();
    pdl_wait();
    lut_build_part<KP, kBtcWarps>(lut, hr, X, s, K, lane, warp);
    __syncthreads();
    if (t >= Nt) return;

    const int64_t J = s * 16 + (lane >> 1);                 // this lane's 16-column group
    const bool col_ok = s * 256 + lane * 8 < K;
    const int64_t bit = J * w;
    const int64_t wi = bit >> 5;
    const uint32_t sh = (uint32_t)(bit & 31), mask = (1u << w) - 1u, bsh = 8u * (lane & 1);
    const uint32_t tb = smem_u32(lut) + (uint32_t)lane * 4u;
    float acc[KP][32];
#pragma unroll
    for (int r = 0; r < 32; ++r) {
        const int64_t row = min(t * 32 + r, (int64_t)N - 1);   // rows past N: any valid row, not stored
#pragma unroll
        for (int i = 0; i < KP; ++i) {
            const uint32_t* st = indices + ((int64_t)i * N + row) * rw;
            const uint32_t lo = col_ok ? __ldg(st + wi) : 0u;
            const uint32_t hi = (col_ok && wi + 1 < rw) ? __ldg(st + wi + 1) : 0u;
            const uint32_t idx = min(__funnelshift_r(lo, hi, sh) & mask, (uint32_t)c_max - 1u);
            const uint32_t pat = __ldg(codebooks + (int64_t)i * c_max + idx);
            const uint32_t byte = (pat >> bsh) & 0xFFu;
            acc[i][r] = col_ok ? lds_f32(tb + (uint32_t)(i & 1) * 128u + byte * 256u) : 0.0f;
        }
    }
    const int64_t row = t * 32 + lane;
    float y = 0.0f;
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        const float sum = warp_transpose_sum(acc[i], lane);
        y += row < N ? __half2float(__ushort_as_half(g16[(int64_t)i * N + row])) * sum : 0.0f;
    }
    if (row < N) part[s * N + row] = y;
}

// Y[layer][n] = sum over slices of the partials, in slice order
__global__ void btc_reduce_kernel(const __grid_constant__ BtcBatch B, int count, const float* __restrict__ part,
                                  int N, int S, int ydt)
{
    pdl_launch_dependents();
    pdl_wait();
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < (int64_t)count * N;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int layer = (int)(x / N);
        const int64_t n = x - (int64_t)layer * N;
        const float* p = part + (int64_t)layer * S * N + n;
        float y = 0.0f;
        for (int s = 0; s < S; ++s) y += p[(int64_t)s * N];
        store_y(B.Y[layer], ydt, n, y);
    }
}

// ---------------------------------------------------------------- tensor-core decode kernel
// M >= 2 (up to 64), and M = 1 with k > 4.  mma.sync m16n8k16, fp16 operands,
// fp32 accumulation: A = the signed scales +-h_i expanded from the sign words in
// registers, B = the activations converted to fp16, D = one accumulator per
// plane; Y = sum_i g_i * D_i.  Products of two fp16 values are exact in fp32.
//
// K order inside a 32-column word: MMA k index 2j + e is column j + 16e (the
// order of the h pairs (h[j], h[j+16])), so one shift brings sign bits j and
// j+16 to the sign positions of an fp16 pair and one LOP3 applies them; the
// staged activations use the same order.
//
// Grid: per layer, row groups of 8 tiles (one 32-row tile per warp) x CS CTAs
// along K (a cluster; rank j takes the contiguous slices [j*spc, (j+1)*spc)) x
// token groups of 8*NT tokens (grid.y).  Partial sums of a row group go over
// distributed shared memory to the rank that owns the row and are added there
// in rank order (deterministic, no workspace).
constexpr int kMmaWarps = 8;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kMmaRows = kMmaWarps * 32;        // rows per CTA

__host__ __device__ constexpr int mma_xs(int spc) { return spc * 256 + 8; }   // halves per staged token row
__host__ __device__ inline int mma_smem_bytes(int kp, int nt, int spc, int CS)
{
    const int x = 8 * nt * mma_xs(spc) * 2;                  // staged X, fp16
    const int hq = kp * spc * 8 * 4 * 16;                    // h pairs, 16 B per (plane, word, t)
    const int recv = CS > 1 ? kMmaRows * 8 * nt * 4 : 0;     // partial sums received from the cluster
    return (x + 15) / 16 * 16 + hq + recv;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (~shifted & 0x80008000) ^ hpair: a clear sign bit turns +h into -h.
__device__ __forceinline__ uint32_t sign_pair(uint32_t shifted, uint32_t hpair)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xA6;" : "=r"(d) : "r"(shifted), "r"(0x80008000u), "r"(hpair));
    return d;
}

// The 8 logical words of plane i, slice s, tile T for row `lane` (zero past the tiles).
template <int KP>
__device__ __forceinline__ void mma_load_words(uint32_t (&w)[KP][8], const uint32_t* __restrict__ planes,
                                               int64_t s, int64_t T, int64_t S, int64_t Nt, int lane)
{
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        const uint32_t* blk = planes + block_index(i, s, T, S, Nt) * 256 + lane;
#pragma unroll
        for (int q = 0; q < 8; ++q) w[i][q] = T < Nt ? __ldcs(blk + ((q ^ (lane >> 2)) * 32)) : 0u;
    }
}

// Two CTAs per SM where the accumulators allow it (k * NT <= 4: at most 128
// registers per thread), so each SM has 16 warps to hide the shuffle ->
// shift -> LOP3 -> HMMA latency chain.
template <int KP, int NT>
__global__ void __launch_bounds__(kMmaThreads, (KP * NT <= 4) ? 2 : 1)
gemv_mma_kernel(const __grid_constant__ LutBatch batch, int N, int K, int M, int CS, int groups, int ydt,
                int32_t* dev_status)
{
    constexpr int TG = 8 * NT;
    extern __shared__ __align__(16) uint8_t msm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int rank = CS > 1 ? (int)cluster_rank() : 0;
    const int cl = blockIdx.x / CS;
    const int layer = cl / groups, grp = cl % groups;
    const uint32_t* __restrict__ planes = batch.planes[layer];
    const uint16_t* __restrict__ g16 = batch.g16[layer];
    const uint16_t* __restrict__ h16 = batch.h16[layer];
    const uint16_t* __restrict__ X = batch.X[layer];
    void* __restrict__ Y = batch.Y[layer];
    const int spc = (int)((S + CS - 1) / CS);
    const int64_t s0 = (int64_t)rank * spc;
    const int nsl = (int)(s0 < S ? (S - s0 < spc ? S - s0 : spc) : 0);
    const int m0 = blockIdx.y * TG;
    const int XS = mma_xs(spc);
    uint16_t* xs = reinterpret_cast<uint16_t*>(msm);                                  // [TG][XS]
    uint4* hq = reinterpret_cast<uint4*>(msm + (TG * XS * 2 + 15) / 16 * 16);         // [KP][spc*8][4]
    float* recv = reinterpret_cast<float*>(hq + KP * spc * 8 * 4);                     // [CS][rows/CS][TG]
    const int64_t T = (int64_t)grp * kMmaWarps + warp;                               // this warp's tile

    // ---- before the dependency wait: the first slice's sign words and the h pairs
    uint32_t cw[KP][8];
    if (nsl > 0) mma_load_words<KP>(cw, planes, s0, T, S, Nt, lane);
    // one (plane, word) per item: 64 B of h, 16 pairs (h[j], h[j+16]), four 16 B entries
    for (int idx = threadIdx.x; idx < KP * nsl * 8; idx += kMmaThreads) {
        const int i = idx / (nsl * 8), wl = idx % (nsl * 8);
        const int64_t c0 = s0 * 256 + 32 * wl;
        uint32_t hw[16];                              // h[c0 + 2e], h[c0 + 2e + 1] in word e
        if (c0 < K) {
            const uint4* hb = reinterpret_cast<const uint4*>(h16 + (int64_t)i * K + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 v = hb[q];
                hw[4 * q] = v.x; hw[4 * q + 1] = v.y; hw[4 * q + 2] = v.z; hw[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) hw[e] = 0u;
        }
        uint4* dst = hq + (i * spc * 8 + wl) * 4;
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
            uint32_t pr[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = tt + 4 * q;             // pair (h[j], h[j+16])
                pr[q] = prmt(hw[j >> 1], hw[(j + 16) >> 1], (j & 1) ? 0x7632u : 0x5410u);
            }
            dst[tt] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
        }
    }
    pdl_launch_dependents();
    pdl_wait();
    // ---- activations of the CTA's columns, fp16, pair order (j, j+16) per word;
    // one item = token m, word wl, half q: pairs j = 8q .. 8q+7 from two 16 B loads.
    // A value that is infinite in fp16 (|x| >= 65520, or x infinite) raises RB_DEV_RANGE.
    int x_range = 0;
    for (int idx = threadIdx.x; idx < TG * nsl * 16; idx += kMmaThreads) {
        const int m = idx / (nsl * 16), rem = idx % (nsl * 16), wl = rem >> 1, q = rem & 1;
        const int64_t c0 = s0 * 256 + 32 * wl + 8 * q;
        uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
        if (m0 + m < M && c0 < K) {
            const uint16_t* xr = X + (int64_t)(m0 + m) * K + c0;
            lo = *reinterpret_cast<const uint4*>(xr);          // columns 8q .. 8q+7 of the word
            hi = *reinterpret_cast<const uint4*>(xr + 16);     // columns 16+8q .. 16+8q+7
        }
        const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w}, hw[4] = {hi.x, hi.y, hi.z, hi.w};
        uint32_t pr[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t a = (e & 1) ? (lw[e >> 1] & 0xffff0000u) : (lw[e >> 1] << 16);
            const uint32_t b = (e & 1) ? (hw[e >> 1] & 0xffff0000u) : (hw[e >> 1] << 16);
            const __half2 h2 = __floats2half2_rn(__uint_as_float(a), __uint_as_float(b));
            x_range |= __hisinf(__low2half(h2)) | __hisinf(__high2half(h2));
            pr[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        uint4* dst = reinterpret_cast<uint4*>(xs + m * XS + 32 * wl + 16 * q);
        dst[0] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
        dst[1] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
    }
    if (__syncthreads_or(x_range) && threadIdx.x == 0) set_dev_status(dev_status, RB_DEV_RANGE);

    float acc[KP][2][NT][4];
#pragma unroll
    for (int i = 0; i < KP; ++i)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][hf][nt][q] = 0.0f;

    const uint16_t* xg = xs + g * XS + 2 * t;       // this thread's token row g, k pair 2t
    for (int sl = 0; sl < nsl; ++sl) {
        uint32_t nw[KP][8];
        if (sl + 1 < nsl) mma_load_words<KP>(nw, planes, s0 + sl + 1, T, S, Nt, lane);
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const int wl = sl * 8 + w;
            uint32_t b[2][NT][2];
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint16_t* xp = xg + nt * 8 * XS + 32 * wl + 16 * ks;
                    b[ks][nt][0] = *reinterpret_cast<const uint32_t*>(xp);
                    b[ks][nt][1] = *reinterpret_cast<const uint32_t*>(xp + 8);
                }
#pragma unroll
            for (int i = 0; i < KP; ++i) {
                const uint4 hv = hq[(i * spc * 8 + wl) * 4 + t];      // pairs j = t, t+4, t+8, t+12
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t wa = __shfl_sync(0xffffffffu, cw[i][w], 16 * hf + g);
                    const uint32_t wb = __shfl_sync(0xffffffffu, cw[i][w], 16 * hf + g + 8);
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const int j0 = 8 * ks + t;
                        const uint32_t h0 = ks ? hv.z : hv.x, h1 = ks ? hv.w : hv.y;
                        const uint32_t a0 = sign_pair(wa << (15 - j0), h0), a1 = sign_pair(wb << (15 - j0), h0);
                        const uint32_t a2 = sign_pair(wa << (11 - j0), h1), a3 = sign_pair(wb << (11 - j0), h1);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_16816(acc[i][hf][nt], a0, a1, a2, a3, b[ks][nt][0], b[ks][nt][1]);
                    }
                }
            }
        }
        if (sl + 1 < nsl) {
#pragma unroll
            for (int i = 0; i < KP; ++i)
#pragma unroll
                for (int q = 0; q < 8; ++q) cw[i][q] = nw[i][q];
        }
    }

    // ---- y[row][token] = sum_i g_i[row] * acc_i; thread rows 16hf + g + 8e, tokens 8nt + 2t + q
    float y[2][2][NT][2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int64_t r = T * 32 + 16 * hf + g + 8 * e;
            float gi[KP];
#pragma unroll
            for (int i = 0; i < KP; ++i)
                gi[i] = r < N ? __half2float(__ushort_as_half(g16[(int64_t)i * N + r])) : 0.0f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float v = 0.0f;
#pragma unroll
                    for (int i = 0; i < KP; ++i) v += gi[i] * acc[i][hf][nt][2 * e + q];
                    y[hf][e][nt][q] = v;
                }
        }
    if (CS == 1) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t r = T * 32 + 16 * hf + g + 8 * e;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int m = m0 + 8 * nt + 2 * t + q;
                        if (r < N && m < M) store_y(Y, ydt, (int64_t)m * N + r, y[hf][e][nt][q]);
                    }
            }
        return;
    }
    // Rows [j*RPO, (j+1)*RPO) of the CTA's 256 belong to rank j; slot (source rank, row, token).
    const int RPO = kMmaRows / CS;
    const uint32_t recv_s = smem_u32(recv);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int cr = warp * 32 + 16 * hf + g + 8 * e;
            const int owner = cr / RPO, lr = cr - owner * RPO;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int tok = 8 * nt + 2 * t + q;
                    st_dsmem_f32(recv_s + (uint32_t)(((rank * RPO + lr) * TG + tok) * 4), (uint32_t)owner,
                                 y[hf][e][nt][q]);
                }
        }
    cluster_sync_all();
    for (int idx = threadIdx.x; idx < RPO * TG; idx += kMmaThreads) {
        const int tok = idx / RPO, lr = idx % RPO;
        float v = 0.0f;
        for (int j = 0; j < CS; ++j) v += recv[(j * RPO + lr) * TG + tok];
        const int64_t r = (int64_t)grp * kMmaRows + rank * RPO + lr;
        const int m = m0 + tok;
        if (r < N && m < M) store_y(Y, ydt, (int64_t)m * N + r, v);
    }
}

// ---------------------------------------------------------------- host side
struct LutPlan {
    int CS;          // CTAs per cluster (slice groups)
    int R;           // clusters (row chunks)
    int smem;        // dynamic shared memory bytes
};

cudaLaunchConfig_t lut_config(const LutPlan& p, int count, int threads, cudaLaunchAttribute* attr, bool pdl,
                              cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(count * p.CS * p.R));
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = stream;
    int na = 0;
    if (p.CS > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)p.CS;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cfg;
}

template <int KP>
bool lut_set_attributes()
{
    static std::atomic<bool> attr_set[64];       // per device; setting the attributes twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return false;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(gemv_lut_kernel<KP>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
            return false;
        if (cudaFuncSetAttribute(gemv_lut_kernel<KP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
            return false;
        attr_set[dev].store(true, std::memory_order_release);
    }
    return true;
}

// Clusters of CS CTAs (CTAs when CS = 1) the GPU keeps resident with `smem`
// bytes per CTA, or 0 if the query fails.
template <int KP>
int lut_resident(int CS, int smem)
{
    LutPlan p{CS, 1, smem};
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = lut_config(p, 1, LutCfg<KP>::threads, attr, false, 0);
    int n = 0;
    if (CS > 1) {
        if (cudaOccupancyMaxActiveClusters(&n, gemv_lut_kernel<KP>, &cfg) != cudaSuccess) n = 0;
    } else {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_lut_kernel<KP>, LutCfg<KP>::threads, (size_t)smem) !=
            cudaSuccess)
            n = 0;
        n *= num_sms();
    }
    return n;
}

// Cost of one slice's table build, in units of one row tile's lookups per warp
// (64 stores and ~80 arithmetic instructions per thread plus the barriers).
constexpr int kLutBuildTiles = 8;

// Single layer (count == 1): lowest latency.  Slices per CTA = ceil(S/16),
// CS = ceil(S / that) CTAs per cluster, row chunks (R): one cluster fewer than
// the SMs hold at one CTA each (and no more than stay resident), one wave.
// Batch: CS (a power of two) and R minimise the modelled time waves * (time of
// one CTA), where a CTA builds ceil(S/CS) tables and runs ceil(rows/R) row
// tiles through each, and the count * R clusters run in ceil(count * R /
// resident) waves of the clusters the GPU keeps resident (fewer for larger
// clusters: a cluster's CTAs share a GPC).  A single wave that leaves resident
// slots empty is charged for them in part (x 1 + (empty fraction) / 2): the
// CTAs then crowd some SMs while others idle.  Measured on 4096 x 4096 layers,
// full waves of 8-CTA clusters with all rows per CTA came out fastest.
template <int KP>
rb_status lut_plan_uncached(int N, int K, int count, LutPlan* plan)
{
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    constexpr int kSmemCap = 105 * 1024;        // two CTAs per SM, when the tables leave room
    const int cap = lut_table_bytes(KP) < 96 * 1024 ? kSmemCap : 227 * 1024;
    if (count == 1) {
        const int spc = (int)((S + 15) / 16);
        const int CS = (int)((S + spc - 1) / spc);
        const int sms = num_sms();
        // clusters: one fewer than the SMs hold at one CTA each, which leaves SMs
        // free for the first CTAs of the next layer's launch (PDL): 8 clusters of
        // 16 on 148 SMs measured 4.37 against 4.60 us per layer with 9 in a
        // dependent chain of 4096 x 4096 layers (7 and 6: 4.57 and 5.8 us)
        int R = CS > 1 ? sms / CS - 1 : sms;
        if (R < 1) R = 1;
        if (R > Nt) R = (int)Nt;
        while (R < Nt && lut_table_bytes(KP) + lut_row_bytes(Nt, R, CS) > cap) ++R;
        LutPlan p{CS, R, lut_table_bytes(KP) + lut_row_bytes(Nt, R, CS)};
        if (CS > 1) {
            const int active = lut_resident<KP>(CS, p.smem);
            if (active > 0 && active < R) {
                p.R = active;
                p.smem = lut_table_bytes(KP) + lut_row_bytes(Nt, p.R, CS);
            }
        }
        if (p.smem > 227 * 1024) return RB_ERR_UNSUPPORTED;
        *plan = p;
        return RB_OK;
    }
    LutPlan best{0, 0, 0};
    double best_cost = 1e300;
    for (int CS = 1; CS <= 16 && (CS == 1 || CS <= S); CS *= 2) {
        const int64_t spc = (S + CS - 1) / CS;
        int resident = -1;
        const int rmax = (int)(Nt < 4096 ? Nt : 4096);
        for (int R = 1; R <= rmax; ++R) {
            const int smem = lut_table_bytes(KP) + lut_row_bytes(Nt, R, CS);
            if (smem > cap) continue;
            if (resident < 0) resident = lut_resident<KP>(CS, smem);   // a lower bound for larger R (less smem)
            if (resident <= 0) break;
            const int64_t units = (int64_t)count * R;
            const int64_t waves = (units + resident - 1) / resident;
            const int64_t tiles = (Nt + R - 1) / R;
            const int64_t per_cta = spc * (kLutBuildTiles + (tiles + LutCfg<KP>::warps - 1) / LutCfg<KP>::warps * LutCfg<KP>::warps);
            double cost = (double)(waves * per_cta);
            if (units < resident) cost *= 1.0 + 0.5 * (double)(resident - units) / (double)resident;
            if (cost < best_cost) {
                best_cost = cost;
                best = LutPlan{CS, R, smem};
            }
            if (units >= 4 * (int64_t)resident) break;      // later R only add waves
        }
    }
    if (best.CS == 0) return RB_ERR_UNSUPPORTED;
    *plan = best;
    return RB_OK;
}

// Plans are cached per (device, k, N, K, count): the occupancy queries behind
// them cost more host time than a launch.
struct LutPlanKey {
    int dev, kp, N, K, count;
    bool operator==(const LutPlanKey& o) const {
        return dev == o.dev && kp == o.kp && N == o.N && K == o.K && count == o.count;
    }
};
constexpr int kPlanCache = 256;
std::mutex g_plan_mu;
LutPlanKey g_plan_keys[kPlanCache];
LutPlan g_plan_vals[kPlanCache];
int g_plan_n = 0;

template <int KP>
rb_status lut_plan(int N, int K, int count, LutPlan* plan)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RB_ERR_CUDA;
    if (!lut_set_attributes<KP>()) return RB_ERR_CUDA;
    const LutPlanKey key{dev, KP, N, K, count};
    {
        std::lock_guard<std::mutex> lk(g_plan_mu);
        for (int j = 0; j < g_plan_n; ++j)
            if (g_plan_keys[j] == key) {
                *plan = g_plan_vals[j];
                return RB_OK;
            }
    }
    rb_status st = lut_plan_uncached<KP>(N, K, count, plan);
    if (st != RB_OK) return st;
    std::lock_guard<std::mutex> lk(g_plan_mu);
    const int j = g_plan_n < kPlanCache ? g_plan_n++ : (int)((unsigned)(N ^ K ^ count) % kPlanCache);
    g_plan_keys[j] = key;
    g_plan_vals[j] = *plan;
    return RB_OK;
}

template <int KP>
rb_status launch_lut(const rb_layer_t* const* layers, const uint16_t* const* X, void* const* Y, int count,
                     int ydt, bool pdl, cudaStream_t stream)
{
    const rb_layer_t* L0 = layers[0];
    for (int base = 0; base < count; base += kMaxBatch) {
        const int n = count - base < kMaxBatch ? count - base : kMaxBatch;
        LutBatch b = {};
        for (int j = 0; j < n; ++j) {
            b.planes[j] = layers[base + j]->planes;
            b.g16[j] = layers[base + j]->g16;
            b.h16[j] = layers[base + j]->h16;
            b.X[j] = X[base + j];
            b.Y[j] = Y[base + j];
        }
        LutPlan plan;
        rb_status st = lut_plan<KP>(L0->n_out, L0->k_in, n, &plan);
        if (st != RB_OK) return st;
        cudaLaunchAttribute attr[2];
        cudaLaunchConfig_t cfg = lut_config(plan, n, LutCfg<KP>::threads, attr, pdl, stream);
        if (cudaLaunchKernelEx(&cfg, gemv_lut_kernel<KP>, b, (int)L0->n_out, (int)L0->k_in, plan.CS, plan.R, ydt) !=
            cudaSuccess)
            return RB_ERR_CUDA;
    }
    return RB_OK;
}

// Tensor-core decode: tokens per group 8*NT with k*NT <= 8 (accumulator
// registers); CS = the smallest power of two that fits the staged activations
// (at most 96 KB) and gives about two CTAs per SM, at most min(16, S).
template <int KP, int NT>
rb_status launch_mma_nt(const LutBatch& b, int n, int N, int K, int M, int ydt, int32_t* dev_status, bool pdl,
                        cudaStream_t stream)
{
    static std::atomic<bool> attr_set[64];       // per device; setting the attributes twice is harmless
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RB_ERR_CUDA;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(gemv_mma_kernel<KP, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess ||
            cudaFuncSetAttribute(gemv_mma_kernel<KP, NT>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess)
            return RB_ERR_CUDA;
        attr_set[dev].store(true, std::memory_order_release);
    }
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int groups = (int)((Nt + kMmaWarps - 1) / kMmaWarps);
    const int tgroups = (M + 8 * NT - 1) / (8 * NT);
    const int64_t want = 2LL * num_sms();
    int CS = 1;
    while (CS < 16 && CS < S &&
           (8 * NT * mma_xs((int)((S + CS - 1) / CS)) * 2 > 96 * 1024 || (int64_t)n * groups * tgroups * CS < want))
        CS *= 2;
    const int spc = (int)((S + CS - 1) / CS);
    const int smem = mma_smem_bytes(KP, NT, spc, CS);
    if (smem > 227 * 1024) return RB_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n * groups * CS), (unsigned)tgroups);
    cfg.blockDim = dim3(kMmaThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (CS > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)CS;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, gemv_mma_kernel<KP, NT>, b, N, K, M, CS, groups, ydt, dev_status) != cudaSuccess)
        return RB_ERR_CUDA;
    return RB_OK;
}

template <int KP>
rb_status launch_mma(const rb_layer_t* const* layers, const uint16_t* const* X, void* const* Y, int count, int M,
                     int ydt, int32_t* dev_status, bool pdl, cudaStream_t stream)
{
    // 16 tokens per CTA at most: at k <= 2 two such CTAs share an SM, which beats one
    // 32-token CTA per SM (4096 x 4096, k = 2, 96 layers at M = 64: 17.1 vs 24.8 us)
    constexpr int NTMAX = KP <= 4 ? 2 : 1;
    const rb_layer_t* L0 = layers[0];
    for (int base = 0; base < count; base += kMaxBatch) {
        const int n = count - base < kMaxBatch ? count - base : kMaxBatch;
        LutBatch b = {};
        for (int j = 0; j < n; ++j) {
            b.planes[j] = layers[base + j]->planes;
            b.g16[j] = layers[base + j]->g16;
            b.h16[j] = layers[base + j]->h16;
            b.X[j] = X[base + j];
            b.Y[j] = Y[base + j];
        }
        const int need = (M + 7) / 8;                 // n-tiles for all tokens in one group
        rb_status st;
        if (need >= 2 && NTMAX >= 2)
            st = launch_mma_nt<KP, (NTMAX >= 2 ? 2 : 1)>(b, n, L0->n_out, L0->k_in, M, ydt, dev_status, pdl, stream);
        else
            st = launch_mma_nt<KP, 1>(b, n, L0->n_out, L0->k_in, M, ydt, dev_status, pdl, stream);
        if (st != RB_OK) return st;
    }
    return RB_OK;
}

bool use_lut(const rb_layer_t* L, int M) { return M == 1 && L->k_planes <= 4; }

}  // namespace
}  // namespace rbw

using namespace rbw;

// rb_gemv runs on the tcgen05 kernel (K split over a cluster) when the caller
// passes its workspace and the layer is large enough for it: 32 <= M <= 64,
// k <= 4 and N*K*k*M above 4.5e9 multiply-adds.  Measured single-layer times
// (back-to-back launches over layers that do not fit in L2), tcgen05 against
// mma.sync: 4096 x 4096 k = 2, M = 64: 43.4 against 38.4 us; 14336 x 4096
// k = 2, M = 64: 64.9 against 86.9 us; 28672 x 8192 k = 2, M = 32: 139
// against 153 us; 11008 x 4096 k = 2, M = 48 (4.3e9): 61.3 against 51.9 us.
constexpr int kTcMinM = 32;
constexpr double kTcMinWork = 4.5e9;

static bool use_tc_decode(int n_out, int k_in, int k_planes, int M)
{
    return M >= kTcMinM && M <= 64 && k_planes <= 4 &&
           (double)n_out * (double)k_in * (double)k_planes * (double)M > kTcMinWork;
}

extern "C" size_t rb_gemv_workspace_bytes(int n_out, int k_in, int k_planes, int M)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 4) return 0;
    if (!use_tc_decode(n_out, k_in, k_planes, M)) return 0;
    return gemm_workspace(k_in, k_planes, M);
}

static rb_status gemv_dispatch(const rb_layer_t* const* layers, const uint16_t* const* X, void* const* Y,
                               int count, int M, rb_dtype y_dtype, int32_t* dev_status, unsigned flags,
                               cudaStream_t stream)
{
    const rb_layer_t* L0 = layers[0];
    for (int j = 0; j < count; ++j) {
        rb_status st = check_apply_args(layers[j], X[j], M, Y[j], y_dtype, flags);
        if (st != RB_OK) return st;
        if (layers[j]->n_out != L0->n_out || layers[j]->k_in != L0->k_in || layers[j]->k_planes != L0->k_planes)
            return RB_ERR_SHAPE;
    }
    if (M > 64) return RB_ERR_SHAPE;
    if (dev_status && !aligned16(dev_status)) return RB_ERR_ALIGN;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    const bool pdl = (flags & RB_LAUNCH_PDL) != 0;
    const int ydt = (int)y_dtype;
    if (use_lut(L0, M)) {
        switch (L0->k_planes) {
            case 1: return launch_lut<1>(layers, X, Y, count, ydt, pdl, stream);
            case 2: return launch_lut<2>(layers, X, Y, count, ydt, pdl, stream);
            case 3: return launch_lut<3>(layers, X, Y, count, ydt, pdl, stream);
            default: return launch_lut<4>(layers, X, Y, count, ydt, pdl, stream);
        }
    }
    switch (L0->k_planes) {
        case 1: return launch_mma<1>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
        case 2: return launch_mma<2>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
        case 3: return launch_mma<3>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
        case 4: return launch_mma<4>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
        case 5: return launch_mma<5>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
        case 6: return launch_mma<6>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
        case 7: return launch_mma<7>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
        default: return launch_mma<8>(layers, X, Y, count, M, ydt, dev_status, pdl, stream);
    }
}

extern "C" rb_status rb_gemv(const rb_layer_t* layer, const uint16_t* X, int M, void* Y,
                             rb_dtype y_dtype, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, unsigned flags, cudaStream_t stream)
{
    if (!layer) return RB_ERR_ARG;
    if (use_tc_decode(layer->n_out, layer->k_in, layer->k_planes, M) && workspace != nullptr &&
        workspace_bytes >= rb_gemv_workspace_bytes(layer->n_out, layer->k_in, layer->k_planes, M))
        return gemm_with_timeout(layer, X, M, Y, y_dtype, workspace, workspace_bytes, dev_status, flags, stream,
                                 kWaitTimeoutNs, true);
    return gemv_dispatch(&layer, &X, &Y, 1, M, y_dtype, dev_status, flags, stream);
}

extern "C" rb_status rb_gemv_batch(const rb_layer_t* const* layers, const uint16_t* const* X, void* const* Y,
                                   int count, int M, rb_dtype y_dtype, int32_t* dev_status, unsigned flags,
                                   cudaStream_t stream)
{
    if (!layers || !X || !Y || count < 1) return RB_ERR_ARG;
    for (int j = 0; j < count; ++j)
        if (!layers[j]) return RB_ERR_ARG;
    return gemv_dispatch(layers, X, Y, count, M, y_dtype, dev_status, flags, stream);
}

extern "C" size_t rb_btc_gemv_workspace_bytes(int n_out, int k_in)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0) return 0;
    return (size_t)num_slices(k_in) * (size_t)n_out * 4;
}

extern "C" size_t rb_btc_gemv_batch_workspace_bytes(int n_out, int k_in, int count)
{
    if (count < 1) return 0;
    return rb_btc_gemv_workspace_bytes(n_out, k_in) * (size_t)(count < kBtcMaxBatch ? count : kBtcMaxBatch);
}

extern "C" rb_status rb_btc_gemv_batch(const rb_btc_layer_t* const* layers, const uint16_t* const* X,
                                       void* const* Y, int count, rb_dtype y_dtype, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status, unsigned flags,
                                       cudaStream_t stream)
{
    (void)dev_status;
    if (!layers || !X || !Y || count < 1) return RB_ERR_ARG;
    if ((y_dtype != RB_F32 && y_dtype != RB_BF16) || (flags & ~RB_LAUNCH_PDL)) return RB_ERR_ARG;
    const rb_btc_layer_t* L0 = layers[0];
    if (!L0) return RB_ERR_ARG;
    for (int j = 0; j < count; ++j) {
        const rb_btc_layer_t* L = layers[j];
        if (!L || !X[j] || !Y[j] || !L->codebooks || !L->indices || !L->g16 || !L->h16 || L->reserved != 0)
            return RB_ERR_ARG;
        if (L->c_max < 1 || L->c_max > 65536 || L->index_bits != rb_btc_index_bits(L->c_max)) return RB_ERR_ARG;
        if (L->k_planes < 1 || L->k_planes > 8) return RB_ERR_ARG;
        if (L->n_out != L0->n_out || L->k_in != L0->k_in || L->k_planes != L0->k_planes || L->c_max != L0->c_max)
            return RB_ERR_SHAPE;
        const void* ptrs[] = {L->codebooks, L->indices, L->g16, L->h16, X[j], Y[j]};
        for (const void* q : ptrs)
            if (!aligned16(q)) return RB_ERR_ALIGN;
    }
    if (L0->k_planes > 2) return RB_ERR_UNSUPPORTED;
    const int N = L0->n_out, K = L0->k_in;
    if (N < 1 || K < 32 || K % 32 != 0) return RB_ERR_SHAPE;
    if (!workspace || workspace_bytes < rb_btc_gemv_batch_workspace_bytes(N, K, count)) return RB_ERR_WORKSPACE;
    if (!aligned16(workspace)) return RB_ERR_ALIGN;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    const bool pdl = (flags & RB_LAUNCH_PDL) != 0;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int64_t per_layer = (Nt + kBtcWarps - 1) / kBtcWarps * S;
    if (per_layer * kBtcMaxBatch > INT32_MAX) return RB_ERR_UNSUPPORTED;
    const int smem = lut_table_bytes(2);
    float* part = static_cast<float*>(workspace);
    static std::atomic<bool> attr_set[64][2];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RB_ERR_CUDA;
    const int kk = L0->k_planes - 1;
    if (!attr_set[dev][kk].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kk ? btc_gemv_kernel<2> : btc_gemv_kernel<1>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return RB_ERR_CUDA;
        attr_set[dev][kk].store(true, std::memory_order_release);
    }
    for (int base = 0; base < count; base += kBtcMaxBatch) {
        const int n = count - base < kBtcMaxBatch ? count - base : kBtcMaxBatch;
        BtcBatch b = {};
        for (int j = 0; j < n; ++j) {
            const rb_btc_layer_t* L = layers[base + j];
            b.indices[j] = L->indices;
            b.codebooks[j] = L->codebooks;
            b.g16[j] = L->g16;
            b.h16[j] = L->h16;
            b.X[j] = X[base + j];
            b.Y[j] = Y[base + j];
        }
        const dim3 grid((unsigned)(per_layer * n));
        rb_status st = kk ? launch(btc_gemv_kernel<2>, grid, dim3(kBtcWarps * 32), (size_t)smem, stream, pdl, b, N, K,
                                   L0->c_max, L0->index_bits, part)
                          : launch(btc_gemv_kernel<1>, grid, dim3(kBtcWarps * 32), (size_t)smem, stream, pdl, b, N, K,
                                   L0->c_max, L0->index_bits, part);
        if (st != RB_OK) return st;
        int64_t rb = ((int64_t)n * N + 255) / 256;
        if (rb > 4 * num_sms()) rb = 4 * num_sms();
        st = launch(btc_reduce_kernel, dim3((unsigned)rb), dim3(256), 0, stream, true, b, n, (const float*)part, N,
                    (int)S, (int)y_dtype);
        if (st != RB_OK) return st;
    }
    return RB_OK;
}

extern "C" rb_status rb_btc_gemv(const rb_btc_layer_t* layer, const uint16_t* X, void* Y, rb_dtype y_dtype,
                                 void* workspace, size_t workspace_bytes, int32_t* dev_status, unsigned flags,
                                 cudaStream_t stream)
{
    return rb_btc_gemv_batch(&layer, &X, &Y, 1, y_dtype, workspace, workspace_bytes, dev_status, flags, stream);
}

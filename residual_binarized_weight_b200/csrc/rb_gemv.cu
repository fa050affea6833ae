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
// Any M <= 64, any k <= 8: generic CUDA-core kernel (lane = row, one signed
// fused add per bit and token); it keeps every plane and token block in
// registers and needs no workspace.
#include "rbw_internal.cuh"

#include <mutex>

namespace rbw {
namespace {

constexpr int kLutThreads = 256;
constexpr int kLutWarps = kLutThreads / 32;
constexpr int kLutPF = 2;              // row tiles per warp held in registers ahead of use
constexpr int kLutPD = 6;              // row tiles per warp prefetched into L2 ahead of use

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

// L2 prefetch of one row tile's sign words (KP blocks of 1 KB = 8 lines each):
// lane l < 8*KP touches line l%8 of plane l/8.  Keeps DRAM busy further ahead
// than the register-held tiles can.
template <int KP>
__device__ __forceinline__ void lut_prefetch_tile(const uint32_t* __restrict__ planes, int64_t s, int64_t t,
                                                  int64_t S, int64_t Nt, int lane)
{
    if (lane < 8 * KP) {
        const uint32_t* p = planes + block_index(lane >> 3, s, t, S, Nt) * 256 + (lane & 7) * 32;
        asm volatile("prefetch.global.L2 [%0];" :: "l"(p));
    }
}

// g as raw fp16 bits: converting here would stall on the load before the wait.
template <int KP>
__device__ __forceinline__ void lut_load_g(uint16_t (&gv)[KP], const uint16_t* __restrict__ g16, int64_t r, int N)
{
#pragma unroll
    for (int i = 0; i < KP; ++i) gv[i] = r < N ? g16[(int64_t)i * N + r] : (uint16_t)0;
}

// Shared-window address of dynamic shared memory in a kernel without static
// shared memory on sm_100 (the first 1 KB is reserved).  The byte tables start
// there, so a lookup is one LDS with the PRMT result as register and the table
// base folded into the immediate.  The kernel checks the base at entry and uses
// a register add instead if it ever differs.
constexpr uint32_t kDynSmemBase = 1024;

template <uint32_t IMM>
__device__ __forceinline__ float lds_imm(uint32_t off) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(off), "n"(IMM));
    return v;
}

template <bool FAST, int I>
__device__ __forceinline__ float lut_entry(uint32_t tbase, uint32_t off) {
    constexpr uint32_t C = (uint32_t)((I >> 1) * 65536 + (I & 1) * 128);
    if constexpr (FAST) return lds_imm<kDynSmemBase + C>(off);
    else return lds_f32(tbase + C + off);
}

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

// Per-row sums (red) plus, with a cluster, the receive area of the rows this CTA
// sums: CS slots of at most ceil(rows/CS) rows, which never exceeds rows + CS;
// rounded up to 16 bytes.
__host__ __device__ inline int lut_row_bytes(int64_t Nt, int R, int CS)
{
    const int64_t rows = ((Nt + R - 1) / R) * 32;
    return (int)(((CS > 1 ? 2 * rows + CS : rows) + 3) / 4 * 16);
}

// Byte tables of slice s for all KP planes (256 threads: thread (group gg,
// part) writes bytes 32*part .. 32*part+31 of group gg).  Plane i's entry
// (byte, group) sits at region(i/2) + byte*256 + (i%2)*128 + group*4.
template <int KP>
__device__ __forceinline__ void lut_load_h(uint4 (&hr)[KP], const uint16_t* __restrict__ h16, int64_t s, int K)
{
    const int64_t c0 = s * 256 + (threadIdx.x & 31) * 8;
#pragma unroll
    for (int i = 0; i < KP; ++i)
        hr[i] = c0 < K ? *reinterpret_cast<const uint4*>(h16 + (int64_t)i * K + c0) : make_uint4(0, 0, 0, 0);
}

template <int KP>
__device__ __forceinline__ void lut_build(float* lut, const uint4 (&hrr)[KP], const uint16_t* __restrict__ X,
                                          int64_t s, int K)
{
    const int gg = threadIdx.x & 31, part = threadIdx.x >> 5;
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
        float Hh[2];                              // signed sums of columns 4..7 for this part's high nibbles
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = 2 * part + e;
            float acc = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) acc += ((n >> q) & 1) ? v[4 + q] : -v[4 + q];
            Hh[e] = acc;
        }
        char* base = reinterpret_cast<char*>(lut) + (i >> 1) * 65536 + (i & 1) * 128 + gg * 4;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int b = 32 * part + j;
            *reinterpret_cast<float*>(base + b * 256) = L[b & 15] + Hh[(b >> 4) & 1];
        }
    }
}

// All lookups of the kLutPF register-held tiles: for each word slot, the PRMT
// offsets of 4 bytes x kLutPF tiles x KP planes are formed first, then all the
// LDS are issued, then the FADDs, so each warp keeps 4*kLutPF*KP independent
// table reads in flight.
template <int KP, bool FAST>
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
                e[b][p][0] = lut_entry<FAST, 0>(tbase, off[b][p][0]);
                if constexpr (KP > 1) e[b][p][1] = lut_entry<FAST, 1>(tbase, off[b][p][1]);
                if constexpr (KP > 2) e[b][p][2] = lut_entry<FAST, 2>(tbase, off[b][p][2]);
                if constexpr (KP > 3) e[b][p][3] = lut_entry<FAST, 3>(tbase, off[b][p][3]);
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
// L2 prefetches run kLutPD tiles ahead in the same sequence, on into the next
// slice.  Tile validity only gates the red[] update, so no load is guarded by
// a branch.
template <int KP, bool FAST>
__device__ __forceinline__ void lut_tiles(uint32_t (&wd)[kLutPF][KP][8], uint16_t (&gv)[kLutPF][KP],
                                          const uint32_t (&G)[8], const uint32_t (&SEL)[4], uint32_t tbase,
                                          float* red, const uint32_t* __restrict__ planes,
                                          const uint16_t* __restrict__ g16, int64_t s, int64_t s_next,
                                          int64_t S, int64_t Nt, int N, int tb, int te, int warp, int lane)
{
    const int nw = te - tb > warp ? (te - tb - warp + kLutWarps - 1) / kLutWarps : 0;
    const int iters = (nw + kLutPF - 1) / kLutPF;
    const bool has_next = s_next < S;
    const uint32_t* cur[KP];
    const uint32_t* nxt[KP];
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        cur[i] = planes + block_index(i, s, 0, S, Nt) * 256 + lane;
        nxt[i] = has_next ? planes + block_index(i, s_next, 0, S, Nt) * 256 + lane : cur[i];
    }
    // this lane's L2-prefetch line: plane lane/8, line lane%8 of a tile block
    const bool pf_lane = lane < 8 * KP;
    const uint32_t* pf_cur = planes + block_index(pf_lane ? lane >> 3 : 0, s, 0, S, Nt) * 256 + (lane & 7) * 32;
    const uint32_t* pf_nxt = has_next
        ? planes + block_index(pf_lane ? lane >> 3 : 0, s_next, 0, S, Nt) * 256 + (lane & 7) * 32 : pf_cur;
    const int t_w = tb + warp;                    // the warp's first tile
    for (int it = 0; it < iters; ++it) {
        float acc[kLutPF][KP][2];
#pragma unroll
        for (int p = 0; p < kLutPF; ++p)
#pragma unroll
            for (int i = 0; i < KP; ++i) acc[p][i][0] = acc[p][i][1] = 0.0f;
        lut_lookups<KP, FAST>(acc, wd, G, SEL, tbase);
        const bool last = it + 1 == iters;
#pragma unroll
        for (int p = 0; p < kLutPF; ++p) {
            const int j = it * kLutPF + p;
            float pr = 0.0f;
#pragma unroll
            for (int i = 0; i < KP; ++i)
                pr += __half2float(__ushort_as_half(gv[p][i])) * (acc[p][i][0] + acc[p][i][1]);
            if (j < nw) red[(j * kLutWarps + warp) * 32 + lane] += pr;
            const int jp = j + kLutPD;
            const bool pf_here = jp < nw;
            if (pf_lane && (pf_here || (has_next && jp - nw < nw))) {
                const uint32_t* q = pf_here ? pf_cur + (size_t)(t_w + jp * kLutWarps) * 256
                                            : pf_nxt + (size_t)(t_w + (jp - nw) * kLutWarps) * 256;
                asm volatile("prefetch.global.L2 [%0];" :: "l"(q));
            }
            if (!last || (has_next && p < nw)) {
                const int jn = last ? p : min(j + kLutPF, nw - 1);
                const size_t tn = (size_t)(t_w + jn * kLutWarps);
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
__global__ void __launch_bounds__(kLutThreads, 2)
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
        const int64_t t = t_begin + warp + (int64_t)p * kLutWarps;
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
    if (s_first < S) {
        lut_load_h<KP>(hr, h16, s_first, K);
#pragma unroll
        for (int p = kLutPF; p < kLutPD; ++p) {
            const int64_t t = t_begin + warp + (int64_t)p * kLutWarps;
            if (t < t_end) lut_prefetch_tile<KP>(planes, s_first, t, S, Nt, lane);
        }
    }
    for (int64_t x = threadIdx.x; x < chunk_rows; x += kLutThreads) red[x] = 0.0f;

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
    const bool fast_base = tbase == kDynSmemBase;
    pdl_launch_dependents();
    pdl_wait();

    for (int64_t s = s_first; s < S; s += CS) {
        if (s != s_first) {
            __syncthreads();                      // the previous slice's lookups are done with the tables
            lut_load_h<KP>(hr, h16, s, K);        // (its tiles are in registers already)
        }
        lut_build<KP>(lut, hr, X, s, K);
        __syncthreads();

        if (fast_base)
            lut_tiles<KP, true>(wd, gv, G, SEL, tbase, red, planes, g16, s, s + CS, S, Nt, N, (int)t_begin,
                                (int)t_end, warp, lane);
        else
            lut_tiles<KP, false>(wd, gv, G, SEL, tbase, red, planes, g16, s, s + CS, S, Nt, N, (int)t_begin,
                                 (int)t_end, warp, lane);
    }

    // ---- cross-slice sum
    if (CS == 1) {
        __syncthreads();
        for (int64_t x = threadIdx.x; x < chunk_rows; x += kLutThreads) {
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
        const int tpo = kLutThreads / CS;         // threads per destination rank
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
    for (int xo = threadIdx.x; xo < my_span; xo += kLutThreads) {
        float y = 0.0f;
        for (int j = 0; j < CS; ++j) y += recv[j * my_span + xo];
        const int64_t r = t_begin * 32 + x0 + xo;
        if (r < N) store_y(Y, ydt, r, y);
    }
}

// ---------------------------------------------------------------- generic kernel
constexpr int kGenThreads = 128;       // 4 warps = 4 row tiles
constexpr int kGenMT = 4;              // tokens per CTA

template <int KP>
__global__ void __launch_bounds__(kGenThreads)
gemv_generic_kernel(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ g16,
                    const uint16_t* __restrict__ h16, const uint16_t* __restrict__ X,
                    int N, int K, int M, void* __restrict__ Y, int ydt)
{
    __shared__ float hx[KP][kGenMT][8][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int64_t t = (int64_t)blockIdx.x * (kGenThreads / 32) + warp;
    const int m0 = blockIdx.y * kGenMT;
    pdl_launch_dependents();
    pdl_wait();

    float acc[KP][kGenMT];
#pragma unroll
    for (int i = 0; i < KP; ++i)
#pragma unroll
        for (int m = 0; m < kGenMT; ++m) acc[i][m] = 0.0f;

    for (int64_t s = 0; s < S; ++s) {
        for (int idx = threadIdx.x; idx < KP * kGenMT * 256; idx += kGenThreads) {
            const int cc = idx & 255, m = (idx >> 8) % kGenMT, i = idx / (256 * kGenMT);
            const int64_t c = s * 256 + cc;
            float v = 0.0f;
            if (c < K && m0 + m < M)
                v = __half2float(__ushort_as_half(h16[(int64_t)i * K + c])) *
                    bf16_bits_to_f32(X[(int64_t)(m0 + m) * K + c]);
            hx[i][m][cc >> 5][cc & 31] = v;
        }
        __syncthreads();
        if (t < Nt) {
#pragma unroll
            for (int i = 0; i < KP; ++i) {
                const uint32_t* blk = planes + block_index(i, s, t, S, Nt) * 256 + lane;
                for (int sl = 0; sl < 8; ++sl) {
                    const uint32_t word = blk[sl * 32];
                    const int wl = sl ^ (lane >> 2);
#pragma unroll 8
                    for (int j = 0; j < 32; ++j) {
                        const float sg = ((word >> j) & 1u) ? 1.0f : -1.0f;
#pragma unroll
                        for (int m = 0; m < kGenMT; ++m) acc[i][m] = fmaf(sg, hx[i][m][wl][j], acc[i][m]);
                    }
                }
            }
        }
        __syncthreads();
    }
    const int64_t r = t * 32 + lane;
    if (t < Nt && r < N) {
#pragma unroll
        for (int m = 0; m < kGenMT; ++m) {
            if (m0 + m >= M) break;
            float y = 0.0f;
#pragma unroll
            for (int i = 0; i < KP; ++i)
                y += __half2float(__ushort_as_half(g16[(int64_t)i * N + r])) * acc[i][m];
            store_y(Y, ydt, (int64_t)(m0 + m) * N + r, y);
        }
    }
}

// ---------------------------------------------------------------- host side
struct LutPlan {
    int CS;          // CTAs per cluster (slice groups)
    int R;           // clusters (row chunks)
    int smem;        // dynamic shared memory bytes
};

cudaLaunchConfig_t lut_config(const LutPlan& p, int count, cudaLaunchAttribute* attr, bool pdl, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(count * p.CS * p.R));
    cfg.blockDim = dim3(kLutThreads);
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
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return false;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(gemv_lut_kernel<KP>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
            return false;
        if (cudaFuncSetAttribute(gemv_lut_kernel<KP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
            return false;
        attr_set[dev] = true;
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
    cudaLaunchConfig_t cfg = lut_config(p, 1, attr, false, 0);
    int n = 0;
    if (CS > 1) {
        if (cudaOccupancyMaxActiveClusters(&n, gemv_lut_kernel<KP>, &cfg) != cudaSuccess) n = 0;
    } else {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_lut_kernel<KP>, kLutThreads, (size_t)smem) !=
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
// CS = ceil(S / that) CTAs per cluster, as many row chunks (R) as the GPU keeps
// clusters resident, one wave.
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
        int R = CS > 1 ? sms / CS : sms;
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
            const int64_t per_cta = spc * (kLutBuildTiles + (tiles + kLutWarps - 1) / kLutWarps * kLutWarps);
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
        LutPlan plan;
        rb_status st = lut_plan<KP>(L0->n_out, L0->k_in, n, &plan);
        if (st != RB_OK) return st;
        LutBatch b = {};
        for (int j = 0; j < n; ++j) {
            b.planes[j] = layers[base + j]->planes;
            b.g16[j] = layers[base + j]->g16;
            b.h16[j] = layers[base + j]->h16;
            b.X[j] = X[base + j];
            b.Y[j] = Y[base + j];
        }
        cudaLaunchAttribute attr[2];
        cudaLaunchConfig_t cfg = lut_config(plan, n, attr, pdl, stream);
        if (cudaLaunchKernelEx(&cfg, gemv_lut_kernel<KP>, b, (int)L0->n_out, (int)L0->k_in, plan.CS, plan.R, ydt) !=
            cudaSuccess)
            return RB_ERR_CUDA;
    }
    return RB_OK;
}

template <int KP>
rb_status launch_generic(const rb_layer_t* L, const uint16_t* X, int M, void* Y, int ydt,
                         bool pdl, cudaStream_t stream)
{
    const int64_t Nt = num_row_tiles(L->n_out);
    dim3 grid((unsigned)((Nt + 3) / 4), (unsigned)((M + kGenMT - 1) / kGenMT));
    return launch(gemv_generic_kernel<KP>, grid, dim3(kGenThreads), 0, stream, pdl,
                  L->planes, L->g16, L->h16, X, L->n_out, L->k_in, M, Y, ydt);
}

bool use_lut(const rb_layer_t* L, int M) { return M == 1 && L->k_planes <= 4; }

}  // namespace
}  // namespace rbw

using namespace rbw;

extern "C" size_t rb_gemv_workspace_bytes(int n_out, int k_in, int k_planes, int M)
{
    (void)n_out; (void)k_in; (void)k_planes; (void)M;
    return 0;          // every rb_gemv path keeps its partial sums on chip
}

static rb_status gemv_dispatch(const rb_layer_t* const* layers, const uint16_t* const* X, void* const* Y,
                               int count, int M, rb_dtype y_dtype, unsigned flags, cudaStream_t stream)
{
    const rb_layer_t* L0 = layers[0];
    for (int j = 0; j < count; ++j) {
        rb_status st = check_apply_args(layers[j], X[j], M, Y[j], y_dtype, flags);
        if (st != RB_OK) return st;
        if (layers[j]->n_out != L0->n_out || layers[j]->k_in != L0->k_in || layers[j]->k_planes != L0->k_planes)
            return RB_ERR_SHAPE;
    }
    if (M > 64) return RB_ERR_SHAPE;
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
    for (int j = 0; j < count; ++j) {
        rb_status st;
        switch (L0->k_planes) {
            case 1: st = launch_generic<1>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
            case 2: st = launch_generic<2>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
            case 3: st = launch_generic<3>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
            case 4: st = launch_generic<4>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
            case 5: st = launch_generic<5>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
            case 6: st = launch_generic<6>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
            case 7: st = launch_generic<7>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
            default: st = launch_generic<8>(layers[j], X[j], M, Y[j], ydt, pdl, stream); break;
        }
        if (st != RB_OK) return st;
    }
    return RB_OK;
}

extern "C" rb_status rb_gemv(const rb_layer_t* layer, const uint16_t* X, int M, void* Y,
                             rb_dtype y_dtype, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, unsigned flags, cudaStream_t stream)
{
    (void)dev_status;
    (void)workspace;
    (void)workspace_bytes;
    if (!layer) return RB_ERR_ARG;
    return gemv_dispatch(&layer, &X, &Y, 1, M, y_dtype, flags, stream);
}

extern "C" rb_status rb_gemv_batch(const rb_layer_t* const* layers, const uint16_t* const* X, void* const* Y,
                                   int count, int M, rb_dtype y_dtype, int32_t* dev_status, unsigned flags,
                                   cudaStream_t stream)
{
    (void)dev_status;
    if (!layers || !X || !Y || count < 1) return RB_ERR_ARG;
    for (int j = 0; j < count; ++j)
        if (!layers[j]) return RB_ERR_ARG;
    return gemv_dispatch(layers, X, Y, count, M, y_dtype, flags, stream);
}

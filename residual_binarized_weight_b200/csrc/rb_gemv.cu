// rb_gemv.cu -- decode-time application Y = sum_i g_i .* (B_i (h_i .* x))
// (RaBiT, "Residual binarization": matmul-free inference with additions and
// element-wise scaling; the k paths run side by side).
//
// M = 1, k <= 4: byte-table kernel.  For each 256-column slice the CTA builds,
// per plane, T_i[byte][group] = sum_{q<8} (bit q of byte ? +1 : -1) * hx_i[8*group + q]
// with hx_i = h_i .* x formed exactly in fp32 (a bf16 x fp16 product has at
// most 19 significant bits).  One table lookup then stands for eight signed
// additions.  Lane l of a warp owns row l of a 32-row tile; the XOR-swizzled
// storage layout hands it logical word (slot ^ l/4), so at every step the 32
// lanes read 32 different groups: group (4*slot + b) ^ l lives in smem bank
// ((4*slot + b) ^ l) and the lookups are conflict-free.  One PRMT forms the
// byte offset (byte << 8 | group << 2), one LDS fetches the entry, one FADD
// accumulates: three instructions per eight weights.  Row sums across the
// slices go through a small fp32 workspace; the last warp to finish a row tile
// (per-tile arrival counter) adds the slice partials in slice order, so the
// result is deterministic.
//
// Any M <= 64, any k <= 8: generic CUDA-core kernel (lane = row, one signed
// fused add per bit and token); it keeps every plane and token block in
// registers and needs no workspace.
#include "rbw_internal.cuh"

namespace rbw {
namespace {

constexpr int kLutThreads = 256;
constexpr int kLutWarps = kLutThreads / 32;

// smem bytes of the byte tables: planes (2p, 2p+1) share a 64 KB region with
// entry (byte, group) of plane i at region(i/2) + byte*256 + (i%2)*128 + group*4.
__host__ __device__ constexpr int lut_smem_bytes(int kp) { return ((kp + 1) / 2) * 65536; }

// Prefetch depth of the byte-table kernel: row tiles per warp held in registers.
constexpr int kLutPF = 2;

template <int KP>
__device__ __forceinline__ void lut_load_tile(uint32_t (&wd)[KP][8], const uint32_t* __restrict__ planes,
                                              int s, int64_t t, int64_t S, int64_t Nt, int lane)
{
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        const uint32_t* blk = planes + block_index(i, s, t, S, Nt) * 256 + lane;
#pragma unroll
        for (int sl = 0; sl < 8; ++sl) wd[i][sl] = __ldcs(blk + sl * 32);
    }
}

template <int KP>
__global__ void __launch_bounds__(kLutThreads, 2)
gemv_lut_kernel(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ g16,
                const uint16_t* __restrict__ h16, const uint16_t* __restrict__ X,
                int N, int K, int C, float* __restrict__ partial,
                unsigned* __restrict__ counters, void* __restrict__ Y, int ydt)
{
    extern __shared__ __align__(1024) float lut[];
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const int s = blockIdx.x / C, cta = blockIdx.x % C;
    const int64_t t_begin = Nt * cta / C, t_end = Nt * (cta + 1) / C;

    // ---- before the dependency wait: everything that does not depend on X.
    // Weights of this warp's first kLutPF row tiles, their g values, this
    // thread's h values for the table build.
    uint32_t wd[kLutPF][KP][8];
    float gv[kLutPF][KP];
#pragma unroll
    for (int p = 0; p < kLutPF; ++p) {
        const int64_t t = t_begin + warp + (int64_t)p * kLutWarps;
        if (t < t_end) {
            lut_load_tile<KP>(wd[p], planes, s, t, S, Nt, lane);
            const int64_t r = t * 32 + lane;
#pragma unroll
            for (int i = 0; i < KP; ++i)
                gv[p][i] = r < N ? __half2float(__ushort_as_half(g16[(int64_t)i * N + r])) : 0.0f;
        }
    }
    const int gg = threadIdx.x & 31, part = threadIdx.x >> 5;
    const int64_t c0 = (int64_t)s * 256 + gg * 8;
    const bool col_ok = c0 < K;
    uint4 hr[KP];
#pragma unroll
    for (int i = 0; i < KP; ++i)
        hr[i] = col_ok ? *reinterpret_cast<const uint4*>(h16 + (int64_t)i * K + c0) : make_uint4(0, 0, 0, 0);

    pdl_launch_dependents();
    pdl_wait();

    // ---- byte tables of slice s: thread (group gg, part) writes bytes 32*part .. +31
    {
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
            float v[8];
            const uint32_t hw[4] = {hr[i].x, hr[i].y, hr[i].z, hr[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[2 * q] = __half2float(__ushort_as_half((unsigned short)(hw[q] & 0xffffu))) * xv[2 * q];
                v[2 * q + 1] = __half2float(__ushort_as_half((unsigned short)(hw[q] >> 16))) * xv[2 * q + 1];
            }
            float L[16];                       // signed sums of columns 0..3 of the group
            L[0] = -((v[0] + v[1]) + (v[2] + v[3]));
#pragma unroll
            for (int n = 1; n < 16; ++n) {
                const int low = n & -n;
                const int q = low == 1 ? 0 : low == 2 ? 1 : low == 4 ? 2 : 3;
                L[n] = L[n & (n - 1)] + 2.0f * v[q];
            }
            float Hh[2];                       // signed sums of columns 4..7 for this part's high nibbles
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
    __syncthreads();

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
    const char* tb = reinterpret_cast<const char*>(lut);
    const int64_t Ntp = Nt * 32;

    for (int64_t t0 = t_begin + warp; t0 < t_end; t0 += (int64_t)kLutPF * kLutWarps) {
#pragma unroll
        for (int p = 0; p < kLutPF; ++p) {
            const int64_t t = t0 + (int64_t)p * kLutWarps;
            if (t >= t_end) break;
            float acc[KP];
#pragma unroll
            for (int i = 0; i < KP; ++i) {
                float a0 = 0.0f, a1 = 0.0f;
                const char* tp = tb + (i >> 1) * 65536 + (i & 1) * 128;
#pragma unroll
                for (int sl = 0; sl < 8; ++sl) {
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const uint32_t off = prmt(wd[p][i][sl], G[sl], SEL[b]);
                        const float e = *reinterpret_cast<const float*>(tp + off);
                        if (b & 1) a1 += e; else a0 += e;
                    }
                }
                acc[i] = a0 + a1;
            }
            float pr = 0.0f;
#pragma unroll
            for (int i = 0; i < KP; ++i) pr += gv[p][i] * acc[i];
            const int64_t r = t * 32 + lane;
            if (S == 1) {
                if (r < N) store_y(Y, ydt, r, pr);
            } else {
                partial[(int64_t)s * Ntp + r] = pr;
            }
            // refill this slot with the tile kLutPF rounds ahead
            const int64_t tn = t + (int64_t)kLutPF * kLutWarps;
            if (tn < t_end) {
                lut_load_tile<KP>(wd[p], planes, s, tn, S, Nt, lane);
                const int64_t rn = tn * 32 + lane;
#pragma unroll
                for (int i = 0; i < KP; ++i)
                    gv[p][i] = rn < N ? __half2float(__ushort_as_half(g16[(int64_t)i * N + rn])) : 0.0f;
            }
        }
    }
    if (S == 1) return;

    // ---- cross-slice sum: the last of the S CTAs that own row tiles [t_begin, t_end)
    // adds the slice partials in slice order.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(counters + cta, 1u) == (unsigned)(S - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int64_t r = t_begin * 32 + threadIdx.x; r < t_end * 32; r += kLutThreads) {
        float y = 0.0f;
        for (int64_t sb = 0; sb < S; sb += 16) {        // 16 independent L2 loads in flight
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = (sb + j < S) ? __ldcg(partial + (sb + j) * Ntp + r) : 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) y += v[j];
        }
        if (r < N) store_y(Y, ydt, r, y);
    }
    if (threadIdx.x == 0) counters[cta] = 0u;
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

// CTAs per slice for the byte-table kernel: minimise the per-SM load
// ceil(S*C / SMs) * (table build + ceil(Nt/C) row tiles); one table build costs
// about as many shared-memory wavefronts as 6.4 row tiles.
int lut_ctas_per_slice(int64_t S, int64_t Nt, int sms, int kp)
{
    const int occ = kp <= 2 ? 3 : 1;
    int best = 1;
    double best_cost = 1e30;
    for (int C = 1; C <= Nt && C <= 4 * sms; ++C) {
        const int64_t ctas = S * C;
        if (ctas > (int64_t)sms * occ) break;
        const double per_sm = (double)((ctas + sms - 1) / sms);
        const double cost = per_sm * (6.4 + (double)((Nt + C - 1) / C));
        if (cost < best_cost - 1e-9) { best_cost = cost; best = C; }
    }
    return best;
}

struct GemvWs {
    unsigned* counters;
    float* partial;
    size_t bytes;
};

GemvWs gemv_ws_layout(int N, int K, void* base)
{
    const int64_t S = num_slices(K), Nt = num_row_tiles(N);
    const size_t cnt_bytes = ((size_t)Nt * 4 + 255) / 256 * 256;
    const size_t part_bytes = (size_t)S * Nt * 32 * 4;
    GemvWs w;
    w.counters = reinterpret_cast<unsigned*>(base);
    w.partial = reinterpret_cast<float*>(reinterpret_cast<char*>(base) + cnt_bytes);
    w.bytes = S > 1 ? cnt_bytes + part_bytes : 0;
    return w;
}

template <int KP>
rb_status launch_lut(const rb_layer_t* L, const uint16_t* X, void* Y, int ydt,
                     const GemvWs& ws, bool pdl, cudaStream_t stream)
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int smem = lut_smem_bytes(KP);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(gemv_lut_kernel<KP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return RB_ERR_CUDA;
        attr_set[dev] = true;
    }
    const int64_t S = num_slices(L->k_in), Nt = num_row_tiles(L->n_out);
    const int C = lut_ctas_per_slice(S, Nt, num_sms(), KP);
    return launch(gemv_lut_kernel<KP>, dim3((unsigned)(S * C)), dim3(kLutThreads), (size_t)smem,
                  stream, pdl, L->planes, L->g16, L->h16, X, L->n_out, L->k_in, C,
                  ws.partial, ws.counters, Y, ydt);
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
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 8 || M < 1 || M > 64)
        return 0;
    rb_layer_t L = {n_out, k_in, k_planes, 0, nullptr, nullptr, nullptr};
    if (!use_lut(&L, M)) return 0;
    return gemv_ws_layout(n_out, k_in, nullptr).bytes;
}

extern "C" rb_status rb_gemv(const rb_layer_t* layer, const uint16_t* X, int M, void* Y,
                             rb_dtype y_dtype, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, unsigned flags, cudaStream_t stream)
{
    (void)dev_status;
    rb_status st = check_apply_args(layer, X, M, Y, y_dtype, flags);
    if (st != RB_OK) return st;
    if (M > 64) return RB_ERR_SHAPE;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    const bool pdl = (flags & RB_LAUNCH_PDL) != 0;
    const int ydt = (int)y_dtype;
    if (use_lut(layer, M)) {
        GemvWs ws = gemv_ws_layout(layer->n_out, layer->k_in, workspace);
        if (ws.bytes && (!workspace || workspace_bytes < ws.bytes)) return RB_ERR_WORKSPACE;
        if (workspace && !aligned16(workspace)) return RB_ERR_ALIGN;
        switch (layer->k_planes) {
            case 1: return launch_lut<1>(layer, X, Y, ydt, ws, pdl, stream);
            case 2: return launch_lut<2>(layer, X, Y, ydt, ws, pdl, stream);
            case 3: return launch_lut<3>(layer, X, Y, ydt, ws, pdl, stream);
            default: return launch_lut<4>(layer, X, Y, ydt, ws, pdl, stream);
        }
    }
    switch (layer->k_planes) {
        case 1: return launch_generic<1>(layer, X, M, Y, ydt, pdl, stream);
        case 2: return launch_generic<2>(layer, X, M, Y, ydt, pdl, stream);
        case 3: return launch_generic<3>(layer, X, M, Y, ydt, pdl, stream);
        case 4: return launch_generic<4>(layer, X, M, Y, ydt, pdl, stream);
        case 5: return launch_generic<5>(layer, X, M, Y, ydt, pdl, stream);
        case 6: return launch_generic<6>(layer, X, M, Y, ydt, pdl, stream);
        case 7: return launch_generic<7>(layer, X, M, Y, ydt, pdl, stream);
        default: return launch_generic<8>(layer, X, M, Y, ydt, pdl, stream);
    }
}

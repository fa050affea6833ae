// rb_gemm.cu -- batched application Y = X . What^T on the tcgen05 tensor cores,
// What = sum_i diag(g_i) B_i diag(h_i)  (RaBiT, "Residual binarization"; the
// k binary paths run side by side and are summed with their row scales).
//
// Per plane i the contraction D_i[n][m] = sum_c (s_i[n][c] h_i[c]) * X[m][c] is
// a dense fp16 GEMM with fp32 accumulation:
//   A_i = +-h_i  (sign expanded in registers, 128 output rows x 64 columns per
//                 stage, written to tensor memory with tcgen05.st: the MMA
//                 reads A straight from TMEM, so the expansion costs no shared
//                 memory bandwidth),
//   B   = X in fp16 (a pre-pass converts bf16 -> fp16, exact in the normal
//                 range, and interleaves each 32-column group so that column
//                 pair (j, j+16) of a sign word becomes one fp16x2 TMEM cell:
//                 one shift + one LOP3 per two weights), loaded by TMA with a
//                 128-byte swizzle,
//   D_i = one fp32 accumulator per plane in TMEM (128 lanes x BT columns).
// Epilogue: Y[m][n] = sum_i g_i[n] * D_i[n][m], one output row per TMEM lane,
// so every store instruction writes 32 consecutive outputs.
//
// Warp roles (64 + 32 EW threads): warp 0 = TMA producer + TMEM allocator,
// warp 1 = MMA issuer (one thread), warps 2 .. 1 + EW = sign expansion, then
// epilogue (warp w owns TMEM lanes 32*(w%4) .. +31; with EW = 8 two warps share
// a lane quarter and take one 32-column word of each k-block, and every other
// 32-token chunk of the epilogue).  Every mbarrier wait is bounded: on expiry
// the kernel raises RB_DEV_TIMEOUT in dev_status, drains what it issued,
// frees its tensor memory and returns.
#include <atomic>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "rbw_internal.cuh"
#include "rb_tcgen05.cuh"

namespace rbw {
namespace {

constexpr int kBR = 128;          // output rows per CTA (MMA M, TMEM lanes)
constexpr int kBK = 64;           // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int kSX = 8;            // X stages (at most; fewer when h pairs of a long K need the room)
__host__ __device__ constexpr int gemm_threads(int ew) { return 64 + 32 * ew; }

// Instruction descriptor, kind::f16: fp32 D, fp16 A and B, both K-major, N = bt, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int bt) {
    return (1u << 4) | ((uint32_t)(bt >> 3) << 17) | ((uint32_t)(kBR >> 4) << 24);
}

__host__ __device__ constexpr int gemm_bt(int kp) { return kp <= 2 ? 128 : 64; }
__host__ __device__ constexpr int gemm_sa(int kp) { return kp <= 2 ? 4 : 2; }
// With three or more planes the expansion warps are the bottleneck and read the
// h pairs of the whole layer from shared memory (one bulk copy per CTA) with the
// sign words a slice ahead; with one or two planes the k-block-ahead loads from
// global memory measured faster.
__host__ __device__ constexpr bool gemm_hp_in_smem(int kp) { return kp >= 3; }
// Shared memory: nsx X stages, the h pairs when they live there (kp * K/2 words), barriers.
__host__ __device__ inline int gemm_hp_bytes(int kp, int K) {
    return gemm_hp_in_smem(kp) ? ((kp * (K / 2) * 4) + 127) / 128 * 128 : 0;
}
// ks > 1 adds the receive area of the cluster reduction (128 rows x bt tokens fp32).
__host__ __device__ inline int gemm_smem_bytes(int kp, int bt, int K, int nsx, int ks) {
    return nsx * bt * 128 + gemm_hp_bytes(kp, K) + 1024 + 256 + (ks > 1 ? ks * ((kBR + ks - 1) / ks) * bt * 4 : 0);
}

// ---------------------------------------------------------------- pre-pass
// X16[m][32q + 2j + e] = fp16(X[m][32q + j + 16e]);  hperm[i][16q + j] = (h[32q+j], h[32q+j+16]),
// from the stored fp16 h16, or (h32 != nullptr, training forward) from fp32 h rounded to nearest even.
__global__ void gemm_prepass_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ h16,
                                    int M, int K, int kp, uint16_t* __restrict__ X16,
                                    uint32_t* __restrict__ hperm, int32_t* dev_status,
                                    const float* __restrict__ h32)
{
    pdl_launch_dependents();
    pdl_wait();
    const int64_t groups = (int64_t)K / 32;
    const int64_t nx = (int64_t)M * groups, nh = (int64_t)kp * groups;
    int flags = 0;
    for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < nx + nh;
         it += (int64_t)gridDim.x * blockDim.x) {
        if (it < nx) {
            const int64_t m = it / groups, q = it % groups;
            const uint4* src = reinterpret_cast<const uint4*>(X + m * K + q * 32);
            uint32_t in[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 u = src[v];
                in[4 * v] = u.x; in[4 * v + 1] = u.y; in[4 * v + 2] = u.z; in[4 * v + 3] = u.w;
            }
            uint32_t out[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t lo = (j & 1) ? (in[j >> 1] >> 16) : (in[j >> 1] & 0xffffu);
                const uint32_t hi = (j & 1) ? (in[8 + (j >> 1)] >> 16) : (in[8 + (j >> 1)] & 0xffffu);
                const __half a = __float2half_rn(bf16_bits_to_f32(lo));
                const __half b = __float2half_rn(bf16_bits_to_f32(hi));
                if (__hisinf(a) || __hisinf(b)) flags |= RB_DEV_RANGE;
                out[j] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
            }
            uint4* dst = reinterpret_cast<uint4*>(X16 + m * K + q * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(out[4 * v], out[4 * v + 1], out[4 * v + 2], out[4 * v + 3]);
        } else {
            const int64_t x = it - nx, i = x / groups, q = x % groups;
            uint32_t* hd = hperm + i * (K / 2) + q * 16;
            if (h32) {
                const float* hs = h32 + i * K + q * 32;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const __half a = __float2half_rn(hs[j]), b = __float2half_rn(hs[j + 16]);
                    if (__hisnan(a) || __hisnan(b)) flags |= RB_DEV_NONFINITE;
                    else if (__hisinf(a) || __hisinf(b)) flags |= RB_DEV_RANGE;
                    hd[j] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
                }
            } else {
                const uint16_t* hs = h16 + i * K + q * 32;
#pragma unroll
                for (int j = 0; j < 16; ++j) hd[j] = (uint32_t)hs[j] | ((uint32_t)hs[j + 16] << 16);
            }
        }
    }
    if (flags) set_dev_status(dev_status, flags);
}

// ---------------------------------------------------------------- main kernel
// BT tokens per tile (the MMA's N), SA A stages.  gridDim.z = ks > 1 splits K:
// the ks CTAs of a cluster (1, 1, ks) take kb_per k-blocks each, push their
// partial sums (Y contributions of 128 rows x BT tokens) over distributed
// shared memory to the rank that owns the row, and that rank adds them in
// rank order.
// g32 != nullptr (training forward): the epilogue scales row n of plane i by
// the fp32 g32[i][n] instead of the stored fp16 g16.
template <int KP, int BT, int SA, int EW>
__global__ void __launch_bounds__(gemm_threads(EW), (KP <= 2 && BT <= 64) ? 2 : 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint32_t* __restrict__ planes,
               const uint16_t* __restrict__ g16, const uint32_t* __restrict__ hperm,
               int N, int K, int M, void* __restrict__ Y, int ydt, int32_t* dev_status, uint64_t timeout_ns,
               int nsx, int kb_per, const float* __restrict__ g32)
{
    constexpr int NCOLS = (KP * BT + SA * KP * 32) <= 256 ? 256 : 512;
    constexpr uint32_t X_STAGE = BT * 128;
    constexpr uint32_t IDESC = idesc_f16(BT);
    static_assert(KP * BT + SA * KP * 32 <= NCOLS, "tensor memory budget");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base for the swizzled X stages
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t xs0 = sbase;
    const uint32_t hp_bytes = (uint32_t)gemm_hp_bytes(KP, K);
    const uint32_t hps = sbase + (uint32_t)nsx * X_STAGE;           // h pairs, [plane][K/2]
    const uint32_t* hsm = reinterpret_cast<const uint32_t*>(gbase + (size_t)nsx * X_STAGE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + (size_t)nsx * X_STAGE + hp_bytes);
    const uint32_t bar0 = smem_u32(bars);
    auto full_x = [&](int s) { return bar0 + 8u * s; };
    auto empty_x = [&](int s) { return bar0 + 8u * (kSX + s); };
    auto full_a = [&](int s) { return bar0 + 8u * (2 * kSX + s); };
    auto empty_a = [&](int s) { return bar0 + 8u * (2 * kSX + SA + s); };
    const uint32_t acc_full = bar0 + 8u * (2 * kSX + 2 * SA);
    const uint32_t hp_full = bar0 + 8u * (2 * kSX + 2 * SA + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kSX + 2 * SA + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kBR, m0 = blockIdx.y * BT;
    const int nkb = (K + kBK - 1) / kBK;
    const int ks = (int)gridDim.z, rank = (int)blockIdx.z;
    const int kb0 = rank * kb_per;
    const int kb1 = kb0 + kb_per < nkb ? kb0 + kb_per : nkb;      // kb0 < kb1 (host guarantees)
    const int nloc = kb1 - kb0;
    float* recv = reinterpret_cast<float*>(gbase + (size_t)nsx * X_STAGE + hp_bytes + 256);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSX; ++s) { mbar_init(full_x(s), 1); mbar_init(empty_x(s), 1); }
        for (int s = 0; s < SA; ++s) { mbar_init(full_a(s), 32 * EW); mbar_init(empty_a(s), 1); }
        mbar_init(acc_full, 1);
        mbar_init(hp_full, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(&tmap_x) : "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"((uint32_t)NCOLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();
    pdl_wait();                                   // X16 / hperm come from the pre-pass

    if (warp == 0) {
        if (lane == 0) {                          // ---------------- TMA producer
            if constexpr (gemm_hp_in_smem(KP)) {
                mbar_arrive_expect_tx(hp_full, (uint32_t)(KP * (K / 2) * 4));
                bulk_load(hps, hperm, (uint32_t)(KP * (K / 2) * 4), hp_full);
            }
            // stage s and its fill count j (phase = j & 1) advance without divisions
            int issued = 0, s = 0, j = 0;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (j > 0 && !mbar_wait(empty_x(s), (j - 1) & 1, abort_flag, dev_status, timeout_ns)) break;
                mbar_arrive_expect_tx(full_x(s), X_STAGE);
                tma_load_2d(xs0 + s * X_STAGE, &tmap_x, full_x(s), kb * kBK, m0);
                ++issued;
                if (++s == nsx) { s = 0; ++j; }
            }
            if (*abort_flag) {                    // drain the loads this thread issued: they always land
                const uint64_t t0 = globaltimer_ns();
                for (int kb = issued - nsx < 0 ? 0 : issued - nsx; kb < issued; ++kb)
                    mbar_drain(full_x(kb % nsx), (kb / nsx) & 1, t0);
                if constexpr (gemm_hp_in_smem(KP)) mbar_drain(hp_full, 0, t0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {                          // ---------------- MMA issuer
            int s = 0;
            uint32_t xphase = 0;
            for (int it = 0; it < nloc; ++it) {
                const int sa = it % SA;
                if (!mbar_wait(full_x(s), xphase, abort_flag, dev_status, timeout_ns)) break;
                if (!mbar_wait(full_a(sa), (it / SA) & 1, abort_flag, dev_status, timeout_ns)) break;
                tc_fence_after();
                const uint32_t xaddr = xs0 + s * X_STAGE;
#pragma unroll
                for (int i = 0; i < KP; ++i) {
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t a_t = tmem + (uint32_t)(KP * BT + (sa * KP + i) * 32 + kk * 8);
                        const uint32_t d_t = tmem + (uint32_t)(i * BT);
                        tc_mma_f16_ts(d_t, a_t, smem_desc_sw128(xaddr + kk * 32), IDESC,
                                      (it > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc_commit(empty_x(s));
                tc_commit(empty_a(sa));
                if (++s == nsx) { s = 0; xphase ^= 1u; }
            }
            tc_commit(acc_full);                  // arrives once every MMA issued above is done
        }
    } else {                                      // ---------------- expansion, then epilogue
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const int64_t n = (int64_t)n0 + r;
        const int64_t S = num_slices(K), Nt = num_row_tiles(N);
        const int64_t tile = n >> 5;
        const bool tile_ok = tile < Nt;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        static_assert(EW == 4 || EW == 8, "four or eight expansion warps");
        constexpr int NWW = EW == 8 ? 1 : 2;     // 32-column words of a k-block per thread
        const int hh = EW == 8 ? (warp - 2) >> 2 : 0;   // with EW = 8: this warp's word of the k-block
        bool ok = true;
        if constexpr (!gemm_hp_in_smem(KP)) {
            // Sign words and +-h pairs of one k-block, fetched one k-block ahead from
            // global memory (L1/L2 hits: every row of the CTA reads the same h pairs).
            auto load_kb = [&](int kb, uint32_t (&wv)[KP][NWW], uint32_t (&hp)[KP][16 * NWW]) {
                const int64_t sl = kb / 4;
                const int w0 = (kb & 3) * 2;
#pragma unroll
                for (int i = 0; i < KP; ++i) {
#pragma unroll
                    for (int w2 = 0; w2 < NWW; ++w2) {
                        const int ww = NWW == 1 ? hh : w2;
                        const int64_t col0 = (int64_t)kb * kBK + ww * 32;
                        wv[i][w2] = (tile_ok && col0 < K)
                            ? planes[block_index(i, sl, tile, S, Nt) * 256 + (((w0 + ww) ^ (lane >> 2)) * 32) + lane]
                            : 0u;
                        const int64_t hbase = (int64_t)i * (K / 2) + (int64_t)kb * 32 + ww * 16;
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 u = make_uint4(0, 0, 0, 0);
                            if (col0 < K) u = *reinterpret_cast<const uint4*>(hperm + hbase + 4 * v);
                            hp[i][16 * w2 + 4 * v] = u.x; hp[i][16 * w2 + 4 * v + 1] = u.y;
                            hp[i][16 * w2 + 4 * v + 2] = u.z; hp[i][16 * w2 + 4 * v + 3] = u.w;
                        }
                    }
                }
            };
            uint32_t wv[KP][NWW], hp[KP][16 * NWW];
            load_kb(kb0, wv, hp);
            for (int kb = kb0; kb < kb1 && ok; ++kb) {
                const int it = kb - kb0, sa = it % SA;
                uint32_t cw[KP][NWW], ch[KP][16 * NWW];
#pragma unroll
                for (int i = 0; i < KP; ++i) {
#pragma unroll
                    for (int w2 = 0; w2 < NWW; ++w2) cw[i][w2] = wv[i][w2];
#pragma unroll
                    for (int j = 0; j < 16 * NWW; ++j) ch[i][j] = hp[i][j];
                }
                if (kb + 1 < kb1) load_kb(kb + 1, wv, hp);
                if (it >= SA) {
                    if (!mbar_wait_warp(empty_a(sa), ((it / SA) - 1) & 1, abort_flag, dev_status, timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
#pragma unroll
                for (int i = 0; i < KP; ++i) {
                    uint32_t a[16 * NWW];
#pragma unroll
                    for (int w2 = 0; w2 < NWW; ++w2)
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            a[w2 * 16 + j] = lop3_sign(cw[i][w2] << (15 - j), ch[i][w2 * 16 + j]);
                    const uint32_t col = (uint32_t)(KP * BT + (sa * KP + i) * 32);
                    if constexpr (NWW == 2) tc_st_32x32b_x32(tmem + lane_base + col, a);
                    else tc_st_32x32b_x16(tmem + lane_base + col + (uint32_t)(hh * 16), a);
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(full_a(sa));
            }
        } else {
            // Sign words: the 8 logical words of a 256-column slice (4 k-blocks) per
            // plane, loaded one slice ahead.  h pairs: from shared memory.
            auto load_slice = [&](int64_t sl, uint32_t (&wv)[KP][8]) {
    #pragma unroll
                for (int i = 0; i < KP; ++i) {
                    const uint32_t* blk = planes + block_index(i, sl, tile, S, Nt) * 256 + lane;
    #pragma unroll
                    for (int w = 0; w < 8; ++w)
                        wv[i][w] = (tile_ok && sl * 256 + w * 32 < K) ? blk[((w ^ (lane >> 2)) * 32)] : 0u;
                }
            };
            uint32_t cur[KP][8], nxt[KP][8];
            load_slice(kb0 / 4, cur);
            ok = mbar_wait_warp(hp_full, 0, abort_flag, dev_status, timeout_ns);
            for (int64_t sl = kb0 / 4; sl * 4 < kb1 && ok; ++sl) {
                if ((sl + 1) * 4 < kb1) load_slice(sl + 1, nxt);
    #pragma unroll
                for (int qk = 0; qk < 4; ++qk) {
                    const int kb = (int)sl * 4 + qk;
                    if (kb >= kb1 || !ok) break;
                    const int it = kb - kb0, sa = it % SA;
                    if (it >= SA) {
                        if (!mbar_wait_warp(empty_a(sa), ((it / SA) - 1) & 1, abort_flag, dev_status, timeout_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
    #pragma unroll
                    for (int i = 0; i < KP; ++i) {
                        uint32_t hp[16 * NWW];
                        uint32_t a[16 * NWW];
    #pragma unroll
                        for (int w2 = 0; w2 < NWW; ++w2) {
                            const int ww = NWW == 1 ? hh : w2;
                            const uint32_t* hrow = hsm + (size_t)i * (K / 2) + (size_t)kb * 32 + ww * 16;
    #pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                uint4 u = make_uint4(0, 0, 0, 0);
                                if (kb * 64 + ww * 32 < K) u = *reinterpret_cast<const uint4*>(hrow + 4 * v);
                                hp[16 * w2 + 4 * v] = u.x; hp[16 * w2 + 4 * v + 1] = u.y;
                                hp[16 * w2 + 4 * v + 2] = u.z; hp[16 * w2 + 4 * v + 3] = u.w;
                            }
    #pragma unroll
                            for (int j = 0; j < 16; ++j)
                                a[w2 * 16 + j] = lop3_sign(cur[i][2 * qk + ww] << (15 - j), hp[w2 * 16 + j]);
                        }
                        const uint32_t col = (uint32_t)(KP * BT + (sa * KP + i) * 32);
                        if constexpr (NWW == 2) tc_st_32x32b_x32(tmem + lane_base + col, a);
                        else tc_st_32x32b_x16(tmem + lane_base + col + (uint32_t)(hh * 16), a);
                    }
                    tc_wait_st();
                    tc_fence_before();
                    mbar_arrive(full_a(sa));
                }
    #pragma unroll
                for (int i = 0; i < KP; ++i)
    #pragma unroll
                    for (int w = 0; w < 8; ++w) cur[i][w] = nxt[i][w];
            }
        }
        // ---- epilogue
        if (ok && mbar_wait_warp(acc_full, 0, abort_flag, dev_status, timeout_ns)) {
            tc_fence_after();
            float gi[KP];
#pragma unroll
            for (int i = 0; i < KP; ++i)
                gi[i] = n >= N ? 0.0f : g32 ? g32[(int64_t)i * N + n]
                                            : __half2float(__ushort_as_half(g16[(int64_t)i * N + n]));
            constexpr int CW = BT < 32 ? BT : 32;            // tokens per TMEM load
            constexpr int PB = KP <= 4 ? KP : 2;             // planes per batch of TMEM loads (registers)
#pragma unroll 1
            for (int c = NWW == 1 ? hh : 0; c < BT / CW; c += 3 - NWW) {
                float y[CW];
#pragma unroll
                for (int j = 0; j < CW; ++j) y[j] = 0.0f;
#pragma unroll
                for (int i0 = 0; i0 < KP; i0 += PB) {
                    uint32_t v[PB][CW];
#pragma unroll
                    for (int ii = 0; ii < PB; ++ii) {
                        if (i0 + ii >= KP) break;
                        const uint32_t col = (uint32_t)((i0 + ii) * BT + c * CW);
                        if constexpr (CW == 32) tc_ld_32x32b_x32(tmem + lane_base + col, v[ii]);
                        else tc_ld_32x32b_x16(tmem + lane_base + col, v[ii]);
                    }
                    tc_wait_ld();
#pragma unroll
                    for (int ii = 0; ii < PB; ++ii) {
                        if (i0 + ii >= KP) break;
#pragma unroll
                        for (int j = 0; j < CW; ++j) y[j] = fmaf(gi[i0 + ii], __uint_as_float(v[ii][j]), y[j]);
                    }
                }
                if (ks == 1) {
                    if (n < N) {
#pragma unroll
                        for (int j = 0; j < CW; ++j) {
                            const int64_t m = (int64_t)m0 + c * CW + j;
                            if (m < M) store_y(Y, ydt, m * N + n, y[j]);
                        }
                    }
                } else {                          // slot (this rank, row, tokens c*CW ..) at the row's owner
                    // rank j owns rows [ceil(128 j / ks), ceil(128 (j+1) / ks)); any ks <= 16
                    const int rpo = (kBR + ks - 1) / ks, owner = (r * ks) / kBR;
                    const int lr = r - (kBR * owner + ks - 1) / ks;
                    const uint32_t dst = smem_u32(recv) + (uint32_t)(((rank * rpo + lr) * BT + c * CW) * 4);
#pragma unroll
                    for (int j = 0; j < CW; j += 4)
                        st_dsmem_v4(dst + (uint32_t)(j * 4), (uint32_t)owner, y[j], y[j + 1], y[j + 2], y[j + 3]);
                }
            }
        }
    }

    if (ks > 1) {                                 // every CTA arrives, also one that gave up
        cluster_sync_all();
        const int rpo = (kBR + ks - 1) / ks;
        const int row0 = (kBR * rank + ks - 1) / ks, nrow = (kBR * (rank + 1) + ks - 1) / ks - row0;
        for (int idx = threadIdx.x; idx < nrow * BT; idx += (int)blockDim.x) {
            const int tok = idx / nrow, lr = idx - tok * nrow;
            float v = 0.0f;
            for (int j = 0; j < ks; ++j) v += recv[(j * rpo + lr) * BT + tok];
            const int64_t n = (int64_t)n0 + row0 + lr, m = (int64_t)m0 + tok;
            if (n < N && m < M) store_y(Y, ydt, m * N + n, v);
        }
    }

    // ---- teardown: every MMA has completed (acc_full) or the CTA gave up
    if (warp == 1 && lane == 0 && *abort_flag)      // no MMA may still run when TMEM is freed:
        mbar_drain(acc_full, 0, globaltimer_ns());  // acc_full is committed after the last MMA, always
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) set_dev_status(dev_status, RB_DEV_TIMEOUT);
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem), "r"((uint32_t)NCOLS) : "memory");
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn()
{
    // Looked up once per process; host threads may race here, and every racer
    // stores the same driver address.
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

struct GemmWs {
    uint16_t* x16;
    uint32_t* hperm;
    size_t bytes;
};

GemmWs gemm_ws_layout(int K, int kp, int M, void* base)
{
    GemmWs w;
    const size_t xb = ((size_t)M * K * 2 + 255) / 256 * 256;
    const size_t hb = ((size_t)kp * K * 2 + 255) / 256 * 256;
    w.x16 = reinterpret_cast<uint16_t*>(base);
    w.hperm = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(base) + xb);
    w.bytes = xb + hb;
    return w;
}

// ks > 1: K split over clusters of (1, 1, ks); every rank gets a whole number
// of 256-column slices and at least one k-block.
template <int KP, int BT, int SA, int EW = 4>
rb_status launch_gemm(const rb_layer_t* L, int M, void* Y, int ydt, const GemmWs& ws,
                      int32_t* dev_status, bool pdl, cudaStream_t stream, uint64_t timeout_ns, int ks,
                      const float* g32 = nullptr, bool dry = false)
{
    if (dry) {                                   // only the shared-memory check, nothing launched
        int kb_per = ((L->k_in + kBK - 1) / kBK + ks - 1) / ks;
        kb_per = (kb_per + 3) / 4 * 4;
        ks = ((L->k_in + kBK - 1) / kBK + kb_per - 1) / kb_per;
        return gemm_smem_bytes(KP, BT, L->k_in, 2, ks) > 227 * 1024 ? RB_ERR_UNSUPPORTED : RB_OK;
    }
    PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
    if (!enc) return RB_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)L->k_in, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)L->k_in * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BT};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ws.x16, gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return RB_ERR_CUDA;
    const int nkb = (L->k_in + kBK - 1) / kBK;
    int kb_per = (nkb + ks - 1) / ks;
    kb_per = (kb_per + 3) / 4 * 4;                            // whole slices per rank
    ks = (nkb + kb_per - 1) / kb_per;                         // no rank without k-blocks
    static std::atomic<bool> attr_set[64];       // per device; setting the attributes twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    constexpr int kMaxSmem = 227 * 1024;
    int nsx = kSX;
    while (nsx > 2 && gemm_smem_bytes(KP, BT, L->k_in, nsx, ks) > kMaxSmem) --nsx;
    const int smem = gemm_smem_bytes(KP, BT, L->k_in, nsx, ks);
    if (smem > kMaxSmem) return RB_ERR_UNSUPPORTED;          // K too long for the h pairs in shared memory
    if (dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(gemm_tc_kernel<KP, BT, SA, EW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxSmem) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_tc_kernel<KP, BT, SA, EW>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess)
            return RB_ERR_CUDA;
        attr_set[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((L->n_out + kBR - 1) / kBR), (unsigned)((M + BT - 1) / BT), (unsigned)ks);
    cfg.blockDim = dim3(gemm_threads(EW));
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (ks > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = (unsigned)ks;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, gemm_tc_kernel<KP, BT, SA, EW>, map, L->planes, L->g16, (const uint32_t*)ws.hperm,
                           (int)L->n_out, (int)L->k_in, M, Y, ydt, dev_status, timeout_ns, nsx, kb_per, g32) !=
        cudaSuccess)
        return RB_ERR_CUDA;
    return RB_OK;
}

// Decode-sized M (<= 64): tokens per tile 16, 32 or 64, two A stages, and the
// K split that gives about two CTAs per SM (at most 16 ranks).
template <int KP>
rb_status launch_gemm_decode(const rb_layer_t* L, int M, void* Y, int ydt, const GemmWs& ws,
                             int32_t* dev_status, cudaStream_t stream, uint64_t timeout_ns)
{
    const int bt = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    const int64_t ctas = (int64_t)((L->n_out + kBR - 1) / kBR) * ((M + bt - 1) / bt);
    const int nkb = (L->k_in + kBK - 1) / kBK;
    int ks = 1;
    while (ks < 16 && ks * 4 < nkb && ctas * ks < 2LL * num_sms()) ks *= 2;
    if (bt == 16) return launch_gemm<KP, 16, 2>(L, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, ks);
    if (bt == 32) return launch_gemm<KP, 32, 2>(L, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, ks);
    return launch_gemm<KP, 64, 2>(L, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, ks);
}

// Expansion warps of the prefill tiles: eight for k = 4 (its expansion is the
// longest; 614 against 549 TFLOP/s at M = 2048 on 4096 x 4096), four below
// (eight measured within +-3 % for k <= 2 and 5 % slower for k = 3).
template <int KP> constexpr int kPrefillEW = KP == 4 ? 8 : 4;

// Tile shape per k and M for the prefill kernel (the prepass has run).
rb_status gemm_dispatch(const rb_layer_t* layer, int M, void* Y, int ydt, const GemmWs& ws, int32_t* dev_status,
                        cudaStream_t stream, uint64_t timeout_ns, const float* g32, bool dry = false)
{
    // Wider token tiles amortise each k-block's fixed cost (expansion, barriers)
    // over more MMA work: 256 tokens for k = 1, 192 for k = 2 and 96 for k = 3
    // (the widest the 512 tensor-memory columns hold next to the A stages) once
    // M fills them; narrower below that, where a wide last tile pads more.
    switch (layer->k_planes) {
        case 1:
            if (M >= 1024) return launch_gemm<1, 256, 4, kPrefillEW<1>>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
            return launch_gemm<1, gemm_bt(1), gemm_sa(1), kPrefillEW<1>>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
        case 2:
            if (M >= 1536) return launch_gemm<2, 192, 2, kPrefillEW<2>>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
            return launch_gemm<2, gemm_bt(2), gemm_sa(2), kPrefillEW<2>>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
        case 3:
            if (M >= 1024) return launch_gemm<3, 96, 2, kPrefillEW<3>>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
            return launch_gemm<3, gemm_bt(3), gemm_sa(3), kPrefillEW<3>>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
        case 4: return launch_gemm<4, gemm_bt(4), gemm_sa(4), kPrefillEW<4>>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
        // k = 5..8: the accumulators (k x BT columns) and the A stages (SA x k x 32)
        // share the 512 tensor-memory columns, so the tiles narrow and the
        // pipeline shortens as k grows.
        case 5: return launch_gemm<5, 32, 2>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
        case 6: return launch_gemm<6, 16, 2>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
        case 7: return launch_gemm<7, 32, 1>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
        default: return launch_gemm<8, 32, 1>(layer, M, Y, ydt, ws, dev_status, true, stream, timeout_ns, 1, g32, dry);
    }
}

}  // namespace

// rb_gemm with a caller-chosen bound on every device-side wait; decode = the
// small-M tile shapes with the K split (rb_gemv for M >= 2 with a workspace).
rb_status gemm_with_timeout(const rb_layer_t* layer, const uint16_t* X, int M, void* Y, rb_dtype y_dtype,
                               void* workspace, size_t workspace_bytes, int32_t* dev_status, unsigned flags,
                               cudaStream_t stream, uint64_t timeout_ns, bool decode)
{
    rb_status st = check_apply_args(layer, X, M, Y, y_dtype, flags);
    if (st != RB_OK) return st;
    if (decode && (M > 64 || layer->k_planes > 4)) return RB_ERR_UNSUPPORTED;
    if (dev_status && !aligned16(dev_status)) return RB_ERR_ALIGN;
    GemmWs ws = gemm_ws_layout(layer->k_in, layer->k_planes, M, workspace);
    if (!workspace || workspace_bytes < ws.bytes) return RB_ERR_WORKSPACE;
    if (!aligned16(workspace)) return RB_ERR_ALIGN;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    const bool pdl = (flags & RB_LAUNCH_PDL) != 0;
    const int64_t groups = layer->k_in / 32;
    int64_t items = (int64_t)M * groups + (int64_t)layer->k_planes * groups;
    int64_t ctas = (items + 255) / 256;
    if (ctas > 8 * num_sms()) ctas = 8 * num_sms();
    st = launch(gemm_prepass_kernel, dim3((unsigned)ctas), dim3(256), 0, stream, pdl, X, layer->h16, M,
                layer->k_in, layer->k_planes, ws.x16, ws.hperm, dev_status, (const float*)nullptr);
    if (st != RB_OK) return st;
    const int ydt = (int)y_dtype;
    if (decode) {
        switch (layer->k_planes) {
            case 1: return launch_gemm_decode<1>(layer, M, Y, ydt, ws, dev_status, stream, timeout_ns);
            case 2: return launch_gemm_decode<2>(layer, M, Y, ydt, ws, dev_status, stream, timeout_ns);
            case 3: return launch_gemm_decode<3>(layer, M, Y, ydt, ws, dev_status, stream, timeout_ns);
            default: return launch_gemm_decode<4>(layer, M, Y, ydt, ws, dev_status, stream, timeout_ns);
        }
    }
    return gemm_dispatch(layer, M, Y, ydt, ws, dev_status, stream, timeout_ns, nullptr);
}

size_t gemm_workspace(int k_in, int k_planes, int M) { return gemm_ws_layout(k_in, k_planes, M, nullptr).bytes; }

}  // namespace rbw

using namespace rbw;

extern "C" size_t rb_gemm_workspace_bytes(int n_out, int k_in, int k_planes, int M)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 8 || M < 1) return 0;
    return gemm_ws_layout(k_in, k_planes, M, nullptr).bytes;
}

extern "C" rb_status rb_gemm(const rb_layer_t* layer, const uint16_t* X, int M, void* Y, rb_dtype y_dtype,
                             void* workspace, size_t workspace_bytes, int32_t* dev_status, unsigned flags,
                             cudaStream_t stream)
{
    return gemm_with_timeout(layer, X, M, Y, y_dtype, workspace, workspace_bytes, dev_status, flags,
                             stream, kTimeoutNs, false);
}

// Training forward: the planes of this step's latent W are derived once into
// the workspace by the pack kernel (one read of W), then the prefill kernel
// runs on them with the fp32 g in its epilogue and the h pairs rounded from
// the fp32 h.  Deriving the signs inside the GEMM's operand expansion instead
// re-reads W once per token tile; at M = 2048 on a 4096 x 4096, k = 2 layer it
// measured 515 us against 19 + 168 us for these two steps.
namespace rbw {
namespace {
size_t qat_planes_bytes(int n_out, int k_in, int k_planes)
{
    return (rb_packed_words(n_out, k_in, k_planes) * 4 + 255) / 256 * 256;
}
}  // namespace
}  // namespace rbw

extern "C" size_t rb_qat_forward_workspace_bytes(int n_out, int k_in, int k_planes, int M)
{
    const size_t g = rb_gemm_workspace_bytes(n_out, k_in, k_planes, M);
    return g ? qat_planes_bytes(n_out, k_in, k_planes) + g : 0;
}

extern "C" rb_status rb_qat_forward(const float* W, const float* g, const float* h, int n_out, int k_in,
                                    int k_planes, const uint16_t* X, int M, void* Y, rb_dtype y_dtype,
                                    void* workspace, size_t workspace_bytes, int32_t* dev_status, unsigned flags,
                                    cudaStream_t stream)
{
    if (!W || !g || !h || !X || !Y) return RB_ERR_ARG;
    if (k_planes < 1 || k_planes > 8) return RB_ERR_ARG;
    if ((y_dtype != RB_F32 && y_dtype != RB_BF16) || (flags & ~RB_LAUNCH_PDL)) return RB_ERR_ARG;
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || M < 1) return RB_ERR_SHAPE;
    const void* ptrs[] = {W, g, h, X, Y};
    for (const void* q : ptrs)
        if (!aligned16(q)) return RB_ERR_ALIGN;
    if (dev_status && !aligned16(dev_status)) return RB_ERR_ALIGN;
    if (!workspace || workspace_bytes < rb_qat_forward_workspace_bytes(n_out, k_in, k_planes, M))
        return RB_ERR_WORKSPACE;
    if (!aligned16(workspace)) return RB_ERR_ALIGN;
    if (!device_is_sm100()) return RB_ERR_UNSUPPORTED;
    uint32_t* planes = static_cast<uint32_t*>(workspace);
    const size_t pb = qat_planes_bytes(n_out, k_in, k_planes);
    GemmWs ws = gemm_ws_layout(k_in, k_planes, M, static_cast<uint8_t*>(workspace) + pb);
    // a layer view of the derived planes; its fp16 scales are not read (g32 and the prepass's h pairs are)
    const rb_layer_t L{n_out, k_in, k_planes, 0, planes, nullptr, nullptr};
    // the GEMM's shared-memory limit on K is checked before anything is launched
    rb_status st = gemm_dispatch(&L, M, Y, (int)y_dtype, ws, dev_status, stream, kTimeoutNs, g, true);
    if (st != RB_OK) return st;
    st = pack_planes(W, g, h, n_out, k_in, k_planes, planes, dev_status, stream);
    if (st != RB_OK) return st;
    const bool pdl = (flags & RB_LAUNCH_PDL) != 0;
    const int64_t groups = k_in / 32;
    int64_t ctas = ((int64_t)M * groups + (int64_t)k_planes * groups + 255) / 256;
    if (ctas > 8 * num_sms()) ctas = 8 * num_sms();
    st = launch(gemm_prepass_kernel, dim3((unsigned)ctas), dim3(256), 0, stream, pdl, X,
                (const uint16_t*)nullptr, M, k_in, k_planes, ws.x16, ws.hperm, dev_status, h);
    if (st != RB_OK) return st;
    return gemm_dispatch(&L, M, Y, (int)y_dtype, ws, dev_status, stream, kTimeoutNs, g);
}

extern "C" rb_status rb_gemm_wait_limit(const rb_layer_t* layer, const uint16_t* X, int M, void* Y,
                                        rb_dtype y_dtype, void* workspace, size_t workspace_bytes,
                                        int32_t* dev_status, unsigned flags, uint64_t wait_limit_ns,
                                        cudaStream_t stream)
{
    if (wait_limit_ns > kTimeoutNs) return RB_ERR_ARG;
    return gemm_with_timeout(layer, X, M, Y, y_dtype, workspace, workspace_bytes, dev_status, flags,
                             stream, wait_limit_ns, false);
}

// ---------------------------------------------------------------------------
// rb_gemm_noalloc: rb_gemm for callers that must not allocate device memory.
//
// Some hosts hand this library a fixed device-memory budget up front and do
// not allow further allocations: embedded and real-time deployments that size
// everything at start-up, plugin hosts whose own allocator owns the GPU, or
// code that must not block on the allocator's device-wide synchronisation.
// Such callers cannot provide rb_gemm's workspace.  This entry point uses a
// file-scope device array instead (kNoAllocScratchBytes, held by every GPU
// that loads the library until the process exits).  It calls no cudaMalloc,
// cudaFree or any other allocating routine.
//
// The array's name is only a host-side stand-in in host code; its device
// address is looked up once per device with cudaGetSymbolAddress, with that
// device current, by the first call on that device (so the first call on a
// device should come before any stream capture).  Every call shares the array
// and the kernels fully rewrite the part they use before reading it, so no
// state carries over; calls that overlap on the GPU (for example on two
// streams at once) race on it and must be serialised by the caller.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;    // 32 MiB
static __device__ __align__(256) uint8_t g_gemm_scratch[kNoAllocScratchBytes];

void* noalloc_scratch_address()
{
    static std::atomic<void*> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    void* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_gemm_scratch) != cudaSuccess || !p) return nullptr;
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}
}  // namespace

extern "C" rb_status rb_gemm_noalloc(const rb_layer_t* layer, const uint16_t* X, int M, void* Y, rb_dtype y_dtype,
                                     int32_t* dev_status, unsigned flags, cudaStream_t stream)
{
    rb_status st = rbw::check_apply_args(layer, X, M, Y, y_dtype, flags);
    if (st != RB_OK) return st;
    if (rb_gemm_workspace_bytes(layer->n_out, layer->k_in, layer->k_planes, M) > kNoAllocScratchBytes)
        return RB_ERR_WORKSPACE;                 // problem larger than the fixed scratch array
    if (!rbw::device_is_sm100()) return RB_ERR_UNSUPPORTED;
    void* scratch = noalloc_scratch_address();
    if (!scratch) return RB_ERR_CUDA;
    return rbw::gemm_with_timeout(layer, X, M, Y, y_dtype, scratch, kNoAllocScratchBytes, dev_status, flags,
                                  stream, rbw::kTimeoutNs, false);
}

/*
 * rbw.h -- C ABI of the residual dual-scale binarized linear layer for
 * NVIDIA B200 (sm_100a).
 *
 * The method (RaBiT: Residual-Aware Binarization Training for Accurate and
 * Efficient LLMs; "Residual binarization" background section and Algorithm 2):
 *
 *   W ~= sum_{i=1..k} diag(g_i) B_i diag(h_i),   B_i in {-1,+1}^{N x K}
 *   R_0 = W;  B_i = sign(R_{i-1}) (sign(0) = +1);  R_i = R_{i-1} - g_i h_i^T .* B_i
 *   Y   = sum_i g_i .* (B_i (h_i .* X))              ("matmul-free" inference)
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller (allocated
 *     with cudaMalloc or a framework allocator).  The library allocates no
 *     memory and keeps no global state besides the kernel attributes it sets
 *     once per process.
 *   - Row-major: W is [N out][K in]; X is [M][K]; Y is [M][N].
 *   - Calls are asynchronous on `stream`.  Argument, shape and alignment
 *     errors are returned synchronously and launch nothing.  CUDA launch
 *     errors return RB_ERR_CUDA.  Data-dependent errors (non-finite input,
 *     fp16 overflow of a scale, a bounded device wait that expired) are OR-ed
 *     as RB_DEV_* bits into *dev_status (nullable, caller-zeroed), which the
 *     caller reads after synchronising.
 *   - Every pointer must be 16-byte aligned (RB_ERR_ALIGN otherwise).
 *   - K must be a positive multiple of 32 (RB_ERR_SHAPE otherwise).
 *   - Launch flags: RB_LAUNCH_PDL launches with programmatic dependent launch
 *     so that a kernel may start streaming its weights while the previous
 *     kernel on the stream finishes; the kernels wait for the previous grid
 *     before reading X or writing anything.
 *
 * Packed sign-plane storage layout (the "32 columns packed into one
 * uint32_t" format of RaBiT's kernel paragraph, with a word order chosen for
 * this library):
 *   - bit = 1 <=> B = +1; column c of a word is bit c % 32 (LSB first).
 *   - plane i is cut into S = ceil(K/256) column slices and ceil(N/32) row
 *     tiles of 32 rows; each (plane, slice, row tile) block is 256 words:
 *       word(i, s, r, w) = ((((i*S + s)*Nt + r/32) * 256)
 *                           + ((w ^ ((r % 32) / 4)) * 32) + r % 32
 *     holds columns 256*s + 32*w .. 256*s + 32*w + 31 of row r (w = 0..7,
 *     Nt = ceil(N/32)).  Bits of columns >= K and words of rows >= N are 0.
 *   - scales are IEEE fp16: g16 [k][N], h16 [k][K].
 */
#ifndef RBW_H_
#define RBW_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define RB_API __attribute__((visibility("default")))
#else
#define RB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RB_OK = 0,
    RB_ERR_ARG = 1,          /* null pointer, bad count, bad enum            */
    RB_ERR_SHAPE = 2,        /* K not a multiple of 32, sizes out of range   */
    RB_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned             */
    RB_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required   */
    RB_ERR_UNSUPPORTED = 5,  /* no sm_100 device current, or k/M not served  */
    RB_ERR_CUDA = 6          /* a CUDA runtime call failed                   */
} rb_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define RB_DEV_NONFINITE 0x1  /* W, g or h held a NaN or infinity            */
#define RB_DEV_RANGE 0x2      /* a value rounds to infinity in fp16: a scale
                                 g or h (rb_pack), or an activation x on a
                                 tensor-core path (rb_gemm; rb_gemv and
                                 rb_gemv_batch for M >= 2 or k > 4)          */
#define RB_DEV_TIMEOUT 0x4    /* a bounded device-side wait expired          */

typedef enum { RB_F32 = 0, RB_BF16 = 1 } rb_dtype;

#define RB_LAUNCH_PDL 0x1u

/* A packed layer: all pointers are device pointers owned by the caller. */
typedef struct {
    int32_t n_out;            /* N */
    int32_t k_in;             /* K (multiple of 32) */
    int32_t k_planes;         /* k, 1..8 */
    int32_t reserved;         /* must be 0 */
    const uint32_t *planes;   /* rb_packed_words(N, K, k) words */
    const uint16_t *g16;      /* [k][N] fp16 */
    const uint16_t *h16;      /* [k][K] fp16 */
} rb_layer_t;

/* Library version, 10000*major + 100*minor + patch. */
RB_API int rb_version(void);

/* Human-readable name of a status code (static string). */
RB_API const char *rb_status_string(int status);

/* Number of uint32 words of the sign planes of an N x K layer with k planes
 * (layout above): k * ceil(K/256) * ceil(N/32) * 256.  Returns 0 for invalid
 * sizes. */
RB_API size_t rb_packed_words(int n_out, int k_in, int k_planes);

/*
 * Plain row-major packing <-> storage layout.  RaBiT's kernel paragraph
 * ("Technical novelty": 32 columns packed into one uint32_t) fixes only the
 * word contents; the plain form of it is words [k][N][K/32]: row r, column c
 * at bit c % 32 of word c / 32 (LSB first), bit = 1 meaning B = +1 -- e.g.
 * numpy's packbits(B >= 0, bitorder="little") viewed as little-endian uint32.
 * These calls permute whole words between that form and the storage layout
 * above, so planes packed elsewhere can be applied here and planes derived
 * here can be exported.
 *   rowmajor   rb_rowmajor_words(N, K, k) = k * N * K/32 uint32 words.
 *   planes     rb_packed_words(N, K, k) words in the storage layout; from the
 *              plain form every word is written (padding words zero).
 * The two buffers must not overlap (RB_ERR_ARG).  Asynchronous on `stream`;
 * HBM-bound (one read and one write of k N K / 8 bytes).
 */
RB_API size_t rb_rowmajor_words(int n_out, int k_in, int k_planes);
RB_API rb_status rb_planes_from_rowmajor(const uint32_t *rowmajor, int n_out, int k_in, int k_planes,
                                         uint32_t *planes, cudaStream_t stream);
RB_API rb_status rb_planes_to_rowmajor(const uint32_t *planes, int n_out, int k_in, int k_planes,
                                       uint32_t *rowmajor, cudaStream_t stream);

/*
 * rb_shard_rows -- rows [row0, row0 + rows) of a packed layer as a packed layer
 * of their own, for a row-parallel split over P GPUs: rank r applies its shard
 * to the full X and the [M][rows] outputs are concatenated along N (an
 * all-gather).  The pages give no multi-GPU scheme; since every output row of
 * Y = sum_i g_i .* (B_i (h_i .* X)) depends only on its own sign rows and g
 * values, the split needs no other exchange.
 *   row0         a multiple of 32 (RB_ERR_SHAPE otherwise), rows >= 1,
 *                row0 + rows <= N.
 *   planes_out   rb_packed_words(rows, K, k) words (every word written; rows
 *                past `rows` in the last tile are zero).
 *   g16_out      [k][rows] fp16, copied from layer->g16.
 * The shard's h16 is layer->h16 itself.  Must not overlap layer->planes.
 */
RB_API rb_status rb_shard_rows(const rb_layer_t *layer, int row0, int rows, uint32_t *planes_out,
                               uint16_t *g16_out, cudaStream_t stream);

/*
 * rb_pack -- derive and bit-pack the residual sign planes (RaBiT, Algorithm 2
 * forward pass; deployment freezes these planes and drops W).
 *   W        [N][K] fp32 latent weight.
 *   g, h     [k][N], [k][K] fp32 per-plane scales (any sign; normally >= 0).
 *   planes   out, rb_packed_words(N,K,k) uint32 words (layout above).
 *   g16, h16 out, fp16 copies of g, h (round to nearest even).
 * The residual runs in fp32 with the product g_i[r]*h_i[c] rounded on its own
 * before the single add/subtract (no fused multiply-add), using the fp32
 * scales: b = (R >= 0) (so -0.0 gives +1); R <- b ? R - t : R + t.
 * dev_status gets RB_DEV_NONFINITE / RB_DEV_RANGE.
 */
RB_API rb_status rb_pack(const float *W, const float *g, const float *h,
                  int n_out, int k_in, int k_planes,
                  uint32_t *planes, uint16_t *g16, uint16_t *h16,
                  int32_t *dev_status, cudaStream_t stream);

/*
 * rb_gemv -- decode-time Y = sum_i g_i .* (B_i (h_i .* X)) for 1 <= M <= 64
 * tokens (RaBiT, "Residual binarization": the k binary paths run side by side
 * and are summed after the element-wise scaling).
 *   X   [M][K] bfloat16 bit patterns.
 *   Y   [M][N] fp32 or bfloat16 (y_dtype), written, never read.
 *   workspace: rb_gemv_workspace_bytes(N, K, k, M) bytes of 16-byte aligned
 *   device memory (0 when no path needs one; then NULL is fine).  It holds X
 *   converted to fp16 and the h pairs for the tcgen05 path; no clearing needed.
 *   Calls that share a workspace must not overlap on the GPU.
 * M = 1 and k <= 4: byte tables; h_i .* x is formed exactly in fp32 and every
 * sum is accumulated in fp32 (CUDA cores, additions only).
 * 32 <= M <= 64, k <= 4, N*K*k*M > 4.5e9, with the workspace: the tcgen05
 * kernel of rb_gemm with 16/32/64-token tiles and K split over a thread-block
 * cluster (the measured crossover: below it the mma.sync kernel is faster,
 * and rb_gemv_workspace_bytes returns 0).
 * Otherwise (no workspace, smaller layers, or k > 4): mma.sync kernel.  Both tensor-core paths
 * use fp16 operands with fp32 accumulation: the +-h_i operands are exact in
 * fp16 and X is converted to fp16 (exact for bf16 values of magnitude
 * 2^-14 .. 65504; smaller ones lose low bits; |x| >= 65520 overflows and
 * both paths raise RB_DEV_RANGE in *dev_status), so every product is exact
 * and only the accumulation rounds.  The byte-table path forms h*x in fp32
 * and raises nothing.
 */
RB_API size_t rb_gemv_workspace_bytes(int n_out, int k_in, int k_planes, int M);
RB_API rb_status rb_gemv(const rb_layer_t *layer, const uint16_t *X, int M,
                  void *Y, rb_dtype y_dtype, void *workspace, size_t workspace_bytes,
                  int32_t *dev_status, unsigned flags, cudaStream_t stream);

/*
 * rb_gemv_batch -- rb_gemv applied to `count` independent layers of one shape
 * (same N, K, k) in as few launches as possible, e.g. the q/k/v or gate/up
 * projections of one decode step, or the layers of several models served at
 * once.  layers[j], X[j], Y[j] (host arrays of device pointers) describe
 * application j; Y[j] must not alias any other input or output of the call.
 * For M = 1 one launch serves up to 128 layers; its shape (CTAs per cluster,
 * row chunks per layer) is chosen for the whole batch so that every SM stays
 * busy and each CTA's table builds are spread over many rows.  The per-slice
 * sums are therefore associated differently than in rb_gemv for the same layer,
 * so results may differ from rb_gemv's in the last bits; both are
 * deterministic for a given count.  Needs no workspace.  dev_status
 * (nullable, 16-byte aligned) gets RB_DEV_RANGE as for rb_gemv.
 */
RB_API rb_status rb_gemv_batch(const rb_layer_t *const *layers, const uint16_t *const *X, void *const *Y,
                               int count, int M, rb_dtype y_dtype, int32_t *dev_status, unsigned flags,
                               cudaStream_t stream);

/*
 * rb_gemm -- batched (prefill) Y = X . What^T for any M >= 1 (tuned for
 * M >= 64) on the tcgen05 tensor cores.  It computes the same product as
 * rb_gemv (RaBiT, "Residual binarization": Y = sum_i g_i .* (B_i (h_i .* X)),
 * the k paths side by side) from the bit-packed planes of RaBiT's kernel
 * paragraph ("Technical novelty": 32 columns per uint32_t), organised as a
 * dense contraction: sign tiles are expanded to +-h_i
 * (fp16, exact) and multiplied with X converted to fp16 (exact in the normal
 * range), fp32 accumulation in tensor memory, one accumulator per plane,
 * epilogue Y = sum_i g_i . acc_i.  Every k = 1..8 is served: the k
 * accumulators and the sign-expansion stages share the 512 tensor-memory
 * columns, so the token tile narrows from 192-256 (k <= 2) to 16-32 (k >= 5).
 * For k >= 3 the h pairs of the whole layer sit in shared memory, which
 * bounds k * K (k = 4: K <= 26848; k = 8: K <= 13920); beyond that
 * RB_ERR_UNSUPPORTED.
 *   workspace: rb_gemm_workspace_bytes(N, K, k, M) bytes (holds X in fp16).
 */
RB_API size_t rb_gemm_workspace_bytes(int n_out, int k_in, int k_planes, int M);
RB_API rb_status rb_gemm(const rb_layer_t *layer, const uint16_t *X, int M,
                  void *Y, rb_dtype y_dtype, void *workspace, size_t workspace_bytes,
                  int32_t *dev_status, unsigned flags, cudaStream_t stream);

/*
 * rb_gemm_wait_limit -- rb_gemm with a caller-chosen bound on every
 * device-side pipeline wait (rb_gemm uses 1 s), for callers that run their
 * own watchdog and want the kernel to give up sooner, and for tests of the
 * error path.  The pages have no counterpart.  When a wait expires the
 * kernel stops issuing work, lets the copies
 * and MMAs it already issued finish, frees its tensor memory, raises
 * RB_DEV_TIMEOUT in *dev_status and returns; Y is then undefined, and the
 * stream and context stay usable.
 *   wait_limit_ns  0 .. 1e9.  0 waits not at all: any pipeline stage that is
 *                  not ready at its first probe ends the call with
 *                  RB_DEV_TIMEOUT (useful only to exercise the error path).
 *                  Larger values return RB_ERR_ARG.
 * Other arguments as rb_gemm.
 */
RB_API rb_status rb_gemm_wait_limit(const rb_layer_t *layer, const uint16_t *X, int M,
                                    void *Y, rb_dtype y_dtype, void *workspace, size_t workspace_bytes,
                                    int32_t *dev_status, unsigned flags, uint64_t wait_limit_ns,
                                    cudaStream_t stream);

/*
 * rb_gemm_noalloc -- rb_gemm for callers that must not allocate device memory.
 * The paper has no counterpart: this is a deployment convenience of the
 * library.  Some hosts give the library a fixed device-memory budget at
 * start-up and allow no further allocations (embedded or real-time
 * deployments, plugin hosts whose own allocator owns the GPU, code that must
 * not block on the allocator), so they cannot supply rb_gemm's workspace.
 * This call takes the same arguments minus the workspace and uses a fixed
 * 32 MiB array compiled into the library instead (every GPU that loads the
 * library holds it until the process exits).  It allocates nothing.
 *   - Sizes whose rb_gemm_workspace_bytes(N, K, k, M) exceeds 32 MiB (about
 *     M*K <= 16.7 million) return RB_ERR_WORKSPACE; other limits as for
 *     rb_gemm.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - All calls share the array.  Each call rewrites what it uses before
 *     reading it, so nothing carries over between calls, but calls that
 *     overlap on the GPU (two streams at once) race on it: serialise them.
 */
RB_API rb_status rb_gemm_noalloc(const rb_layer_t *layer, const uint16_t *X, int M,
                                 void *Y, rb_dtype y_dtype, int32_t *dev_status, unsigned flags,
                                 cudaStream_t stream);

/*
 * rb_transpose_planes -- sign planes of the transposed layer, for the
 * gradient that reaches the layer input in training (RaBiT, Algorithm 2
 * backward pass): dX = dY . What.  Since What^T = sum_i diag(h_i) B_i^T
 * diag(g_i), the K x N layer {n_out = K, k_in = N, k, planes_t, g16 = h16,
 * h16 = g16} (the same scale arrays, exchanged) is a packed layer whose
 * forward product is the input gradient: rb_gemv / rb_gemm on it with
 * X = dY ([M][N] bfloat16) give dX [M][K].
 *   layer     the forward layer (N x K); N must be a multiple of 32
 *             (RB_ERR_SHAPE otherwise), as it becomes the input width.
 *   planes_t  out, rb_packed_words(K, N, k) uint32 words in the storage
 *             layout of a K x N layer; every word is written.  It must not
 *             overlap layer->planes (RB_ERR_ARG).
 * The bits are exactly those rb_pack derives from (W^T, h, g): the
 * recurrence is element-wise and fl(g h) = fl(h g).
 */
RB_API rb_status rb_transpose_planes(const rb_layer_t *layer, uint32_t *planes_t, cudaStream_t stream);

/*
 * Binary-codebook layer (BTC-LLM, "Binary codebook" and "LUT-GEMM"): every
 * 16-column group (v = 16) of sign plane i is replaced by the index of a
 * 16-bit codebook pattern (bit q = column 16 j + q is +1), stored in
 * w = rb_btc_index_bits(c_max) = ceil(log2 c_max) bits: w / 16 bits per weight
 * (13 / 16 = 0.8125 at the page's c = 7132).
 *   codebooks  [k][c_max] uint16 patterns (entries past a plane's size unused).
 *   indices    [k][N][rb_btc_row_words(K, w)] uint32 streams: index j of row r
 *              at bits [j w, j w + w) of the row's words, LSB-first.
 *   g16, h16   as rb_layer_t.
 */
typedef struct {
    int32_t n_out;              /* N */
    int32_t k_in;               /* K (multiple of 32) */
    int32_t k_planes;           /* k, 1 or 2 for rb_btc_gemv */
    int32_t c_max;              /* codebook entries per plane, 1..65536 */
    int32_t index_bits;         /* rb_btc_index_bits(c_max) */
    int32_t reserved;           /* must be 0 */
    const uint16_t *codebooks;
    const uint32_t *indices;
    const uint16_t *g16;
    const uint16_t *h16;
} rb_btc_layer_t;

RB_API int rb_btc_index_bits(int c_max);                 /* 0 for c_max outside 1..65536 */
RB_API size_t rb_btc_row_words(int k_in, int index_bits);
RB_API size_t rb_btc_encode_workspace_bytes(int c_max);

/*
 * rb_btc_encode -- codebook and index stream of sign plane `plane` of a packed
 * layer by binary k-means (BTC-LLM, "Binary codebook": Hamming assignment by
 * XOR + popcount, majority-vote centroids with sign(0) = +1, codebook size
 * c = min(c_max, number of distinct patterns)).  The initial centroids are
 * the c most frequent patterns (count descending, then pattern ascending);
 * `iters` rounds of assignment (ties to the smaller index) and majority update
 * (a centroid without members is kept) precede the final assignment.
 *   codebook   [c_max] out (2-byte aligned); entries past c are 0.
 *   c_out      device int32 (4-byte aligned), nullable: c.
 *   indices    [N][rb_btc_row_words(K, w)] out (4-byte aligned),
 *              w = rb_btc_index_bits(c_max).
 *   workspace  rb_btc_encode_workspace_bytes(c_max) bytes, 16-byte aligned.
 * Integer arithmetic throughout: bit-exact and deterministic.  iters <= 1000;
 * N * K / 16 < 2^31.
 */
RB_API rb_status rb_btc_encode(const rb_layer_t *layer, int plane, int c_max, int iters, uint16_t *codebook,
                               int32_t *c_out, uint32_t *indices, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * rb_btc_gemv -- Y = sum_i g_i .* (Bhat_i (h_i .* x)) for one token (M = 1),
 * Bhat_i the codebook reconstruction of plane i (BTC-LLM, "LUT-GEMM": dot
 * products of the input blocks with the weight patterns are precomputed and
 * the weights only select them).  The tables are this library's byte tables
 * (sum of +-h x over 8 columns for all 256 sign bytes, fp32, exact products);
 * a codebook pattern's product is the sum of the entries of its two bytes.
 * One CTA per (256-row block, 256-column slice) writes row partials to the
 * workspace; a second launch adds them in slice order (deterministic).
 *   X [K] bfloat16 bits.  Y [N] fp32 or bf16.  k = 1 or 2 (else UNSUPPORTED).
 *   workspace  rb_btc_gemv_workspace_bytes(N, K) bytes.  dev_status: unused
 *   (nullable); flags: RB_LAUNCH_PDL.
 */
RB_API size_t rb_btc_gemv_workspace_bytes(int n_out, int k_in);
RB_API rb_status rb_btc_gemv(const rb_btc_layer_t *layer, const uint16_t *X, void *Y, rb_dtype y_dtype,
                             void *workspace, size_t workspace_bytes, int32_t *dev_status, unsigned flags,
                             cudaStream_t stream);

/*
 * rb_btc_gemv_batch -- rb_btc_gemv for `count` independent codebook layers of
 * one shape (same N, K, k, c_max), up to 64 per launch pair (more are cut into
 * groups of 64 that reuse the workspace in stream order).  layers[j], X[j],
 * Y[j] are host arrays of device pointers; each Y[j] equals rb_btc_gemv's
 * result for that layer bit for bit (the same per-slice partials, added in
 * the same order).
 *   workspace  rb_btc_gemv_batch_workspace_bytes(N, K, count) bytes.
 */
RB_API size_t rb_btc_gemv_batch_workspace_bytes(int n_out, int k_in, int count);
RB_API rb_status rb_btc_gemv_batch(const rb_btc_layer_t *const *layers, const uint16_t *const *X, void *const *Y,
                                   int count, rb_dtype y_dtype, void *workspace, size_t workspace_bytes,
                                   int32_t *dev_status, unsigned flags, cudaStream_t stream);

/*
 * rb_qat_forward -- forward pass of one coupled-training layer (RaBiT,
 * Algorithm 2 forward: the binary cores are derived from the latent weight
 * at every step): Y = X What^T with What = sum_i diag(g_i) B_i diag(h_i), the
 * B_i taken from W by the same fp32 recurrence as rb_pack and the trainable
 * fp32 scales used as they are.  The planes are derived once into the
 * workspace (one read of W), then the prefill GEMM runs on them with fp32 g
 * in its epilogue: no fp16 copy of g is made.
 *   W        [N][K] fp32 latent weight.   g, h  [k][N], [k][K] fp32.
 *   X        [M][K] bfloat16 bits.        Y     [M][N] fp32 or bf16.
 *   workspace  rb_qat_forward_workspace_bytes(N, K, k, M) bytes, 16-byte
 *              aligned: the derived planes (rb_packed_words(N, K, k) words in
 *              the storage layout, left there for the caller) followed by
 *              rb_gemm's workspace.
 * k = 1..8 with rb_gemm's limits on K (RB_ERR_UNSUPPORTED before any launch).
 * Precision: the MMA operands are +-fp16(h_i) (round to nearest even) and
 * fp16(x) with fp32 accumulation, g is applied in fp32, so |Y - exact| <=
 * 2^-11 sum |g h x| plus the accumulation error.  dev_status gets
 * RB_DEV_RANGE when an x or h overflows fp16, RB_DEV_NONFINITE for a NaN h or
 * a NaN / infinite W, RB_DEV_TIMEOUT as rb_gemm.
 */
RB_API size_t rb_qat_forward_workspace_bytes(int n_out, int k_in, int k_planes, int M);
RB_API rb_status rb_qat_forward(const float *W, const float *g, const float *h, int n_out, int k_in,
                                int k_planes, const uint16_t *X, int M, void *Y, rb_dtype y_dtype,
                                void *workspace, size_t workspace_bytes, int32_t *dev_status, unsigned flags,
                                cudaStream_t stream);

/*
 * rb_qat_backward -- gradients of one coupled-training layer (RaBiT,
 * Algorithm 2 backward pass: the signs derived on the fly from the latent
 * weight W are held constant, W takes the gradient of the effective weight,
 * the scales follow by the chain rule).  With G = dY^T X:
 *   dW[n][c] = G[n][c]
 *   dg_i[n]  = sum_c G[n][c] B_i[n][c] h_i[c]
 *   dh_i[c]  = sum_n G[n][c] g_i[n] B_i[n][c]
 * (the input gradient dX = dY What comes from rb_transpose_planes + rb_gemm).
 *   planes   the signs of W: rb_pack(W, g, h) output, storage layout above.
 *   g, h     [k][N], [k][K] fp32 trainable scales (the same ones rb_pack used).
 *   X, dY    [M][K], [M][N] bfloat16 bit patterns (layer input, output gradient).
 *   dW       out, [N][K] fp32: G, on the tcgen05 tensor cores (bf16 products are
 *            exact, accumulation in fp32 over the M tokens).
 *   dg, dh   out, [k][N], [k][K] fp32: one pass over G and the planes, partial
 *            sums added in a fixed order (deterministic).
 *   workspace  rb_qat_backward_workspace_bytes(N, K, k) bytes (partial sums).
 * N must be a multiple of 32 (RB_ERR_SHAPE otherwise): dY rows are read by TMA.
 * dev_status gets RB_DEV_TIMEOUT if a bounded pipeline wait expires.
 */
RB_API size_t rb_qat_backward_workspace_bytes(int n_out, int k_in, int k_planes);
RB_API rb_status rb_qat_backward(const uint32_t *planes, const float *g, const float *h,
                                 int n_out, int k_in, int k_planes,
                                 const uint16_t *X, const uint16_t *dY, int M,
                                 float *dW, float *dg, float *dh,
                                 void *workspace, size_t workspace_bytes,
                                 int32_t *dev_status, cudaStream_t stream);

/*
 * rb_svid_greedy -- greedy SVID scales for each plane (RaBiT names Greedy
 * SVID as the traditional initialiser): for i = 1..k, (g_i, h_i) is the
 * rank-1 approximation of |R_{i-1}| by `iters` rounds of power iteration in
 * float64 (v0 = 1/sqrt(K); u = A v/|A v|; v = A^T u/|A^T u|; sigma = u^T A v;
 * g_i = fp32(sqrt(sigma) u), h_i = fp32(sqrt(sigma) v)), with R_{i-1} from
 * the same fp32 recurrence as rb_pack.
 *   g, h out [k][N], [k][K] fp32.
 *   workspace: rb_svid_workspace_bytes(N, K) bytes.
 */
RB_API size_t rb_svid_workspace_bytes(int n_out, int k_in);
RB_API rb_status rb_svid_greedy(const float *W, int n_out, int k_in, int k_planes, int iters,
                         float *g, float *h, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * rb_svid_iterative -- iterative residual SVID (RaBiT, Algorithm 1 without
 * the I/O channel preprocessing): the greedy scales, then `sweeps`
 * Gauss-Seidel sweeps (the pages run 20).  Sweep t refits plane i = 1..k to
 * T_i = W - sum_{j != i} diag(g_j) B_j diag(h_j) with the latest scales and
 * signs of the other planes: B_i = sign(T_i) (sign(0) = +1) and (g_i, h_i) =
 * the rank-1 of |T_i| by the same float64 power iteration as rb_svid_greedy.
 * T_i is formed in float64 (each g_j[r] h_j[c] is exact there), planes in
 * order.  The signs are internal: rb_pack derives the deployed planes from W
 * and the returned scales by the residual recurrence.
 *   g, h out [k][N], [k][K] fp32 (also hold the state between sweeps).
 *   workspace: rb_svid_iterative_workspace_bytes(N, K, k) bytes (scratch of
 *   the power iteration and the k sign planes); no clearing needed.
 *   sweeps = 0 gives exactly rb_svid_greedy's scales.
 */
RB_API size_t rb_svid_iterative_workspace_bytes(int n_out, int k_in, int k_planes);
RB_API rb_status rb_svid_iterative(const float *W, int n_out, int k_in, int k_planes, int sweeps, int iters,
                                   float *g, float *h, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/*
 * rb_svid_pack -- the deployment path of a trained latent weight in one call,
 * on the device with no host round trip: scales by iterative residual SVID
 * (RaBiT, Algorithm 1 without the I/O preprocessing; `sweeps` = 0 gives the
 * greedy SVID), then the residual sign planes and fp16 scales by rb_pack
 * (Algorithm 2 forward; deployment freezes the planes).  The result equals
 * rb_svid_iterative followed by rb_pack on the same stream.
 *   g, h                out, [k][N], [k][K] fp32 scales (also returned).
 *   planes, g16, h16    out, as rb_pack.
 *   workspace           rb_svid_pack_workspace_bytes(N, K, k) bytes.
 * dev_status gets rb_pack's RB_DEV_* bits.
 */
RB_API size_t rb_svid_pack_workspace_bytes(int n_out, int k_in, int k_planes);
RB_API rb_status rb_svid_pack(const float *W, int n_out, int k_in, int k_planes, int sweeps, int iters,
                              float *g, float *h, uint32_t *planes, uint16_t *g16, uint16_t *h16,
                              void *workspace, size_t workspace_bytes, int32_t *dev_status,
                              cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* RBW_H_ */

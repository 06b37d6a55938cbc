/*
 * rot_b200.h -- C ABI of the B200 (sm_100a) rotation / group-quantisation / W4A4 library.
 *
 * The library implements the online hot path of rotation-based low-bit quantisation:
 * each activation row a = A[m,:] is mapped to y = T a by an orthonormal rotation T,
 * quantised in groups of G contiguous rotated coordinates with symmetric absmax
 * scales, packed, and fed to a W4A4 linear whose weights went through the same T
 * offline, so that A.B = (A.T^T)(T.B).
 *
 *   T = randomized Hadamard transform (RHT): random +-1 signs D, a fast Walsh-Hadamard
 *       transform of size K, scaled by 1/sqrt(K)            [Hadamard-Int4-Accuracy wiki,
 *       Hypothesis and Method (fwht_norm); HARP abstract and gist.science summary,
 *       section 1]; or
 *   T = HARP processor (P_{m-1} S_{m-1}) ... (P_0 S_0) D: a product of block-diagonal
 *       orthogonal stages over a mixed-radix schedule prod b_t = K, with optional
 *       permutations between stages                         [HARP gist.science summary,
 *       sections 2.1 and 2.2; HARP abstract].
 *
 * Conventions shared by every call:
 *   - Device pointers are caller-owned CUDA device memory on the device that is current
 *     when the call is made (for rot_plan_create: the device the plan lives on). The
 *     library never frees or keeps caller pointers.
 *   - Calls that take a stream are asynchronous on that stream (a cudaStream_t passed as
 *     void*, NULL = legacy default stream) and never synchronise; argument errors are
 *     detected on the host and returned before any launch.
 *   - The fused rotation kernels (rot_apply / rot_quant on RHT-type plans) and the linear
 *     kernels are launched with programmatic dependent launch: their prologue (barrier
 *     set-up, copying the plan's sign table, TMEM allocation, an L2 prefetch of the weight
 *     rows) may overlap the tail of the previous kernel in the stream, and every other
 *     global access waits for that kernel to complete (an L2 prefetch is safe: L2 is the
 *     device's point of coherence). Setting ROT_B200_PDL=0 in the environment launches them
 *     normally. Stream capture into CUDA graphs is supported (the dependency becomes a
 *     programmatic graph edge).
 *   - Device pointers must be 16-byte aligned; leading dimensions are in elements and
 *     lda * sizeof(element) must be a multiple of 16 bytes.
 *   - Layouts (row-major):
 *       activations  A      [M, lda]  bf16 or fp32
 *       codes        uint8  [M, K*bits/8]  int4: byte j = q[2j] | q[2j+1] << 4
 *                                          int2: byte j holds q[4j+i] in bits 2i..2i+1
 *                                          int8: byte j = q[j]
 *                           (two's complement, symmetric levels -qmax..qmax,
 *                            qmax = 2^(bits-1) - 1)
 *       scales       uint16 [M, K/G]  IEEE binary16 bit patterns, one per (row, group)
 *   - Quantisation [Hadamard-Int4-Accuracy wiki, Method: q_dequant_vec]: per group
 *       s = fp16_rn(fp32(max|y| / qmax)),  q = clamp(round_half_away(y / s), +-qmax),
 *       s == 0 (or not finite) gives q = 0.
 *   - On failure a call returns a non-zero rot_status and rot_last_error() (per host
 *     thread) holds a one-line message.
 */
#ifndef ROT_B200_H
#define ROT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct rot_plan_s* rot_plan_t;

typedef enum {
  ROT_OK = 0,
  ROT_EINVAL = 1,        /* invalid argument (shape, alignment, null pointer, bad plan) */
  ROT_EUNSUPPORTED = 2,  /* valid but outside what this build implements */
  ROT_ECUDA = 3,         /* a CUDA runtime call failed */
  ROT_ETIMEOUT = 4,      /* a bounded device-side wait gave up (reported by rot_check_device) */
  ROT_ENOMEM = 5         /* device allocation failed (plan creation only) */
} rot_status;

enum { ROT_F32 = 0, ROT_BF16 = 1 };

/* Build a rotation plan and copy its parameters to the current device.
 *
 * Defines T = (P_{m-1} S_{m-1}) ... (P_0 S_0) D [HARP gist.science summary, 2.1-2.2].
 *   K            dimension, K = prod radices[t]
 *   n_stages     m >= 1
 *   radices      host int[m], every b_t >= 2
 *   stage_params host array of m pointers; stage_params[t] is NULL (base mixer:
 *                H_b / sqrt(b) for a power-of-two b, the identity otherwise) or a host fp32
 *                array of n_blocks[t] * b * b row-major b x b orthogonal blocks
 *   n_blocks     host int64[m] (may be NULL when every stage_params[t] is NULL):
 *                1 (one block shared by the stage) or K / b_t (block c for coordinates
 *                base + r * s_t, s_t = prod_{u<t} b_u, c = low + high * s_t where low/high
 *                are the digits below/above t)
 *   perms        NULL or host array of m pointers; perms[t] NULL or a host int32[K]
 *                permutation applied after stage t as a gather x''[j] = x'[P_t[j]]
 *   signs        NULL (all +1) or host int8[K] with entries +1 / -1 (the D of the RHT)
 * The RHT of size K is radices = {2, ..., 2}, stage_params all NULL, signs = the random
 * signs. Host arrays are copied; the caller may free them after the call.
 * Errors: ROT_EINVAL (product != K, radix < 2, n_blocks not 1 or K/b, perms not a
 * permutation, signs not +-1), ROT_ENOMEM, ROT_ECUDA. */
rot_status rot_plan_create(rot_plan_t* out, int K, int n_stages, const int* radices,
                           const float* const* stage_params, const int64_t* n_blocks,
                           const int32_t* const* perms, const int8_t* signs);

/* Release a plan's device memory (synchronises the device). NULL is accepted. */
rot_status rot_plan_destroy(rot_plan_t plan);

/* Which kernel a plan uses: *chunk = 2^n > 0 when T acts as independent signed
 * Walsh-Hadamard transforms on contiguous chunks of 2^n coordinates (the fused
 * butterfly kernel), 0 when the generic stage kernel runs. *K receives the plan's K. */
rot_status rot_plan_info(rot_plan_t plan, int* K, int* chunk);

/* y = T a (inverse = 0) or y = T^T a (inverse = 1) for every row: fp32 output.
 * A: [M, lda] of a_dtype; Y: fp32 [M, ldy]. M may be 0. In-place (A == Y, fp32, lda == ldy)
 * is allowed. */
rot_status rot_apply(const void* A, int a_dtype, int64_t M, int64_t lda, rot_plan_t plan,
                     int inverse, float* Y, int64_t ldy, void* stream);

/* Fused rotate + quantise + pack, one HBM pass [HARP abstract; Hadamard-Int4-Accuracy
 * wiki, Method]: codes [M, K*bits/8], scales [M, K/G] (binary16 bits).
 * bits in {2, 4, 8}; G must divide K and be a multiple of 16 (int2), 8 (int4) or 4 (int8).
 * Errors: ROT_EINVAL for a bad G / bits / pointer / leading dimension. */
rot_status rot_quant(const void* A, int a_dtype, int64_t M, int64_t lda, rot_plan_t plan,
                     int bits, int G, uint8_t* codes, uint16_t* scales, void* stream);

/* Dequantise: x_hat = q * s (inverse = 0: in the rotated basis) or T^T (q * s)
 * (inverse = 1: back in the original basis). out: fp32 [M, K] dense. */
rot_status rot_dequant(const uint8_t* codes, const uint16_t* scales, int64_t M, rot_plan_t plan,
                       int bits, int G, int inverse, float* out, void* stream);

/* W4A4 linear [Hadamard-Int4-Accuracy wiki, Hypothesis: same-precision int4 MAC]:
 *   C[m, n] = sum_g float(As[m, g]) * float(Ws[n, g]) * P[m, n, g],
 *   P[m, n, g] = sum_{k in group g} qA[m, k] * qW[n, k]   (exact int32)
 * Aq: uint8 [M, K/2], As: binary16 [M, K/G] (rot_quant output, int4);
 * Wq: uint8 [N, K/2], Ws: binary16 [N, K/G] (rows of W^T through the same plan, int4);
 * C:  [M, N] fp32 (c_dtype = ROT_F32) or bf16 (ROT_BF16), row-major, ldc = N.
 * Requires K % G == 0, G % 32 == 0, K % 64 == 0, N % 16 == 0; M >= 0 arbitrary.
 * Decode-sized M (M <= 64 with G % 128 == 0) runs a weight-streaming kernel (mma.sync int8 per 8
 * weight rows; each CTA streams its rows into shared memory with bulk copies -- for M <= 16 also the
 * activation rows and the scale rows -- and sums its K-slices itself, so C is written directly). Other shapes run a persistent tcgen05 kernel over 128 x 128
 * output tiles, and shapes whose tiles leave most SMs idle split K into ranges aligned to
 * lcm(G, 128); their partial results are added with fp32 atomics: C is zeroed on the stream first
 * (fp32 output), or, for bf16 output, a stream-ordered temporary of M * N floats is allocated
 * (cudaMallocAsync), accumulated, converted into C and freed on the stream. The summation order then
 * varies between runs (fp32 rounding). The kernels wait for the previous kernel in the stream
 * (griddepcontrol.wait) before touching global memory. */
rot_status w4a4_linear(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq,
                       const uint16_t* Ws, int64_t M, int64_t N, int64_t K, int G, void* C,
                       int c_dtype, void* stream);

/* w4a4_linear without any device allocation: on the split-K path with bf16 output the
 * fp32 partial results accumulate in a static device buffer of 2^20 floats owned by the
 * library (located once per device with cudaGetSymbolAddress and zeroed on the stream
 * before each use) instead of a stream-ordered temporary. Same arguments, results and
 * constraints as w4a4_linear; ROT_EINVAL when that path is taken with M * N > 2^20.
 * Calls that take that path share the buffer: issue them on one stream (or otherwise
 * serialise them). */
rot_status w4a4_linear_noalloc(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq,
                               const uint16_t* Ws, int64_t M, int64_t N, int64_t K, int G, void* C,
                               int c_dtype, void* stream);

/* W4A4 linear with a two-sided processor [HARP abstract: a two-sided orthogonal processor;
 * HARP gist.science summary, sections 1 and 3]. With an input-side plan T (size K) and an
 * output-side plan U (size N), the weights are prepared offline as B~ = T B U^T (the rows of B,
 * length N, through U; then the columns through T; quantised as the rows of B~^T), so that
 * (A T^T) B~ = A B U^T: every output row comes out as c~ = U c. This call runs w4a4_linear on
 * (Aq, As) and (Wq, Ws) = the quantised rows of B~^T and then returns each row to c = U^T c~
 * with the rotation kernels (in place on fp32; for bf16 output on a stream-ordered fp32
 * temporary of M * N floats, converted afterwards).
 *   out_plan  the output-side plan U on the current device, out_plan K == N
 * Other arguments, layouts and constraints as for w4a4_linear. */
rot_status w4a4_linear_rot(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq, const uint16_t* Ws,
                           int64_t M, int64_t N, int64_t K, int G, rot_plan_t out_plan, void* C,
                           int c_dtype, void* stream);

/* The online path in one call: rot_quant of the activations (int4, group G) into a caller
 * workspace, then w4a4_linear against the prepared weights [Hadamard-Int4-Accuracy wiki,
 * Hypothesis: A.B = (A.Q)(Q.B) with both operands quantised; HARP gist.science summary 2.4: stage
 * kernels fused to keep the overhead low]. The linear is launched with programmatic dependent
 * launch: its set-up (barriers, tensor-memory allocation) overlaps the rotation's tail and it
 * reads the packed codes once the rotation has completed, while they are still in L2 at
 * prefill sizes (M * K / 2 bytes: 4 MB for A[2048, 4096]).
 *   A, a_dtype, M, lda, plan   as for rot_quant (plan K = the linear's K)
 *   Wq, Ws, N, G, C, c_dtype   as for w4a4_linear
 *   workspace                  caller-owned device memory, 16-byte aligned, of at least
 *                              w4a4_linear_act_workspace(M, K, G) bytes: the packed codes
 *                              [M, K/2] then (16-byte aligned) the scales [M, K/G]; they keep
 *                              the rotated codes after the call.
 * Errors: as rot_quant and w4a4_linear; ROT_EINVAL for a missing or short workspace. */
rot_status w4a4_linear_act_workspace(int64_t M, int64_t K, int G, size_t* bytes);
rot_status w4a4_linear_act(const void* A, int a_dtype, int64_t M, int64_t lda, rot_plan_t plan,
                           const uint8_t* Wq, const uint16_t* Ws, int64_t N, int G, void* C, int c_dtype,
                           void* workspace, size_t workspace_bytes, void* stream);

/* W4A8 linear: int8 activations, int4 weights [Hadamard-Int4-Accuracy wiki, Method
 * (matmul_q_err with abits = 8, bbits = 4) and Results ("W4A8 (act8/wt4)", a diagnostic that
 * isolates which operand's int4 hurts); fact 3: int8 activations absorb the outliers]:
 *   C[m, n] = sum_g float(As[m, g]) * float(Ws[n, g]) * P[m, n, g],
 *   P[m, n, g] = sum_{k in group g} qA[m, k] * qW[n, k]   (exact int32)
 * Aq: int8 [M, K] (rot_quant with bits = 8: one two's-complement code per byte, natural order),
 * As: binary16 [M, K/G]; Wq, Ws, C and every constraint as for w4a4_linear. The same kernels run
 * with the int8 activation tile loaded as is (tcgen05 kind::i8; mma.sync s8 for decode-sized M)
 * and only the weights unpacked. */
rot_status w4a8_linear(const int8_t* Aq, const uint16_t* As, const uint8_t* Wq, const uint16_t* Ws,
                       int64_t M, int64_t N, int64_t K, int G, void* C, int c_dtype, void* stream);

/* The exact int32 group partial sums P[m, n, g] of the W4A8 contraction (int8 Aq [M, K]),
 * written to P: int32 [M, N, K/G]. For checking only. */
rot_status w4a8_group_partials(const int8_t* Aq, const uint8_t* Wq, int64_t M, int64_t N, int64_t K,
                               int G, int32_t* P, void* stream);

/* Host only (no device work): the work list the tcgen05 tile kernel of w4a4_linear uses for a
 * shape (M > 64 or G % 128 != 0), given the device's SM count. out: int64 [6] =
 * {tiles_m, tiles_n, splits, kb_per_split, units, grid}: 128 x 128 output tiles; K split into
 * `splits` ranges of kb_per_split K-blocks of 128 (a multiple of lcm(G, 128) / 128, so every range
 * starts and ends on a K-block and a group boundary; none is empty) when the tiles alone leave
 * more than half of the SMs idle and partials == 0; units = tiles * splits; grid = min(units,
 * sms) persistent CTAs. ROT_EINVAL for the shapes w4a4_linear rejects, M <= 0 or sms <= 0. */
rot_status w4a4_tile_plan(int64_t M, int64_t N, int64_t K, int G, int sms, int partials, int64_t* out);

/* The exact int32 group partial sums P[m, n, g] of the same contraction, written to
 * P: int32 [M, N, K/G]. Same constraints as w4a4_linear. For checking only. */
rot_status w4a4_group_partials(const uint8_t* Aq, const uint8_t* Wq, int64_t M, int64_t N,
                               int64_t K, int G, int32_t* P, void* stream);

/* Host helpers building HARP stage blocks from their parameters
 * [HARP gist.science summary, 2.2: B = Q(theta) G_b]:
 *   rot_harp_givens_blocks: out[i] = R(theta_i) . H_2 / sqrt(2) (fp32 2x2 row-major),
 *     R(t) = [[cos t, -sin t], [sin t, cos t]]; out holds n * 4 floats.
 *   rot_harp_qr_block: the Q factor (diag(R) > 0) of the b x b row-major matrix g
 *     (Householder QR in double), out holds b * b floats. */
rot_status rot_harp_givens_blocks(const double* theta, int64_t n, float* out);
rot_status rot_harp_qr_block(const double* g, int b, float* out);

/* rot_harp_cayley_block: B = Q(theta) G for one b x b block (b >= 2), Q(theta) = (I + S)^{-1}
 *   (I - S) the Cayley map of the skew-symmetric S whose strictly upper entries are params
 *   (b(b-1)/2 doubles, row-major order: S[i][j] = params[k] for i < j, S[j][i] = -params[k]),
 *   G = mixer (b x b row-major fp32) or, when mixer is NULL, the base mixer (H_b / sqrt(b) for a
 *   power of two, else the identity). Q(0) = I, so B(0) = G [HARP gist.science summary, 2.2:
 *   Cayley map for b_t > 2]. out: b * b floats. Host only, double precision. */
rot_status rot_harp_cayley_block(const double* params, int b, const float* mixer, float* out);

/* Build a plan from HARP parameters stored in int8 [HARP gist.science summary, 2.4 (storage in
 * int8) and 4 (2.00 -> 2.05 bits per parameter)]: stage t's parameters are
 * theta = codes[t][i] * scales[t] (one fp32 scale per stage).
 *   codes[t]   NULL (theta = 0: the block is the stage's mixer) or host int8:
 *              b_t == 2: n_blocks[t] Givens angles, B = R(theta) H_2 / sqrt(2);
 *              b_t >  2: n_blocks[t] * b(b-1)/2 Cayley parameters per block (rot_harp_cayley_block
 *              order), B = Q(theta) G_b
 *   scales     host fp32[n_stages] (read for stages with codes)
 *   n_blocks   host int64[n_stages]: 1 or K / b_t for stages with codes
 *   mixers     NULL or host array of n_stages pointers: NULL (base mixer) or a b x b fp32 G_b
 *              (e.g. the QR fallback, rot_harp_qr_block); radix-2 stages take none
 *   perms, signs as for rot_plan_create.
 * The Givens blocks are computed on the device from the int8 codes when the plan is loaded
 * (sincosf in fp32); Cayley blocks are built on the host in double. The kernels then read the
 * expanded fp32 blocks, so rot_apply / rot_quant cost the same as with an fp32 plan.
 * Errors: as rot_plan_create; ROT_EINVAL for a missing scale / n_blocks or a radix-2 mixer. */
rot_status rot_plan_create_q8(rot_plan_t* out, int K, int n_stages, const int* radices,
                              const int8_t* const* codes, const float* scales, const int64_t* n_blocks,
                              const float* const* mixers, const int32_t* const* perms, const int8_t* signs);

/* Synchronise the current device and report device-side errors recorded by bounded
 * waits (ROT_ETIMEOUT) since the last call; clears the record. */
rot_status rot_check_device(void);

/* Testing hook for the bounded-wait failure path (the pages have no counterpart). Every
 * device-side wait of the fused rotation kernels (staging copies) and of the W4A4 tile kernel
 * (its mbarrier pipeline) gives up after a bound of wall time, records ROT_ETIMEOUT for
 * rot_check_device and returns without leaving a copy or an MMA in flight. This call makes
 * that happen on purpose, so tests can check the path without faulting the GPU:
 *   fault = 0  no fault (only sets the bound)
 *   fault = 1  ROT_TEST_ROTATION_COPY: the next rot_quant / rot_apply launch of the fused
 *              rotation kernel does not issue the first staging copy of CTA 0's first slot;
 *              that slot's waits run out, every other slot completes normally (the few-row
 *              kernel for 4096-coordinate chunks -- at most 512 chunks, bf16 in, quantised
 *              out -- stages nothing and waits on nothing: the fault is consumed and has no
 *              effect there)
 *   fault = 2  ROT_TEST_W4A4_LOADS: the next launch of the W4A4 tile kernel (M > 64 or
 *              G % 128 != 0) issues no TMA load; every role's waits run out
 * The fault is one-shot (consumed by the next launch of that kernel family on any thread).
 * wait_ns > 0 sets the bound of those waits (default: 1 s rotation, 2 s W4A4) until the
 * next call; 0 restores the defaults. Outputs of a launch that gave up are unspecified.
 * ROT_EINVAL for an unknown fault or wait_ns < 0. Host only. */
enum { ROT_TEST_NONE = 0, ROT_TEST_ROTATION_COPY = 1, ROT_TEST_W4A4_LOADS = 2 };
rot_status rot_test_inject(int fault, int64_t wait_ns);

/* Last error message of the calling host thread ("" if none). */
const char* rot_last_error(void);

/* Library version string. */
const char* rot_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ROT_B200_H */

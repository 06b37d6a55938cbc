// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <string>
#include <vector>

#include "rot_b200.h"

namespace rotb {

// ---------------------------------------------------------------- errors (host)
rot_status set_error(rot_status st, const std::string& msg);
rot_status cuda_error(cudaError_t e, const char* what);
#define ROT_CUDA_TRY(expr)                                   \
  do {                                                       \
    cudaError_t _e = (expr);                                 \
    if (_e != cudaSuccess) return ::rotb::cuda_error(_e, #expr); \
  } while (0)

int sm_count();  // SMs of the current device (cached per device)

// Testing hook (rot_test_inject): a one-shot fault for the next launch of one kernel family
// and an optional bound for the kernels' device-side waits.
enum { TEST_FAULT_NONE = 0, TEST_FAULT_ROTATION_COPY = 1, TEST_FAULT_W4A4_LOADS = 2 };
bool take_test_fault(int which);                        // true once after rot_test_inject(which, .)
unsigned long long wait_limit_ns(unsigned long long dflt);  // the injected bound, else dflt

// ---------------------------------------------------------------- plan
struct Stage {
  int b = 0;            // radix
  int stride = 1;       // s_t = prod_{u<t} b_u
  int64_t n_blocks = 0; // 1 or K/b (0 when the stage is the identity and skipped)
  bool identity = false;
  bool hadamard = false;  // blocks equal H_b / sqrt(b) (power-of-two b)
  float* d_blocks = nullptr;   // [n_blocks, b, b] fp32 row-major (base mixer materialised)
  float* d_blocks_pad = nullptr;  // per-block stages of radix 3..48: [n_blocks, b, bp] rows padded
                                  // to bp = a multiple of 4 floats (zeros), for 16-byte loads
  int32_t* d_perm = nullptr;   // gather after the stage, or nullptr
  int32_t* d_iperm = nullptr;  // inverse permutation (for T^T)
};

}  // namespace rotb

struct rot_plan_s {
  int K = 0;
  int device = 0;
  bool has_signs = false;
  // fused butterfly path: T = blockdiag over K/chunk chunks of H_chunk D_c / sqrt(chunk)
  int chunk_log2 = -1;          // >= 0 when the fused path applies, else -1
  uint32_t* d_signmask = nullptr;  // K/2 words: bit 15 = sign of coord 2p, bit 31 = of 2p+1
  float* d_signf = nullptr;        // K entries +-1.0f (generic stage kernel)
  std::vector<rotb::Stage> stages;  // generic path (always built)
  int max_radix = 0;
};

namespace rotb {

// ---------------------------------------------------------------- launchers
// fused butterfly path (rot_fwht.cu)
rot_status fwht_apply(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda,
                      int inverse, float* Y, int64_t ldy, cudaStream_t s);
rot_status fwht_quant(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda,
                      int bits, int G, uint8_t* codes, uint16_t* scales, cudaStream_t s);
bool fwht_quant_supported(const rot_plan_s* p, int bits, int G);
rot_status fwht_fetch_device_error();
// generic stage path (rot_stages.cu)
rot_status stages_apply(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda,
                        int inverse, float* Y, int64_t ldy, cudaStream_t s);
rot_status stages_quant(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda,
                        int bits, int G, uint8_t* codes, uint16_t* scales, cudaStream_t s);
// dequantisation (rot_dequant.cu)
rot_status dequant_launch(const uint8_t* codes, const uint16_t* scales, int64_t M, int K, int bits,
                          int G, float* out, cudaStream_t s);
// W4A4 / W4A8 linear (w4a4_linear.cu); a8: Aq holds int8 codes [M, K] instead of packed int4
// split-K accumulation: `scratch` (scratch_floats floats) if non-null, else a stream-ordered
// temporary; only used for bf16 output on the split path
constexpr int64_t W4A4_NOALLOC_SCRATCH_FLOATS = int64_t(1) << 20;
// Programmatic dependent launch for the library's kernels (a kernel's prologue may overlap the
// previous kernel in the stream; every kernel orders its global accesses after griddepcontrol.wait,
// L2 prefetches of constant operands aside); ROT_B200_PDL=0 in the environment turns it off.
bool pdl_default();

rot_status w4a4_launch(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq,
                       const uint16_t* Ws, int64_t M, int64_t N, int64_t K, int G, void* C,
                       int c_dtype, int32_t* partials, cudaStream_t s, float* scratch = nullptr,
                       int64_t scratch_floats = 0, bool a8 = false, bool pdl = false);
rot_status w4a4_noalloc_scratch(float** out);
rot_status f32_to_bf16_launch(const float* src, void* dst, int64_t n, cudaStream_t s);
struct W4A4TilePlan {
  int64_t tiles_m, tiles_n, units, grid;
  int splits, kb_per_split;
};
rot_status w4a4_tile_plan_compute(int64_t M, int64_t N, int64_t K, int G, int sms, bool partials,
                                  W4A4TilePlan* out);

// ---------------------------------------------------------------- device helpers
#ifdef __CUDACC__
// (a, b) <- (a + b, a - b) on two register pairs with packed fp32x2 adds
__device__ __forceinline__ void bfly_x2(float& a0, float& a1, float& b0, float& b1) {
  unsigned long long A, B, S, D;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(S) : "l"(A), "l"(B));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(S));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(D));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// byte permute
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Scale / code-factor of one quantisation group.
//   m_z   : max |z| over the group, z the un-normalised rotated values (y = z * norm)
//   c_div : fp32(norm / qmax);  c_f : fp32(norm * (1 + 2^-22))
// Returns the binary16 scale bits, s = binary16(m_z * c_div): the quotient absmax / qmax
// within an fp32 ulp or two of the correctly rounded one, so s differs from the rounding
// of the exact quotient only for quotients within ~1e-7 relative of a binary16 midpoint.
// *f receives the factor with v = z * f ~= y / s (approximate reciprocal, within about
// 2 ulp), nudged up by 2^-22 relative so that exact ties of z * f round away from zero;
// *slow is set when the scale is zero, subnormal or not finite (codes need clamping then).
__device__ __forceinline__ uint16_t group_scale(float m_z, float c_div, float c_f, float* f,
                                                bool* slow) {
  const __half s16 = __float2half_rn(m_z * c_div);
  const uint32_t hb = __half_as_ushort(s16);
  const float s = __half2float(s16);
  // normal finite binary16 <=> magnitude bits in [0x0400, 0x7bff]
  *slow = ((hb & 0x7fffu) - 0x0400u) >= 0x7800u;
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  *f = (s > 0.0f && s <= 65504.0f) ? r * c_f : 0.0f;
  return (uint16_t)hb;
}

// Per bit width: qmax = 2^(bits-1) - 1, the rounding constant 2^23 + qmax + 1 (its low bits
// hold the offset code qmax + 1 + q after an fma), and the XOR that turns packed offset codes
// (qmax + 1 + q, the high bit of each field set for q >= 0) into two's complement fields.
__host__ __device__ constexpr float qmax_of_bits(int bits) { return bits == 8 ? 127.0f : bits == 4 ? 7.0f : 1.0f; }
__host__ __device__ constexpr float magic_of_bits(int bits) {
  return bits == 8 ? 8388736.0f : bits == 4 ? 8388616.0f : 8388610.0f;
}
__host__ __device__ constexpr uint32_t offset_xor_of_bits(int bits) {
  return bits == 8 ? 0x80808080u : bits == 4 ? 0x88888888u : 0xAAAAAAAAu;
}

// Offset code u = qmax + 1 + rne(v) in the low bits of the result (magic-number rounding);
// with clamping for the slow path. v = z * f.
__device__ __forceinline__ uint32_t code_magic(float z, float f, float magic) {
  return __float_as_uint(__fmaf_rn(z, f, magic));
}
__device__ __forceinline__ uint32_t code_magic_clamped(float z, float f, float qmax, float magic) {
  float v = fminf(fmaxf(__fmul_rn(z, f), -qmax), qmax);
  return __float_as_uint(__fadd_rn(v, magic));
}
#endif

}  // namespace rotb

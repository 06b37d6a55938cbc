// Generic HARP stage kernel: any mixed-radix schedule, shared or per-block orthogonal
// blocks, permutations between stages [HARP gist.science summary, 2.1: block-diagonal
// orthogonal stages B_t on coordinate groups separated by stride permutations; mixed-radix
// schedules with prod b_t = d; HARP abstract].
//
// One CTA owns one row at a time; the row lives in shared memory (fp32, two buffers).
//   load:   x = D a (signs), coalesced;
//   stage:  x'[base + r s_t] = sum_r' B_{t,c}[r][r'] x[base + r' s_t]; radix-2 stages use
//           one thread per 2x2 block, larger radices one thread per output coordinate;
//           blocks come from global memory (L1/L2 resident across rows);
//   gather: x''[j] = x'[P_t[j]];
//   then either store y (fp32) or quantise groups of G coordinates (one warp per group).
// The inverse T^T runs the stages in reverse order with transposed blocks and inverse
// permutations, and applies the signs last.
#include "rot_internal.cuh"

namespace rotb {
namespace {

struct StageDev {
  const float* blocks;
  const int32_t* perm;   // gather applied after the stage (forward) / before (inverse: iperm)
  int b;
  int stride;
  int per_block;         // 1: block c, 0: one shared block
  int identity;
};

constexpr int MAX_STAGES = 32;

struct Args {
  const void* A;
  int a_bf16;
  int64_t lda;
  int64_t M;
  int K;
  const float* signs;    // K entries +-1
  int n_stages;
  int inverse;
  StageDev st[MAX_STAGES];
  float* Y;
  int64_t ldy;
  uint8_t* codes;
  uint16_t* scales;
  int G;
  int bits;              // 0: apply (fp32 out)
};

constexpr int THREADS = 512;

__device__ __forceinline__ void run_stage(const StageDev& s, const float* in, float* out, int K,
                                          bool transpose) {
  const int b = s.b, st = s.stride;
  if (b == 2) {
    for (int c = threadIdx.x; c < K / 2; c += THREADS) {
      // block c: low = c % st, high = c / st; base = low + high * 2 * st
      const int low = c % st, high = c / st;
      const int base = low + high * 2 * st;
      const float* B = s.blocks + (s.per_block ? 4 * c : 0);
      const float x0 = in[base], x1 = in[base + st];
      float b00 = B[0], b01 = B[1], b10 = B[2], b11 = B[3];
      if (transpose) { const float tmp = b01; b01 = b10; b10 = tmp; }
      out[base] = fmaf(b00, x0, b01 * x1);
      out[base + st] = fmaf(b10, x0, b11 * x1);
    }
  } else {
    for (int e = threadIdx.x; e < K; e += THREADS) {
      const int r = (e / st) % b;
      const int base = e - r * st;
      const int low = base % st, high = base / (st * b);
      const int c = low + high * st;
      const float* B = s.blocks + (s.per_block ? (int64_t)c * b * b : 0);
      float acc = 0.0f;
      if (!transpose) {
        for (int k = 0; k < b; ++k) acc = fmaf(B[r * b + k], in[base + k * st], acc);
      } else {
        for (int k = 0; k < b; ++k) acc = fmaf(B[k * b + r], in[base + k * st], acc);
      }
      out[e] = acc;
    }
  }
}

__global__ void __launch_bounds__(THREADS) stages_kernel(const Args a) {
  extern __shared__ __align__(16) float smem[];
  float* buf0 = smem;
  float* buf1 = smem + a.K;
  const int K = a.K;
  for (int64_t row = blockIdx.x; row < a.M; row += gridDim.x) {
    float* cur = buf0;
    float* nxt = buf1;
    // load (+ signs in the forward direction)
    if (a.a_bf16) {
      const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(a.A) + row * a.lda;
      for (int i = threadIdx.x; i < K; i += THREADS) {
        const float v = __bfloat162float(src[i]);
        cur[i] = a.inverse ? v : v * a.signs[i];
      }
    } else {
      const float* src = static_cast<const float*>(a.A) + row * a.lda;
      for (int i = threadIdx.x; i < K; i += THREADS) cur[i] = a.inverse ? src[i] : src[i] * a.signs[i];
    }
    __syncthreads();
    for (int q = 0; q < a.n_stages; ++q) {
      const int t = a.inverse ? a.n_stages - 1 - q : q;
      const StageDev& s = a.st[t];
      if (a.inverse && s.perm) {  // inverse of the gather: x[j] = x'[iperm[j]]
        for (int i = threadIdx.x; i < K; i += THREADS) nxt[i] = cur[s.perm[i]];
        __syncthreads();
        float* tmp = cur; cur = nxt; nxt = tmp;
      }
      if (!s.identity) {
        run_stage(s, cur, nxt, K, a.inverse != 0);
        __syncthreads();
        float* tmp = cur; cur = nxt; nxt = tmp;
      }
      if (!a.inverse && s.perm) {
        for (int i = threadIdx.x; i < K; i += THREADS) nxt[i] = cur[s.perm[i]];
        __syncthreads();
        float* tmp = cur; cur = nxt; nxt = tmp;
      }
    }
    if (a.inverse) {
      for (int i = threadIdx.x; i < K; i += THREADS) cur[i] *= a.signs[i];
      __syncthreads();
    }
    if (a.bits == 0) {
      float* dst = a.Y + row * a.ldy;
      for (int i = threadIdx.x; i < K; i += THREADS) dst[i] = cur[i];
    } else {
      // one warp per group: absmax by warp reduction, then one lane per 32-bit code word
      const float qmax = a.bits == 4 ? 7.0f : 1.0f;
      const float magic = a.bits == 4 ? 8388616.0f : 8388610.0f;
      const int cpw = 32 / a.bits;
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
      const int ngr = K / a.G;
      for (int g = warp; g < ngr; g += THREADS / 32) {
        const float* gx = cur + (int64_t)g * a.G;
        float m = 0.0f;
        for (int i = lane; i < a.G; i += 32) m = fmaxf(m, fabsf(gx[i]));
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float f;
        bool slow;
        const uint16_t s16 = group_scale(m, a.bits == 4 ? 1.0f / 7.0f : 1.0f, 1.0f + 0x1p-22f, &f, &slow);
        if (lane == 0) a.scales[row * ngr + g] = s16;
        uint32_t* cw = reinterpret_cast<uint32_t*>(a.codes + row * (int64_t)(K / cpw) * 4) +
                       (int64_t)g * a.G / cpw;
        for (int w = lane; w < a.G / cpw; w += 32) {
          uint32_t word = 0;
          for (int j = 0; j < cpw; ++j) {
            const uint32_t u = slow ? code_magic_clamped(gx[w * cpw + j], f, qmax, magic)
                                    : code_magic(gx[w * cpw + j], f, magic);
            word |= (u & ((1u << a.bits) - 1u)) << (a.bits * j);
          }
          cw[w] = word ^ (a.bits == 4 ? 0x88888888u : 0xAAAAAAAAu);
        }
      }
    }
    __syncthreads();
  }
}

rot_status launch(const rot_plan_s* p, Args& a, cudaStream_t s) {
  if ((int)p->stages.size() > MAX_STAGES) return set_error(ROT_EUNSUPPORTED, "generic rotation: too many stages");
  const size_t smem = (size_t)2 * p->K * sizeof(float);
  if (smem > 227 * 1024) return set_error(ROT_EUNSUPPORTED, "generic rotation: K too large for shared memory");
  a.K = p->K;
  a.signs = p->d_signf;
  a.n_stages = (int)p->stages.size();
  for (int t = 0; t < a.n_stages; ++t) {
    const Stage& S = p->stages[t];
    a.st[t].blocks = S.d_blocks;
    a.st[t].perm = a.inverse ? S.d_iperm : S.d_perm;
    a.st[t].b = S.b;
    a.st[t].stride = S.stride;
    a.st[t].per_block = S.n_blocks > 1;
    a.st[t].identity = S.identity;
  }
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    ROT_CUDA_TRY(cudaFuncSetAttribute(stages_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
    configured[dev] = 1;
  }
  if (a.M == 0) return ROT_OK;
  const int per_sm = smem <= 110 * 1024 ? 2 : 1;
  int64_t grid = std::min<int64_t>(a.M, (int64_t)sm_count() * per_sm);
  stages_kernel<<<(unsigned)grid, THREADS, smem, s>>>(a);
  ROT_CUDA_TRY(cudaGetLastError());
  return ROT_OK;
}

}  // namespace

rot_status stages_apply(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda,
                        int inverse, float* Y, int64_t ldy, cudaStream_t s) {
  Args a{};
  a.A = A;
  a.a_bf16 = a_dtype == ROT_BF16;
  a.lda = lda;
  a.M = M;
  a.inverse = inverse;
  a.Y = Y;
  a.ldy = ldy;
  a.bits = 0;
  return launch(p, a, s);
}

rot_status stages_quant(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda,
                        int bits, int G, uint8_t* codes, uint16_t* scales, cudaStream_t s) {
  Args a{};
  a.A = A;
  a.a_bf16 = a_dtype == ROT_BF16;
  a.lda = lda;
  a.M = M;
  a.inverse = 0;
  a.codes = codes;
  a.scales = scales;
  a.G = G;
  a.bits = bits;
  return launch(p, a, s);
}

}  // namespace rotb

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
#include <cstdlib>

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
      const float qmax = qmax_of_bits(a.bits);
      const float magic = magic_of_bits(a.bits);
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
        const uint16_t s16 = group_scale(m, 1.0f / qmax, 1.0f + 0x1p-22f, &f, &slow);
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
          cw[w] = word ^ offset_xor_of_bits(a.bits);
        }
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- multi-row forward kernel
// Forward rotation (+ quantisation) of ROWS rows at a time per CTA, so that every stage
// parameter read from L2 serves ROWS rows. Stages:
//   radix 2:  in place, one thread per 2 x 2 block (per-block or shared parameters);
//   radix b:  (3 <= b <= MR_MAXB) each work item holds the b inputs of one block in registers
//             and produces a range of outputs, written back in place after a barrier; a shared
//             block is kept in shared memory (read as broadcasts), per-block blocks are read
//             from a copy with rows padded to a multiple of 4 floats (16-byte loads, L2/L1);
//   gather:   x''[j] = x'[P[j]] into the second buffer.
// The block index c = low + high * s of coordinate base = low + high * b * s uses a
// multiply-high division by s (exact for c < 2^16).
constexpr int MR_ROWS = 2;
constexpr int MR_THREADS = 512;
constexpr int MR_MAXB = 48;
constexpr int MR_UB = 12;          // 2 x 2 blocks per thread per batch (K/2 <= 6144: one batch)
constexpr int MR_UG = 24;          // gather indices per thread per batch (K <= 12288: one batch)

struct MrStage {
  const float* blocks;   // radix 2: [n_blocks][4]; radix b: [b][b] (shared) or [n_blocks][b][bp] (padded)
  const int32_t* perm;   // gather after the stage or nullptr
  const int32_t* iperm;  // its inverse: a non-identity stage scatters output j to iperm[j]
  int b, stride;
  uint32_t magic;        // ceil(2^32 / stride) for stride >= 2 (stride 1 divides trivially)
  int per_block, identity;
  int sh_off;            // radix b > 2, shared block: its offset (floats) in the shared-memory block area
};

struct MrArgs {
  const void* A;
  int a_bf16;
  int64_t lda, M;
  int K;
  const float* signs;
  int n_stages;
  MrStage st[MAX_STAGES];
  int sh_floats;         // shared-memory block area (floats): the shared dense blocks, rows padded
  float* Y;
  int64_t ldy;
  uint8_t* codes;
  uint16_t* scales;
  int G, bits;
};

// PB: the plan has per-block dense stages (a separate instance, so that plans without them run
// the shared-block code alone)
template <bool PB>
__global__ void __launch_bounds__(MR_THREADS, 1) stages_rows_kernel(const MrArgs a) {
  extern __shared__ __align__(16) float smem[];
  const int K = a.K;
  float* bufA = smem;                          // [MR_ROWS][K]
  float* bufB = smem + MR_ROWS * K;            // [MR_ROWS][K]
  float* sblk = smem + 2 * MR_ROWS * K;        // shared dense blocks, rows padded to a multiple of 4
  for (int t = 0; t < a.n_stages; ++t) {
    const MrStage& S = a.st[t];
    if (S.identity || S.b == 2 || S.per_block) continue;
    const int b = S.b, bp = (b + 3) & ~3;
    for (int i = threadIdx.x; i < b * bp; i += MR_THREADS) {
      const int r = i / bp, k = i - r * bp;
      sblk[S.sh_off + i] = k < b ? S.blocks[r * b + k] : 0.0f;
    }
  }

  for (int64_t row0 = (int64_t)blockIdx.x * MR_ROWS; row0 < a.M; row0 += (int64_t)gridDim.x * MR_ROWS) {
    const int nr = (int)(a.M - row0 < MR_ROWS ? a.M - row0 : MR_ROWS);
    float* cur = bufA;
    float* nxt = bufB;
    for (int r = 0; r < MR_ROWS; ++r) {
      const int64_t row = row0 + (r < nr ? r : 0);
      if (a.a_bf16) {
        const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(a.A) + row * a.lda;
        if ((K & 7) == 0 && (a.lda & 7) == 0 && (reinterpret_cast<uintptr_t>(a.A) & 15) == 0) {
          for (int i = 8 * threadIdx.x; i < K; i += 8 * MR_THREADS) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + i);
            const float4 s0 = *reinterpret_cast<const float4*>(a.signs + i);
            const float4 s1 = *reinterpret_cast<const float4*>(a.signs + i + 4);
            float* d = cur + r * K + i;
            d[0] = __uint_as_float(v.x << 16) * s0.x; d[1] = __uint_as_float(v.x & 0xffff0000u) * s0.y;
            d[2] = __uint_as_float(v.y << 16) * s0.z; d[3] = __uint_as_float(v.y & 0xffff0000u) * s0.w;
            d[4] = __uint_as_float(v.z << 16) * s1.x; d[5] = __uint_as_float(v.z & 0xffff0000u) * s1.y;
            d[6] = __uint_as_float(v.w << 16) * s1.z; d[7] = __uint_as_float(v.w & 0xffff0000u) * s1.w;
          }
        } else {
          for (int i = threadIdx.x; i < K; i += MR_THREADS) cur[r * K + i] = __bfloat162float(src[i]) * a.signs[i];
        }
      } else {
        const float* src = static_cast<const float*>(a.A) + row * a.lda;
        for (int i = threadIdx.x; i < K; i += MR_THREADS) cur[r * K + i] = src[i] * a.signs[i];
      }
    }
    __syncthreads();
    for (int t = 0; t < a.n_stages; ++t) {
      const MrStage& S = a.st[t];
      if (!S.identity) {
        const int st = S.stride;
        // a stage followed by a permutation writes its outputs straight to their permuted places
        // in the other buffer (x''[P^-1[j]] = x'[j]): no separate gather pass
        const bool scat = S.perm != nullptr;
        float* dst = scat ? nxt : cur;
        if (S.b == 2) {
          // MR_UB blocks per thread per batch: their parameter (and scatter index) loads from L2
          // are all in flight before the first is used
          for (int c0 = threadIdx.x; c0 < K / 2; c0 += MR_THREADS * MR_UB) {
            float4 B[MR_UB];
            int base[MR_UB], o0[MR_UB], o1[MR_UB];
#pragma unroll
            for (int u = 0; u < MR_UB; ++u) {
              const int c = c0 + u * MR_THREADS;
              const bool on = c < K / 2;
              const int high = st == 1 ? c : (int)__umulhi((uint32_t)c, S.magic);
              base[u] = (c - high * st) + high * 2 * st;
              B[u] = on ? __ldg(reinterpret_cast<const float4*>(S.blocks + (S.per_block ? 4 * c : 0)))
                        : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              o0[u] = scat && on ? __ldg(S.iperm + base[u]) : base[u];
              o1[u] = scat && on ? __ldg(S.iperm + base[u] + st) : base[u] + st;
            }
#pragma unroll
            for (int u = 0; u < MR_UB; ++u) {
              if (c0 + u * MR_THREADS < K / 2) {
#pragma unroll
                for (int r = 0; r < MR_ROWS; ++r) {
                  const float x0 = cur[r * K + base[u]], x1 = cur[r * K + base[u] + st];
                  dst[r * K + o0[u]] = fmaf(B[u].x, x0, B[u].y * x1);
                  dst[r * K + o1[u]] = fmaf(B[u].z, x0, B[u].w * x1);
                }
              }
            }
          }
        } else {
          // dense radix-b stage: work item (block c, output half h). h is uniform within a
          // warp (warps alternate halves), so every shared-memory load of a block row is one
          // broadcast; both halves of a block lie in the same pass (a pass covers 32-block
          // groups times 2 halves), so the in-place writes are safe.
          const int b = S.b, nb = K / b, bp = (b + 3) & ~3;
          const int nb32 = (nb + 31) & ~31;
          const float* sbl = sblk + S.sh_off;   // shared block (rows padded to bp floats)
          const float* pbk = S.blocks;          // per-block: the padded copy
          for (int r = 0; r < MR_ROWS; ++r) {
            float* x = cur + r * K;
            for (int item0 = 0; item0 < 2 * nb32; item0 += MR_THREADS) {
              const int item = item0 + (int)threadIdx.x;
              const int h = (item >> 5) & 1;
              const int c0 = ((item >> 6) << 5) + (item & 31);
              const bool on = c0 < nb;
              const int c = on ? c0 : 0;
              const int high = st == 1 ? c : (int)__umulhi((uint32_t)c, S.magic);
              const int low = c - high * st;
              const int base = low + high * b * st;
              float in[MR_MAXB];
#pragma unroll
              for (int k = 0; k < MR_MAXB; ++k) in[k] = (on && k < b) ? x[base + k * st] : 0.0f;
              __syncthreads();   // every input of this pass is in registers before any write
              if (on) {
                const int r0 = h ? (b + 1) / 2 : 0, r1 = h ? b : (b + 1) / 2;
                if (PB && S.per_block) {
                  // per-block blocks: the padded copy, read through L1/L2
                  for (int o = r0; o < r1; ++o) {
                    const float4* brow = reinterpret_cast<const float4*>(pbk + ((size_t)c * b + o) * bp);
                    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;   // four independent chains
#pragma unroll
                    for (int k4 = 0; k4 < MR_MAXB / 4; ++k4) {
                      if (4 * k4 < b) {
                        const float4 w = __ldg(brow + k4);
                        a0 = fmaf(w.x, in[4 * k4], a0);
                        a1 = fmaf(w.y, in[4 * k4 + 1], a1);
                        a2 = fmaf(w.z, in[4 * k4 + 2], a2);
                        a3 = fmaf(w.w, in[4 * k4 + 3], a3);
                      }
                    }
                    const int oi = base + o * st;
                    dst[r * K + (scat ? __ldg(S.iperm + oi) : oi)] = (a0 + a1) + (a2 + a3);
                  }
                } else {
                  // one shared block: its rows in shared memory, every load a broadcast
                  for (int o = r0; o < r1; ++o) {
                    const float4* brow = reinterpret_cast<const float4*>(sbl + o * bp);
                    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;   // four independent chains
#pragma unroll
                    for (int k4 = 0; k4 < MR_MAXB / 4; ++k4) {
                      if (4 * k4 < b) {
                        const float4 w = brow[k4];
                        a0 = fmaf(w.x, in[4 * k4], a0);
                        a1 = fmaf(w.y, in[4 * k4 + 1], a1);
                        a2 = fmaf(w.z, in[4 * k4 + 2], a2);
                        a3 = fmaf(w.w, in[4 * k4 + 3], a3);
                      }
                    }
                    const int oi = base + o * st;
                    dst[r * K + (scat ? __ldg(S.iperm + oi) : oi)] = (a0 + a1) + (a2 + a3);
                  }
                }
              }
              __syncthreads();
            }
          }
        }
        __syncthreads();
        if (scat) {
          float* tmp = cur; cur = nxt; nxt = tmp;
        }
      }
      if (S.perm && S.identity) {   // a permutation after an identity stage: plain gather
        for (int i0 = threadIdx.x; i0 < K; i0 += MR_THREADS * MR_UG) {
          int src[MR_UG];
#pragma unroll
          for (int u = 0; u < MR_UG; ++u) src[u] = i0 + u * MR_THREADS < K ? __ldg(S.perm + i0 + u * MR_THREADS) : 0;
#pragma unroll
          for (int u = 0; u < MR_UG; ++u)
            if (i0 + u * MR_THREADS < K) {
#pragma unroll
              for (int r = 0; r < MR_ROWS; ++r) nxt[r * K + i0 + u * MR_THREADS] = cur[r * K + src[u]];
            }
        }
        __syncthreads();
        float* tmp = cur; cur = nxt; nxt = tmp;
      }
    }
    for (int r = 0; r < nr; ++r) {
      const int64_t row = row0 + r;
      const float* xr = cur + r * K;
      if (a.bits == 0) {
        float* dst = a.Y + row * a.ldy;
        for (int i = threadIdx.x; i < K; i += MR_THREADS) dst[i] = xr[i];
      } else {
        // one warp per group; lane l takes 4 consecutive values per 128-value slice (one
        // 16-byte load), neighbouring lanes' code bits are merged with shuffles
        const float qmax = qmax_of_bits(a.bits);
        const float magic = magic_of_bits(a.bits);
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        const int ngr = K / a.G;
        const int lpw = 8 / a.bits;            // lanes per 32-bit code word (4 codes per lane)
        for (int g = warp; g < ngr; g += MR_THREADS / 32) {
          const float* gx = xr + (int64_t)g * a.G;
          float m = 0.0f;
          for (int i = 4 * lane; i < a.G; i += 128) {
            const float4 v = *reinterpret_cast<const float4*>(gx + i);
            m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
          }
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          float f;
          bool slow;
          const uint16_t s16 = group_scale(m, 1.0f / qmax, 1.0f + 0x1p-22f, &f, &slow);
          if (lane == 0) a.scales[row * ngr + g] = s16;
          uint32_t* cw = reinterpret_cast<uint32_t*>(a.codes + row * (int64_t)(K * a.bits / 8)) +
                         (int64_t)g * a.G * a.bits / 32;
          for (int i0 = 0; i0 < a.G; i0 += 128) {
            const int i = i0 + 4 * lane;
            uint32_t part = 0;
            if (i < a.G) {
              const float4 v = *reinterpret_cast<const float4*>(gx + i);
              const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t u = slow ? code_magic_clamped(vv[j], f, qmax, magic) : code_magic(vv[j], f, magic);
                part |= (u & ((1u << a.bits) - 1u)) << (a.bits * j);
              }
            }
            // lane l holds bits [4 l * bits, 4 (l + 1) * bits) of the slice; merge lpw lanes
            uint32_t word = part << (4 * a.bits * (lane % lpw));
            for (int o = 1; o < lpw; o <<= 1) word |= __shfl_down_sync(0xffffffffu, word, o);
            if (lane % lpw == 0 && i < a.G)
              cw[(i0 + 4 * lane) * a.bits / 32] = word ^ offset_xor_of_bits(a.bits);
          }
        }
      }
    }
    __syncthreads();
  }
}

// The multi-row kernel applies to forward plans whose non-identity stages are radix 2 or dense
// of radix 3..MR_MAXB (shared blocks in shared memory, per-block blocks from their padded copy),
// with K < 2^16 and the two row buffers in shared memory.
bool rows_kernel_fits(const rot_plan_s* p, int inverse, size_t* smem_out) {
  if (inverse || p->K >= 65536 || (p->K & 3) || (int)p->stages.size() > MAX_STAGES) return false;
  size_t sh = 0;
  for (const Stage& S : p->stages) {
    if (S.identity) continue;
    if (S.b == 2) continue;
    if (S.b > MR_MAXB) return false;
    // per-block blocks of small radix: the generic kernel (one row per CTA) is faster
    if (S.n_blocks != 1 && (!S.d_blocks_pad || S.b < 16)) return false;
    if (S.n_blocks == 1) sh += (size_t)S.b * ((S.b + 3) & ~3);
  }
  const size_t smem = (size_t)2 * MR_ROWS * p->K * sizeof(float) + sh * sizeof(float);
  if (smem > 227 * 1024) return false;
  *smem_out = smem;
  return true;
}

rot_status launch_rows(const rot_plan_s* p, const Args& a0, size_t smem, cudaStream_t s) {
  MrArgs a{};
  a.A = a0.A;
  a.a_bf16 = a0.a_bf16;
  a.lda = a0.lda;
  a.M = a0.M;
  a.K = p->K;
  a.signs = p->d_signf;
  a.n_stages = (int)p->stages.size();
  for (int t = 0; t < a.n_stages; ++t) {
    const Stage& S = p->stages[t];
    MrStage& d = a.st[t];
    d.blocks = S.d_blocks;
    d.perm = S.d_perm;
    d.iperm = S.d_iperm;
    d.b = S.b;
    d.stride = S.stride;
    d.magic = S.stride > 1 ? (uint32_t)(((1ull << 32) + (uint64_t)S.stride - 1) / (uint64_t)S.stride) : 0u;
    d.per_block = S.n_blocks > 1;
    d.identity = S.identity;
    d.sh_off = 0;
    if (!S.identity && S.b > 2) {
      if (d.per_block) {
        d.blocks = S.d_blocks_pad;
      } else {
        d.sh_off = a.sh_floats;
        a.sh_floats += S.b * ((S.b + 3) & ~3);
      }
    }
  }
  a.Y = a0.Y;
  a.ldy = a0.ldy;
  a.codes = a0.codes;
  a.scales = a0.scales;
  a.G = a0.G;
  a.bits = a0.bits;
  bool pb = false;
  for (int t = 0; t < a.n_stages; ++t) pb = pb || (!a.st[t].identity && a.st[t].b > 2 && a.st[t].per_block);
  static int configured[64][2] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev][pb]) {
    ROT_CUDA_TRY(cudaFuncSetAttribute(pb ? stages_rows_kernel<true> : stages_rows_kernel<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
    configured[dev][pb] = 1;
  }
  if (a.M == 0) return ROT_OK;
  const int64_t units = (a.M + MR_ROWS - 1) / MR_ROWS;
  const int64_t grid = std::min<int64_t>(units, (int64_t)sm_count());
  if (pb) stages_rows_kernel<true><<<(unsigned)grid, MR_THREADS, smem, s>>>(a);
  else stages_rows_kernel<false><<<(unsigned)grid, MR_THREADS, smem, s>>>(a);
  ROT_CUDA_TRY(cudaGetLastError());
  return ROT_OK;
}

rot_status launch(const rot_plan_s* p, Args& a, cudaStream_t s) {
  if ((int)p->stages.size() > MAX_STAGES) return set_error(ROT_EUNSUPPORTED, "generic rotation: too many stages");
  {
    size_t rsmem = 0;
    const char* e = std::getenv("ROT_B200_ROWS");
    if (!(e && e[0] == '0') && rows_kernel_fits(p, a.inverse, &rsmem)) return launch_rows(p, a, rsmem, s);
  }
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

// Fused signed Walsh-Hadamard rotation (+ group quantisation + packing), one HBM pass.
//
// Computes, for every contiguous chunk of N = 2^n coordinates of every row,
//     y = H_N D x / sqrt(N)
// (the randomized Hadamard transform: random signs, fast Walsh-Hadamard transform,
// times 1/sqrt(N) [Hadamard-Int4-Accuracy wiki, Method: fwht_norm; HARP abstract]),
// then optionally the per-group symmetric absmax quantisation of y with fp16 scales and
// two's-complement packing [same wiki, Method: q_dequant_vec].
//
// Work decomposition (sm_100a): a chunk is owned by TPC = 2^(n-e) consecutive threads
// of one warp (or two warps for n = 13), each holding E = 2^e values in registers.
//   phase A  thread t holds coordinates lo + (t << VA) + (hi << e), lo < 2^VA, hi < 2^(n-e)
//            (VA = 2e - n): contiguous runs of 2^VA elements, read straight from HBM with
//            vector loads that are coalesced across the chunk's threads; the e butterfly
//            stages over these register bits run in registers.
//   transpose through shared memory (fp32, XOR-swizzled 16-byte chunks: conflict-free
//            stores and loads).
//   phase B  thread t holds the contiguous coordinates (t << e) + j, j < E; the remaining
//            n - e stages (register bits VA..e-1) run in registers, with packed
//            add/sub.f32x2. Quantisation then sees whole groups (or group fragments
//            reduced with warp shuffles) in contiguous registers and writes packed codes
//            and scales with vector stores.
// Scaling by 1/sqrt(N) is folded into the output (apply) or into the group factor (quant).
#include <cmath>
#include <cstdlib>

#include "rot_internal.cuh"

namespace rotb {
namespace {

#ifndef ROT_FWHT_THREADS_E128
#define ROT_FWHT_THREADS_E128 384   // threads per CTA for the 128-register-value layouts
#endif
#ifndef ROT_FWHT_THREADS_N11
#define ROT_FWHT_THREADS_N11 640    // one warp per 2048-coordinate chunk, 20 chunks per CTA
#endif

// log2 of the values each thread holds for a chunk of 2^n coordinates
constexpr int elog_of(int n) { return n <= 7 ? n : (n == 8 ? 5 : (n == 9 || n == 11) ? 6 : 7); }
// threads per CTA
constexpr int threads_of(int n) {
  return n <= 7 ? 256 : (n == 8 ? 768 : (n == 9 ? 512 : (n == 11 ? ROT_FWHT_THREADS_N11 : ROT_FWHT_THREADS_E128)));
}

template <int LOGN>
struct Cfg {
  static constexpr int N = 1 << LOGN;
  static constexpr int ELOG = elog_of(LOGN);
  static constexpr int E = 1 << ELOG;
  static constexpr int HB = LOGN - ELOG;   // thread bits (= high register bits of phase A)
  static constexpr int VA = ELOG - HB;     // contiguous run bits of phase A
  static constexpr int TPC = 1 << HB;      // threads per chunk
  static constexpr int NV = 1 << VA;       // run length
  static constexpr int NH = 1 << HB;       // runs per thread
  static constexpr int THREADS = threads_of(LOGN);
  static constexpr int SLOTS = THREADS / TPC;
  static constexpr int SSTRIDE = N + 4;    // floats per slot buffer (16-byte pad)
  static_assert(VA >= 1, "phase A needs element pairs");
};

// Physical float index of chunk-local coordinate i in a slot buffer: 16-byte chunks are
// XOR-swizzled by the three coordinate bits above the phase-B thread's run (and, for
// n = 9 and 11, also by coordinate bit 5), which makes phase-A stores and phase-B loads
// conflict-free (n = 10 keeps 4-way conflicts on the stores).
template <int LOGN>
__device__ __forceinline__ int swz(int i) {
  constexpr int ELOG = Cfg<LOGN>::ELOG;
  int x = ((i >> ELOG) & 7) << 2;
  if constexpr (LOGN == 9 || LOGN == 11) x ^= ((i >> 5) & 1) << 2;
  return i ^ x;
}

struct Args {
  const void* A;
  int64_t lda;
  int64_t M;
  int chunks;       // chunks per row (K / N)
  int K;
  const uint32_t* signmask;  // K/2 words or nullptr
  float* Y;
  int64_t ldy;
  uint8_t* codes;
  uint16_t* scales;
  int G;
  int log2G;
  int64_t ngroups;   // K / G
  float norm;
  float cdiv;        // fp32(norm / qmax)
  float cf;          // fp32(norm * (1 + 2^-22))
  unsigned long long wait_ns;  // bound of the staging waits
  int skip_first;    // testing hook: slot 0 of CTA 0 never issues its first staging copy
};

enum { MODE_APPLY = 0, MODE_APPLY_INV = 1, MODE_QUANT = 2 };


// NW consecutive sign-mask words starting at word w0 (w0 a multiple of NW), vector loads.
template <int NW>
__device__ __forceinline__ void load_masks(uint32_t (&m)[NW], const uint32_t* smask, int w0, bool on) {
  if (!on) {
#pragma unroll
    for (int w = 0; w < NW; ++w) m[w] = 0u;
    return;
  }
  if constexpr (NW >= 4) {
#pragma unroll
    for (int v = 0; v < NW / 4; ++v) {
      const uint4 q = reinterpret_cast<const uint4*>(smask + w0)[v];
      m[4 * v] = q.x; m[4 * v + 1] = q.y; m[4 * v + 2] = q.z; m[4 * v + 3] = q.w;
    }
  } else if constexpr (NW == 2) {
    const uint2 q = *reinterpret_cast<const uint2*>(smask + w0);
    m[0] = q.x; m[1] = q.y;
  } else {
    m[0] = smask[w0];
  }
}

// Lanes of this thread's slot within its warp.
template <int TPC>
__device__ __forceinline__ unsigned slot_lanes() {
  if constexpr (TPC >= 32) {
    return 0xffffffffu;
  } else {
    const unsigned lane = threadIdx.x & 31;
    return ((1u << TPC) - 1u) << (lane & ~(TPC - 1));
  }
}

template <int TPC>
__device__ __forceinline__ void slot_sync(int slot) {
  if constexpr (TPC > 32) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + slot), "r"(TPC) : "memory");
  } else if constexpr (TPC > 1) {
    __syncwarp(slot_lanes<TPC>());
  }
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Pack 8 offset codes (low bytes of t[0..7], each 8 + q) into one int4 word: byte j holds
// codes 2j (low nibble) and 2j+1 (high nibble), two's complement.
__device__ __forceinline__ uint32_t pack8_int4(const uint32_t (&t)[8]) {
  const uint32_t x01 = t[1] * 16u + t[0], x23 = t[3] * 16u + t[2];
  const uint32_t x45 = t[5] * 16u + t[4], x67 = t[7] * 16u + t[6];
  return prmt(prmt(x01, x23, 0x0040u), prmt(x45, x67, 0x0040u), 0x5410u) ^ 0x88888888u;
}
// Pack 4 offset codes (low bytes of t[0..3], each 128 + q) into one int8 word, two's complement.
__device__ __forceinline__ uint32_t pack4_int8(const uint32_t (&t)[4]) {
  return prmt(prmt(t[0], t[1], 0x0040u), prmt(t[2], t[3], 0x0040u), 0x5410u) ^ 0x80808080u;
}
// Pack 16 offset codes (each 2 + q) into one int2 word: byte j holds codes 4j .. 4j+3.
__device__ __forceinline__ uint32_t pack16_int2(const uint32_t (&t)[16]) {
  uint32_t b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) b[i] = ((t[4 * i + 3] * 4u + t[4 * i + 2]) * 4u + t[4 * i + 1]) * 4u + t[4 * i];
  return prmt(prmt(b[0], b[1], 0x0040u), prmt(b[2], b[3], 0x0040u), 0x5410u) ^ 0xAAAAAAAAu;
}

__device__ int g_fwht_error = 0;

#ifndef ROT_STAGE_SLEEP
#define ROT_STAGE_SLEEP 0
#endif

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bounded wait on a slot's staging barrier (the bulk copy always completes; the bound only
// protects against a programming error, and lets the testing hook check this path). Returns
// false after limit_ns of wall time (1 s by default) and records ROT_ETIMEOUT.
__device__ __forceinline__ bool stage_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
  const uint32_t addr = smem_addr(bar);
  unsigned long long t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
#if ROT_STAGE_SLEEP > 0
    __nanosleep(ROT_STAGE_SLEEP);
#endif
    if ((it & 255) == 255) {
      unsigned long long now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) {
        atomicExch(&g_fwht_error, (int)ROT_ETIMEOUT);
        return false;
      }
    }
  }
}

// One elected thread: announce the bytes and start the bulk copy global -> slot buffer.
__device__ __forceinline__ void stage_issue(uint64_t* bar, void* dst, const void* src, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}


// Radix-2 butterflies along pair-index bit b: (P, Q) <- (P + Q, P - Q) on fp32 pairs.
template <int NP>
__device__ __forceinline__ void stage_pairs(float2 (&xp)[NP], int b) {
  const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int i = 0; i < NP; ++i)
    if (!(i & (1 << b))) {
      const float2 P = xp[i], Q = xp[i + (1 << b)];
      xp[i] = __fadd2_rn(P, Q);
      xp[i + (1 << b)] = __ffma2_rn(Q, m1, P);
    }
}

// Quantise the E values a thread holds (coordinates c0 .. c0+E-1 of one row) and store
// packed codes and scales. GT > 0: compile-time group size; GT == 0: runtime a.G.
// srow: the scales of the row (or of the chunk: any base whose group 0 starts at coordinate 0 of
// c0's frame); dst: this thread's first code word; c0: its first coordinate in that frame.
template <int BITS, int GT, int E, int TPC>
__device__ __forceinline__ void quantise_store_at(const Args& a, const float2 (&xp)[E / 2], uint16_t* srow,
                                                  uint32_t* dst, int c0, int t) {
  constexpr float QMAX = qmax_of_bits(BITS);
  constexpr float MAGIC = magic_of_bits(BITS);  // 2^23 + qmax + 1
  constexpr int CPW = 32 / BITS;   // codes per 32-bit word
  constexpr int NWD = E / CPW;     // words per thread
  uint32_t words[NWD];
  if constexpr (GT > 0) {
    constexpr int GE = GT <= E ? GT : E;     // elements of one group held by this thread
    constexpr int NGT = E / GE;              // groups (or group fragments) per thread
    float f[NGT];
    uint16_t sv[NGT];
    bool any_slow = false;
#pragma unroll
    for (int g = 0; g < NGT; ++g) {
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < GE / 2; ++j) {
        const float2 p = xp[g * (GE / 2) + j];
        m = max3(m, fabsf(p.x), fabsf(p.y));
      }
      if constexpr (GT > E) {
        const unsigned lanes = slot_lanes<TPC>();
#pragma unroll
        for (int o = 1; o < GT / E; o <<= 1) m = fmaxf(m, __shfl_xor_sync(lanes, m, o));
      }
      bool slow;
      sv[g] = group_scale(m, a.cdiv, a.cf, &f[g], &slow);
      any_slow |= slow;
    }
    if constexpr (GT > E) {
      if ((t & (GT / E - 1)) == 0) srow[c0 / GT] = sv[0];
    } else {
      // NGT consecutive scales: one vector store when the address allows it
      uint16_t* sp = srow + c0 / GT;
      const bool vec = NGT >= 2 && NGT <= 8 && (reinterpret_cast<uintptr_t>(sp) & (2 * NGT - 1)) == 0;
      if constexpr (NGT == 2) {
        if (vec) { *reinterpret_cast<uint32_t*>(sp) = sv[0] | ((uint32_t)sv[1] << 16); }
        else { sp[0] = sv[0]; sp[1] = sv[1]; }
      } else if constexpr (NGT == 4) {
        if (vec) {
          *reinterpret_cast<uint2*>(sp) = make_uint2(sv[0] | ((uint32_t)sv[1] << 16), sv[2] | ((uint32_t)sv[3] << 16));
        } else {
#pragma unroll
          for (int g = 0; g < 4; ++g) sp[g] = sv[g];
        }
      } else {
#pragma unroll
        for (int g = 0; g < NGT; ++g) sp[g] = sv[g];
      }
    }
    const float2 mg = make_float2(MAGIC, MAGIC);
    if (!any_slow) {
#pragma unroll
      for (int w = 0; w < NWD; ++w) {
        const float fg = f[(w * CPW) / GE];
        const float2 ff = make_float2(fg, fg);
        uint32_t tt[CPW];
#pragma unroll
        for (int j = 0; j < CPW; j += 2) {
          const float2 r = __ffma2_rn(xp[(CPW * w + j) / 2], ff, mg);
          tt[j] = __float_as_uint(r.x);
          tt[j + 1] = __float_as_uint(r.y);
        }
        if constexpr (BITS == 8) words[w] = pack4_int8(*reinterpret_cast<const uint32_t(*)[4]>(tt));
        else if constexpr (BITS == 4) words[w] = pack8_int4(*reinterpret_cast<const uint32_t(*)[8]>(tt));
        else words[w] = pack16_int2(*reinterpret_cast<const uint32_t(*)[16]>(tt));
      }
    } else {
#pragma unroll
      for (int w = 0; w < NWD; ++w) {
        const float fg = f[(w * CPW) / GE];
        uint32_t tt[CPW];
#pragma unroll
        for (int j = 0; j < CPW; j += 2) {
          tt[j] = code_magic_clamped(xp[(CPW * w + j) / 2].x, fg, QMAX, MAGIC);
          tt[j + 1] = code_magic_clamped(xp[(CPW * w + j) / 2].y, fg, QMAX, MAGIC);
        }
        if constexpr (BITS == 8) words[w] = pack4_int8(*reinterpret_cast<const uint32_t(*)[4]>(tt));
        else if constexpr (BITS == 4) words[w] = pack8_int4(*reinterpret_cast<const uint32_t(*)[8]>(tt));
        else words[w] = pack16_int2(*reinterpret_cast<const uint32_t(*)[16]>(tt));
      }
    }
  } else {
    // runtime group size: max per granule of 8, predicated tree, shuffles across threads
    constexpr int NG = E / 8;
    const int G = a.G;
    const int gg = G >> 3;
    float gm[NG];
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) m = max3(m, fabsf(xp[4 * i + j].x), fabsf(xp[4 * i + j].y));
      gm[i] = m;
    }
#pragma unroll
    for (int st = 1; st < NG; st <<= 1) {
      if (st < gg) {
#pragma unroll
        for (int i = 0; i + st < NG; i += 2 * st) gm[i] = fmaxf(gm[i], gm[i + st]);
      }
    }
    if (G > E) {
      const unsigned lanes = slot_lanes<TPC>();
      for (int o = 1; o < G / E; o <<= 1) gm[0] = fmaxf(gm[0], __shfl_xor_sync(lanes, gm[0], o));
    }
    float fw[NG];
    bool slow[NG];
    uint16_t sc[NG];
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      if ((i & (gg - 1)) == 0) {
        sc[i] = group_scale(gm[i], a.cdiv, a.cf, &fw[i], &slow[i]);
      } else {
        fw[i] = fw[i - 1];
        slow[i] = slow[i - 1];
        sc[i] = sc[i - 1];
      }
    }
    if (G > E) {
      if ((t & (G / E - 1)) == 0) srow[c0 >> a.log2G] = sc[0];
    } else {
#pragma unroll
      for (int i = 0; i < NG; ++i)
        if ((i & (gg - 1)) == 0) srow[(c0 + 8 * i) >> a.log2G] = sc[i];
    }
    const float2 mg = make_float2(MAGIC, MAGIC);
#pragma unroll
    for (int w = 0; w < NWD; ++w) {
      const int gi = (w * CPW) / 8;        // granule of 8 codes holding the word's first code
      uint32_t tt[CPW];
      if (!slow[gi]) {
        const float2 ff = make_float2(fw[gi], fw[gi]);
#pragma unroll
        for (int j = 0; j < CPW; j += 2) {
          const float2 r = __ffma2_rn(xp[(CPW * w + j) / 2], ff, mg);
          tt[j] = __float_as_uint(r.x);
          tt[j + 1] = __float_as_uint(r.y);
        }
      } else {
#pragma unroll
        for (int j = 0; j < CPW; j += 2) {
          tt[j] = code_magic_clamped(xp[(CPW * w + j) / 2].x, fw[gi], QMAX, MAGIC);
          tt[j + 1] = code_magic_clamped(xp[(CPW * w + j) / 2].y, fw[gi], QMAX, MAGIC);
        }
      }
      if constexpr (BITS == 8) words[w] = pack4_int8(*reinterpret_cast<const uint32_t(*)[4]>(tt));
      else if constexpr (BITS == 4) words[w] = pack8_int4(*reinterpret_cast<const uint32_t(*)[8]>(tt));
      else words[w] = pack16_int2(*reinterpret_cast<const uint32_t(*)[16]>(tt));
    }
  }
  if constexpr (NWD >= 4) {
#pragma unroll
    for (int v = 0; v < NWD / 4; ++v)
      reinterpret_cast<uint4*>(dst)[v] = make_uint4(words[4 * v], words[4 * v + 1], words[4 * v + 2], words[4 * v + 3]);
  } else if constexpr (NWD == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
  } else {
    dst[0] = words[0];
  }
}

template <int LOGN, int BITS, int GT, int E, int TPC>
__device__ __forceinline__ void quantise_store(const Args& a, const float2 (&xp)[E / 2], int64_t row, int c0, int t) {
  constexpr int CPW = 32 / BITS;
  uint32_t* dst = reinterpret_cast<uint32_t*>(a.codes + row * (int64_t)(a.K / CPW) * 4) + c0 / CPW;
  quantise_store_at<BITS, GT, E, TPC>(a, xp, a.scales + row * a.ngroups, dst, c0, t);
}

// Sign masks in shared memory: one word per bf16 pair (bits 15 and 31), or, for the bf16
// quantise path, two words per pair (the low element's sign moved to bit 31, and the high
// element's sign at bit 31), so that sign flip and bf16 -> fp32 widening take one integer
// instruction per element: (w << 16) + lo_mask and (w ^ hi_mask) & 0xffff0000.
template <int LOGN, bool BF16, int MODE>
constexpr bool dual_masks() {
  return BF16 && MODE == MODE_QUANT && LOGN <= 12;
}

template <int LOGN, bool BF16, int MODE, int BITS, int GT>
__global__ void __launch_bounds__(Cfg<LOGN>::THREADS, 1) fwht_kernel(const Args a) {
  constexpr bool DUAL = dual_masks<LOGN, BF16, MODE>();
  using C = Cfg<LOGN>;
  constexpr int N = C::N, ELOG = C::ELOG, E = C::E, HB = C::HB, VA = C::VA, TPC = C::TPC;
  constexpr int NV = C::NV, NH = C::NH, SLOTS = C::SLOTS, SSTRIDE = C::SSTRIDE;
  constexpr int NP = E / 2;   // fp32 pairs per thread: xp[i] = layout coordinates (2i, 2i+1)
  constexpr int NW = NV / 2;  // pairs per phase-A run
  extern __shared__ __align__(128) float smem[];
  float* sbuf = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SLOTS * SSTRIDE);
  uint32_t* smask = reinterpret_cast<uint32_t*>(bars + ((SLOTS + 1) & ~1));  // 16-byte aligned

  const int slot = threadIdx.x / TPC;
  const int t = threadIdx.x % TPC;
  float* buf = sbuf + slot * SSTRIDE;
  uint64_t* bar = bars + slot;
  const bool has_signs = a.signmask != nullptr;

  const int64_t units = a.M * a.chunks;
  const int64_t stride = (int64_t)gridDim.x * SLOTS;
  int64_t u = (int64_t)blockIdx.x * SLOTS + slot;
  const int64_t drow = stride / a.chunks;
  const int dchunk = (int)(stride - drow * a.chunks);
  int64_t row = u / a.chunks;
  int chunk = (int)(u - row * a.chunks);
  constexpr uint32_t ELEM = BF16 ? 2 : 4;
  const uint32_t chunk_bytes = (uint32_t)N * ELEM;
  auto src_of = [&](int64_t r, int c) -> const void* {
    return static_cast<const uint8_t*>(a.A) + ((int64_t)r * a.lda + (int64_t)c * N) * ELEM;
  };

  // Prologue that touches no memory written by earlier kernels: the slot barriers and the
  // sign table (plan memory). Under programmatic dependent launch it overlaps the tail of
  // the previous kernel in the stream; griddepcontrol.wait then orders every access to A
  // and to the outputs after that kernel's completion (a no-op for an ordinary launch).
  if (t == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (has_signs) {
    if constexpr (DUAL) {
      for (int i = threadIdx.x; i < a.K / 2; i += C::THREADS) {
        const uint32_t m = a.signmask[i];
        smask[2 * i] = m << 16;
        smask[2 * i + 1] = m & 0x80000000u;
      }
    } else {
      for (int i = threadIdx.x; i < a.K / 2; i += C::THREADS) smask[i] = a.signmask[i];
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the slot leader initialised its own barrier: it can start the first copy at once
  if (t == 0 && u < units && !(a.skip_first && blockIdx.x == 0 && slot == 0))
    stage_issue(bar, buf, src_of(row, chunk), chunk_bytes);
  __syncthreads();

  // per-thread shared-memory bases (loop invariant); compile-time offsets are added per access
  const int T = t << VA;                       // first coordinate of this thread's phase-A runs
  constexpr int NPA = VA >= 5 ? 1 : (1 << (5 - (VA < 2 ? 2 : VA)));
  constexpr bool B5 = (LOGN == 9 || LOGN == 11);  // extra swizzle term from coordinate bit 5
  // phase-A store bases: pa[k] = T ^ (k << max(VA, 2)); with the bit-5 term (bit 5 of the
  // coordinate is a thread bit) the XOR on coordinate bit 2 also depends on the thread.
  const int tb = B5 ? ((T >> 5) & 1) << 2 : 0;
  int pa[NPA];
#pragma unroll
  for (int k = 0; k < NPA; ++k) pa[k] = (T ^ (k << (VA < 2 ? 2 : VA))) ^ tb;
  int qb[8];                                    // phase-B load bases
#pragma unroll
  for (int r = 0; r < 8; ++r) qb[r] = (t << ELOG) + ((4 * r) ^ ((t & 7) << 2));

  uint32_t parity = 0;

  for (; u < units; u += stride) {
    const int cbase = chunk * N;
    float2 xp[NP];
    if (!stage_wait(bar, parity, a.wait_ns)) break;
    parity ^= 1u;

    // ---------------- phase A: runs of NV elements from the staged chunk, signs, fp32 pairs
    if constexpr (DUAL) {
      const uint32_t* sraw = reinterpret_cast<const uint32_t*>(buf) + (T >> 1);
      const uint32_t* smk = smask + cbase + T;   // two mask words per pair
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        uint32_t raw[NW], m[2 * NW];
        load_masks<NW>(raw, sraw + h * (E / 2), 0, true);
        load_masks<2 * NW>(m, smk + h * E, 0, has_signs);
#pragma unroll
        for (int w = 0; w < NW; ++w)
          xp[h * NW + w] = make_float2(__uint_as_float((raw[w] << 16) + m[2 * w]),
                                       __uint_as_float((raw[w] ^ m[2 * w + 1]) & 0xffff0000u));
      }
    } else if constexpr (BF16) {
      const uint32_t* sraw = reinterpret_cast<const uint32_t*>(buf) + (T >> 1);
      const uint32_t* smk = smask + ((cbase + T) >> 1);
      const bool sg = MODE != MODE_APPLY_INV && has_signs;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        uint32_t raw[NW], m[NW];
        load_masks<NW>(raw, sraw + h * (E / 2), 0, true);
        load_masks<NW>(m, smk + h * (E / 2), 0, sg);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const uint32_t v = raw[w] ^ m[w];
          xp[h * NW + w] = make_float2(bf16lo(v), bf16hi(v));
        }
      }
    } else {
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float* src = buf + T + (h << ELOG);
        if constexpr (NV >= 4) {
#pragma unroll
          for (int v = 0; v < NV / 4; ++v) {
            const float4 q = reinterpret_cast<const float4*>(src)[v];
            xp[h * NW + 2 * v] = make_float2(q.x, q.y);
            xp[h * NW + 2 * v + 1] = make_float2(q.z, q.w);
          }
        } else {
          xp[h * NW] = *reinterpret_cast<const float2*>(src);
        }
        if (MODE != MODE_APPLY_INV && has_signs) {
          uint32_t m[NW];
          load_masks<NW>(m, smask + ((cbase + T) >> 1) + h * (E / 2), 0, true);
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            xp[h * NW + w].x = __uint_as_float(__float_as_uint(xp[h * NW + w].x) ^ (m[w] << 16));
            xp[h * NW + w].y = __uint_as_float(__float_as_uint(xp[h * NW + w].y) ^ (m[w] & 0x80000000u));
          }
        }
      }
    }

    // ---------------- phase A butterflies: register bit 0 (inside the pairs), then bits 1..e-1
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float p = xp[i].x, q = xp[i].y;
      xp[i] = make_float2(p + q, p - q);
    }
#pragma unroll
    for (int b = 0; b < ELOG - 1; ++b) stage_pairs<NP>(xp, b);

    // ---------------- transpose through the slot buffer
    if constexpr (HB > 0) {
      slot_sync<TPC>(slot);  // every thread has read its staged runs
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        constexpr int SH = VA < 2 ? 2 : VA;        // lowest XOR bit not inside a run
        const int X = (h & 7) << 2;                // phys = i ^ X, i = T + (h << ELOG) + 4v
        const int base = pa[(X >> SH) & (NPA - 1)] + (h << ELOG);
        if constexpr (NV >= 4) {
#pragma unroll
          for (int v = 0; v < NV / 4; ++v) {
            const float2 p0 = xp[h * NW + 2 * v], p1 = xp[h * NW + 2 * v + 1];
            // bit 2 of the physical index: (4v ^ X) bit 2, flipped by tb (folded into base)
            const int off = (4 * v) ^ (X & ((1 << SH) - 1));
            const int adr = B5 ? (base ^ (off & 4)) + (off & ~4) : base + off;
            *reinterpret_cast<float4*>(buf + adr) = make_float4(p0.x, p0.y, p1.x, p1.y);
          }
        } else {
          *reinterpret_cast<float2*>(buf + base) = xp[h * NW];
        }
      }
      slot_sync<TPC>(slot);
#pragma unroll
      for (int jc = 0; jc < E / 4; ++jc) {
        // coordinate (t << ELOG) + 4jc; bit 5 of it is bit 3 of jc (compile-time)
        const int r = B5 ? ((jc & 7) ^ ((jc >> 3) & 1)) : (jc & 7);
        const float4 q = *reinterpret_cast<const float4*>(buf + qb[r] + 32 * (jc >> 3));
        xp[2 * jc] = make_float2(q.x, q.y);
        xp[2 * jc + 1] = make_float2(q.z, q.w);
      }
    }
    // the slot buffer is free: stage the next unit while this one finishes
    int64_t nrow = row + drow;
    int nchunk = chunk + dchunk;
    if (nchunk >= a.chunks) { nchunk -= a.chunks; ++nrow; }
    if (u + stride < units) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      slot_sync<TPC>(slot);
      if (t == 0) stage_issue(bar, buf, src_of(nrow, nchunk), chunk_bytes);
    }
    // ---------------- phase B butterflies: register bits VA..e-1 (pair-index bits VA-1..e-2)
    if constexpr (HB > 0) {
#pragma unroll
      for (int b = VA - 1; b < ELOG - 1; ++b) stage_pairs<NP>(xp, b);
    }
    const int64_t cur_row = row;
    row = nrow;
    chunk = nchunk;

    const int c0 = cbase + (t << ELOG);  // row coordinate of the first element
    if constexpr (MODE == MODE_APPLY || MODE == MODE_APPLY_INV) {
      float* dst = a.Y + cur_row * a.ldy + c0;
      const float2 nn = make_float2(a.norm, a.norm);
#pragma unroll
      for (int jc = 0; jc < E / 4; ++jc) {
        const float2 p0 = __fmul2_rn(xp[2 * jc], nn), p1 = __fmul2_rn(xp[2 * jc + 1], nn);
        float4 q = make_float4(p0.x, p0.y, p1.x, p1.y);
        if (MODE == MODE_APPLY_INV && has_signs) {
          const uint32_t m0 = smask[(c0 >> 1) + 2 * jc], m1 = smask[(c0 >> 1) + 2 * jc + 1];
          q.x = __uint_as_float(__float_as_uint(q.x) ^ (m0 << 16));
          q.y = __uint_as_float(__float_as_uint(q.y) ^ (m0 & 0x80000000u));
          q.z = __uint_as_float(__float_as_uint(q.z) ^ (m1 << 16));
          q.w = __uint_as_float(__float_as_uint(q.w) ^ (m1 & 0x80000000u));
        }
        *reinterpret_cast<float4*>(dst + 4 * jc) = q;
      }
    } else {
      quantise_store<LOGN, BITS, GT, E, TPC>(a, xp, cur_row, c0, t);
    }
  }
}

// ---------------------------------------------------------------- tensor-core first stage
// Chunks of 2048 coordinates, bf16 input, quantised output. H_2048 = H_2^(x)11 factors over
// the 11 coordinate bits e0..e10 (e = sum e_b 2^b), so the butterfly stages can be taken in
// any order. The stages over {e0, e1, e2, e6} form one H_16, applied on the tensor cores to
// the signed bf16 input (products with +-1 are exact, sums in fp32); the other seven stages
// run on fp32 pairs in registers.
//   MMA     m16n8k16 (bf16 in, fp32 out), D = X H_16 with X the 16 x 16 block of the chunk
//           whose rows are coordinate blocks (row bits e3, e4, e5, e7) and columns the
//           H_16 coordinates (k bits e0, e1, e2, e6); eight row tiles (e8, e9, e10).
//           The A fragments come straight from the staged bf16 row with ldmatrix; the signs
//           are XORed into them from a table kept in fragment order.
//   phase A lane 4g + c holds e1e2 = c and e3e4e5 = g; its registers hold e0 (inside each
//           fp32 pair), e6 (which of the two MMAs), e7 and e8..e10: butterflies over e7..e10.
//   phase B after a transpose through shared memory (XOR-swizzled 16-byte chunks, no bank
//           conflicts either way) lane l holds the contiguous coordinates 64 l .. 64 l + 63:
//           butterflies over e3..e5, then group quantisation and packing as in fwht_kernel.
#ifndef ROT_MMA_WARPS
#define ROT_MMA_WARPS 20
#endif
constexpr int MMA_SLOTS = ROT_MMA_WARPS;          // warps per CTA, one chunk each
constexpr int MMA_THREADS = MMA_SLOTS * 32;
constexpr int MMA_BARS = (MMA_SLOTS + 1) & ~1;    // even: the sign table after them stays 16-byte aligned
constexpr int MMA_SSTRIDE = 2048 + 64;         // floats per slot buffer (256-byte multiple)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void mma_h16(float2& d01, float2& d23, const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d01.x), "=f"(d01.y), "=f"(d23.x), "=f"(d23.y)
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// bf16 +-1 of the Sylvester entry (-1)^popcount(k & o)
__host__ __device__ constexpr uint32_t h16_bf16(int k, int o) {
  int v = k & o, par = 0;
  while (v) { par ^= 1; v &= v - 1; }
  return par ? 0xBF80u : 0x3F80u;
}

// 32-bit shared-state-space accesses (addresses computed once per lane, offsets folded in)
__device__ __forceinline__ void sts64(uint32_t addr, float2 v) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y) : "memory");
}
__device__ __forceinline__ float4 lds128f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 lds128u(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}

template <int BITS, int GT>
__global__ void __launch_bounds__(MMA_THREADS, 1) fwht_mma_kernel(const Args a) {
  constexpr int N = 2048, NP = 32;
  constexpr int CPW = 32 / BITS;
  extern __shared__ __align__(128) float smem[];
  // slot buffers start on a 256-byte boundary (the transpose addresses below rely on it)
  const uint32_t sm_raw = smem_addr(smem);
  const uint32_t sm0 = (sm_raw + 255u) & ~255u;
  float* sbase_ptr = smem + (sm0 - sm_raw) / 4;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sbase_ptr + MMA_SLOTS * MMA_SSTRIDE);
  uint32_t* smf = reinterpret_cast<uint32_t*>(bars + MMA_BARS);   // sign masks, fragment order

  const int slot = threadIdx.x >> 5;
  const int l = threadIdx.x & 31;
  const int g = l >> 2, c = l & 3;
  const uint32_t buf_b = sm0 + (uint32_t)(slot * MMA_SSTRIDE * 4);   // this warp's slot buffer
  uint64_t* bar = bars + slot;
  const bool has_signs = a.signmask != nullptr;

  const int64_t units = a.M * a.chunks;
  const int64_t stride = (int64_t)gridDim.x * MMA_SLOTS;
  int64_t u = (int64_t)blockIdx.x * MMA_SLOTS + slot;
  const int64_t drow = stride / a.chunks;
  const int dchunk = (int)(stride - drow * a.chunks);
  int64_t row = u / a.chunks;
  int chunk = (int)(u - row * a.chunks);
  auto src_of = [&](int64_t r, int ch) -> const void* {
    return static_cast<const uint8_t*>(a.A) + ((int64_t)r * a.lda + (int64_t)ch * N) * 2;
  };
  // outputs of unit u (chunk `chunk` of row `row`) are contiguous in u: codes at u * N * bits / 8
  // bytes, scales at u * N / G (G divides N); this lane's part advances by a constant per unit
  uint32_t* cdst = reinterpret_cast<uint32_t*>(a.codes) + u * (N / CPW) + (64 * l) / CPW;
  uint16_t* sdst = a.scales + u * (N / GT);
  const int64_t cstep = stride * (N / CPW), sstep = stride * (N / GT);

  // prologue on plan memory only (see fwht_kernel): barrier, sign table in fragment order
  if (l == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (has_signs) {
    // word (ch * 1024 + i * 128 + lane * 4 + r): register r of lane's A fragment, tile i
    for (int idx = threadIdx.x; idx < a.K / 2; idx += MMA_THREADS) {
      const int ch = idx >> 10, i = (idx >> 7) & 7, ln = (idx >> 2) & 31, r = idx & 3;
      const int off = ch * N + 8 * (ln >> 2) + 2 * (ln & 3) + 256 * i + ((r & 1) << 7) + ((r & 2) << 5);
      smf[idx] = a.signmask[off >> 1];
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (l == 0 && u < units && !(a.skip_first && blockIdx.x == 0 && slot == 0))
    stage_issue(bar, sbase_ptr + slot * MMA_SSTRIDE, src_of(row, chunk), N * 2);
  __syncthreads();

  // B fragments of H_16 for the two MMAs (outputs o3 = 0 / 1): n = g, k = 2c + {0,1} (+8)
  uint32_t hb[2][2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int o = 8 * q + g;
    hb[q][0] = h16_bf16(2 * c, o) | (h16_bf16(2 * c + 1, o) << 16);
    hb[q][1] = h16_bf16(2 * c + 8, o) | (h16_bf16(2 * c + 9, o) << 16);
  }
  // ldmatrix row address of this lane: matrix l >> 3, row l & 7
  const uint32_t ldsm_b = buf_b + (uint32_t)(8 * (l & 7) + ((l >> 3) & 1) * 128 + ((l >> 4) & 1) * 64) * 2;
  // transpose, phase-A stores: element 2c + 8g + 64 p (+ e0), 16-byte chunks XOR-swizzled by
  // (p & 7): byte address (buf_b + 8 (c + 4 g)) ^ ((p & 7) << 4) + 256 p (buf_b is 256-aligned
  // and 8 (c + 4 g) < 256, so the XOR only touches bits 4..6 of the in-buffer offset)
  const uint32_t wbase = buf_b + (uint32_t)(4 * (2 * c + 8 * g));
  // phase-B loads: lane l reads floats 64 l + ((4 j) ^ ((l & 7) << 2)): byte address
  // ((buf_b + 256 l + 16 (l & 7)) ^ (16 (j & 7))) + 128 (j >> 3)
  const uint32_t rbase = buf_b + (uint32_t)(256 * l + 16 * (l & 7));
  const uint32_t sgn_b = smem_addr(smf) + 16u * (uint32_t)l;
  const uint32_t bar_b = smem_addr(bar);
  uint32_t parity = 0;

  for (; u < units; u += stride) {
    const int cbase = chunk * N;
    float2 xp[NP];
    if (!stage_wait(bar, parity, a.wait_ns)) break;
    parity ^= 1u;

    // ---------------- MMA: H_16 over {e0, e1, e2, e6} for the 8 row tiles
    const uint32_t sg = sgn_b + 2u * (uint32_t)cbase;      // this chunk's sign words (fragment order)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t af[4];
      ldsm_x4(ldsm_b + i * 512, af);
      if (has_signs) {
        const uint4 m = lds128u(sg + i * 512);
        af[0] ^= m.x; af[1] ^= m.y; af[2] ^= m.z; af[3] ^= m.w;
      }
      // xp index p = e6 + 2 e7 + 4 (e8..e10): MMA q gives e6 = q; rows g / g + 8 give e7
      mma_h16(xp[4 * i + 0], xp[4 * i + 2], af, hb[0][0], hb[0][1]);
      mma_h16(xp[4 * i + 1], xp[4 * i + 3], af, hb[1][0], hb[1][1]);
    }
    // ---------------- phase A: e7 .. e10 (pair-index bits 1 .. 4)
#pragma unroll
    for (int b = 1; b < 5; ++b) stage_pairs<NP>(xp, b);

    // ---------------- transpose through the slot buffer (XOR-swizzled 16-byte chunks)
    __syncwarp();   // every lane's ldmatrix reads of the staged row are done
#pragma unroll
    for (int p = 0; p < NP; ++p) sts64((wbase ^ (uint32_t)((p & 7) << 4)) + 256u * p, xp[p]);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float4 q = lds128f((rbase ^ (uint32_t)(16 * (j & 7))) + 128u * (j >> 3));
      xp[2 * j] = make_float2(q.x, q.y);
      xp[2 * j + 1] = make_float2(q.z, q.w);
    }
    // the slot buffer is free: stage the next chunk while this one finishes
    int64_t nrow = row + drow;
    int nchunk = chunk + dchunk;
    if (nchunk >= a.chunks) { nchunk -= a.chunks; ++nrow; }
    if (u + stride < units) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (l == 0) {
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_b), "r"(N * 2) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                         buf_b),
                     "l"(src_of(nrow, nchunk)), "r"(N * 2), "r"(bar_b)
                     : "memory");
      }
    }
    // ---------------- phase B: e3 .. e5 (pair-index bits 2 .. 4)
#pragma unroll
    for (int b = 2; b < 5; ++b) stage_pairs<NP>(xp, b);
    row = nrow;
    chunk = nchunk;
    quantise_store_at<BITS, GT, 64, 32>(a, xp, sdst, cdst, 64 * l, l);
    cdst += cstep;
    sdst += sstep;
  }
}

// Few-row kernel for 4096-coordinate chunks (bf16 in, quantised out): one CTA of 256 threads per
// chunk, 16 values per thread, so a handful of rows (decode) is spread over many SMs instead of one
// warp per row. The chunk lives in shared memory between three radix-16 passes:
//   pass 0  thread t holds coordinates 16 t + j (loaded from HBM): butterflies over bits 0..3;
//   pass 1  thread t holds (t & 15) + 16 j + 256 (t >> 4): bits 4..7;
//   pass 2  thread t holds t + 256 j: bits 8..11;
// then thread t reads 16 t + j again and quantises as the other kernels do. Float i is stored at
// i + (i >> 4) (one pad per 16): every pass's accesses of a warp fall in distinct banks (pass 2:
// one two-way pair).
constexpr int SMALL_THREADS = 256;
constexpr int SMALL_N = 4096;
constexpr int SMALL_SMEM = (SMALL_N + SMALL_N / 16) * 4;

__device__ __forceinline__ int small_pad(int i) { return i + (i >> 4); }

// 16-point Walsh-Hadamard butterflies on the 16 values of a thread (pairs: bit 0 inside a pair)
__device__ __forceinline__ void fwht16(float2 (&xp)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) xp[i] = make_float2(xp[i].x + xp[i].y, xp[i].x - xp[i].y);
#pragma unroll
  for (int b = 0; b < 3; ++b) stage_pairs<8>(xp, b);
}

template <int BITS, int GT>
__global__ void __launch_bounds__(SMALL_THREADS) fwht_small_kernel(const Args a) {
  extern __shared__ __align__(16) float sfl[];
  const int t = threadIdx.x;
  const int64_t u = blockIdx.x;               // chunk `chunk` of row `row`
  const int64_t row = u / a.chunks;
  const int chunk = (int)(u - row * a.chunks);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  float2 xp[8];
  {
    // 16 bf16 values (two 16-byte loads), signs XORed into the pairs, widened to fp32
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.A) +
                                                      ((int64_t)row * a.lda + (int64_t)chunk * SMALL_N + 16 * t) * 2);
    const uint4 v0 = src[0], v1 = src[1];
    uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    if (a.signmask) {
      const uint4* sm = reinterpret_cast<const uint4*>(a.signmask + (chunk * SMALL_N + 16 * t) / 2);
      const uint4 m0 = sm[0], m1 = sm[1];
      const uint32_t m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] ^= m[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) xp[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
  }
  // pass 0: bits 0..3
  fwht16(xp);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sfl[small_pad(16 * t + 2 * j)] = xp[j].x;
    sfl[small_pad(16 * t + 2 * j + 1)] = xp[j].y;
  }
  __syncthreads();
  // pass 1: bits 4..7
  const int b1 = (t & 15) + 256 * (t >> 4);
#pragma unroll
  for (int j = 0; j < 8; ++j) xp[j] = make_float2(sfl[small_pad(b1 + 32 * j)], sfl[small_pad(b1 + 32 * j + 16)]);
  fwht16(xp);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sfl[small_pad(b1 + 32 * j)] = xp[j].x;
    sfl[small_pad(b1 + 32 * j + 16)] = xp[j].y;
  }
  __syncthreads();
  // pass 2: bits 8..11
#pragma unroll
  for (int j = 0; j < 8; ++j) xp[j] = make_float2(sfl[small_pad(t + 512 * j)], sfl[small_pad(t + 512 * j + 256)]);
  fwht16(xp);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sfl[small_pad(t + 512 * j)] = xp[j].x;
    sfl[small_pad(t + 512 * j + 256)] = xp[j].y;
  }
  __syncthreads();
  // contiguous again: quantise coordinates 16 t .. 16 t + 15 of the chunk
#pragma unroll
  for (int j = 0; j < 8; ++j) xp[j] = make_float2(sfl[small_pad(16 * t + 2 * j)], sfl[small_pad(16 * t + 2 * j + 1)]);
  constexpr int CPW = 32 / BITS;
  const int c0 = chunk * SMALL_N + 16 * t;                 // coordinate within the row
  uint32_t* dst = reinterpret_cast<uint32_t*>(a.codes + row * (int64_t)(a.K / CPW) * 4) + c0 / CPW;
  quantise_store_at<BITS, GT, 16, SMALL_THREADS>(a, xp, a.scales + row * a.ngroups, dst, c0, t);
}

size_t mma_smem_bytes(int K) {
  return 256 + (size_t)MMA_SLOTS * MMA_SSTRIDE * 4 + (size_t)MMA_BARS * 8 + (size_t)(K / 2) * 4;
}


template <int LOGN>
size_t fused_smem_bytes(int K, bool dual) {
  using C = Cfg<LOGN>;
  return (size_t)C::SLOTS * C::SSTRIDE * 4 + (size_t)((C::SLOTS + 1) & ~1) * 8 + (size_t)(dual ? K : K / 2) * 4;
}

size_t fused_smem_any(int logn, int K, bool dual) {
  switch (logn) {
    case 5: return fused_smem_bytes<5>(K, dual);
    case 6: return fused_smem_bytes<6>(K, dual);
    case 7: return fused_smem_bytes<7>(K, dual);
    case 8: return fused_smem_bytes<8>(K, dual);
    case 9: return fused_smem_bytes<9>(K, dual);
    case 10: return fused_smem_bytes<10>(K, dual);
    case 11: return fused_smem_bytes<11>(K, dual);
    case 12: return fused_smem_bytes<12>(K, dual);
    case 13: return fused_smem_bytes<13>(K, dual);
    default: return ~(size_t)0;
  }
}

template <int LOGN, bool BF16, int MODE, int BITS, int GT>
rot_status launch_one(const Args& a, cudaStream_t s) {
  using C = Cfg<LOGN>;
  const size_t smem = fused_smem_bytes<LOGN>(a.K, dual_masks<LOGN, BF16, MODE>());
  if (smem > 227 * 1024) return set_error(ROT_EUNSUPPORTED, "fused rotation: sign table too large for shared memory");
  auto kern = fwht_kernel<LOGN, BF16, MODE, BITS, GT>;
  static int configured[64] = {0};  // per device: the opt-in limit is set once
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    ROT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
    configured[dev] = 1;
  }
  const int64_t units = a.M * a.chunks;
  int64_t grid = (units + C::SLOTS - 1) / C::SLOTS;
  const int64_t cap = (int64_t)sm_count();
  if (grid > cap) grid = cap;
  if (grid < 1) return ROT_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_default() ? 1 : 0;
  ROT_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, a));
  ROT_CUDA_TRY(cudaGetLastError());
  return ROT_OK;
}

// Tensor-core first stage for 2048-coordinate chunks (ROT_B200_TC=0 in the environment
// selects the all-CUDA-core kernel instead).
bool tc_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("ROT_B200_TC");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <int BITS, int GT>
rot_status launch_mma(const Args& a, cudaStream_t s) {
  const size_t smem = mma_smem_bytes(a.K);
  if (smem > 227 * 1024) return set_error(ROT_EUNSUPPORTED, "fused rotation: sign table too large for shared memory");
  auto kern = fwht_mma_kernel<BITS, GT>;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    ROT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
    configured[dev] = 1;
  }
  const int64_t units = a.M * a.chunks;
  int64_t grid = (units + MMA_SLOTS - 1) / MMA_SLOTS;
  const int64_t cap = (int64_t)sm_count();
  if (grid > cap) grid = cap;
  if (grid < 1) return ROT_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(MMA_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_default() ? 1 : 0;
  ROT_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, a));
  return ROT_OK;
}

// Few rows of 4096-coordinate chunks: one CTA per chunk (ROT_B200_SMALL=0 / 1 in the environment
// turns the choice off / on for every row count; by default up to SMALL_MAX_UNITS chunks).
constexpr int64_t SMALL_MAX_UNITS = 512;
int small_mode() {
  static const int mode = [] {
    const char* e = std::getenv("ROT_B200_SMALL");
    return e ? (e[0] == '0' ? 0 : 1) : -1;
  }();
  return mode;
}

template <int BITS, int GT>
rot_status launch_small(const Args& a, cudaStream_t s) {
  const int64_t units = a.M * a.chunks;
  if (units < 1) return ROT_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units);
  cfg.blockDim = dim3(SMALL_THREADS);
  cfg.dynamicSmemBytes = SMALL_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_default() ? 1 : 0;
  ROT_CUDA_TRY(cudaLaunchKernelEx(&cfg, fwht_small_kernel<BITS, GT>, a));
  return ROT_OK;
}

template <int LOGN, bool BF16, int MODE, int BITS>
rot_status launch_g(const Args& a, cudaStream_t s) {
  if constexpr (MODE == MODE_QUANT && BF16 && LOGN == 12) {
    const int sm = small_mode();
    // 16-byte row loads (lda a multiple of 8 elements, 16-byte aligned A) and G <= 512 (a group
    // spans at most one warp of 16-value threads)
    const bool fits = (a.lda % 8) == 0 && (reinterpret_cast<uintptr_t>(a.A) & 15) == 0 && a.G <= 512 && a.G >= 8;
    if (fits && (sm == 1 || (sm == -1 && a.M * a.chunks <= SMALL_MAX_UNITS))) {
      if (a.G == 32) return launch_small<BITS, 32>(a, s);
      if (a.G == 64) return launch_small<BITS, 64>(a, s);
      if (a.G == 128) return launch_small<BITS, 128>(a, s);
      return launch_small<BITS, 0>(a, s);
    }
  }
  if constexpr (MODE == MODE_QUANT && BF16 && LOGN == 11) {
    if (tc_enabled() && mma_smem_bytes(a.K) <= 227 * 1024) {
      if (a.G == 32) return launch_mma<BITS, 32>(a, s);
      if (a.G == 64) return launch_mma<BITS, 64>(a, s);
      if (a.G == 128) return launch_mma<BITS, 128>(a, s);
    }
  }
  // compile-time group sizes for the common shapes (bf16 quantisation on large chunks)
  if constexpr (MODE == MODE_QUANT && BF16 && (LOGN == 8 || LOGN >= 11)) {
    if (a.G == 32) return launch_one<LOGN, BF16, MODE, BITS, 32>(a, s);
    if (a.G == 64) return launch_one<LOGN, BF16, MODE, BITS, 64>(a, s);
    if (a.G == 128) return launch_one<LOGN, BF16, MODE, BITS, 128>(a, s);
  }
  return launch_one<LOGN, BF16, MODE, BITS, 0>(a, s);
}

template <bool BF16, int MODE, int BITS>
rot_status dispatch_logn(int logn, const Args& a, cudaStream_t s) {
  switch (logn) {
    case 5: return launch_g<5, BF16, MODE, BITS>(a, s);
    case 6: return launch_g<6, BF16, MODE, BITS>(a, s);
    case 7: return launch_g<7, BF16, MODE, BITS>(a, s);
    case 8: return launch_g<8, BF16, MODE, BITS>(a, s);
    case 9: return launch_g<9, BF16, MODE, BITS>(a, s);
    case 10: return launch_g<10, BF16, MODE, BITS>(a, s);
    case 11: return launch_g<11, BF16, MODE, BITS>(a, s);
    case 12: return launch_g<12, BF16, MODE, BITS>(a, s);
    case 13: return launch_g<13, BF16, MODE, BITS>(a, s);
    default: return set_error(ROT_EUNSUPPORTED, "fused rotation: chunk size out of range");
  }
}

Args make_args(const rot_plan_s* p, const void* A, int64_t M, int64_t lda) {
  Args a{};
  a.A = A;
  a.lda = lda;
  a.M = M;
  a.K = p->K;
  a.chunks = p->K >> p->chunk_log2;
  a.signmask = p->has_signs ? p->d_signmask : nullptr;
  a.norm = (float)(1.0 / std::sqrt((double)(1 << p->chunk_log2)));
  a.wait_ns = wait_limit_ns(1000000000ull);
  a.skip_first = take_test_fault(TEST_FAULT_ROTATION_COPY) ? 1 : 0;
  return a;
}

}  // namespace

rot_status fwht_fetch_device_error() {
  int v = 0;
  ROT_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_fwht_error, sizeof(int)));
  if (v) {
    int z = 0;
    ROT_CUDA_TRY(cudaMemcpyToSymbol(g_fwht_error, &z, sizeof(int)));
    return set_error((rot_status)v, "a bounded wait in the fused rotation kernel gave up");
  }
  return ROT_OK;
}

bool fwht_quant_supported(const rot_plan_s* p, int bits, int G) {
  if (p->chunk_log2 < 5) return false;
  // shared memory for the bf16 layout (the larger of the two sign-table layouts)
  if (fused_smem_any(p->chunk_log2, p->K, p->chunk_log2 <= 12) > 227 * 1024) return false;
  const int N = 1 << p->chunk_log2;
  if (G < 8 || (G & (G - 1)) != 0 || G > N) return false;
  if (bits == 2 && G < 16) return false;
  const int e = elog_of(p->chunk_log2);
  if (G > (1 << e) && G / (1 << e) > 32) return false;
  return true;
}

rot_status fwht_apply(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda,
                      int inverse, float* Y, int64_t ldy, cudaStream_t s) {
  Args a = make_args(p, A, M, lda);
  a.Y = Y;
  a.ldy = ldy;
  const int n = p->chunk_log2;
  if (a_dtype == ROT_BF16)
    return inverse ? dispatch_logn<true, MODE_APPLY_INV, 4>(n, a, s) : dispatch_logn<true, MODE_APPLY, 4>(n, a, s);
  return inverse ? dispatch_logn<false, MODE_APPLY_INV, 4>(n, a, s) : dispatch_logn<false, MODE_APPLY, 4>(n, a, s);
}

rot_status fwht_quant(const rot_plan_s* p, const void* A, int a_dtype, int64_t M, int64_t lda, int bits,
                      int G, uint8_t* codes, uint16_t* scales, cudaStream_t s) {
  Args a = make_args(p, A, M, lda);
  a.codes = codes;
  a.scales = scales;
  a.G = G;
  a.log2G = 0;
  while ((1 << a.log2G) < G) ++a.log2G;
  a.ngroups = p->K / G;
  {
    const double nd = 1.0 / std::sqrt((double)(1 << p->chunk_log2));
    a.cdiv = (float)(nd / (bits == 8 ? 127.0 : bits == 4 ? 7.0 : 1.0));
    a.cf = (float)(nd * (1.0 + 0x1p-22));
  }
  const int n = p->chunk_log2;
  if (a_dtype == ROT_BF16) {
    if (bits == 8) return dispatch_logn<true, MODE_QUANT, 8>(n, a, s);
    return bits == 4 ? dispatch_logn<true, MODE_QUANT, 4>(n, a, s) : dispatch_logn<true, MODE_QUANT, 2>(n, a, s);
  }
  if (bits == 8) return dispatch_logn<false, MODE_QUANT, 8>(n, a, s);
  return bits == 4 ? dispatch_logn<false, MODE_QUANT, 4>(n, a, s) : dispatch_logn<false, MODE_QUANT, 2>(n, a, s);
}

}  // namespace rotb

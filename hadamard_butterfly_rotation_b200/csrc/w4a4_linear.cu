// W4A4 linear on sm_100a tensor cores (tcgen05, int8 MMA, TMEM accumulators).
//
//   C[m, n] = sum_g sA[m, g] * sW[n, g] * P[m, n, g],
//   P[m, n, g] = sum_{k in group g} qA[m, k] * qW[n, k]        (exact integers)
// [Hadamard-Int4-Accuracy wiki, Hypothesis: W4A4 is a same-precision int4 MAC; the
//  rotated operands A.Q and Q^T.B are group-quantised, A.B = (A.Q)(Q^T.B)].
//
// sm_100 has no 4-bit integer MMA, so codes are unpacked to int8 on the fly. The packed
// byte q[2j] | q[2j+1] << 4 gives 16*q[2j+1] as (byte & 0xF0) and 16*q[2j] as
// ((byte << 4) & 0xF0): both operands are fed as 16*q (products 256*q_a*q_w, still exact
// in int32), with the even codes of every 32-code chunk placed before the odd ones. The
// same K permutation is applied to both operands, so every group sum is unchanged.
//
// Tile: 128 rows of A x 256 rows of W per CTA; K in blocks of 128 (one 128-byte swizzle
// atom of int8 per row), 4 UMMAs of K = 32 per block, 3-stage smem ring. (A 128 x 128 tile
// avoids the epilogue's register spills but re-reads A twice as often and measured slower.)
// Warp roles (512 threads, launched with 128 registers each). setmaxnreg acts on whole
// warpgroups, so roles are aligned to them: warpgroups 0-1 (epilogue) grow to 168 registers,
// warpgroups 2-3 (producers + MMA warp) shrink to 88: 256*168 + 256*88 = 512*128.
//   warps 0-7   epilogue: two warpgroups, 128 columns each; after each group they read
//               the int32 partials from TMEM, apply the group scales and accumulate in
//               fp32 registers (packed f32x2 FMAs);
//   warps 8-14  producers: load packed codes from global memory (register prefetch two
//               K-blocks ahead), unpack, store into the swizzled K-major smem layout, then
//               fence.proxy.async + mbarrier arrive;
//   warp 15     TMEM allocation and MMA issue (one elected lane).
// TMEM holds two group accumulators (2 x 256 columns). Before a group's MMAs accumulate
// into a buffer, the epilogue fills it with the bit pattern of 1.5 * 2^23; adding the
// integer partial sum 256*P keeps the exponent, so the accumulator bits read back as the
// fp32 value 1.5 * 2^23 + 256*P: fma(u, sW/256, -1.5*2^23*sW/256) then gives P*sW exactly,
// with no integer-to-float conversion. (|256*P| < 2^22 requires G <= 256.)
//
// Every mbarrier wait is bounded (about 2 s of wall time); a wait that gives up records
// ROT_ETIMEOUT in a device flag, and the CTA skips its remaining work and exits.
#include <cstdint>

#include "rot_internal.cuh"

namespace rotb {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KB = 128;                  // K elements per stage
constexpr int STAGES = 3;
constexpr int A_STAGE_BYTES = BM * KB;   // unpacked int8
constexpr int B_STAGE_BYTES = BN * KB;
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int N_EPI = 256;               // epilogue threads (2 warpgroups)
constexpr int N_PROD = 224;              // producer threads
constexpr int THREADS = N_EPI + N_PROD + 32;
constexpr int N_CHUNKS = (BM + BN) * (KB / 32);                  // 16-byte packed chunks / stage
constexpr int PROD_CHUNKS = (N_CHUNKS + N_PROD - 1) / N_PROD;     // per producer thread
constexpr int EPI_COLS = BN / 2;         // columns per epilogue warpgroup
constexpr int MMA_WARP = (N_EPI + N_PROD) / 32;
constexpr int LAUNCH_REGS = 128;         // 65536 / THREADS
constexpr int EPI_REGS = 168, PROD_REGS = 88;  // per warpgroup role
static_assert(THREADS == 512, "register split assumes 512 threads");
static_assert(N_EPI == 256 && N_PROD + 32 == 256, "roles must fill whole warpgroups");
static_assert(N_EPI * EPI_REGS + (N_PROD + 32) * PROD_REGS <= THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t TMEM_COLS = 2 * BN;   // two group accumulators (all 512 columns)
constexpr uint32_t BIAS_BITS = 0x4B400000u;  // 1.5 * 2^23
constexpr float BIAS_F = 12582912.0f;
constexpr unsigned long long WAIT_NS = 2000000000ull;

// smem layout (offsets from a 1024-byte aligned base)
constexpr int OFF_STAGES = 0;
constexpr int OFF_SCALES = STAGES * STAGE_BYTES;          // [2][2][BN] fp32: sW/256 and -1.5*2^23*sW/256
constexpr int OFF_BARS = OFF_SCALES + 2 * BN * 8;
constexpr int OFF_TMEM = OFF_BARS + 16 * 8;
constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;          // + alignment slack

__device__ int g_w4a4_error = 0;

struct Params {
  const uint8_t* Aq;
  const uint16_t* As;
  const uint8_t* Wq;
  const uint16_t* Ws;
  void* C;
  int32_t* P;
  int M, N, K, G;
  int c_bf16;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait for the phase with the given parity; returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint32_t addr = smem_u32(bar);
  uint32_t done = 0;
  unsigned long long t0 = 0;
  for (uint32_t it = 0;; ++it) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity), "r"(20000u)   // suspend up to 20 us per try (no spinning)
        : "memory");
    if (done) return true;
    if ((it & 7) == 7) {
      if (*abort_flag) return false;
      unsigned long long now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      else if (now - t0 > WAIT_NS) {
        *abort_flag = 1;
        atomicExch(&g_w4a4_error, (int)ROT_ETIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// K-major, 128-byte swizzled operand descriptor (rows of 128 bytes, 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);        // start address
  d |= (uint64_t)1u << 16;                         // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024u >> 4) << 32;               // stride byte offset: 8-row atom pitch
  d |= (uint64_t)1u << 46;                         // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                         // SWIZZLE_128B
  return d;
}

// int8 x int8 -> int32, K-major A and B, M = 128, N = BN.
constexpr uint32_t IDESC = (2u << 4)            // D format: s32
                           | (1u << 7)          // A: signed int8
                           | (1u << 10)         // B: signed int8
                           | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(IDESC), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st16_const(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Ordered shared-memory vector load: kept next to the TMEM load it serves, so the scale loads
// of all column chunks are not hoisted ahead (which would need a register per loaded value).
__device__ __forceinline__ float4 lds128(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

template <bool PARTIALS>
__global__ void __launch_bounds__(THREADS, 1) w4a4_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BARS);
  uint64_t* full = bars;                 // [STAGES] producers -> MMA
  uint64_t* empty = bars + STAGES;       // [STAGES] MMA commit -> producers
  uint64_t* tfull = bars + 2 * STAGES;   // [2] MMA commit -> epilogue
  uint64_t* tempty = bars + 2 * STAGES + 2;  // [2] epilogue -> MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_TMEM + 8);
  float* sc = reinterpret_cast<float*>(smem + OFF_SCALES);  // [buf][0: sW/256, 1: c][BN]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int KS = p.K / 32;                 // UMMA k-steps
  const int NKB = (p.K + KB - 1) / KB;     // K blocks
  const int NG = p.K / p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], N_PROD);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], N_EPI);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < N_EPI / 32) {
    // ======================= epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 168;");
    const int wg = warp >> 2;                 // column block of EPI_COLS
    const int row = (warp & 3) * 32 + lane;   // TMEM lane = tile row
    const int m = m0 + row;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int ep_tid = threadIdx.x;           // 0..N_EPI-1
    // initial bias in both accumulators, then release them to the MMA warp
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int c = 0; c < EPI_COLS / 16; ++c) tmem_st16_const(lane_addr + b * BN + wg * EPI_COLS + c * 16, BIAS_BITS);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&tempty[0]);
    mbar_arrive(&tempty[1]);

    // fp32 accumulators as pairs of adjacent columns
    float2 acc[EPI_COLS / 2];
#pragma unroll
    for (int j = 0; j < EPI_COLS / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
    const bool row_ok = m < p.M;
    const int n_col = n0 + ep_tid;            // the column whose scale this thread stages
    // scales of the next group are fetched one group ahead
    float sw_next = 0.0f, sa_next = 0.0f;
    if (!PARTIALS) {
      if (ep_tid < BN && n_col < p.N) sw_next = __half2float(__ushort_as_half(p.Ws[(int64_t)n_col * NG]));
      if (row_ok) sa_next = __half2float(__ushort_as_half(p.As[(int64_t)m * NG]));
    }
    bool ok = true;
    for (int g = 0; g < NG; ++g) {
      const float sa = sa_next;
      if (!PARTIALS) {
        if (ep_tid < BN) {
          const float sw = sw_next * (1.0f / 256.0f);
          sc[((g & 1) * 2 + 0) * BN + ep_tid] = sw;
          sc[((g & 1) * 2 + 1) * BN + ep_tid] = -BIAS_F * sw;
        }
        if (g + 1 < NG) {
          if (ep_tid < BN && n_col < p.N) sw_next = __half2float(__ushort_as_half(p.Ws[(int64_t)n_col * NG + g + 1]));
          if (row_ok) sa_next = __half2float(__ushort_as_half(p.As[(int64_t)m * NG + g + 1]));
        }
      }
      named_bar(1, N_EPI);
      const int b = g & 1;
      if (!ok || !mbar_wait(&tfull[b], (g >> 1) & 1, abort_flag)) { ok = false; continue; }
      tc_fence_after();
      const uint32_t base = lane_addr + b * BN + wg * EPI_COLS;
      const float* scw = sc + ((g & 1) * 2 + 0) * BN + wg * EPI_COLS;
      const float* scc = sc + ((g & 1) * 2 + 1) * BN + wg * EPI_COLS;
      const float2 sa2 = make_float2(sa, sa);
#pragma unroll
      for (int c = 0; c < EPI_COLS / 8; ++c) {
        uint32_t rr[8];
        tmem_ld8(base + c * 8, rr);
        tmem_wait_ld();
        if constexpr (!PARTIALS) {
#pragma unroll
          for (int j = 0; j < 8; j += 4) {
            const float4 w4 = lds128(scw + c * 8 + j);
            const float4 c4 = lds128(scc + c * 8 + j);
            const float2 u0 = make_float2(__uint_as_float(rr[j]), __uint_as_float(rr[j + 1]));
            const float2 u1 = make_float2(__uint_as_float(rr[j + 2]), __uint_as_float(rr[j + 3]));
            // exact P*sW (the bias cancels inside one rounding), then acc += (P*sW)*sA
            const float2 t0 = __ffma2_rn(u0, make_float2(w4.x, w4.y), make_float2(c4.x, c4.y));
            const float2 t1 = __ffma2_rn(u1, make_float2(w4.z, w4.w), make_float2(c4.z, c4.w));
            acc[(c * 8 + j) / 2] = __ffma2_rn(t0, sa2, acc[(c * 8 + j) / 2]);
            acc[(c * 8 + j) / 2 + 1] = __ffma2_rn(t1, sa2, acc[(c * 8 + j) / 2 + 1]);
          }
        } else {
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int n = n0 + wg * EPI_COLS + c * 8 + j;
              if (n < p.N) p.P[((int64_t)m * p.N + n) * NG + g] = ((int32_t)(rr[j] - BIAS_BITS)) / 256;
            }
          }
        }
      }
      // reset the accumulator to the bias for the group after next, then release it
#pragma unroll
      for (int c = 0; c < EPI_COLS / 16; ++c) tmem_st16_const(base + c * 16, BIAS_BITS);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&tempty[b]);
    }
    if (!PARTIALS && ok && row_ok) {
      const int nb = n0 + wg * EPI_COLS;
      if (!p.c_bf16) {
        float* crow = static_cast<float*>(p.C) + (int64_t)m * p.N + nb;
#pragma unroll
        for (int j = 0; j < EPI_COLS; j += 4)
          if (nb + j < p.N)
            *reinterpret_cast<float4*>(crow + j) =
                make_float4(acc[j / 2].x, acc[j / 2].y, acc[j / 2 + 1].x, acc[j / 2 + 1].y);
      } else {
        __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(p.C) + (int64_t)m * p.N + nb;
#pragma unroll
        for (int j = 0; j < EPI_COLS; j += 8) {
          if (nb + j < p.N) {
            uint4 v;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j / 2].x, acc[j / 2].y);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j / 2 + 1].x, acc[j / 2 + 1].y);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j / 2 + 2].x, acc[j / 2 + 2].y);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j / 2 + 3].x, acc[j / 2 + 3].y);
            v.x = *reinterpret_cast<uint32_t*>(&h0);
            v.y = *reinterpret_cast<uint32_t*>(&h1);
            v.z = *reinterpret_cast<uint32_t*>(&h2);
            v.w = *reinterpret_cast<uint32_t*>(&h3);
            *reinterpret_cast<uint4*>(crow + j) = v;
          }
        }
      }
    }
  } else if (warp < MMA_WARP) {
    // ======================= producers
    asm volatile("setmaxnreg.dec.sync.aligned.u32 88;");
    const int pt = threadIdx.x - N_EPI;    // 0..N_PROD-1
    const int64_t ldp = p.K / 2;           // packed bytes per row
    // chunk q = pt + N_PROD*i: rows 0..BM-1 of A then 0..BN-1 of W, 4 chunks (16 B = 32 codes)
    // per row. The global row pointers are fixed for the CTA; nullptr marks rows beyond M / N.
    const uint8_t* gsrc[PROD_CHUNKS];
#pragma unroll
    for (int i = 0; i < PROD_CHUNKS; ++i) {
      const int q = pt + N_PROD * i;
      const int r = q >> 2, c = q & 3;
      const uint8_t* src = nullptr;
      if (q < N_CHUNKS) {
        if (r < BM) {
          if (m0 + r < p.M) src = p.Aq + (int64_t)(m0 + r) * ldp + c * 16;
        } else {
          if (n0 + r - BM < p.N) src = p.Wq + (int64_t)(n0 + r - BM) * ldp + c * 16;
        }
      }
      gsrc[i] = src;
    }
    auto load = [&](int kb, uint4 (&dst)[PROD_CHUNKS]) {
      const int64_t koff = (int64_t)kb * (KB / 2);
#pragma unroll
      for (int i = 0; i < PROD_CHUNKS; ++i) {
        const int c = (pt + N_PROD * i) & 3;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (gsrc[i] != nullptr && koff + c * 16 < ldp) v = __ldg(reinterpret_cast<const uint4*>(gsrc[i] + koff));
        dst[i] = v;
      }
    };
    // unpack one stage from registers, publish it, then refill the registers with K-block kb+2
    auto stage = [&](int kb, uint4 (&cur)[PROD_CHUNKS]) -> bool {
      const int s = kb % STAGES;
      if (kb >= STAGES && !mbar_wait(&empty[s], ((kb / STAGES) + 1) & 1, abort_flag)) return false;
      uint8_t* st = smem + OFF_STAGES + s * STAGE_BYTES;
#pragma unroll
      for (int i = 0; i < PROD_CHUNKS; ++i) {
        const int q = pt + N_PROD * i;
        if (q >= N_CHUNKS) continue;
        const int r = q >> 2, c = q & 3;
        uint8_t* tile = r < BM ? st : st + A_STAGE_BYTES;
        const int rr = r < BM ? r : r - BM;
        const uint4 w = cur[i];
        const uint4 lo = make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u, (w.z << 4) & 0xF0F0F0F0u,
                                    (w.w << 4) & 0xF0F0F0F0u);
        const uint4 hi = make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
        uint8_t* rowp = tile + (rr >> 3) * 1024 + (rr & 7) * 128;
        *reinterpret_cast<uint4*>(rowp + (((2 * c) ^ (rr & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(rowp + (((2 * c + 1) ^ (rr & 7)) << 4)) = hi;
      }
      fence_proxy_async();
      mbar_arrive(&full[s]);
      if (kb + 2 < NKB) load(kb + 2, cur);
      return true;
    };
    uint4 b0[PROD_CHUNKS], b1[PROD_CHUNKS];
    load(0, b0);
    if (NKB > 1) load(1, b1);
    for (int kb = 0; kb < NKB; kb += 2) {
      if (!stage(kb, b0)) break;
      if (kb + 1 < NKB && !stage(kb + 1, b1)) break;
    }
  } else {
    // ======================= MMA issue
    asm volatile("setmaxnreg.dec.sync.aligned.u32 88;");  // same value as the producers of its warpgroup
    const bool leader = lane == 0;
    const uint32_t sbase = smem_u32(smem + OFF_STAGES);
    for (int ks = 0; ks < KS; ++ks) {
      const int kb = ks >> 2, k4 = ks & 3, s = kb % STAGES;
      if (k4 == 0) {
        if (!mbar_wait(&full[s], (kb / STAGES) & 1, abort_flag)) break;
        tc_fence_after();
      }
      const int g = (ks * 32) / p.G;
      const bool first = (ks * 32) % p.G == 0;
      const bool last = ((ks + 1) * 32) % p.G == 0;
      const int b = g & 1;
      if (first) {
        if (!mbar_wait(&tempty[b], (g >> 1) & 1, abort_flag)) break;
        tc_fence_after();
      }
      if (leader) {
        const uint32_t a_addr = sbase + s * STAGE_BYTES + k4 * 32;
        const uint32_t b_addr = sbase + s * STAGE_BYTES + A_STAGE_BYTES + k4 * 32;
        umma_i8(tmem + b * BN, make_desc(a_addr), make_desc(b_addr), 1u);
        if (last) umma_commit(&tfull[b]);
        if (k4 == 3 || ks == KS - 1) umma_commit(&empty[s]);
      }
      __syncwarp();
    }
    // the last stage-release commit must have landed before the CTA (and its smem) goes away
    if (!*abort_flag && NKB > 0) {
      const int kl = NKB - 1;
      mbar_wait(&empty[kl % STAGES], (kl / STAGES) & 1, abort_flag);
    }
  }

  __syncthreads();
  if (warp == MMA_WARP) {
    if (*abort_flag) {
      // let any in-flight MMA drain before the columns are released
      unsigned long long t0, now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
      do { asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now)); } while (now - t0 < 1000000ull);
    }
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace

rot_status w4a4_launch(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq, const uint16_t* Ws, int64_t M,
                       int64_t N, int64_t K, int G, void* C, int c_dtype, int32_t* partials, cudaStream_t s) {
  if (G > 256) return set_error(ROT_EUNSUPPORTED, "w4a4_linear: G > 256 is not supported");
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return set_error(ROT_EUNSUPPORTED, "w4a4_linear: size too large");
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    // The setmaxnreg split is only valid for the register count it was sized for: refuse
    // to launch otherwise (an over-subscribed split would wait for registers forever).
    for (int v = 0; v < 2; ++v) {
      const void* k = v ? (const void*)w4a4_kernel<true> : (const void*)w4a4_kernel<false>;
      cudaFuncAttributes fa;
      ROT_CUDA_TRY(cudaFuncGetAttributes(&fa, k));
      if (fa.numRegs != LAUNCH_REGS)
        return set_error(ROT_EUNSUPPORTED, "w4a4_linear: kernel built with an unexpected register count");
      ROT_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    }
    configured[dev] = 1;
  }
  Params p{};
  p.Aq = Aq;
  p.As = As;
  p.Wq = Wq;
  p.Ws = Ws;
  p.C = C;
  p.P = partials;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.G = G;
  p.c_bf16 = c_dtype == ROT_BF16;
  dim3 grid((unsigned)((N + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
  if (partials) w4a4_kernel<true><<<grid, THREADS, SMEM_BYTES, s>>>(p);
  else w4a4_kernel<false><<<grid, THREADS, SMEM_BYTES, s>>>(p);
  ROT_CUDA_TRY(cudaGetLastError());
  return ROT_OK;
}

rot_status w4a4_fetch_device_error() {
  int v = 0;
  ROT_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_w4a4_error, sizeof(int)));
  if (v) {
    int z = 0;
    ROT_CUDA_TRY(cudaMemcpyToSymbol(g_w4a4_error, &z, sizeof(int)));
    return set_error((rot_status)v, "a bounded device wait in w4a4_linear gave up");
  }
  return ROT_OK;
}

}  // namespace rotb

extern "C" rot_status rot_check_device(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return rotb::cuda_error(e, "rot_check_device");
  rot_status st = rotb::fwht_fetch_device_error();
  rot_status st2 = rotb::w4a4_fetch_device_error();
  return st != ROT_OK ? st : st2;
}

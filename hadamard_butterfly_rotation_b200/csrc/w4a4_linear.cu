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
// atom of int8 per row), 4 UMMAs of K = 32 per block.
// Warp roles (512 threads, launched with 128 registers each). setmaxnreg acts on whole
// warpgroups, so roles are aligned to them: warpgroups 0-1 (epilogue) grow to 168 registers,
// warpgroups 2-3 (producers + MMA warp) shrink to 88: 256*168 + 256*88 = 512*128.
//   warps 0-7   epilogue: two warpgroups, 128 columns each; after each group they read
//               the int32 partials from TMEM, apply the group scales and accumulate in
//               fp32 registers;
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
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t BIAS_BITS = 0x4B400000u;  // 1.5 * 2^23
constexpr float BIAS_F = 12582912.0f;
constexpr unsigned long long WAIT_NS = 2000000000ull;

// smem layout (offsets from a 1024-byte aligned base)
constexpr int OFF_STAGES = 0;
constexpr int OFF_SCALES = STAGES * STAGE_BYTES;          // [2][BN] float2 (sW/256, -bias*sW/256)
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
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    if ((it & 63) == 63) {
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

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
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

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

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
  float2* sc = reinterpret_cast<float2*>(smem + OFF_SCALES);

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

    float acc[EPI_COLS];
#pragma unroll
    for (int j = 0; j < EPI_COLS; ++j) acc[j] = 0.0f;
    const bool row_ok = m < p.M;
    const int n_col = n0 + ep_tid;            // the column whose scale this thread stages
    bool ok = true;
    for (int g = 0; g < NG; ++g) {
      // stage the column scales of group g: (sW/256, -1.5*2^23 * sW/256)
      if (p.Ws && ep_tid < BN) {
        float sw = 0.0f;
        if (n_col < p.N) sw = __half2float(__ushort_as_half(p.Ws[(int64_t)n_col * NG + g])) * (1.0f / 256.0f);
        sc[(g & 1) * BN + ep_tid] = make_float2(sw, -BIAS_F * sw);
      }
      const float sa = (p.As && row_ok) ? __half2float(__ushort_as_half(p.As[(int64_t)m * NG + g])) : 0.0f;
      named_bar(1, N_EPI);
      const int b = g & 1;
      if (!ok || !mbar_wait(&tfull[b], (g >> 1) & 1, abort_flag)) { ok = false; continue; }
      tc_fence_after();
      const uint32_t base = lane_addr + b * BN + wg * EPI_COLS;
      const float2* scg = sc + (g & 1) * BN + wg * EPI_COLS;
      uint32_t rr[16];
#pragma unroll
      for (int c = 0; c < EPI_COLS / 16; ++c) {
        tmem_ld16(base + c * 16, rr);
        tmem_wait_ld();
        if (p.P == nullptr) {
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float4 s2 = *reinterpret_cast<const float4*>(scg + c * 16 + j);
            const float t0 = fmaf(__uint_as_float(rr[j]), s2.x, s2.y);
            const float t1 = fmaf(__uint_as_float(rr[j + 1]), s2.z, s2.w);
            acc[c * 16 + j] = fmaf(t0, sa, acc[c * 16 + j]);
            acc[c * 16 + j + 1] = fmaf(t1, sa, acc[c * 16 + j + 1]);
          }
        } else if (row_ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + wg * EPI_COLS + c * 16 + j;
            if (n < p.N) p.P[((int64_t)m * p.N + n) * NG + g] = ((int32_t)(rr[j] - BIAS_BITS)) / 256;
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
    if (ok && p.P == nullptr && row_ok) {
      const int nb = n0 + wg * EPI_COLS;
      if (!p.c_bf16) {
        float* crow = static_cast<float*>(p.C) + (int64_t)m * p.N + nb;
#pragma unroll
        for (int j = 0; j < EPI_COLS; j += 4)
          if (nb + j < p.N) *reinterpret_cast<float4*>(crow + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
      } else {
        __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(p.C) + (int64_t)m * p.N + nb;
#pragma unroll
        for (int j = 0; j < EPI_COLS; j += 8) {
          if (nb + j < p.N) {
            uint4 v;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j], acc[j + 1]);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
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
    // chunk q = pt + N_PROD*i: rows 0..BM-1 of A then 0..BN-1 of W, 4 chunks (16 B = 32 codes) per row
    auto load = [&](int kb, uint4 (&dst)[PROD_CHUNKS]) {
#pragma unroll
      for (int i = 0; i < PROD_CHUNKS; ++i) {
        const int q = pt + N_PROD * i;
        const int r = q >> 2, c = q & 3;
        const int64_t kbyte = (int64_t)kb * (KB / 2) + c * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (q >= N_CHUNKS) {
        } else if (r < BM) {
          const int mm = m0 + r;
          if (mm < p.M && kbyte < ldp) v = __ldg(reinterpret_cast<const uint4*>(p.Aq + (int64_t)mm * ldp + kbyte));
        } else {
          const int nn = n0 + r - BM;
          if (nn < p.N && kbyte < ldp) v = __ldg(reinterpret_cast<const uint4*>(p.Wq + (int64_t)nn * ldp + kbyte));
        }
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
    cudaFuncAttributes fa;
    ROT_CUDA_TRY(cudaFuncGetAttributes(&fa, w4a4_kernel));
    if (fa.numRegs != LAUNCH_REGS)
      return set_error(ROT_EUNSUPPORTED, "w4a4_linear: kernel built with an unexpected register count");
    ROT_CUDA_TRY(cudaFuncSetAttribute(w4a4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
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
  w4a4_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(p);
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

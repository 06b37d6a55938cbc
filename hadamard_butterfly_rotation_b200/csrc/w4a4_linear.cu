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
// atom of int8 per row), 4 UMMAs of K = 32 per block, 3-stage ring of unpacked int8 tiles fed
// by a 2-stage ring of packed tiles. (A 128 x 128 tile re-reads A twice as often and
// measured slower.)
// Warp roles (512 threads, launched with 128 registers each). setmaxnreg acts on whole
// warpgroups, so roles are aligned to them: warpgroups 0-1 (epilogue) grow to 216 registers,
// warpgroups 2-3 (loader, unpackers, MMA warp) shrink to 40: 256*216 + 256*40 = 512*128.
//   warps 0-7   epilogue: two warpgroups, 128 columns each; after each group they read
//               the int32 partials from TMEM (32 columns per load), apply the group scales
//               and accumulate in fp32 registers (packed f32x2 FMAs);
//   warp 8      loader: one bulk copy (cp.async.bulk) per tile row and K-block brings the
//               packed codes into the packed ring, completing on an mbarrier;
//   warps 9-14  unpackers: read a packed stage from shared memory, unpack, store into the
//               swizzled K-major int8 layout, fence.proxy.async, then release both stages;
//   warp 15     TMEM allocation and MMA issue (one elected lane).
// Measured on B200 at M=2048, N=K=4096 (timestamps and role-by-role variants): the MMA warp
// alone reaches 1529 TOPS; the epilogue's per-group TMEM traffic (read 256 partial columns,
// rewrite the bias) slows the MMAs on the other accumulator several-fold while it runs, so
// at G = 128 the epilogue's TMEM time, not the unpacking, bounds the kernel (G = 256 halves
// it). Per-row bulk copies of the packed codes were 5x slower than the two 2-D TMA boxes.
// TMEM holds two group accumulators (2 x 256 columns); a group's first MMA overwrites its
// accumulator. The epilogue adds the bit pattern of 1.5 * 2^23 to the int32 partial 256*P
// (one integer add): the sum is the bit pattern of the fp32 value 1.5 * 2^23 + 256*P, and
// fma(u, sW/256, -1.5*2^23*sW/256) then gives P*sW exactly, with no integer-to-float
// conversion. (|256*P| < 2^22 requires G <= 256.)
//
// Every mbarrier wait is bounded (about 2 s of wall time); a wait that gives up records
// ROT_ETIMEOUT in a device flag, and the CTA skips its remaining work and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>

#include "rot_internal.cuh"

namespace rotb {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KB = 128;                  // K elements per stage
constexpr int STAGES = 3;                // unpacked int8 stages
constexpr int PSTAGES = 2;               // packed stages
constexpr int A_STAGE_BYTES = BM * KB;   // unpacked int8
constexpr int B_STAGE_BYTES = BN * KB;
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int PROW_BYTES = KB / 2;       // packed bytes of one row in one K-block
constexpr int PSTAGE_BYTES = (BM + BN) * PROW_BYTES;
constexpr int N_EPI = 256;               // epilogue threads (2 warpgroups)
constexpr int LOADER_WARP = N_EPI / 32;  // warp 8
constexpr int N_UNP = 192;               // unpacker threads (warps 9-14)
constexpr int N_UNP_WARPS = N_UNP / 32;
constexpr int THREADS = N_EPI + 32 + N_UNP + 32;
constexpr int N_CHUNKS = (BM + BN) * (KB / 32);                  // 16-byte packed chunks / stage
constexpr int UNP_CHUNKS = N_CHUNKS / N_UNP;                     // per unpacker thread
constexpr int EPI_COLS = BN / 2;         // columns per epilogue warpgroup
constexpr int MMA_WARP = (N_EPI + 32 + N_UNP) / 32;
constexpr int LAUNCH_REGS = 128;         // 65536 / THREADS
constexpr int EPI_REGS = 216, PROD_REGS = 40;  // per warpgroup role
static_assert(THREADS == 512, "register split assumes 512 threads");
static_assert(N_CHUNKS % N_UNP == 0, "unpack work divides evenly");
static_assert(N_EPI * EPI_REGS + (THREADS - N_EPI) * PROD_REGS <= THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t TMEM_COLS = 2 * BN;   // two group accumulators (all 512 columns)
constexpr uint32_t BIAS_BITS = 0x4B400000u;  // 1.5 * 2^23
constexpr float BIAS_F = 12582912.0f;
constexpr unsigned long long WAIT_NS = 2000000000ull;

// smem layout (offsets from a 1024-byte aligned base)
constexpr int OFF_STAGES = 0;
constexpr int OFF_PSTAGES = STAGES * STAGE_BYTES;
constexpr int OFF_SCALES = OFF_PSTAGES + PSTAGES * PSTAGE_BYTES;  // [2][2][BN] fp32: sW/256, -1.5*2^23*sW/256
constexpr int OFF_BARS = OFF_SCALES + 2 * BN * 8;
constexpr int OFF_TMEM = OFF_BARS + 16 * 8;
constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;          // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

__device__ int g_w4a4_error = 0;

// Static split-K accumulation buffer for w4a4_linear_noalloc (bf16 output on the split path).
__device__ __align__(256) float g_w4a4_scratch[W4A4_NOALLOC_SCRATCH_FLOATS];

struct Params {
  CUtensorMap tmA;   // packed A codes [M, K/2] uint8, box {64 bytes, BM rows}
  CUtensorMap tmW;   // packed W codes [N, K/2] uint8, box {64 bytes, BN rows}
  const uint8_t* Aq;
  const uint16_t* As;
  const uint8_t* Wq;
  const uint16_t* Ws;
  void* C;
  int32_t* P;
  int M, N, K, G;
  int c_bf16;
  int kb_per_split;  // K-blocks per split (blockIdx.z); a multiple of the K-blocks per group
  float* Cacc;       // split-K: fp32 [M, N] accumulated with atomics (zeroed beforehand), else null
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

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// 2-D tiled TMA load (no multicast) of box (x, y) of `tmap` into shared memory; the box's
// bytes (out-of-range elements zero-filled) complete on `bar`
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Warp-uniform bounded wait: lane 0 waits on the mbarrier, the result is broadcast and the
// warp re-converges (its memory accesses are ordered after lane 0's acquire by __syncwarp).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int lane) {
  int w = 1;
  if (lane == 0) w = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
  w = __shfl_sync(0xffffffffu, w, 0);
  __syncwarp();
  return w != 0;
}

template <bool PARTIALS>
__global__ void __launch_bounds__(THREADS, 1) w4a4_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BARS);
  uint64_t* full = bars;                      // [STAGES]  unpackers -> MMA (one arrival per warp)
  uint64_t* empty = bars + STAGES;            // [STAGES]  MMA commit -> unpackers
  uint64_t* tfull = bars + 2 * STAGES;        // [2]       MMA commit -> epilogue
  uint64_t* tempty = bars + 2 * STAGES + 2;   // [2]       epilogue -> MMA
  uint64_t* pfull = bars + 2 * STAGES + 4;    // [PSTAGES] bulk copies -> unpackers
  uint64_t* pempty = bars + 2 * STAGES + 4 + PSTAGES;  // [PSTAGES] unpackers -> loader
  static_assert(2 * STAGES + 4 + 2 * PSTAGES <= 16, "barrier slots");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_TMEM + 8);
  float* sc = reinterpret_cast<float*>(smem + OFF_SCALES);  // [buf][0: sW/256, 1: c][BN]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int NG = p.K / p.G;                // groups of the whole K (scale row length)
  // this CTA's K range (split-K over blockIdx.z; the split is at group boundaries)
  const int NKB_ALL = (p.K + KB - 1) / KB;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int kb1 = min(NKB_ALL, kb0 + p.kb_per_split);
  const int NKB = kb1 - kb0;                       // K blocks of this CTA
  const int ks0 = kb0 * (KB / 32);
  const int KS = min(p.K / 32, kb1 * (KB / 32)) - ks0;   // UMMA k-steps of this CTA
  const int g0 = (ks0 * 32) / p.G;                 // first group
  const int NGL = (KS * 32) / p.G;                 // groups of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], N_UNP_WARPS);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], N_EPI);
    }
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], N_UNP_WARPS);
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
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;");
    const int wg = warp >> 2;                 // column block of EPI_COLS
    const int row = (warp & 3) * 32 + lane;   // TMEM lane = tile row
    const int m = m0 + row;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int ep_tid = threadIdx.x;           // 0..N_EPI-1
    // both accumulators start free (a group's first MMA overwrites its accumulator)
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
      if (ep_tid < BN && n_col < p.N) sw_next = __half2float(__ushort_as_half(p.Ws[(int64_t)n_col * NG + g0]));
      if (row_ok) sa_next = __half2float(__ushort_as_half(p.As[(int64_t)m * NG + g0]));
    }
    bool ok = true;
    for (int gl = 0; gl < NGL; ++gl) {
      const int g = g0 + gl;
      const float sa = sa_next;
      if (!PARTIALS) {
        if (ep_tid < BN) {
          const float sw = sw_next * (1.0f / 256.0f);
          sc[((gl & 1) * 2 + 0) * BN + ep_tid] = sw;
          sc[((gl & 1) * 2 + 1) * BN + ep_tid] = -BIAS_F * sw;
        }
        if (gl + 1 < NGL) {
          if (ep_tid < BN && n_col < p.N) sw_next = __half2float(__ushort_as_half(p.Ws[(int64_t)n_col * NG + g + 1]));
          if (row_ok) sa_next = __half2float(__ushort_as_half(p.As[(int64_t)m * NG + g + 1]));
        }
      }
      named_bar(1, N_EPI);
      const int b = gl & 1;
      ok = ok && warp_wait(&tfull[b], (gl >> 1) & 1, abort_flag, lane);   // warp-uniform
      if (!ok) continue;
      tc_fence_after();
      const uint32_t base = lane_addr + b * BN + wg * EPI_COLS;
      const float* scw = sc + ((gl & 1) * 2 + 0) * BN + wg * EPI_COLS;
      const float* scc = sc + ((gl & 1) * 2 + 1) * BN + wg * EPI_COLS;
      const float2 sa2 = make_float2(sa, sa);
#pragma unroll
      for (int c = 0; c < EPI_COLS / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(base + c * 32, rr);
        tmem_wait_ld();
        if constexpr (!PARTIALS) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 w4 = lds128(scw + c * 32 + j);
            const float4 c4 = lds128(scc + c * 32 + j);
            // 256*P + bits(1.5 * 2^23) = bits of the float 1.5 * 2^23 + 256*P
            const float2 u0 = make_float2(__uint_as_float(rr[j] + BIAS_BITS), __uint_as_float(rr[j + 1] + BIAS_BITS));
            const float2 u1 =
                make_float2(__uint_as_float(rr[j + 2] + BIAS_BITS), __uint_as_float(rr[j + 3] + BIAS_BITS));
            // exact P*sW (the bias cancels inside one rounding), then acc += (P*sW)*sA
            const float2 t0 = __ffma2_rn(u0, make_float2(w4.x, w4.y), make_float2(c4.x, c4.y));
            const float2 t1 = __ffma2_rn(u1, make_float2(w4.z, w4.w), make_float2(c4.z, c4.w));
            acc[(c * 32 + j) / 2] = __ffma2_rn(t0, sa2, acc[(c * 32 + j) / 2]);
            acc[(c * 32 + j) / 2 + 1] = __ffma2_rn(t1, sa2, acc[(c * 32 + j) / 2 + 1]);
          }
        } else {
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int n = n0 + wg * EPI_COLS + c * 32 + j;
              if (n < p.N) p.P[((int64_t)m * p.N + n) * NG + g] = ((int32_t)rr[j]) / 256;
            }
          }
        }
      }
      // the partials are in registers: release the accumulator for the group after next
      tc_fence_before();
      mbar_arrive(&tempty[b]);
    }
    if (!PARTIALS && ok && row_ok) {
      const int nb = n0 + wg * EPI_COLS;
      if (p.Cacc) {
        // split-K: add this K range's contribution (fp32 vector atomics)
        float* crow = p.Cacc + (int64_t)m * p.N + nb;
#pragma unroll
        for (int j = 0; j < EPI_COLS; j += 4)
          if (nb + j < p.N)
            atomicAdd(reinterpret_cast<float4*>(crow + j),
                      make_float4(acc[j / 2].x, acc[j / 2].y, acc[j / 2 + 1].x, acc[j / 2 + 1].y));
      } else if (!p.c_bf16) {
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
  } else if (warp == LOADER_WARP) {
    // ======================= loader: the packed A and W tiles of one K-block -> packed stage
    // (two 2-D TMA boxes; rows beyond M / N and bytes beyond K/2 arrive as zeros)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    for (int j = 0; j < NKB; ++j) {
      const int kb = kb0 + j, ps = j % PSTAGES;
      if (j >= PSTAGES && !warp_wait(&pempty[ps], ((j / PSTAGES) + 1) & 1, abort_flag, lane)) break;
      if (lane == 0) {
        uint8_t* pst = smem + OFF_PSTAGES + ps * PSTAGE_BYTES;
        mbar_arrive_expect_tx(&pfull[ps], (uint32_t)PSTAGE_BYTES);
        // x = kb * 64 bytes: a multiple of 16, as a tiled TMA requires of the inner coordinate
        tma_load_2d(pst, &p.tmA, kb * PROW_BYTES, m0, &pfull[ps]);
        tma_load_2d(pst + BM * PROW_BYTES, &p.tmW, kb * PROW_BYTES, n0, &pfull[ps]);
      }
      __syncwarp();
    }
  } else if (warp < MMA_WARP) {
    // ======================= unpackers: packed stage -> swizzled int8 stage
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    const int ut = threadIdx.x - (LOADER_WARP + 1) * 32;   // 0..N_UNP-1
    for (int j = 0; j < NKB; ++j) {
      const int s = j % STAGES, ps = j % PSTAGES;
      if (!warp_wait(&pfull[ps], (j / PSTAGES) & 1, abort_flag, lane)) break;
      if (j >= STAGES && !warp_wait(&empty[s], ((j / STAGES) + 1) & 1, abort_flag, lane)) break;
      const uint8_t* pst = smem + OFF_PSTAGES + ps * PSTAGE_BYTES;
      uint8_t* st = smem + OFF_STAGES + s * STAGE_BYTES;
#pragma unroll 4
      for (int i = 0; i < UNP_CHUNKS; ++i) {
        // chunk q: row r (A rows 0..BM-1, then W rows), 16-byte piece c of the row's 64 bytes
        const int q = ut + N_UNP * i;
        const int r = q >> 2, c = q & 3;
        const uint4 w = *reinterpret_cast<const uint4*>(pst + q * 16);
        uint8_t* tile = r < BM ? st : st + A_STAGE_BYTES;
        const int rr = r < BM ? r : r - BM;
        const uint4 lo = make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u, (w.z << 4) & 0xF0F0F0F0u,
                                    (w.w << 4) & 0xF0F0F0F0u);
        const uint4 hi = make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
        uint8_t* rowp = tile + (rr >> 3) * 1024 + (rr & 7) * 128;
        *reinterpret_cast<uint4*>(rowp + (((2 * c) ^ (rr & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(rowp + (((2 * c + 1) ^ (rr & 7)) << 4)) = hi;
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full[s]);
        mbar_arrive(&pempty[ps]);
      }
    }
  } else {
    // ======================= MMA issue
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");  // same value as the rest of its warpgroup
    const bool leader = lane == 0;
    const uint32_t sbase = smem_u32(smem + OFF_STAGES);
    for (int ks = 0; ks < KS; ++ks) {
      // local k-step / K-block / group indices drive the rings; the split is group-aligned
      const int kb = ks >> 2, k4 = ks & 3, s = kb % STAGES;
      if (k4 == 0) {
        if (!mbar_wait(&full[s], (kb / STAGES) & 1, abort_flag)) break;
        tc_fence_after();
      }
      const int gl = (ks * 32) / p.G;
      const bool first = (ks * 32) % p.G == 0;
      const bool last = ((ks + 1) * 32) % p.G == 0;
      const int b = gl & 1;
      if (first) {
        if (!mbar_wait(&tempty[b], (gl >> 1) & 1, abort_flag)) break;
        tc_fence_after();
      }
      if (leader) {
        const uint32_t a_addr = sbase + s * STAGE_BYTES + k4 * 32;
        const uint32_t b_addr = sbase + s * STAGE_BYTES + A_STAGE_BYTES + k4 * 32;
        umma_i8(tmem + b * BN, make_desc(a_addr), make_desc(b_addr), first ? 0u : 1u);
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
      // let any in-flight MMA or bulk copy drain before the columns and smem are released
      unsigned long long t0, now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
      do { asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now)); } while (now - t0 < 1000000ull);
    }
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace

// ---------------------------------------------------------------- decode-sized M
// For M <= 64 the contraction is a weight stream: every weight byte is used by at most 64
// tokens. One warp owns 8 weight rows (an n-tile) over a K range; per 64-byte span (128
// codes) of those rows each lane loads one 16-byte piece of its row (lanes 4g..4g+3 cover
// row g), unpacks it to 16*q int8 words (even codes, odd codes), and feeds four
// mma.sync.m16n8k32 s8 MMAs per 16-token tile. A span's 128 codes are split over the four
// MMAs in an order that both operands share, so every group sum is unchanged; the int32
// group partials stay in registers, and the epilogue per group is 4 FMAs per lane.
// Needs G % 128 == 0; the K range of a warp is a whole number of groups.
constexpr int DEC_THREADS = 256;
constexpr int DEC_MAXMT = 4;   // 16-token tiles

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct DecParams {
  const uint8_t* Aq;
  const uint16_t* As;
  const uint8_t* Wq;
  const uint16_t* Ws;
  void* C;           // output when splits == 1
  float* Cacc;       // fp32 accumulation target (zeroed) when splits > 1
  int M, N, K, G;
  int c_bf16;
  int groups_per_split;
};

template <int MT>
__global__ void __launch_bounds__(DEC_THREADS) w4a4_decode_kernel(const DecParams p) {
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int g = l >> 2, c = l & 3;
  const int nt = blockIdx.x * (DEC_THREADS / 32) + warp;   // n-tile of 8 weight rows
  const int n0 = nt * 8;
  if (n0 >= p.N) return;
  const int NG = p.K / p.G;
  const int ga = blockIdx.y * p.groups_per_split;
  const int gb = min(NG, ga + p.groups_per_split);
  if (ga >= gb) return;
  const int64_t ldp = p.K / 2;
  const int spans_per_group = p.G / 128;
  const uint8_t* wrow = p.Wq + (int64_t)(n0 + g) * ldp + 16 * c;
  float acc[MT][4];
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;

  // the next span's weight piece is loaded one span ahead
  int span = ga * spans_per_group;
  const int span_end = gb * spans_per_group;
  uint4 wnext = __ldg(reinterpret_cast<const uint4*>(wrow + (int64_t)span * 64));
  for (int gg = ga; gg < gb; ++gg) {
    int d[MT][4];
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) d[t][i] = 0;
    for (int sp = 0; sp < spans_per_group; ++sp, ++span) {
      const uint4 wv = wnext;
      if (span + 1 < span_end) wnext = __ldg(reinterpret_cast<const uint4*>(wrow + (int64_t)(span + 1) * 64));
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int m_lo = t * 16 + g, m_hi = m_lo + 8;
        uint4 alo = make_uint4(0u, 0u, 0u, 0u), ahi = make_uint4(0u, 0u, 0u, 0u);
        if (m_lo < p.M) alo = __ldg(reinterpret_cast<const uint4*>(p.Aq + (int64_t)m_lo * ldp + (int64_t)span * 64 + 16 * c));
        if (m_hi < p.M) ahi = __ldg(reinterpret_cast<const uint4*>(p.Aq + (int64_t)m_hi * ldp + (int64_t)span * 64 + 16 * c));
        const uint32_t al[4] = {alo.x, alo.y, alo.z, alo.w}, ah[4] = {ahi.x, ahi.y, ahi.z, ahi.w};
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          // A rows g / g + 8: even codes (low nibbles, as 16*q) then odd codes (high nibbles)
          const uint32_t a[4] = {(al[s4] << 4) & 0xF0F0F0F0u, (ah[s4] << 4) & 0xF0F0F0F0u, al[s4] & 0xF0F0F0F0u,
                                 ah[s4] & 0xF0F0F0F0u};
          mma_s8_16832(d[t], a, (ww[s4] << 4) & 0xF0F0F0F0u, ww[s4] & 0xF0F0F0F0u);
        }
      }
    }
    // group scales: D[row][col] with rows m (tokens) and cols n0 + 2c (+1)
    const float sw0 = __half2float(__ushort_as_half(p.Ws[(int64_t)(n0 + 2 * c) * NG + gg])) * (1.0f / 256.0f);
    const float sw1 = __half2float(__ushort_as_half(p.Ws[(int64_t)(n0 + 2 * c + 1) * NG + gg])) * (1.0f / 256.0f);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int m_lo = t * 16 + g, m_hi = m_lo + 8;
      const float sa0 = m_lo < p.M ? __half2float(__ushort_as_half(p.As[(int64_t)m_lo * NG + gg])) : 0.0f;
      const float sa1 = m_hi < p.M ? __half2float(__ushort_as_half(p.As[(int64_t)m_hi * NG + gg])) : 0.0f;
      // exact int32 partials (|256 P| < 2^22) convert exactly; P*sW then acc += (P*sW)*sA
      acc[t][0] = fmaf((float)d[t][0] * sw0, sa0, acc[t][0]);
      acc[t][1] = fmaf((float)d[t][1] * sw1, sa0, acc[t][1]);
      acc[t][2] = fmaf((float)d[t][2] * sw0, sa1, acc[t][2]);
      acc[t][3] = fmaf((float)d[t][3] * sw1, sa1, acc[t][3]);
    }
  }
#pragma unroll
  for (int t = 0; t < MT; ++t) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = t * 16 + g + 8 * h;
      if (m >= p.M) continue;
      const int n = n0 + 2 * c;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      if (p.Cacc) {
        atomicAdd(reinterpret_cast<float2*>(p.Cacc + (int64_t)m * p.N + n), make_float2(v0, v1));
      } else if (p.c_bf16) {
        *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.C) + (int64_t)m * p.N + n) =
            __floats2bfloat162_rn(v0, v1);
      } else {
        *reinterpret_cast<float2*>(static_cast<float*>(p.C) + (int64_t)m * p.N + n) = make_float2(v0, v1);
      }
    }
  }
}

// Split-K factor: only when the output tiles leave most SMs idle (decode-sized M); each
// split then covers a whole number of groups.
int split_count(int64_t tiles, int group_units, int sms) {
  if (tiles * 2 > sms || group_units < 2) return 1;
  int64_t sp = sms / tiles;
  if (sp > group_units) sp = group_units;
  return (int)(sp < 1 ? 1 : sp);
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n4) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(src)[i];
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v.x, v.y), h1 = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&h0);
    o.y = *reinterpret_cast<uint32_t*>(&h1);
    reinterpret_cast<uint2*>(dst)[i] = o;
  }
}

rot_status w4a4_launch(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq, const uint16_t* Ws, int64_t M,
                       int64_t N, int64_t K, int G, void* C, int c_dtype, int32_t* partials, cudaStream_t s,
                       float* scratch, int64_t scratch_floats) {
  if (G > 256) return set_error(ROT_EUNSUPPORTED, "w4a4_linear: G > 256 is not supported");
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return set_error(ROT_EUNSUPPORTED, "w4a4_linear: size too large");
  // fp32 accumulation target for K-split launches: C itself (fp32), the caller's scratch, or a
  // stream-ordered temporary (bf16 output); zeroed on the stream
  float* scratch_owned = nullptr;
  auto acc_target = [&](float** out) -> rot_status {
    if (c_dtype == ROT_F32) {
      *out = static_cast<float*>(C);
    } else if (scratch) {
      if (M * N > scratch_floats)
        return set_error(ROT_EINVAL, "w4a4_linear_noalloc: M * N exceeds the static split-K buffer");
      *out = scratch;
    } else {
      ROT_CUDA_TRY(cudaMallocAsync(reinterpret_cast<void**>(&scratch_owned), (size_t)(M * N) * sizeof(float), s));
      *out = scratch_owned;
    }
    ROT_CUDA_TRY(cudaMemsetAsync(*out, 0, (size_t)(M * N) * sizeof(float), s));
    return ROT_OK;
  };
  auto finish_acc = [&](float* acc) -> rot_status {
    if (c_dtype == ROT_BF16) {
      const int64_t n4 = M * N / 4;   // N % 16 == 0
      const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, (int64_t)sm_count() * 8);
      f32_to_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(acc, static_cast<__nv_bfloat16*>(C), n4);
      ROT_CUDA_TRY(cudaGetLastError());
    }
    if (scratch_owned) ROT_CUDA_TRY(cudaFreeAsync(scratch_owned, s));
    return ROT_OK;
  };
  if (!partials && M <= 16 * DEC_MAXMT && G % 128 == 0) {
    // decode-sized M: weight-streaming kernel, K split until about 16 warps per SM are busy
    const int64_t ntiles = N / 8;
    const int NG = (int)(K / G);
    int64_t want = ((int64_t)sm_count() * 16 + ntiles - 1) / ntiles;
    const int splits0 = (int)std::max<int64_t>(1, std::min<int64_t>(NG, want));
    const int gps = (NG + splits0 - 1) / splits0;
    const int splits = (NG + gps - 1) / gps;
    DecParams d{};
    d.Aq = Aq;
    d.As = As;
    d.Wq = Wq;
    d.Ws = Ws;
    d.C = C;
    d.Cacc = nullptr;
    d.M = (int)M;
    d.N = (int)N;
    d.K = (int)K;
    d.G = G;
    d.c_bf16 = c_dtype == ROT_BF16;
    d.groups_per_split = gps;
    if (splits > 1) {
      rot_status st = acc_target(&d.Cacc);
      if (st) return st;
    }
    const dim3 grid((unsigned)((ntiles + DEC_THREADS / 32 - 1) / (DEC_THREADS / 32)), (unsigned)splits);
    const int mt = (int)((M + 15) / 16);
    if (mt == 1) w4a4_decode_kernel<1><<<grid, DEC_THREADS, 0, s>>>(d);
    else if (mt == 2) w4a4_decode_kernel<2><<<grid, DEC_THREADS, 0, s>>>(d);
    else if (mt == 3) w4a4_decode_kernel<3><<<grid, DEC_THREADS, 0, s>>>(d);
    else w4a4_decode_kernel<4><<<grid, DEC_THREADS, 0, s>>>(d);
    ROT_CUDA_TRY(cudaGetLastError());
    return splits > 1 ? finish_acc(d.Cacc) : ROT_OK;
  }
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
  {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      ROT_CUDA_TRY(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn)
        return set_error(ROT_ECUDA, "w4a4_linear: cuTensorMapEncodeTiled not available");
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t ldp = (cuuint64_t)(K / 2);
    const cuuint32_t estr[2] = {1, 1};
    {
      const cuuint64_t dims[2] = {ldp, (cuuint64_t)(M > 0 ? M : 1)};
      const cuuint64_t strides[1] = {ldp};
      const cuuint32_t box[2] = {(cuuint32_t)PROW_BYTES, (cuuint32_t)BM};
      if (encode(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(Aq), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return set_error(ROT_EINVAL, "w4a4_linear: tensor map for Aq rejected");
    }
    {
      const cuuint64_t dims[2] = {ldp, (cuuint64_t)N};
      const cuuint64_t strides[1] = {ldp};
      const cuuint32_t box[2] = {(cuuint32_t)PROW_BYTES, (cuuint32_t)BN};
      if (encode(&p.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(Wq), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return set_error(ROT_EINVAL, "w4a4_linear: tensor map for Wq rejected");
    }
  }
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
  const int64_t gx = (N + BN - 1) / BN, gy = (M + BM - 1) / BM;
  const int nkb = (int)((K + KB - 1) / KB);
  const int unit = G > KB ? G / KB : 1;            // K-blocks per group (split granularity)
  const int splits = partials ? 1 : split_count(gx * gy, nkb / unit, sm_count());
  p.kb_per_split = ((nkb / unit + splits - 1) / splits) * unit;
  const int zs = (nkb + p.kb_per_split - 1) / p.kb_per_split;
  p.Cacc = nullptr;
  if (zs > 1) {
    rot_status st = acc_target(&p.Cacc);
    if (st) return st;
  }
  dim3 grid((unsigned)gx, (unsigned)gy, (unsigned)zs);
  if (partials) w4a4_kernel<true><<<grid, THREADS, SMEM_BYTES, s>>>(p);
  else w4a4_kernel<false><<<grid, THREADS, SMEM_BYTES, s>>>(p);
  ROT_CUDA_TRY(cudaGetLastError());
  return zs > 1 ? finish_acc(p.Cacc) : ROT_OK;
}

rot_status w4a4_noalloc_scratch(float** out) {
  static float* addr[64] = {nullptr};
  int dev = 0;
  ROT_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 64) return set_error(ROT_EUNSUPPORTED, "w4a4_linear_noalloc: device index too large");
  if (!addr[dev]) ROT_CUDA_TRY(cudaGetSymbolAddress(reinterpret_cast<void**>(&addr[dev]), g_w4a4_scratch));
  *out = addr[dev];
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

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
// Persistent kernel: one CTA per SM walks a static list of work units (128 x 128 output
// tiles, times the K splits when the tiles alone leave SMs idle), M-index fastest so that
// the CTAs running at the same time share weight tiles in L2. Per K-block of 128: the
// loader warp brings the packed A and W tiles (two 2-D TMA boxes) into a 6-deep packed
// ring; 6 unpacker warps expand them into a 3-deep ring of swizzled K-major int8 tiles;
// the MMA warp, converged, issues 4 UMMAs (M = N = 128, K = 32) per K-block under an
// elect.sync predicate into one of four 128-column TMEM accumulators, one per group in
// flight, so the tensor pipe can run three groups ahead of the epilogue.
// Warp roles (512 threads, launched with 128 registers each). setmaxnreg acts on whole
// warpgroups, so roles are aligned to them: warpgroups 0-1 (epilogue) grow to 176 registers,
// warpgroups 2-3 (loader, unpackers, MMA warp) shrink to 80: 256*176 + 256*80 = 512*128.
//   warps 0-7   epilogue: warp w reads TMEM lanes 32*(w%4).. and columns 64*(w/4)..+63 of
//               a group's accumulator (two 32-column loads in flight), scales them and
//               accumulates in fp32 registers (packed f32x2 FMAs); it stages its own
//               columns' scales in a private shared-memory buffer;
//   warp 8      loader;   warps 9-14 unpackers;   warp 15 TMEM allocation and MMA issue.
// Group scaling: the epilogue adds the bit pattern of 1.5 * 2^23 to the int32 partial 256*P
// (one integer add): the sum is the bit pattern of the fp32 value 1.5 * 2^23 + 256*P, so
// fma(u, sA, -1.5*2^23*sA) = 256*P*sA rounded once, with no integer-to-float conversion
// (|256*P| < 2^22 requires G <= 256), and acc += that * sW/256.
// Measured on B200 (a probe with the MMAs and eight warps of TMEM loads running together):
// 128-column int8 UMMAs keep their full rate while the TMEM is read, so the accumulator
// depth, not TMEM bandwidth, sets how far the MMAs can run ahead of the epilogue.
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
constexpr int BN = 128;
constexpr int KB = 128;                  // K elements per stage
constexpr int STAGES = 3;                // unpacked int8 stages
constexpr int PSTAGES = 6;               // packed stages
constexpr int NACC = 4;                  // TMEM accumulators (groups in flight)
constexpr int A_STAGE_BYTES = BM * KB;   // unpacked int8
constexpr int B_STAGE_BYTES = BN * KB;
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int PROW_BYTES = KB / 2;       // packed bytes of one row in one K-block
constexpr int N_EPI = 256;               // epilogue threads (2 warpgroups)
constexpr int N_EPI_WARPS = N_EPI / 32;
constexpr int LOADER_WARP = N_EPI / 32;  // warp 8
constexpr int N_UNP = 192;               // unpacker threads (warps 9-14)
constexpr int N_UNP_WARPS = N_UNP / 32;
constexpr int THREADS = N_EPI + 32 + N_UNP + 32;
constexpr int EPI_COLS = BN / 2;         // columns per epilogue warp
constexpr int MMA_WARP = (N_EPI + 32 + N_UNP) / 32;
constexpr int LAUNCH_REGS = 128;         // 65536 / THREADS
constexpr int EPI_REGS = 176, PROD_REGS = 80;  // per warpgroup role
static_assert(THREADS == 512, "register split assumes 512 threads");
static_assert(N_UNP % 4 == 0 && (N_UNP / 4) % 8 == 0, "an unpacker keeps its chunk column and swizzle phase");
static_assert(N_EPI * EPI_REGS + (THREADS - N_EPI) * PROD_REGS <= THREADS * LAUNCH_REGS, "register split");
static_assert(A_STAGE_BYTES == BM * 128, "A and W int8 tiles are contiguous 128-byte rows");
constexpr uint32_t TMEM_COLS = NACC * BN;   // all 512 columns
static_assert(TMEM_COLS == 512, "TMEM columns");
constexpr uint32_t BIAS_BITS = 0x4B400000u;  // 1.5 * 2^23
constexpr float BIAS_F = 12582912.0f;
constexpr unsigned long long WAIT_NS = 2000000000ull;

// Shared-memory layout (offsets from a 1024-byte aligned base) of the two variants:
//   A8 = false (W4A4): a packed stage holds the packed A and W tiles of one K-block (16 KB), and
//                      the int8 ring stage holds the unpacked A and W tiles (32 KB);
//   A8 = true  (W4A8): a packed stage holds the int8 A tile, landed by TMA in the MMA's 128-byte
//                      swizzled K-major layout (16 KB), and the packed W tile (8 KB); the int8 ring
//                      stage holds only the unpacked W tile (16 KB).
// The int8 operands hold UNIT_A * qA and UNIT_W * qW (unpacking leaves 16 * q), so the int32
// accumulators hold UNIT * P, UNIT = 256 (W4A4) or 16 (W4A8).
constexpr int N_BARS = 2 * STAGES + 2 * PSTAGES + 2 * NACC;
template <bool A8>
struct Lay {
  static constexpr int A_PBYTES = A8 ? BM * KB : BM * PROW_BYTES;   // A part of a packed stage
  static constexpr int W_PBYTES = BN * PROW_BYTES;
  static constexpr int PSTAGE = A_PBYTES + W_PBYTES;
  static constexpr int STAGE = A8 ? B_STAGE_BYTES : STAGE_BYTES;    // int8 ring stage
  static constexpr int B_OFF = A8 ? 0 : A_STAGE_BYTES;              // W tile within an int8 stage
  static constexpr int ROWS_UNP = A8 ? BN : BM + BN;                // rows the unpackers expand
  static constexpr int N_CHUNKS = ROWS_UNP * (KB / 32);             // 16-byte packed chunks / stage
  static constexpr int UNP_ITERS = (N_CHUNKS + N_UNP - 1) / N_UNP;  // per unpacker thread (last partial)
  static constexpr int SRC_OFF = A8 ? A_PBYTES : 0;                 // first unpacked row in a packed stage
  static constexpr int OFF_STAGES = 0;
  static constexpr int OFF_PSTAGES = STAGES * STAGE;
  static constexpr int OFF_SLOTS = OFF_PSTAGES + PSTAGES * PSTAGE;  // per epilogue warp: sW/UNIT of its columns
  static constexpr int OFF_BARS = OFF_SLOTS + N_EPI_WARPS * EPI_COLS * 4;
  static constexpr int OFF_TMEM = OFF_BARS + N_BARS * 8;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;                 // + alignment slack
  static constexpr float UNIT = A8 ? 16.0f : 256.0f;
  static constexpr int PEMPTY_ARRIVALS = N_UNP_WARPS + (A8 ? 1 : 0);  // + the MMA's commit (A8)
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(OFF_PSTAGES % 1024 == 0 && PSTAGE % 1024 == 0 && A_PBYTES % 1024 == 0,
                "TMA destinations and the swizzled A tile stay 1024-byte aligned");
};

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
  int tiles_m;       // output tiles along M
  int splits;        // K splits per tile
  int units;         // tiles * splits
  int kb_per_split;  // K-blocks per split; a multiple of lcm(G, KB) / KB
  float* Cacc;       // split-K: fp32 [M, N] accumulated with atomics (zeroed beforehand), else null
  unsigned long long wait_ns;  // bound of every mbarrier wait
  int skip_loads;    // testing hook: the loader issues no TMA load, so every wait runs out
};

// One work unit: an output tile and a group-aligned K range.
struct Unit {
  int m0, n0;
  int kb0, nkb;      // first K-block, K-blocks
  int ks0, ks;       // first UMMA k-step (K = 32 each), k-steps
  int g0, ngl;       // first group, groups
};

__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
  Unit w;
  const int t = u / p.splits, z = u - t * p.splits;
  const int tm = t % p.tiles_m, tn = t / p.tiles_m;
  w.m0 = tm * BM;
  w.n0 = tn * BN;
  const int nkb_all = (p.K + KB - 1) / KB;
  w.kb0 = z * p.kb_per_split;
  const int kb1 = min(nkb_all, w.kb0 + p.kb_per_split);
  w.nkb = kb1 - w.kb0;
  w.ks0 = w.kb0 * (KB / 32);
  w.ks = min(p.K / 32, kb1 * (KB / 32)) - w.ks0;
  w.g0 = (w.ks0 * 32) / p.G;
  w.ngl = (w.ks * 32) / p.G;
  return w;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait for the phase with the given parity, by every lane of a converged warp; the
// result is warp-uniform. A plain try_wait on a completed phase costs ~13 cycles on B200, where
// one lane waiting with a suspend-time hint and broadcasting by shuffle measured ~130: every
// role here waits once or twice per K-block, so the cheap form matters. Between unsuccessful
// polls the warp sleeps for a few tens of nanoseconds. Gives up after ~2 s (records
// ROT_ETIMEOUT and raises the CTA's abort flag).
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned long long limit_ns) {
  const uint32_t addr = smem_u32(bar);
  bool ok = true;
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
    if (done) break;
    // a polling warp takes issue slots from the epilogue's arithmetic on the same scheduler:
    // back off briefly between polls
    __nanosleep(32);
    if ((it & 63) == 63) {
      if (*abort_flag) {
        ok = false;
        break;
      }
      unsigned long long now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) {
        *abort_flag = 1;
        atomicExch(&g_w4a4_error, (int)ROT_ETIMEOUT);
        ok = false;
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
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

// Issued by the whole (converged) warp: elect.sync picks the one lane that issues, so the
// operands stay warp-uniform (issuing from a diverged lane measured ~40% slower per MMA).
__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(IDESC), "r"(accumulate)
      : "memory");
}

// The same MMA and commit issued by the calling thread alone (inside an elected branch).
__device__ __forceinline__ void umma_i8_one(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(IDESC), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit_one(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}" : "=r"(e));
  return e != 0;
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
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

template <bool PARTIALS, bool A8>
__global__ void __launch_bounds__(THREADS, 1) w4a4_kernel(const __grid_constant__ Params p) {
  using L = Lay<A8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BARS);
  uint64_t* full = bars;                 // [STAGES]  unpackers -> MMA (one arrival per unpacker warp)
  uint64_t* empty = full + STAGES;       // [STAGES]  MMA commit -> unpackers
  uint64_t* pfull = empty + STAGES;      // [PSTAGES] TMA bytes -> unpackers
  uint64_t* pempty = pfull + PSTAGES;    // [PSTAGES] unpackers (and, A8, the MMA commit) -> loader
  uint64_t* tfull = pempty + PSTAGES;    // [NACC]    MMA commit -> epilogue
  uint64_t* tempty = tfull + NACC;       // [NACC]    epilogue warps -> MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_TMEM + 8);
  float* slots = reinterpret_cast<float*>(smem + L::OFF_SLOTS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NG = p.K / p.G;                // groups of the whole K (scale row length)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], N_UNP_WARPS);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], L::PEMPTY_ARRIVALS);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], N_EPI_WARPS);
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
  // Under programmatic dependent launch the set-up above may overlap the previous kernel in the
  // stream (e.g. the rotation that writes Aq and As); every global access comes after this wait
  // (a no-op for an ordinary launch). Dependents may start their own set-up at once.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp < N_EPI_WARPS) {
    // ======================= epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 176;");
    const int qd = warp & 3;                  // TMEM lane quadrant
    const int wg = warp >> 2;                 // column half of the tile
    const int row = qd * 32 + lane;           // TMEM lane = tile row
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16) + wg * EPI_COLS;
    // all accumulators start free (a group's first MMA overwrites its accumulator)
    if (lane == 0)
      for (int b = 0; b < NACC; ++b) mbar_arrive(&tempty[b]);

    // Group scales: each warp stages sW/UNIT of its own EPI_COLS columns in a private
    // shared-memory buffer (lane l: columns l + 32 j), ordered by __syncwarp alone, and keeps sA
    // of its row in a register. The raw binary16 values are loaded two groups ahead into a
    // two-entry register ring addressed statically by the parity of the group, from addresses
    // clamped into the matrix (rows >= M and columns >= N are never stored), so every load is
    // unconditional and no register is read while its load is in flight.
    constexpr int CQ = EPI_COLS / 32;         // column vectors per lane
    float* wsc = slots + warp * EPI_COLS;
    int su = blockIdx.x;                      // load cursor: unit and group within it
    int sg = 0, s_ngl = 0;
    const uint16_t* cw[CQ];                   // the cursor group's scales (dummy past the end)
    const uint16_t* ca = p.Ws;
#pragma unroll
    for (int j = 0; j < CQ; ++j) cw[j] = p.Ws;
    auto cursor_unit = [&]() {
      if (su < p.units) {
        const Unit w = unit_of(p, su);
        s_ngl = w.ngl;
#pragma unroll
        for (int j = 0; j < CQ; ++j) cw[j] = p.Ws + (int64_t)min(w.n0 + wg * EPI_COLS + 32 * j + lane, p.N - 1) * NG + w.g0;
        ca = p.As + (int64_t)min(w.m0 + row, p.M - 1) * NG + w.g0;
      } else {
#pragma unroll
        for (int j = 0; j < CQ; ++j) cw[j] = p.Ws;
        ca = p.Ws;
      }
    };
    auto cursor_step = [&]() {
      if (su < p.units) {
        if (++sg == s_ngl) {
          sg = 0;
          su += gridDim.x;
          cursor_unit();
        } else {
#pragma unroll
          for (int j = 0; j < CQ; ++j) ++cw[j];
          ++ca;
        }
      }
    };
    uint16_t q0w[CQ], q1w[CQ], q0a = 0, q1a = 0;   // groups gc (+1), by parity
#pragma unroll
    for (int j = 0; j < CQ; ++j) q0w[j] = q1w[j] = 0;
    if (!PARTIALS) {
      cursor_unit();
#pragma unroll
      for (int j = 0; j < CQ; ++j) q0w[j] = __ldg(cw[j]);
      q0a = __ldg(ca);
      cursor_step();
#pragma unroll
      for (int j = 0; j < CQ; ++j) q1w[j] = __ldg(cw[j]);
      q1a = __ldg(ca);
      cursor_step();
    }

    float2 acc[EPI_COLS / 2];
#pragma unroll
    for (int j = 0; j < EPI_COLS / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
    bool ok = true;
    int gc = 0;                               // groups accumulated by this CTA so far
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit w = unit_of(p, u);
      const int m = w.m0 + row;
      const bool row_ok = m < p.M;
      for (int gl = 0; gl < w.ngl; ++gl, ++gc) {
        float sa = 0.0f;
        if (!PARTIALS) {
          const uint16_t* nw[CQ];
#pragma unroll
          for (int j = 0; j < CQ; ++j) nw[j] = cw[j];
          const uint16_t* na = ca;
          cursor_step();
          uint16_t rw[CQ], ra;
          if (gc & 1) {
#pragma unroll
            for (int j = 0; j < CQ; ++j) { rw[j] = q1w[j]; q1w[j] = __ldg(nw[j]); }
            ra = q1a;
            q1a = __ldg(na);
          } else {
#pragma unroll
            for (int j = 0; j < CQ; ++j) { rw[j] = q0w[j]; q0w[j] = __ldg(nw[j]); }
            ra = q0a;
            q0a = __ldg(na);
          }
          __syncwarp();                 // every lane has read the previous group's column scales
#pragma unroll
          for (int j = 0; j < CQ; ++j) wsc[lane + 32 * j] = __half2float(__ushort_as_half(rw[j])) * (1.0f / L::UNIT);
          sa = __half2float(__ushort_as_half(ra));
          __syncwarp();
        }
        const int b = gc % NACC;
        ok = ok && bar_wait(&tfull[b], (gc / NACC) & 1, abort_flag, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        if constexpr (!PARTIALS) {
          // The group in chunks of 32 columns: each chunk's TMEM load is in flight while the 8
          // column-scale vectors of that chunk are loaded from shared memory, so the arithmetic
          // waits once per chunk for both (instead of once per scale vector). The accumulator is
          // released as soon as the last chunk is in registers.
          const float2 sa2 = make_float2(sa, sa);
          const float2 d2 = make_float2(-BIAS_F * sa, -BIAS_F * sa);   // exact: 3 * 2^22 * binary16
#pragma unroll
          for (int h = 0; h < CQ; ++h) {
            uint32_t r[32];
            float4 w4[8];
            tmem_ld32(lane_addr + b * BN + 32 * h, r);
#pragma unroll
            for (int q = 0; q < 8; ++q) w4[q] = lds128(wsc + 32 * h + 4 * q);
            tmem_wait_ld();
            if (h == CQ - 1) {
              // the whole group is in registers: release the accumulator for the group NACC ahead
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[b]);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int c = 32 * h + 4 * q;
              // 256*P + bits(1.5 * 2^23) = bits of the float 1.5 * 2^23 + 256*P
              const float2 u0 = make_float2(__uint_as_float(r[4 * q] + BIAS_BITS), __uint_as_float(r[4 * q + 1] + BIAS_BITS));
              const float2 u1 =
                  make_float2(__uint_as_float(r[4 * q + 2] + BIAS_BITS), __uint_as_float(r[4 * q + 3] + BIAS_BITS));
              // 256*P*sA (the bias cancels inside one rounding), then acc += that * sW/256
              const float2 t0 = __ffma2_rn(u0, sa2, d2);
              const float2 t1 = __ffma2_rn(u1, sa2, d2);
              acc[c / 2] = __ffma2_rn(t0, make_float2(w4[q].x, w4[q].y), acc[c / 2]);
              acc[c / 2 + 1] = __ffma2_rn(t1, make_float2(w4[q].z, w4[q].w), acc[c / 2 + 1]);
            }
          }
        } else {
          const int g = w.g0 + gl;
#pragma unroll 1
          for (int h = 0; h < CQ; ++h) {
            uint32_t r[32];
            tmem_ld32(lane_addr + b * BN + 32 * h, r);
            tmem_wait_ld();
            if (h == CQ - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[b]);
            }
            if (row_ok) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int n = w.n0 + wg * EPI_COLS + 32 * h + j;
                if (n < p.N) p.P[((int64_t)m * p.N + n) * NG + g] = ((int32_t)r[j]) / (int32_t)L::UNIT;
              }
            }
          }
        }
      }
      if (PARTIALS || !ok) continue;
      if (row_ok) {
        const int nb = w.n0 + wg * EPI_COLS;
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
#pragma unroll
      for (int j = 0; j < EPI_COLS / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
    }
  } else if (warp == LOADER_WARP) {
    // ======================= loader: the packed A and W tiles of one K-block -> packed stage
    // (two 2-D TMA boxes; rows beyond M / N and bytes beyond K/2 arrive as zeros)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
    int it = 0;
    bool ok = !p.skip_loads;   // testing hook: no load is ever issued (nothing in flight)
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit w = unit_of(p, u);
      for (int j = 0; j < w.nkb; ++j, ++it) {
        const int ps = it % PSTAGES;
        if (it >= PSTAGES && !bar_wait(&pempty[ps], ((it / PSTAGES) + 1) & 1, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* pst = smem + L::OFF_PSTAGES + ps * L::PSTAGE;
          const int kb = w.kb0 + j;
          mbar_arrive_expect_tx(&pfull[ps], (uint32_t)L::PSTAGE);
          // x = kb * 128 (int8 A) or kb * 64 bytes: a multiple of 16, as a tiled TMA requires of the
          // inner coordinate; the int8 A box lands 128-byte swizzled (the MMA's operand layout)
          tma_load_2d(pst, &p.tmA, kb * (A8 ? KB : PROW_BYTES), w.m0, &pfull[ps]);
          tma_load_2d(pst + L::A_PBYTES, &p.tmW, kb * PROW_BYTES, w.n0, &pfull[ps]);
        }
        __syncwarp();
      }
    }
  } else if (warp < MMA_WARP) {
    // ======================= unpackers: packed stage -> swizzled int8 stage
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
    const int ut = threadIdx.x - (LOADER_WARP + 1) * 32;   // 0..N_UNP-1
    // chunk q = ut + N_UNP*i: row (q >> 2) of the A-then-W rows, 16-byte piece (q & 3) of its
    // 64 packed bytes. N_UNP/4 is a multiple of 8, so the piece and the row's swizzle phase
    // are the same for all of a thread's chunks, and the A and W int8 tiles are contiguous
    // 128-byte rows (row r at byte 128*r of the stage).
    const int c = ut & 3, r0 = ut >> 2, r7 = r0 & 7;
    const int lo_off = ((2 * c) ^ r7) << 4, hi_off = ((2 * c + 1) ^ r7) << 4;
    constexpr int UNP_ITERS = L::UNP_ITERS;
    constexpr int UNP_BATCH = 4;
    const bool tail = ut + N_UNP * (UNP_ITERS - 1) < L::N_CHUNKS;   // this thread has a last chunk
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit w = unit_of(p, u);
      for (int j = 0; j < w.nkb; ++j, ++it) {
        const int s = it % STAGES, ps = it % PSTAGES;
        if (!bar_wait(&pfull[ps], (it / PSTAGES) & 1, abort_flag, p.wait_ns) ||
            (it >= STAGES && !bar_wait(&empty[s], ((it / STAGES) + 1) & 1, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        const uint8_t* src = smem + L::OFF_PSTAGES + ps * L::PSTAGE + L::SRC_OFF + ut * 16;
        uint8_t* dst = smem + L::OFF_STAGES + s * L::STAGE + r0 * 128;
        // loads in batches of UNP_BATCH, then their stores: the shared-memory latency is paid
        // once per batch (a batch's loads fit the role's register budget)
#pragma unroll
        for (int i0 = 0; i0 < UNP_ITERS; i0 += UNP_BATCH) {
        uint4 v[UNP_BATCH];
#pragma unroll
        for (int i1 = 0; i1 < UNP_BATCH; ++i1) {
          const int i = i0 + i1;
          if (i < UNP_ITERS - 1 || (i == UNP_ITERS - 1 && tail)) v[i1] = *reinterpret_cast<const uint4*>(src + i * N_UNP * 16);
        }
#pragma unroll
        for (int i1 = 0; i1 < UNP_BATCH; ++i1) {
          const int i = i0 + i1;
          if (i < UNP_ITERS - 1 || (i == UNP_ITERS - 1 && tail)) {
            const uint4 lo = make_uint4((v[i1].x << 4) & 0xF0F0F0F0u, (v[i1].y << 4) & 0xF0F0F0F0u,
                                        (v[i1].z << 4) & 0xF0F0F0F0u, (v[i1].w << 4) & 0xF0F0F0F0u);
            const uint4 hi = make_uint4(v[i1].x & 0xF0F0F0F0u, v[i1].y & 0xF0F0F0F0u, v[i1].z & 0xF0F0F0F0u,
                                        v[i1].w & 0xF0F0F0F0u);
            uint8_t* rowp = dst + i * (N_UNP / 4) * 128;
            if constexpr (A8) {
              // natural K order (the int8 A tile is not permuted): interleave even / odd codes
              *reinterpret_cast<uint4*>(rowp + lo_off) =
                  make_uint4(prmt(lo.x, hi.x, 0x5140u), prmt(lo.x, hi.x, 0x7362u), prmt(lo.y, hi.y, 0x5140u),
                             prmt(lo.y, hi.y, 0x7362u));
              *reinterpret_cast<uint4*>(rowp + hi_off) =
                  make_uint4(prmt(lo.z, hi.z, 0x5140u), prmt(lo.z, hi.z, 0x7362u), prmt(lo.w, hi.w, 0x5140u),
                             prmt(lo.w, hi.w, 0x7362u));
            } else {
              // even codes of the 32-code chunk, then odd codes (the same K order for A and W)
              *reinterpret_cast<uint4*>(rowp + lo_off) = lo;
              *reinterpret_cast<uint4*>(rowp + hi_off) = hi;
            }
          }
        }
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full[s]);
          mbar_arrive(&pempty[ps]);
        }
      }
    }
  } else {
    // ======================= MMA issue (the whole warp runs the loop; elect.sync issues)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");  // same value as the rest of its warpgroup
    // descriptors of stage 0; stage s and k-step k4 add (s * stage bytes + 32 * k4) >> 4 to the
    // start-address field (no carry: shared addresses stay below 2^18). W4A4: A and W in the
    // int8 stage s; W4A8: A in the packed stage ps (landed by TMA), W in the int8 stage s.
    const uint32_t sbase = smem_u32(smem + L::OFF_STAGES);
    const uint64_t dA0 = A8 ? make_desc(smem_u32(smem + L::OFF_PSTAGES)) : make_desc(sbase);
    const uint64_t dB0 = make_desc(sbase + L::B_OFF);
    int ps = 0, pph = 0;                    // packed stage of the K-block (A8: A's stage), its parity
    const int gsteps = p.G / 32;            // k-steps per group
    int s = 0, sph = 0;                     // int8 stage and its phase parity
    int b = 0, tph = 0;                     // accumulator and its phase parity
    int kg = 0;                             // k-step within the current group
    int nblk = 0;                           // K-blocks consumed
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit w = unit_of(p, u);         // K range group-aligned: kg == 0 here
      for (int j = 0; j < w.nkb; ++j) {
        if (!bar_wait(&full[s], sph, abort_flag, p.wait_ns) ||
            (A8 && !bar_wait(&pfull[ps], pph, abort_flag, p.wait_ns))) {   // A8: the A tile has landed
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t soA = (uint64_t)(((A8 ? ps * L::PSTAGE : s * L::STAGE)) >> 4);
        const uint64_t soB = (uint64_t)((s * L::STAGE) >> 4);
        if (gsteps % 4 == 0) {
          // G a multiple of 128: the K-block lies inside one group (and K % 128 == 0, so it has
          // all 4 k-steps). The accumulator wait comes first (warp-wide), then one elected lane
          // issues the 4 MMAs and the commits back to back (no per-MMA branches or elections).
          if (kg == 0) {
            if (!bar_wait(&tempty[b], tph, abort_flag, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const bool last = kg + 4 == gsteps;
          if (elect_one()) {
            const uint32_t td = tmem + b * BN;
            umma_i8_one(td, dA0 + soA, dB0 + soB, kg != 0 ? 1u : 0u);
            umma_i8_one(td, dA0 + soA + 2, dB0 + soB + 2, 1u);
            umma_i8_one(td, dA0 + soA + 4, dB0 + soB + 4, 1u);
            umma_i8_one(td, dA0 + soA + 6, dB0 + soB + 6, 1u);
            if (last) umma_commit_one(&tfull[b]);
            umma_commit_one(&empty[s]);
            if (A8) umma_commit_one(&pempty[ps]);
          }
          __syncwarp();
          kg += 4;
          if (last) {
            kg = 0;
            if (++b == NACC) {
              b = 0;
              tph ^= 1;
            }
          }
          ++nblk;
          if (++s == STAGES) {
            s = 0;
            sph ^= 1;
          }
          if (++ps == PSTAGES) {
            ps = 0;
            pph ^= 1;
          }
          continue;
        }
        const int nk = min(4, w.ks - 4 * j);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          if (k4 < nk) {
            if (kg == 0) {
              if (!bar_wait(&tempty[b], tph, abort_flag, p.wait_ns)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            umma_i8(tmem + b * BN, dA0 + soA + 2 * k4, dB0 + soB + 2 * k4, kg != 0 ? 1u : 0u);
            if (++kg == gsteps) {
              umma_commit(&tfull[b]);
              kg = 0;
              if (++b == NACC) {
                b = 0;
                tph ^= 1;
              }
            }
          }
        }
        if (!ok) break;
        umma_commit(&empty[s]);
        if (A8) umma_commit(&pempty[ps]);   // the A tile of this packed stage is consumed
        ++nblk;
        if (++s == STAGES) {
          s = 0;
          sph ^= 1;
        }
        if (++ps == PSTAGES) {
          ps = 0;
          pph ^= 1;
        }
      }
    }
    // the last stage-release commit must have landed before the CTA (and its smem) goes away
    if (ok && nblk > 0) {
      const int last = s == 0 ? STAGES - 1 : s - 1;
      bar_wait(&empty[last], s == 0 ? sph ^ 1 : sph, abort_flag, p.wait_ns);
      if (A8) {
        const int plast = ps == 0 ? PSTAGES - 1 : ps - 1;
        bar_wait(&pempty[plast], ps == 0 ? pph ^ 1 : pph, abort_flag, p.wait_ns);
      }
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
  unsigned long long wait_ns;   // staged kernel: bound of the weight-slice wait
};

// A8 (W4A8): the activation codes are int8 [M, K] in natural order; per span each lane loads the
// 32 int8 codes of its rows that meet its 16-byte weight piece and splits them into even / odd
// codes (byte permutes), the same order as the unpacked weights; products are 16 * qA * qW.
template <int MT, bool A8>
__global__ void __launch_bounds__(DEC_THREADS) w4a4_decode_kernel(const DecParams p) {
  constexpr float UNIT = A8 ? 16.0f : 256.0f;
  asm volatile("griddepcontrol.wait;" ::: "memory");   // see w4a4_kernel (programmatic launch)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
        if constexpr (A8) {
          // int8 codes 128 * span + 32 c .. + 31 of rows m_lo / m_hi (two 16-byte loads each)
          const int64_t lda8 = p.K;
          uint4 l0 = make_uint4(0u, 0u, 0u, 0u), l1 = l0, h0 = l0, h1 = l0;
          if (m_lo < p.M) {
            const uint4* q = reinterpret_cast<const uint4*>(p.Aq + (int64_t)m_lo * lda8 + (int64_t)span * 128 + 32 * c);
            l0 = __ldg(q);
            l1 = __ldg(q + 1);
          }
          if (m_hi < p.M) {
            const uint4* q = reinterpret_cast<const uint4*>(p.Aq + (int64_t)m_hi * lda8 + (int64_t)span * 128 + 32 * c);
            h0 = __ldg(q);
            h1 = __ldg(q + 1);
          }
          const uint32_t al[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
          const uint32_t ah[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) {
            // codes 8 s4 .. 8 s4 + 7 of the lane's 32: even ones, then odd ones
            const uint32_t a[4] = {prmt(al[2 * s4], al[2 * s4 + 1], 0x6420u), prmt(ah[2 * s4], ah[2 * s4 + 1], 0x6420u),
                                   prmt(al[2 * s4], al[2 * s4 + 1], 0x7531u), prmt(ah[2 * s4], ah[2 * s4 + 1], 0x7531u)};
            mma_s8_16832(d[t], a, (ww[s4] << 4) & 0xF0F0F0F0u, ww[s4] & 0xF0F0F0F0u);
          }
        } else {
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
    }
    // group scales: D[row][col] with rows m (tokens) and cols n0 + 2c (+1)
    const float sw0 = __half2float(__ushort_as_half(p.Ws[(int64_t)(n0 + 2 * c) * NG + gg])) * (1.0f / UNIT);
    const float sw1 = __half2float(__ushort_as_half(p.Ws[(int64_t)(n0 + 2 * c + 1) * NG + gg])) * (1.0f / UNIT);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int m_lo = t * 16 + g, m_hi = m_lo + 8;
      const float sa0 = m_lo < p.M ? __half2float(__ushort_as_half(p.As[(int64_t)m_lo * NG + gg])) : 0.0f;
      const float sa1 = m_hi < p.M ? __half2float(__ushort_as_half(p.As[(int64_t)m_hi * NG + gg])) : 0.0f;
      // exact int32 partials (|UNIT P| < 2^22) convert exactly; P*sW then acc += (P*sW)*sA
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

// Staged decode kernel. A CTA owns NPC n-tiles (8 weight rows each, contiguous in Wq) and splits K
// into KS slices of whole groups: warp (t, k) computes n-tile t over slice k. The first warp of each
// n-tile streams its 8 whole rows into shared memory at the start with one bulk asynchronous copy per
// row, completing on the n-tile's mbarrier that all its slice warps wait on, so every SM has its whole
// share of the weight stream in flight at once; the activation codes (L1/L2-resident) are loaded one
// span ahead and the scales per group. The K-slices are summed through shared memory and the CTA
// writes its tile of C directly (no atomics, no second launch). Rows are staged K/2 + 64 bytes apart:
// the 16-byte reads of a quarter-warp (rows g, g + 1 and pieces 0..3) fall in 8 distinct bank groups.
__device__ int g_dec_error = 0;

constexpr int DEC_HDR = 256;   // mbarriers, then the staged weight rows

struct StagedDec {
  int npc, ks;       // n-tiles per CTA, K-slices
  int pitch;         // bytes between staged weight rows
  int apitch;        // one-tile kernel: bytes between staged activation rows
  int off_acts, off_sa, off_sw, off_red;   // shared-memory offsets (one-tile kernel: all four)
  int scale_copy;    // one-tile kernel: the scale rows arrive by bulk copy (16-byte aligned, NG % 8 == 0)
};

constexpr int staged_threads(int mt) { return mt >= 3 ? 256 : 512; }   // bound on the CTA (registers)

// Bounded wait on phase 0 of a staging mbarrier (one use per launch); false when it gave up.
__device__ __forceinline__ bool dec_wait(uint64_t* bar, unsigned long long wait_ns) {
  const uint32_t addr = smem_u32(bar);
  unsigned long long t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(done)
                 : "r"(addr)
                 : "memory");
    if (done) return true;
    if ((it & 63) == 63) {
      unsigned long long now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      else if (now - t0 > wait_ns) {
        atomicExch(&g_dec_error, (int)ROT_ETIMEOUT);
        return false;
      }
    }
  }
}

// A fragments (m16n8k32, s8) of the four K = 32 steps of one 128-code span: activation pieces lo
// (row g) / hi (row g + 8) of this lane. W4A4: 16 packed bytes per row hold the span's codes of this
// lane's quarter; they become the even codes (times 16, low nibbles moved up) and the odd codes (high
// nibbles in place) of every 8-code word, the K order the weight fragments use too. W4A8: 32 int8
// codes per row, split into even / odd codes by byte permutes.
template <bool A8>
__device__ __forceinline__ void dec_a_frags(uint32_t (&a)[4][4], const uint4 (&lo)[2], const uint4 (&hi)[2]) {
  if constexpr (A8) {
    const uint32_t al[8] = {lo[0].x, lo[0].y, lo[0].z, lo[0].w, lo[1].x, lo[1].y, lo[1].z, lo[1].w};
    const uint32_t ah[8] = {hi[0].x, hi[0].y, hi[0].z, hi[0].w, hi[1].x, hi[1].y, hi[1].z, hi[1].w};
#pragma unroll
    for (int s4 = 0; s4 < 4; ++s4) {
      a[s4][0] = prmt(al[2 * s4], al[2 * s4 + 1], 0x6420u);
      a[s4][1] = prmt(ah[2 * s4], ah[2 * s4 + 1], 0x6420u);
      a[s4][2] = prmt(al[2 * s4], al[2 * s4 + 1], 0x7531u);
      a[s4][3] = prmt(ah[2 * s4], ah[2 * s4 + 1], 0x7531u);
    }
  } else {
    const uint32_t al[4] = {lo[0].x, lo[0].y, lo[0].z, lo[0].w};
    const uint32_t ah[4] = {hi[0].x, hi[0].y, hi[0].z, hi[0].w};
#pragma unroll
    for (int s4 = 0; s4 < 4; ++s4) {
      a[s4][0] = (al[s4] << 4) & 0xF0F0F0F0u;
      a[s4][1] = (ah[s4] << 4) & 0xF0F0F0F0u;
      a[s4][2] = al[s4] & 0xF0F0F0F0u;
      a[s4][3] = ah[s4] & 0xF0F0F0F0u;
    }
  }
}

// The four MMAs of one span against weight piece wv (16 packed bytes of row g of an n-tile).
__device__ __forceinline__ void dec_span_mma(int (&d)[4], const uint32_t (&a)[4][4], uint4 wv) {
  const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
  for (int s4 = 0; s4 < 4; ++s4) mma_s8_16832(d, a[s4], (ww[s4] << 4) & 0xF0F0F0F0u, ww[s4] & 0xF0F0F0F0u);
}

// L2 prefetch of a weight row ahead of griddepcontrol.wait. L2 is the device's point of coherence,
// so the prefetch is safe even if the previous kernel in the stream is still writing the row: the
// shared-memory copies issued after the wait read the current data (from L2 when prefetched).
__device__ __forceinline__ void l2_prefetch(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

template <int MT, bool A8>
__global__ void __launch_bounds__(staged_threads(MT)) w4a4_decode_staged_kernel(const DecParams p, const StagedDec q) {
  constexpr float UNIT = A8 ? 16.0f : 256.0f;
  extern __shared__ __align__(128) uint8_t dsm[];
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int g = l >> 2, c = l & 3;
  const int tl = warp % q.npc, ks = warp / q.npc;
  const int n0 = (blockIdx.x * q.npc + tl) * 8;
  const bool active = n0 < p.N;
  if (ks == 0 && active && l < 8) l2_prefetch(p.Wq + (int64_t)(n0 + l) * (p.K / 2), (uint32_t)(p.K / 2));
  asm volatile("griddepcontrol.wait;" ::: "memory");   // see w4a4_kernel (programmatic launch)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int NG = p.K / p.G;
  const int g0 = (int)((int64_t)NG * ks / q.ks);
  int g1 = (int)((int64_t)NG * (ks + 1) / q.ks);
  uint64_t* bar = reinterpret_cast<uint64_t*>(dsm) + tl;       // one per n-tile
  uint8_t* wsm = dsm + DEC_HDR + (size_t)tl * 8 * q.pitch;
  float* red = reinterpret_cast<float*>(dsm + q.off_red);
  const int64_t ldp = p.K / 2;
  const int64_t arow = A8 ? p.K : ldp;                         // bytes of one activation row
  float acc[MT][4];
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;

  if (ks == 0 && active) {
    // the n-tile's first warp: barrier, then one copy of each whole row (K/2 bytes)
    if (l == 0) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      mbar_arrive_expect_tx(bar, (uint32_t)(8 * ldp));
    }
    __syncwarp();
    if (l < 8)
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       smem_u32(wsm + (size_t)l * q.pitch)),
                   "l"(p.Wq + (int64_t)(n0 + l) * ldp), "r"((uint32_t)ldp), "r"(smem_u32(bar))
                   : "memory");
  }
  __syncthreads();   // the n-tile barriers are initialised before any warp waits on them
  if (active && g1 > g0) {
    const int spans_per_group = p.G / 128;
    const uint8_t* wlane = wsm + (size_t)g * q.pitch + 16 * c;
    // activation codes of the first span, loaded while the weights are in flight
    const int abytes = A8 ? 32 : 16;                     // this lane's activation bytes per span and row
    auto a_load = [&](int span, uint4 (&lo)[MT][2], uint4 (&hi)[MT][2]) {
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int m_lo = t * 16 + g, m_hi = m_lo + 8;
        const int64_t off = (int64_t)span * (A8 ? 128 : 64) + abytes * c;
        lo[t][0] = lo[t][1] = hi[t][0] = hi[t][1] = make_uint4(0u, 0u, 0u, 0u);
        if (m_lo < p.M) {
          const uint4* src = reinterpret_cast<const uint4*>(p.Aq + (int64_t)m_lo * arow + off);
          lo[t][0] = __ldg(src);
          if (A8) lo[t][1] = __ldg(src + 1);
        }
        if (m_hi < p.M) {
          const uint4* src = reinterpret_cast<const uint4*>(p.Aq + (int64_t)m_hi * arow + off);
          hi[t][0] = __ldg(src);
          if (A8) hi[t][1] = __ldg(src + 1);
        }
      }
    };
    uint4 alo[MT][2], ahi[MT][2];
    int span = g0 * spans_per_group;
    a_load(span, alo, ahi);
    // bounded wait for the warp's weight slice
    if (!__all_sync(0xffffffffu, dec_wait(bar, p.wait_ns))) g1 = g0;   // gave up: compute nothing
    for (int gg = g0; gg < g1; ++gg) {
      int d[MT][4];
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) d[t][i] = 0;
      for (int sp = 0; sp < spans_per_group; ++sp, ++span) {
        const uint4 wv = *reinterpret_cast<const uint4*>(wlane + (size_t)span * 64);
        uint4 clo[MT][2], chi[MT][2];
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          clo[t][0] = alo[t][0]; clo[t][1] = alo[t][1]; chi[t][0] = ahi[t][0]; chi[t][1] = ahi[t][1];
        }
        if (span + 1 < g1 * spans_per_group) a_load(span + 1, alo, ahi);   // next span's activations
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          uint32_t a[4][4];
          dec_a_frags<A8>(a, clo[t], chi[t]);
          dec_span_mma(d[t], a, wv);
        }
      }
      const float sw0 = __half2float(__ushort_as_half(p.Ws[(int64_t)(n0 + 2 * c) * NG + gg])) * (1.0f / UNIT);
      const float sw1 = __half2float(__ushort_as_half(p.Ws[(int64_t)(n0 + 2 * c + 1) * NG + gg])) * (1.0f / UNIT);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int m_lo = t * 16 + g, m_hi = m_lo + 8;
        const float sa0 = m_lo < p.M ? __half2float(__ushort_as_half(p.As[(int64_t)m_lo * NG + gg])) : 0.0f;
        const float sa1 = m_hi < p.M ? __half2float(__ushort_as_half(p.As[(int64_t)m_hi * NG + gg])) : 0.0f;
        acc[t][0] = fmaf((float)d[t][0] * sw0, sa0, acc[t][0]);
        acc[t][1] = fmaf((float)d[t][1] * sw1, sa0, acc[t][1]);
        acc[t][2] = fmaf((float)d[t][2] * sw0, sa1, acc[t][2]);
        acc[t][3] = fmaf((float)d[t][3] * sw1, sa1, acc[t][3]);
      }
    }
  }
  // sum the K-slices: slices 1.. park their partial sums in shared memory, slice 0 adds and stores
  if (ks > 0) {
    float* r = red + ((size_t)((ks - 1) * q.npc + tl) * 32 + l) * (4 * MT);
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) r[4 * t + i] = acc[t][i];
  }
  __syncthreads();
  if (ks > 0 || !active) return;
  for (int k = 1; k < q.ks; ++k) {
    const float* r = red + ((size_t)((k - 1) * q.npc + tl) * 32 + l) * (4 * MT);
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][i] += r[4 * t + i];
  }
#pragma unroll
  for (int t = 0; t < MT; ++t) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = t * 16 + g + 8 * h;
      if (m >= p.M) continue;
      const int n = n0 + 2 * c;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      if (p.c_bf16) {
        *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.C) + (int64_t)m * p.N + n) =
            __floats2bfloat162_rn(v0, v1);
      } else {
        *reinterpret_cast<float2*>(static_cast<float*>(p.C) + (int64_t)m * p.N + n) = make_float2(v0, v1);
      }
    }
  }
}

// One-tile decode kernel (M <= 16 tokens): everything the group loop reads sits in shared memory.
// A CTA owns NPC n-tiles; warp 0 issues one bulk copy per weight row of all of them and one per
// activation row, and (q.scale_copy) one copy each of the CTA's weight-scale rows and of the token
// scale rows (binary16, contiguous in Ws and As), completing on two mbarriers; without scale copies
// (unaligned scale tables) the threads load the scales into shared memory instead. Before
// griddepcontrol.wait the CTA's weight rows are prefetched into L2. Warp w computes ALL n-tiles of
// the CTA over K-slice w: each span's activation fragments are built once and used by the MMAs of
// every n-tile. The slices are summed through shared memory, warp t sums n-tile t and writes it.
// Activation rows are staged arow + 64 (W4A4) or + 16 (W4A8) bytes past a 128-byte multiple apart,
// so the quarter-warp reads (rows g, g + 1) are conflict-free.
template <bool A8, int NPC>
__global__ void __launch_bounds__(512) w4a4_decode_tile1_kernel(const DecParams p, const StagedDec q) {
  constexpr float UNIT = A8 ? 16.0f : 256.0f;
  extern __shared__ __align__(128) uint8_t dsm[];
  const int warp = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int g = l >> 2, c = l & 3;
  const int NG = p.K / p.G;
  const int64_t nrow0 = (int64_t)blockIdx.x * NPC * 8;                 // first weight row of the CTA
  const int nrows = (int)(p.N - nrow0 < NPC * 8 ? p.N - nrow0 : NPC * 8);   // a multiple of 8
  const int ntl = nrows / 8;                                           // active n-tiles
  if (warp == 0 && l < nrows) l2_prefetch(p.Wq + (nrow0 + l) * (p.K / 2), (uint32_t)(p.K / 2));
  asm volatile("griddepcontrol.wait;" ::: "memory");   // see w4a4_kernel (programmatic launch)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  uint64_t* wbar = reinterpret_cast<uint64_t*>(dsm);
  uint64_t* abar = wbar + 1;
  uint8_t* wsm = dsm + DEC_HDR;
  uint8_t* asm_ = dsm + q.off_acts;
  uint16_t* sA = reinterpret_cast<uint16_t*>(dsm + q.off_sa);          // [16][NG] binary16
  uint16_t* sW = reinterpret_cast<uint16_t*>(dsm + q.off_sw);          // [NPC * 8][NG] binary16
  float* red = reinterpret_cast<float*>(dsm + q.off_red);
  const int64_t ldp = p.K / 2;
  const int64_t arow = A8 ? p.K : ldp;
  const uint32_t sa_bytes = (uint32_t)(p.M * NG * 2), sw_bytes = (uint32_t)(nrows * NG * 2);

  if (warp == 0) {
    if (l == 0) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(wbar)) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(abar)) : "memory");
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      mbar_arrive_expect_tx(wbar, (uint32_t)(nrows * ldp) + (q.scale_copy ? sw_bytes : 0u));
      mbar_arrive_expect_tx(abar, (uint32_t)(p.M * arow) + (q.scale_copy ? sa_bytes : 0u));
    }
    __syncwarp();
    if (l < nrows)   // NPC * 8 <= 16 rows
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       smem_u32(wsm + (size_t)l * q.pitch)),
                   "l"(p.Wq + (nrow0 + l) * ldp), "r"((uint32_t)ldp), "r"(smem_u32(wbar))
                   : "memory");
    if (l < p.M)     // M <= 16 rows
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       smem_u32(asm_ + (size_t)l * q.apitch)),
                   "l"(p.Aq + (int64_t)l * arow), "r"((uint32_t)arow), "r"(smem_u32(abar))
                   : "memory");
    if (q.scale_copy && l == 16)
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       smem_u32(sW)),
                   "l"(p.Ws + nrow0 * NG), "r"(sw_bytes), "r"(smem_u32(wbar))
                   : "memory");
    if (q.scale_copy && l == 17)
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       smem_u32(sA)),
                   "l"(p.As), "r"(sa_bytes), "r"(smem_u32(abar))
                   : "memory");
  }
  if (!q.scale_copy) {
    for (int i = threadIdx.x; i < p.M * NG; i += blockDim.x) sA[i] = p.As[i];
    for (int i = threadIdx.x; i < nrows * NG; i += blockDim.x) sW[i] = p.Ws[nrow0 * NG + i];
  }
  __syncthreads();   // barriers initialised (and, without scale copies, the scales in shared memory)

  float acc[NPC][4];
#pragma unroll
  for (int t = 0; t < NPC; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;
  // K-slice of this warp (warps past q.ks only help to sum and store)
  const int g0 = warp < q.ks ? (int)((int64_t)NG * warp / q.ks) : 0;
  int g1 = warp < q.ks ? (int)((int64_t)NG * (warp + 1) / q.ks) : 0;
  if (g1 > g0) {
    const bool ok = dec_wait(wbar, p.wait_ns) && dec_wait(abar, p.wait_ns);
    if (!__all_sync(0xffffffffu, ok)) g1 = g0;   // gave up: compute nothing (outputs unspecified)
  }
  const int spans_per_group = p.G / 128;
  const uint8_t* wlane = wsm + (size_t)g * q.pitch + 16 * c;
  const uint8_t* alo = asm_ + (size_t)g * q.apitch + (A8 ? 32 : 16) * c;
  const uint8_t* ahi = alo + (size_t)8 * q.apitch;
  const bool lo_on = g < p.M, hi_on = g + 8 < p.M;   // token rows past M: scale 0 (rows not staged)
  int span = g0 * spans_per_group;
  for (int gg = g0; gg < g1; ++gg) {
    int d[NPC][4];
#pragma unroll
    for (int t = 0; t < NPC; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) d[t][i] = 0;
    for (int sp = 0; sp < spans_per_group; ++sp, ++span) {
      const size_t ao = (size_t)span * (A8 ? 128 : 64);
      uint4 lo[2], hi[2];
      lo[0] = *reinterpret_cast<const uint4*>(alo + ao);
      hi[0] = *reinterpret_cast<const uint4*>(ahi + ao);
      if constexpr (A8) {
        lo[1] = *reinterpret_cast<const uint4*>(alo + ao + 16);
        hi[1] = *reinterpret_cast<const uint4*>(ahi + ao + 16);
      } else {
        lo[1] = hi[1] = make_uint4(0u, 0u, 0u, 0u);
      }
      uint4 wv[NPC];
#pragma unroll
      for (int t = 0; t < NPC; ++t)
        if (t < ntl) wv[t] = *reinterpret_cast<const uint4*>(wlane + (size_t)t * 8 * q.pitch + (size_t)span * 64);
      uint32_t a[4][4];
      dec_a_frags<A8>(a, lo, hi);
#pragma unroll
      for (int t = 0; t < NPC; ++t)
        if (t < ntl) dec_span_mma(d[t], a, wv[t]);
    }
    const float sa0 = lo_on ? __half2float(__ushort_as_half(sA[g * NG + gg])) : 0.0f;
    const float sa1 = hi_on ? __half2float(__ushort_as_half(sA[(g + 8) * NG + gg])) : 0.0f;
#pragma unroll
    for (int t = 0; t < NPC; ++t) {
      if (t < ntl) {
        const float sw0 = __half2float(__ushort_as_half(sW[(t * 8 + 2 * c) * NG + gg])) * (1.0f / UNIT);
        const float sw1 = __half2float(__ushort_as_half(sW[(t * 8 + 2 * c + 1) * NG + gg])) * (1.0f / UNIT);
        acc[t][0] = fmaf((float)d[t][0] * sw0, sa0, acc[t][0]);
        acc[t][1] = fmaf((float)d[t][1] * sw1, sa0, acc[t][1]);
        acc[t][2] = fmaf((float)d[t][2] * sw0, sa1, acc[t][2]);
        acc[t][3] = fmaf((float)d[t][3] * sw1, sa1, acc[t][3]);
      }
    }
  }
  // every slice parks its partial sums (slice-major); warp t then sums n-tile t and writes it
  if (warp < q.ks) {
#pragma unroll
    for (int t = 0; t < NPC; ++t)
      *reinterpret_cast<float4*>(red + ((size_t)(warp * NPC + t) * 32 + l) * 4) =
          make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
  }
  __syncthreads();
  if (warp >= ntl) return;
  float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int k = 0; k < q.ks; ++k) {
    const float4 r = *reinterpret_cast<const float4*>(red + ((size_t)(k * NPC + warp) * 32 + l) * 4);
    v.x += r.x; v.y += r.y; v.z += r.z; v.w += r.w;
  }
  const int64_t n = nrow0 + warp * 8 + 2 * c;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int m = g + 8 * h;
    if (m >= p.M) continue;
    const float v0 = h ? v.z : v.x, v1 = h ? v.w : v.y;
    if (p.c_bf16) {
      *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.C) + (int64_t)m * p.N + n) =
          __floats2bfloat162_rn(v0, v1);
    } else {
      *reinterpret_cast<float2*>(static_cast<float*>(p.C) + (int64_t)m * p.N + n) = make_float2(v0, v1);
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

// Work list of the tile kernel: 128 x 128 output tiles, times K splits when the tiles alone
// would leave more than half of the SMs idle. A split covers a whole number of lcm(G, 128)
// K-ranges, so it starts and ends on both a K-block and a group boundary; every split is
// non-empty; one persistent CTA per SM, at most one per unit.
rot_status w4a4_tile_plan_compute(int64_t M, int64_t N, int64_t K, int G, int sms, bool partials,
                                  W4A4TilePlan* out) {
  if (M <= 0 || N <= 0 || K <= 0 || G <= 0 || G > 256 || K % G != 0 || G % 32 != 0 || sms <= 0)
    return set_error(ROT_EINVAL, "w4a4 tile plan: need M, N, K, sms > 0, 0 < G <= 256, G % 32 == 0, K % G == 0");
  W4A4TilePlan tp;
  tp.tiles_n = (N + BN - 1) / BN;
  tp.tiles_m = (M + BM - 1) / BM;
  const int64_t nkb = (K + KB - 1) / KB;
  int unit = 1;                                    // K-blocks per lcm(G, KB) range
  while ((unit * KB) % G != 0) ++unit;
  const int64_t ranges = (nkb + unit - 1) / unit;  // lcm ranges (the last one may be partial)
  const int64_t want = partials ? 1 : split_count(tp.tiles_n * tp.tiles_m, (int)std::min<int64_t>(ranges, 1 << 20), sms);
  tp.kb_per_split = (int)(((ranges + want - 1) / want) * unit);
  tp.splits = (int)((nkb + tp.kb_per_split - 1) / tp.kb_per_split);
  if (tp.tiles_n * tp.tiles_m * tp.splits > (1ll << 30)) return set_error(ROT_EUNSUPPORTED, "w4a4_linear: too many tiles");
  tp.units = tp.tiles_n * tp.tiles_m * tp.splits;
  tp.grid = std::min<int64_t>(tp.units, sms);
  *out = tp;
  return ROT_OK;
}

// Launch a kernel, with programmatic stream serialization when pdl is set (its prologue may then
// overlap the previous kernel; the kernels wait with griddepcontrol.wait before any global access).
template <typename P>
cudaError_t launch_maybe_pdl(void (*kern)(const P), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                             const P& prm) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
  return e != cudaSuccess ? e : cudaGetLastError();
}

rot_status w4a4_launch(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq, const uint16_t* Ws, int64_t M,
                       int64_t N, int64_t K, int G, void* C, int c_dtype, int32_t* partials, cudaStream_t s,
                       float* scratch, int64_t scratch_floats, bool a8, bool pdl) {
  pdl = pdl || pdl_default();
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
    const int64_t ntiles = N / 8;
    const int NG = (int)(K / G);
    const int mt = (int)((M + 15) / 16);
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
    d.wait_ns = wait_limit_ns(WAIT_NS);
    const int64_t pitch = K / 2 + 64;   // staged weight rows (conflict-free quarter-warp reads)
    const int64_t sms = sm_count();
    auto set_limit = [&](const void* fn, int var) -> rot_status {
      static int dec_configured[64][16] = {};   // per device and variant: the opt-in limit set once
      int dev = 0;
      ROT_CUDA_TRY(cudaGetDevice(&dev));
      if (dev >= 64 || !dec_configured[dev][var]) {
        ROT_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
        if (dev < 64) dec_configured[dev][var] = 1;
      }
      return ROT_OK;
    };
    auto launch_dec = [&](void (*dk)(const DecParams, const StagedDec), int64_t grid, int threads, size_t smem,
                          const StagedDec& q) -> rot_status {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)grid);
      cfg.blockDim = dim3(threads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = pdl ? 1 : 0;
      ROT_CUDA_TRY(cudaLaunchKernelEx(&cfg, dk, d, q));
      ROT_CUDA_TRY(cudaGetLastError());
      return ROT_OK;
    };
    d.groups_per_split = NG;
    // one token tile: weights, activation rows and scales all staged in shared memory, 1 or 2
    // n-tiles per CTA (every CTA resident at once, two per SM), 8 to 16 K-slices
    if (mt == 1) {
      const int64_t need = (ntiles + 2 * sms - 1) / (2 * sms);
      const int npc1 = need <= 1 ? 1 : need <= 2 ? 2 : 0;
      if (npc1) {
        const int64_t arow = a8 ? K : K / 2;
        const int64_t apitch = ((arow + 127) & ~(int64_t)127) + (a8 ? 16 : 64);
        StagedDec q{};
        q.npc = npc1;
        q.pitch = (int)pitch;
        q.apitch = (int)apitch;
        const size_t off_acts = DEC_HDR + (size_t)npc1 * 8 * pitch;
        const size_t off_sa = off_acts + (size_t)16 * apitch;
        const size_t off_sw = off_sa + (((size_t)16 * NG * 2 + 15) & ~(size_t)15);
        const size_t off_red = off_sw + (((size_t)npc1 * 8 * NG * 2 + 15) & ~(size_t)15);
        int kk = std::min(NG, 16);
        while (kk > 1 && off_red + (size_t)kk * npc1 * 512 > 110 * 1024) kk = (kk + 1) / 2;
        const size_t smem = off_red + (size_t)kk * npc1 * 512;
        if (smem <= 110 * 1024 && kk >= std::min(NG, 8)) {   // (too few warps: the other path)
          q.ks = kk;
          q.scale_copy = (NG % 8 == 0 && (reinterpret_cast<uintptr_t>(As) & 15) == 0 &&
                          (reinterpret_cast<uintptr_t>(Ws) & 15) == 0) ? 1 : 0;
          q.off_acts = (int)off_acts;
          q.off_sa = (int)off_sa;
          q.off_sw = (int)off_sw;
          q.off_red = (int)off_red;
          void (*dk)(const DecParams, const StagedDec) =
              a8 ? (npc1 == 1 ? w4a4_decode_tile1_kernel<true, 1> : w4a4_decode_tile1_kernel<true, 2>)
                 : (npc1 == 1 ? w4a4_decode_tile1_kernel<false, 1> : w4a4_decode_tile1_kernel<false, 2>);
          rot_status st = set_limit((const void*)dk, 8 + (a8 ? 2 : 0) + (npc1 - 1));
          if (st) return st;
          return launch_dec(dk, (ntiles + npc1 - 1) / npc1, 32 * std::max(kk, npc1), smem, q);
        }
      }
    }
    // staged weight stream: enough n-tiles per CTA that every CTA is resident at once (two per SM),
    // K-slices to bring the CTA to about 16 warps
    const int max_warps = (mt >= 3 ? 256 : 512) / 32;
    int npc = (int)std::max<int64_t>(1, (ntiles + 2 * sms - 1) / (2 * sms));
    int ksl = std::max(1, std::min(NG, max_warps / std::max(1, npc)));
    const size_t red_unit = (size_t)32 * 4 * mt * 4;   // one warp's partial sums
    auto smem_of = [&](int np, int kk) -> size_t {
      return (size_t)DEC_HDR + (size_t)np * 8 * pitch + (size_t)(kk - 1) * np * red_unit;
    };
    while (npc > 1 && smem_of(npc, ksl) > 110 * 1024) {   // keep two CTAs per SM
      npc = (npc + 1) / 2;
      ksl = std::max(1, std::min(NG, max_warps / npc));
    }
    if (npc * ksl <= max_warps && smem_of(npc, ksl) <= 200 * 1024) {
      StagedDec q{};
      q.npc = npc;
      q.ks = ksl;
      q.pitch = (int)pitch;
      q.off_red = (int)(DEC_HDR + (size_t)npc * 8 * pitch);
      void (*dk)(const DecParams, const StagedDec) = nullptr;
      if (a8) dk = mt == 1 ? w4a4_decode_staged_kernel<1, true> : mt == 2 ? w4a4_decode_staged_kernel<2, true>
                   : mt == 3 ? w4a4_decode_staged_kernel<3, true> : w4a4_decode_staged_kernel<4, true>;
      else dk = mt == 1 ? w4a4_decode_staged_kernel<1, false> : mt == 2 ? w4a4_decode_staged_kernel<2, false>
                : mt == 3 ? w4a4_decode_staged_kernel<3, false> : w4a4_decode_staged_kernel<4, false>;
      rot_status st = set_limit((const void*)dk, (a8 ? 4 : 0) + (mt - 1));
      if (st) return st;
      return launch_dec(dk, (ntiles + npc - 1) / npc, 32 * npc * ksl, smem_of(npc, ksl), q);
    }
    // very long rows: the weights stream through registers, K split until about 32 warps per SM
    // are busy (more bytes in flight)
    int64_t want = ((int64_t)sm_count() * 32 + ntiles - 1) / ntiles;
    const int splits0 = (int)std::max<int64_t>(1, std::min<int64_t>(NG, want));
    const int gps = (NG + splits0 - 1) / splits0;
    const int splits = (NG + gps - 1) / gps;
    d.groups_per_split = gps;
    if (splits > 1) {
      rot_status st = acc_target(&d.Cacc);
      if (st) return st;
    }
    const dim3 grid((unsigned)((ntiles + DEC_THREADS / 32 - 1) / (DEC_THREADS / 32)), (unsigned)splits);
    void (*dk)(const DecParams) = nullptr;
    if (a8) dk = mt == 1 ? w4a4_decode_kernel<1, true> : mt == 2 ? w4a4_decode_kernel<2, true>
                 : mt == 3 ? w4a4_decode_kernel<3, true> : w4a4_decode_kernel<4, true>;
    else dk = mt == 1 ? w4a4_decode_kernel<1, false> : mt == 2 ? w4a4_decode_kernel<2, false>
              : mt == 3 ? w4a4_decode_kernel<3, false> : w4a4_decode_kernel<4, false>;
    ROT_CUDA_TRY(launch_maybe_pdl(dk, grid, dim3(DEC_THREADS), 0, s, pdl && splits == 1, d));
    return splits > 1 ? finish_acc(d.Cacc) : ROT_OK;
  }
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    // The setmaxnreg split is only valid for the register count it was sized for: refuse
    // to launch otherwise (an over-subscribed split would wait for registers forever).
    const void* ks[4] = {(const void*)w4a4_kernel<false, false>, (const void*)w4a4_kernel<true, false>,
                         (const void*)w4a4_kernel<false, true>, (const void*)w4a4_kernel<true, true>};
    for (int v = 0; v < 4; ++v) {
      cudaFuncAttributes fa;
      ROT_CUDA_TRY(cudaFuncGetAttributes(&fa, ks[v]));
      if (fa.numRegs != LAUNCH_REGS)
        return set_error(ROT_EUNSUPPORTED, "w4a4_linear: kernel built with an unexpected register count");
      ROT_CUDA_TRY(cudaFuncSetAttribute(ks[v], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        v < 2 ? Lay<false>::SMEM : Lay<true>::SMEM));
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
      // W4A4: packed A [M, K/2], box {64 bytes, BM rows}; W4A8: int8 A [M, K], box {128 bytes,
      // BM rows}, 128-byte swizzled into the MMA's K-major operand layout
      const cuuint64_t lda = a8 ? (cuuint64_t)K : ldp;
      const cuuint64_t dims[2] = {lda, (cuuint64_t)(M > 0 ? M : 1)};
      const cuuint64_t strides[1] = {lda};
      const cuuint32_t box[2] = {(cuuint32_t)(a8 ? KB : PROW_BYTES), (cuuint32_t)BM};
      if (encode(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(Aq), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, a8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
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
  W4A4TilePlan tp;
  {
    rot_status st = w4a4_tile_plan_compute(M, N, K, G, sm_count(), partials != nullptr, &tp);
    if (st) return st;
  }
  p.kb_per_split = tp.kb_per_split;
  p.splits = tp.splits;
  p.tiles_m = (int)tp.tiles_m;
  p.units = (int)tp.units;
  p.Cacc = nullptr;
  p.wait_ns = wait_limit_ns(WAIT_NS);
  p.skip_loads = take_test_fault(TEST_FAULT_W4A4_LOADS) ? 1 : 0;
  if (p.splits > 1) {
    rot_status st = acc_target(&p.Cacc);
    if (st) return st;
  }
  // persistent: one CTA per SM (the shared-memory footprint admits no second one)
  const unsigned grid = (unsigned)tp.grid;
  void (*tk)(const Params) = a8 ? (partials ? w4a4_kernel<true, true> : w4a4_kernel<false, true>)
                                : (partials ? w4a4_kernel<true, false> : w4a4_kernel<false, false>);
  // (after a split-K memset the launch is an ordinary one: the dependency is not a kernel)
  ROT_CUDA_TRY(launch_maybe_pdl(tk, dim3(grid), dim3(THREADS), a8 ? Lay<true>::SMEM : Lay<false>::SMEM, s,
                                pdl && p.splits == 1, p));
  return p.splits > 1 ? finish_acc(p.Cacc) : ROT_OK;
}

rot_status f32_to_bf16_launch(const float* src, void* dst, int64_t n, cudaStream_t s) {
  if (n % 4 != 0) return set_error(ROT_EINVAL, "f32_to_bf16: n must be a multiple of 4");
  const int64_t n4 = n / 4;
  if (n4 == 0) return ROT_OK;
  const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, (int64_t)sm_count() * 8);
  f32_to_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(src, static_cast<__nv_bfloat16*>(dst), n4);
  ROT_CUDA_TRY(cudaGetLastError());
  return ROT_OK;
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
  int v = 0, vd = 0;
  ROT_CUDA_TRY(cudaMemcpyFromSymbol(&vd, g_dec_error, sizeof(int)));
  if (vd) {
    int z = 0;
    ROT_CUDA_TRY(cudaMemcpyToSymbol(g_dec_error, &z, sizeof(int)));
    return set_error((rot_status)vd, "a bounded wait in the decode-sized w4a4 kernel gave up");
  }
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

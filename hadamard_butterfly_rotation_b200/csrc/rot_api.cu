// C-ABI entry points: argument validation and dispatch to the kernels.
#include <cstdint>

#include "rot_internal.cuh"

using namespace rotb;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

rot_status check_plan(rot_plan_t plan, const char* fn) {
  if (!plan) return set_error(ROT_EINVAL, std::string(fn) + ": plan is NULL");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != plan->device) return set_error(ROT_EINVAL, std::string(fn) + ": plan belongs to another device");
  return ROT_OK;
}

rot_status check_rows(const void* A, int a_dtype, int64_t M, int64_t lda, int K, const char* fn) {
  if (a_dtype != ROT_F32 && a_dtype != ROT_BF16) return set_error(ROT_EINVAL, std::string(fn) + ": a_dtype must be ROT_F32 or ROT_BF16");
  if (M < 0) return set_error(ROT_EINVAL, std::string(fn) + ": M < 0");
  if (M == 0) return ROT_OK;
  if (!A) return set_error(ROT_EINVAL, std::string(fn) + ": A is NULL");
  const int es = a_dtype == ROT_BF16 ? 2 : 4;
  if (lda < K) return set_error(ROT_EINVAL, std::string(fn) + ": lda < K");
  if (!aligned16(A) || (lda * es) % 16 != 0)
    return set_error(ROT_EINVAL, std::string(fn) + ": A must be 16-byte aligned and lda*sizeof a multiple of 16");
  return ROT_OK;
}

rot_status check_quant(int K, int bits, int G, const char* fn) {
  if (bits != 8 && bits != 4 && bits != 2) return set_error(ROT_EINVAL, std::string(fn) + ": bits must be 8, 4 or 2");
  const int cpw = 32 / bits;
  if (G <= 0 || K % G != 0 || G % (bits == 8 ? 4 : bits == 4 ? 8 : 16) != 0)
    return set_error(ROT_EINVAL,
                     std::string(fn) + ": G must divide K and be a multiple of 4 (int8) / 8 (int4) / 16 (int2)");
  if (K % cpw != 0) return set_error(ROT_EINVAL, std::string(fn) + ": K must be a multiple of the codes per word");
  return ROT_OK;
}

}  // namespace

extern "C" rot_status rot_apply(const void* A, int a_dtype, int64_t M, int64_t lda, rot_plan_t plan,
                                int inverse, float* Y, int64_t ldy, void* stream) {
  rot_status st = check_plan(plan, "rot_apply");
  if (st) return st;
  if ((st = check_rows(A, a_dtype, M, lda, plan->K, "rot_apply"))) return st;
  if (M == 0) return ROT_OK;
  if (!Y || !aligned16(Y) || ldy < plan->K || (ldy * 4) % 16 != 0)
    return set_error(ROT_EINVAL, "rot_apply: Y must be 16-byte aligned with ldy >= K, ldy*4 % 16 == 0");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (plan->chunk_log2 >= 5) return fwht_apply(plan, A, a_dtype, M, lda, inverse, Y, ldy, s);
  return stages_apply(plan, A, a_dtype, M, lda, inverse, Y, ldy, s);
}

extern "C" rot_status rot_quant(const void* A, int a_dtype, int64_t M, int64_t lda, rot_plan_t plan,
                                int bits, int G, uint8_t* codes, uint16_t* scales, void* stream) {
  rot_status st = check_plan(plan, "rot_quant");
  if (st) return st;
  if ((st = check_rows(A, a_dtype, M, lda, plan->K, "rot_quant"))) return st;
  if ((st = check_quant(plan->K, bits, G, "rot_quant"))) return st;
  if (M == 0) return ROT_OK;
  if (!codes || !scales || !aligned16(codes) || !aligned16(scales))
    return set_error(ROT_EINVAL, "rot_quant: codes and scales must be non-NULL and 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fwht_quant_supported(plan, bits, G)) return fwht_quant(plan, A, a_dtype, M, lda, bits, G, codes, scales, s);
  return stages_quant(plan, A, a_dtype, M, lda, bits, G, codes, scales, s);
}

extern "C" rot_status rot_dequant(const uint8_t* codes, const uint16_t* scales, int64_t M, rot_plan_t plan,
                                  int bits, int G, int inverse, float* out, void* stream) {
  rot_status st = check_plan(plan, "rot_dequant");
  if (st) return st;
  if ((st = check_quant(plan->K, bits, G, "rot_dequant"))) return st;
  if (M < 0) return set_error(ROT_EINVAL, "rot_dequant: M < 0");
  if (M == 0) return ROT_OK;
  if (!codes || !scales || !out || !aligned16(codes) || !aligned16(out))
    return set_error(ROT_EINVAL, "rot_dequant: pointers must be non-NULL, codes/out 16-byte aligned");
  if ((plan->K * 4) % 16 != 0) return set_error(ROT_EINVAL, "rot_dequant: K*4 must be a multiple of 16");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = dequant_launch(codes, scales, M, plan->K, bits, G, out, s))) return st;
  if (!inverse) return ROT_OK;
  if (plan->chunk_log2 >= 5) return fwht_apply(plan, out, ROT_F32, M, plan->K, 1, out, plan->K, s);
  return stages_apply(plan, out, ROT_F32, M, plan->K, 1, out, plan->K, s);
}

static rot_status check_w4a4(const uint8_t* Aq, const uint8_t* Wq, int64_t M, int64_t N, int64_t K, int G,
                             const char* fn) {
  if (M < 0 || N <= 0 || K <= 0) return set_error(ROT_EINVAL, std::string(fn) + ": need M >= 0, N > 0, K > 0");
  if (G <= 0 || K % G != 0 || G % 32 != 0 || K % 64 != 0 || N % 16 != 0)
    return set_error(ROT_EINVAL, std::string(fn) + ": need K % G == 0, G % 32 == 0, K % 64 == 0, N % 16 == 0");
  if ((M > 0 && (!Aq || !aligned16(Aq))) || !Wq || !aligned16(Wq))
    return set_error(ROT_EINVAL, std::string(fn) + ": Aq / Wq must be non-NULL and 16-byte aligned");
  return ROT_OK;
}

extern "C" rot_status w4a4_linear(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq,
                                  const uint16_t* Ws, int64_t M, int64_t N, int64_t K, int G, void* C,
                                  int c_dtype, void* stream) {
  rot_status st = check_w4a4(Aq, Wq, M, N, K, G, "w4a4_linear");
  if (st) return st;
  if (c_dtype != ROT_F32 && c_dtype != ROT_BF16) return set_error(ROT_EINVAL, "w4a4_linear: c_dtype must be ROT_F32 or ROT_BF16");
  if (M == 0) return ROT_OK;
  if (!As || !Ws || !C || !aligned16(C)) return set_error(ROT_EINVAL, "w4a4_linear: As, Ws, C must be non-NULL, C 16-byte aligned");
  return w4a4_launch(Aq, As, Wq, Ws, M, N, K, G, C, c_dtype, nullptr, static_cast<cudaStream_t>(stream));
}

extern "C" rot_status w4a4_linear_noalloc(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq,
                                          const uint16_t* Ws, int64_t M, int64_t N, int64_t K, int G, void* C,
                                          int c_dtype, void* stream) {
  rot_status st = check_w4a4(Aq, Wq, M, N, K, G, "w4a4_linear_noalloc");
  if (st) return st;
  if (c_dtype != ROT_F32 && c_dtype != ROT_BF16)
    return set_error(ROT_EINVAL, "w4a4_linear_noalloc: c_dtype must be ROT_F32 or ROT_BF16");
  if (M == 0) return ROT_OK;
  if (!As || !Ws || !C || !aligned16(C))
    return set_error(ROT_EINVAL, "w4a4_linear_noalloc: As, Ws, C must be non-NULL, C 16-byte aligned");
  float* scratch = nullptr;
  st = w4a4_noalloc_scratch(&scratch);
  if (st) return st;
  return w4a4_launch(Aq, As, Wq, Ws, M, N, K, G, C, c_dtype, nullptr, static_cast<cudaStream_t>(stream), scratch,
                     W4A4_NOALLOC_SCRATCH_FLOATS);
}

extern "C" rot_status w4a4_linear_rot(const uint8_t* Aq, const uint16_t* As, const uint8_t* Wq,
                                      const uint16_t* Ws, int64_t M, int64_t N, int64_t K, int G,
                                      rot_plan_t out_plan, void* C, int c_dtype, void* stream) {
  rot_status st = check_w4a4(Aq, Wq, M, N, K, G, "w4a4_linear_rot");
  if (st) return st;
  if ((st = check_plan(out_plan, "w4a4_linear_rot"))) return st;
  if (out_plan->K != N) return set_error(ROT_EINVAL, "w4a4_linear_rot: the output-side plan must have K == N");
  if (c_dtype != ROT_F32 && c_dtype != ROT_BF16)
    return set_error(ROT_EINVAL, "w4a4_linear_rot: c_dtype must be ROT_F32 or ROT_BF16");
  if (M == 0) return ROT_OK;
  if (!As || !Ws || !C || !aligned16(C))
    return set_error(ROT_EINVAL, "w4a4_linear_rot: As, Ws, C must be non-NULL, C 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // fp32 target of the linear and of the in-place output-side rotation: C itself, or a
  // stream-ordered temporary converted to bf16 afterwards
  float* tgt = static_cast<float*>(C);
  if (c_dtype == ROT_BF16) ROT_CUDA_TRY(cudaMallocAsync(reinterpret_cast<void**>(&tgt), (size_t)(M * N) * 4, s));
  st = w4a4_launch(Aq, As, Wq, Ws, M, N, K, G, tgt, ROT_F32, nullptr, s);
  if (!st) {
    // rows c~ = U c of the linear's output back to c = U^T c~ (inverse of the output-side plan)
    st = out_plan->chunk_log2 >= 5 ? fwht_apply(out_plan, tgt, ROT_F32, M, N, 1, tgt, N, s)
                                   : stages_apply(out_plan, tgt, ROT_F32, M, N, 1, tgt, N, s);
  }
  if (!st && c_dtype == ROT_BF16) st = f32_to_bf16_launch(tgt, C, M * N, s);
  if (c_dtype == ROT_BF16) {
    const cudaError_t e = cudaFreeAsync(tgt, s);
    if (!st && e != cudaSuccess) st = cuda_error(e, "w4a4_linear_rot: cudaFreeAsync");
  }
  return st;
}

static int64_t align16(int64_t x) { return (x + 15) & ~int64_t(15); }

extern "C" rot_status w4a4_linear_act_workspace(int64_t M, int64_t K, int G, size_t* bytes) {
  if (!bytes || M < 0 || K <= 0 || G <= 0 || K % G != 0 || K % 2 != 0)
    return set_error(ROT_EINVAL, "w4a4_linear_act_workspace: need bytes, M >= 0, K > 0, G | K");
  *bytes = (size_t)(align16(M * (K / 2)) + align16(M * (K / G) * 2));
  return ROT_OK;
}

extern "C" rot_status w4a4_linear_act(const void* A, int a_dtype, int64_t M, int64_t lda, rot_plan_t plan,
                                      const uint8_t* Wq, const uint16_t* Ws, int64_t N, int G, void* C,
                                      int c_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  rot_status st = check_plan(plan, "w4a4_linear_act");
  if (st) return st;
  const int64_t K = plan->K;
  if ((st = check_rows(A, a_dtype, M, lda, (int)K, "w4a4_linear_act"))) return st;
  if ((st = check_quant((int)K, 4, G, "w4a4_linear_act"))) return st;
  if ((st = check_w4a4(nullptr, Wq, 0, N, K, G, "w4a4_linear_act"))) return st;
  if (c_dtype != ROT_F32 && c_dtype != ROT_BF16)
    return set_error(ROT_EINVAL, "w4a4_linear_act: c_dtype must be ROT_F32 or ROT_BF16");
  if (M == 0) return ROT_OK;
  size_t need = 0;
  w4a4_linear_act_workspace(M, K, G, &need);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need)
    return set_error(ROT_EINVAL, "w4a4_linear_act: workspace must be 16-byte aligned and hold "
                                 "w4a4_linear_act_workspace bytes");
  if (!Ws || !C || !aligned16(C)) return set_error(ROT_EINVAL, "w4a4_linear_act: Ws and C must be non-NULL, C 16-byte aligned");
  uint8_t* codes = static_cast<uint8_t*>(workspace);
  uint16_t* scales = reinterpret_cast<uint16_t*>(codes + align16(M * (K / 2)));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = fwht_quant_supported(plan, 4, G) ? fwht_quant(plan, A, a_dtype, M, lda, 4, G, codes, scales, s)
                                        : stages_quant(plan, A, a_dtype, M, lda, 4, G, codes, scales, s);
  if (st) return st;
  // the linear's set-up overlaps the rotation's tail; it reads the codes after that kernel completes
  return w4a4_launch(codes, scales, Wq, Ws, M, N, K, G, C, c_dtype, nullptr, s, nullptr, 0, false, true);
}

extern "C" rot_status w4a8_linear(const int8_t* Aq, const uint16_t* As, const uint8_t* Wq,
                                  const uint16_t* Ws, int64_t M, int64_t N, int64_t K, int G, void* C,
                                  int c_dtype, void* stream) {
  const uint8_t* A = reinterpret_cast<const uint8_t*>(Aq);
  rot_status st = check_w4a4(A, Wq, M, N, K, G, "w4a8_linear");
  if (st) return st;
  if (c_dtype != ROT_F32 && c_dtype != ROT_BF16) return set_error(ROT_EINVAL, "w4a8_linear: c_dtype must be ROT_F32 or ROT_BF16");
  if (M == 0) return ROT_OK;
  if (!As || !Ws || !C || !aligned16(C)) return set_error(ROT_EINVAL, "w4a8_linear: As, Ws, C must be non-NULL, C 16-byte aligned");
  return w4a4_launch(A, As, Wq, Ws, M, N, K, G, C, c_dtype, nullptr, static_cast<cudaStream_t>(stream), nullptr, 0,
                     true);
}

extern "C" rot_status w4a8_group_partials(const int8_t* Aq, const uint8_t* Wq, int64_t M, int64_t N,
                                          int64_t K, int G, int32_t* P, void* stream) {
  const uint8_t* A = reinterpret_cast<const uint8_t*>(Aq);
  rot_status st = check_w4a4(A, Wq, M, N, K, G, "w4a8_group_partials");
  if (st) return st;
  if (M == 0) return ROT_OK;
  if (!P || !aligned16(P)) return set_error(ROT_EINVAL, "w4a8_group_partials: P must be non-NULL and 16-byte aligned");
  return w4a4_launch(A, nullptr, Wq, nullptr, M, N, K, G, nullptr, ROT_F32, P, static_cast<cudaStream_t>(stream),
                     nullptr, 0, true);
}

extern "C" rot_status w4a4_tile_plan(int64_t M, int64_t N, int64_t K, int G, int sms, int partials,
                                     int64_t* out) {
  if (!out) return set_error(ROT_EINVAL, "w4a4_tile_plan: out must be non-NULL");
  if (K % 64 != 0 || N % 16 != 0)
    return set_error(ROT_EINVAL, "w4a4_tile_plan: need K % 64 == 0 and N % 16 == 0");
  W4A4TilePlan tp;
  rot_status st = w4a4_tile_plan_compute(M, N, K, G, sms, partials != 0, &tp);
  if (st) return st;
  out[0] = tp.tiles_m;
  out[1] = tp.tiles_n;
  out[2] = tp.splits;
  out[3] = tp.kb_per_split;
  out[4] = tp.units;
  out[5] = tp.grid;
  return ROT_OK;
}

extern "C" rot_status w4a4_group_partials(const uint8_t* Aq, const uint8_t* Wq, int64_t M, int64_t N,
                                          int64_t K, int G, int32_t* P, void* stream) {
  rot_status st = check_w4a4(Aq, Wq, M, N, K, G, "w4a4_group_partials");
  if (st) return st;
  if (M == 0) return ROT_OK;
  if (!P || !aligned16(P)) return set_error(ROT_EINVAL, "w4a4_group_partials: P must be non-NULL and 16-byte aligned");
  return w4a4_launch(Aq, nullptr, Wq, nullptr, M, N, K, G, nullptr, ROT_F32, P, static_cast<cudaStream_t>(stream));
}

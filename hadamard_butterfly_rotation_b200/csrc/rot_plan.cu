// Rotation plans: validation, stage classification, device upload; host helpers that
// build HARP blocks; error reporting.
//
// A plan describes T = (P_{m-1} S_{m-1}) ... (P_0 S_0) D over a mixed-radix schedule
// [HARP gist.science summary, 2.1 core architecture; 2.2 Hadamard preconditioning].
// Stage t mixes the b_t coordinates base + r*s_t (s_t = prod_{u<t} b_u) with block
// c = low + high*s_t. Plans whose non-identity stages are unpermuted normalised
// Sylvester-Hadamard stages over the leading digits are, per contiguous chunk of
// 2^n coordinates, a signed Walsh-Hadamard transform [HARP abstract: the processor
// initialises to the RHT]; those run on the fused butterfly kernel.
#include <cstdlib>
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "rot_internal.cuh"

namespace rotb {

static thread_local std::string g_last_error;

rot_status set_error(rot_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

rot_status cuda_error(cudaError_t e, const char* what) {
  return set_error(ROT_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int sm_count() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static std::atomic<int> g_test_fault{TEST_FAULT_NONE};
static std::atomic<long long> g_test_wait_ns{0};

bool take_test_fault(int which) {
  int expected = which;
  return which != TEST_FAULT_NONE && g_test_fault.compare_exchange_strong(expected, TEST_FAULT_NONE);
}

unsigned long long wait_limit_ns(unsigned long long dflt) {
  const long long v = g_test_wait_ns.load();
  return v > 0 ? (unsigned long long)v : dflt;
}

bool pdl_default() {
  static const bool on = [] {
    const char* e = std::getenv("ROT_B200_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

static bool is_pow2(int64_t x) { return x >= 1 && (x & (x - 1)) == 0; }

// Entry (r, c) of the Sylvester matrix H_b: (-1)^popcount(r & c).
static int sylv(int r, int c) { return (__builtin_popcount((unsigned)(r & c)) & 1) ? -1 : 1; }

static void free_plan_memory(rot_plan_s* p) {
  if (p->d_signmask) cudaFree(p->d_signmask);
  for (auto& s : p->stages) {
    if (s.d_blocks) cudaFree(s.d_blocks);
    if (s.d_blocks_pad) cudaFree(s.d_blocks_pad);
    if (s.d_perm) cudaFree(s.d_perm);
    if (s.d_iperm) cudaFree(s.d_iperm);
  }
  if (p->d_signf) cudaFree(p->d_signf);
}

}  // namespace rotb

using namespace rotb;

extern "C" const char* rot_last_error(void) { return g_last_error.c_str(); }

extern "C" const char* rot_version(void) { return "rot_b200 1.1 (sm_100a)"; }

extern "C" rot_status rot_test_inject(int fault, int64_t wait_ns) {
  if (fault < TEST_FAULT_NONE || fault > TEST_FAULT_W4A4_LOADS || wait_ns < 0)
    return set_error(ROT_EINVAL, "rot_test_inject: unknown fault or negative wait bound");
  g_test_wait_ns.store(wait_ns);
  g_test_fault.store(fault);
  return ROT_OK;
}

extern "C" rot_status rot_plan_create(rot_plan_t* out, int K, int n_stages, const int* radices,
                                      const float* const* stage_params, const int64_t* n_blocks,
                                      const int32_t* const* perms, const int8_t* signs) {
  if (!out) return set_error(ROT_EINVAL, "rot_plan_create: out is NULL");
  *out = nullptr;
  if (K < 1 || n_stages < 1 || !radices)
    return set_error(ROT_EINVAL, "rot_plan_create: need K >= 1, n_stages >= 1, radices");
  int64_t prod = 1;
  for (int t = 0; t < n_stages; ++t) {
    if (radices[t] < 2) return set_error(ROT_EINVAL, "rot_plan_create: every radix must be >= 2");
    prod *= radices[t];
    if (prod > K) break;
  }
  if (prod != K) return set_error(ROT_EINVAL, "rot_plan_create: product of radices != K");
  if (signs) {
    for (int i = 0; i < K; ++i)
      if (signs[i] != 1 && signs[i] != -1)
        return set_error(ROT_EINVAL, "rot_plan_create: signs must be +1 or -1");
  }

  rot_plan_s* p = new rot_plan_s();
  p->K = K;
  cudaGetDevice(&p->device);
  p->has_signs = signs != nullptr;
  int64_t stride = 1;
  std::vector<float> host;
  for (int t = 0; t < n_stages; ++t) {
    Stage st;
    st.b = radices[t];
    st.stride = (int)stride;
    const int b = st.b;
    const float* prm = stage_params ? stage_params[t] : nullptr;
    if (prm) {
      int64_t nb = n_blocks ? n_blocks[t] : 0;
      if (nb != 1 && nb != K / b) {
        delete p;
        return set_error(ROT_EINVAL, "rot_plan_create: n_blocks[t] must be 1 or K/b_t");
      }
      st.n_blocks = nb;
      host.assign(prm, prm + nb * b * b);
      // classify: identity / normalised Sylvester-Hadamard
      bool ident = true, had = is_pow2(b);
      const float hval = (float)(1.0 / std::sqrt((double)b));
      for (int64_t blk = 0; blk < nb && (ident || had); ++blk)
        for (int r = 0; r < b; ++r)
          for (int c = 0; c < b; ++c) {
            float v = host[(blk * b + r) * b + c];
            if (v != (r == c ? 1.0f : 0.0f)) ident = false;
            if (had && v != sylv(r, c) * hval) had = false;
          }
      st.identity = ident;
      st.hadamard = had && !ident;
    } else {
      st.n_blocks = 1;
      host.assign((size_t)b * b, 0.0f);
      if (is_pow2(b)) {
        const double h = 1.0 / std::sqrt((double)b);
        for (int r = 0; r < b; ++r)
          for (int c = 0; c < b; ++c) host[r * b + c] = (float)(sylv(r, c) * h);
        st.hadamard = true;
      } else {
        for (int r = 0; r < b; ++r) host[r * b + r] = 1.0f;
        st.identity = true;
      }
    }
    if (!st.identity) {
      size_t bytes = host.size() * sizeof(float);
      if (cudaMalloc(&st.d_blocks, bytes) != cudaSuccess) {
        delete p;
        return set_error(ROT_ENOMEM, "rot_plan_create: cudaMalloc(blocks)");
      }
      cudaMemcpy(st.d_blocks, host.data(), bytes, cudaMemcpyHostToDevice);
      if (st.n_blocks > 1 && b > 2 && b <= 48) {
        // padded copy for the multi-row kernel's per-block dense stages
        const int bp = (b + 3) & ~3;
        std::vector<float> pad((size_t)st.n_blocks * b * bp, 0.0f);
        for (int64_t c = 0; c < st.n_blocks; ++c)
          for (int r = 0; r < b; ++r)
            for (int k = 0; k < b; ++k) pad[((size_t)c * b + r) * bp + k] = host[((size_t)c * b + r) * b + k];
        if (cudaMalloc(&st.d_blocks_pad, pad.size() * sizeof(float)) != cudaSuccess) {
          cudaFree(st.d_blocks);
          free_plan_memory(p);
          delete p;
          return set_error(ROT_ENOMEM, "rot_plan_create: cudaMalloc(padded blocks)");
        }
        cudaMemcpy(st.d_blocks_pad, pad.data(), pad.size() * sizeof(float), cudaMemcpyHostToDevice);
      }
    }
    if (perms && perms[t]) {
      std::vector<int32_t> seen(K, 0), inv(K);
      for (int j = 0; j < K; ++j) {
        int32_t v = perms[t][j];
        if (v < 0 || v >= K || seen[v]) {
          free_plan_memory(p);
          delete p;
          return set_error(ROT_EINVAL, "rot_plan_create: perms[t] is not a permutation of 0..K-1");
        }
        seen[v] = 1;
        inv[v] = j;
      }
      if (cudaMalloc(&st.d_perm, K * sizeof(int32_t)) != cudaSuccess ||
          cudaMalloc(&st.d_iperm, K * sizeof(int32_t)) != cudaSuccess) {
        free_plan_memory(p);
        delete p;
        return set_error(ROT_ENOMEM, "rot_plan_create: cudaMalloc(perm)");
      }
      cudaMemcpy(st.d_perm, perms[t], K * sizeof(int32_t), cudaMemcpyHostToDevice);
      cudaMemcpy(st.d_iperm, inv.data(), K * sizeof(int32_t), cudaMemcpyHostToDevice);
    }
    p->max_radix = std::max(p->max_radix, b);
    stride *= b;
    p->stages.push_back(st);
  }

  // sign vectors: +-1.0f per coordinate (generic kernel) and bf16-pair XOR masks (fused kernel)
  std::vector<float> sf(K, 1.0f);
  if (signs)
    for (int i = 0; i < K; ++i) sf[i] = (float)signs[i];
  if (cudaMalloc(&p->d_signf, K * sizeof(float)) != cudaSuccess) {
    free_plan_memory(p);
    delete p;
    return set_error(ROT_ENOMEM, "rot_plan_create: cudaMalloc(signs)");
  }
  cudaMemcpy(p->d_signf, sf.data(), K * sizeof(float), cudaMemcpyHostToDevice);

  // fused path: leading stages Hadamard (power-of-two radices), the rest identity, no perms
  {
    bool ok = true;
    int t = 0;
    int64_t chunk = 1;
    while (t < n_stages && p->stages[t].hadamard && !p->stages[t].d_perm) chunk *= p->stages[t++].b;
    for (; t < n_stages; ++t)
      if (!p->stages[t].identity || p->stages[t].d_perm) ok = false;
    for (auto& s : p->stages)
      if (s.d_perm) ok = false;
    int n = 0;
    while ((int64_t(1) << n) < chunk) ++n;
    if (ok && n >= 5 && n <= 13 && (K % 2) == 0) {
      p->chunk_log2 = n;
      std::vector<uint32_t> mk(K / 2, 0u);
      if (signs)
        for (int i = 0; i < K / 2; ++i)
          mk[i] = (signs[2 * i] < 0 ? 0x8000u : 0u) | (signs[2 * i + 1] < 0 ? 0x80000000u : 0u);
      if (cudaMalloc(&p->d_signmask, (K / 2) * sizeof(uint32_t)) != cudaSuccess) {
        free_plan_memory(p);
        delete p;
        return set_error(ROT_ENOMEM, "rot_plan_create: cudaMalloc(signmask)");
      }
      cudaMemcpy(p->d_signmask, mk.data(), (K / 2) * sizeof(uint32_t), cudaMemcpyHostToDevice);
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    free_plan_memory(p);
    delete p;
    return cuda_error(e, "rot_plan_create");
  }
  *out = p;
  return ROT_OK;
}

extern "C" rot_status rot_plan_destroy(rot_plan_t plan) {
  if (!plan) return ROT_OK;
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(plan->device);
  cudaDeviceSynchronize();
  free_plan_memory(plan);
  cudaSetDevice(cur);
  delete plan;
  return ROT_OK;
}

extern "C" rot_status rot_plan_info(rot_plan_t plan, int* K, int* chunk) {
  if (!plan) return set_error(ROT_EINVAL, "rot_plan_info: plan is NULL");
  if (K) *K = plan->K;
  if (chunk) *chunk = plan->chunk_log2 >= 0 ? (1 << plan->chunk_log2) : 0;
  return ROT_OK;
}

extern "C" rot_status rot_harp_givens_blocks(const double* theta, int64_t n, float* out) {
  if (n < 0 || (n > 0 && (!theta || !out)))
    return set_error(ROT_EINVAL, "rot_harp_givens_blocks: bad arguments");
  const double h = 1.0 / std::sqrt(2.0);
  for (int64_t i = 0; i < n; ++i) {
    const double c = std::cos(theta[i]), s = std::sin(theta[i]);
    // [[c, -s], [s, c]] . [[h, h], [h, -h]]
    out[4 * i + 0] = (float)((c - s) * h);
    out[4 * i + 1] = (float)((c + s) * h);
    out[4 * i + 2] = (float)((s + c) * h);
    out[4 * i + 3] = (float)((s - c) * h);
  }
  return ROT_OK;
}

// Cayley map Q = (I + S)^{-1} (I - S) of the skew-symmetric S with strictly upper entries
// params (row-major order), times the base mixer G: B = Q G [HARP gist.science summary, 2.2:
// B = Q(theta) G, Q a Cayley map for b > 2]. I + S is never singular (the eigenvalues of S are
// imaginary); Gaussian elimination with partial pivoting in double.
extern "C" rot_status rot_harp_cayley_block(const double* params, int b, const float* mixer, float* out) {
  if (b < 2 || !out || (!params && b > 1)) return set_error(ROT_EINVAL, "rot_harp_cayley_block: bad arguments");
  std::vector<double> A((size_t)b * b, 0.0), X((size_t)b * b, 0.0);
  int k = 0;
  for (int i = 0; i < b; ++i) {
    A[i * b + i] = 1.0;
    X[i * b + i] = 1.0;
  }
  for (int i = 0; i < b; ++i)
    for (int j = i + 1; j < b; ++j, ++k) {
      A[i * b + j] += params[k];    // I + S
      A[j * b + i] -= params[k];
      X[i * b + j] -= params[k];    // I - S
      X[j * b + i] += params[k];
    }
  for (int c = 0; c < b; ++c) {
    int piv = c;
    for (int r = c + 1; r < b; ++r)
      if (std::fabs(A[r * b + c]) > std::fabs(A[piv * b + c])) piv = r;
    if (A[piv * b + c] == 0.0) return set_error(ROT_EINVAL, "rot_harp_cayley_block: singular I + S");
    if (piv != c)
      for (int j = 0; j < b; ++j) {
        std::swap(A[c * b + j], A[piv * b + j]);
        std::swap(X[c * b + j], X[piv * b + j]);
      }
    for (int r = 0; r < b; ++r) {
      if (r == c) continue;
      const double f = A[r * b + c] / A[c * b + c];
      if (f == 0.0) continue;
      for (int j = 0; j < b; ++j) {
        A[r * b + j] -= f * A[c * b + j];
        X[r * b + j] -= f * X[c * b + j];
      }
    }
  }
  for (int r = 0; r < b; ++r)
    for (int j = 0; j < b; ++j) X[r * b + j] /= A[r * b + r];
  // B = Q G, G = mixer (row-major b x b) or the base mixer
  std::vector<double> G((size_t)b * b, 0.0);
  if (mixer) {
    for (int i = 0; i < b * b; ++i) G[i] = mixer[i];
  } else if (is_pow2(b)) {
    const double h = 1.0 / std::sqrt((double)b);
    for (int r = 0; r < b; ++r)
      for (int c = 0; c < b; ++c) G[r * b + c] = sylv(r, c) * h;
  } else {
    for (int r = 0; r < b; ++r) G[r * b + r] = 1.0;
  }
  for (int r = 0; r < b; ++r)
    for (int c = 0; c < b; ++c) {
      double acc = 0.0;
      for (int j = 0; j < b; ++j) acc += X[r * b + j] * G[j * b + c];
      out[r * b + c] = (float)acc;
    }
  return ROT_OK;
}

namespace rotb {
namespace {

// Givens blocks of a stage from its int8 codes, on the device: theta = code * scale,
// B = R(theta) H_2 / sqrt(2) [HARP gist.science summary, 2.2 (Givens for b = 2) and 2.4 (int8
// parameter storage)]. One thread per block.
__global__ void givens_expand_kernel(const int8_t* __restrict__ codes, float scale, int64_t n,
                                     float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float th = (float)codes[i] * scale;
    float sn, cs;
    sincosf(th, &sn, &cs);
    const float h = 0.70710678118654752f;
    float4 v;
    v.x = (cs - sn) * h;
    v.y = (cs + sn) * h;
    v.z = (sn + cs) * h;
    v.w = (sn - cs) * h;
    reinterpret_cast<float4*>(out)[i] = v;
  }
}

}  // namespace
}  // namespace rotb

extern "C" rot_status rot_plan_create_q8(rot_plan_t* out, int K, int n_stages, const int* radices,
                                         const int8_t* const* codes, const float* scales,
                                         const int64_t* n_blocks, const float* const* mixers,
                                         const int32_t* const* perms, const int8_t* signs) {
  if (!out) return set_error(ROT_EINVAL, "rot_plan_create_q8: out is NULL");
  *out = nullptr;
  if (K < 1 || n_stages < 1 || n_stages > 64 || !radices)
    return set_error(ROT_EINVAL, "rot_plan_create_q8: need K >= 1, 1 <= n_stages <= 64, radices");
  for (int t = 0; t < n_stages; ++t)
    if (radices[t] < 2 || K % radices[t] != 0) return set_error(ROT_EINVAL, "rot_plan_create_q8: bad radix");
  std::vector<std::vector<float>> host(n_stages);
  std::vector<const float*> params(n_stages, nullptr);
  std::vector<int64_t> nb(n_stages, 0);
  std::vector<int> expand(n_stages, 0);   // Givens stages built on the device after plan creation
  for (int t = 0; t < n_stages; ++t) {
    const int b = radices[t];
    const int8_t* q = codes ? codes[t] : nullptr;
    const float* mix = mixers ? mixers[t] : nullptr;
    if (b == 2 && mix) return set_error(ROT_EINVAL, "rot_plan_create_q8: a radix-2 stage takes no mixer");
    if (!q) {   // theta = 0: the block is the mixer
      if (mix) {
        host[t].assign(mix, mix + (size_t)b * b);
        params[t] = host[t].data();
        nb[t] = 1;
      }
      continue;
    }
    if (!scales || !n_blocks || (n_blocks[t] != 1 && n_blocks[t] != K / b))
      return set_error(ROT_EINVAL, "rot_plan_create_q8: a stage with codes needs a scale and n_blocks 1 or K/b");
    const int64_t n = n_blocks[t];
    const int npb = b == 2 ? 1 : b * (b - 1) / 2;   // codes per block
    bool any = false;
    for (int64_t i = 0; i < n * npb && !any; ++i) any = q[i] != 0;
    if (!any && !mix) continue;                      // all zero: the base mixer
    nb[t] = n;
    host[t].assign((size_t)n * b * b, 0.0f);
    params[t] = host[t].data();
    if (b == 2) {   // placeholder blocks, replaced on the device by the expansion kernel
      expand[t] = 1;
      continue;
    }
    std::vector<double> th(npb);
    for (int64_t c = 0; c < n; ++c) {
      for (int k = 0; k < npb; ++k) th[k] = (double)q[c * npb + k] * (double)scales[t];
      rot_status st = rot_harp_cayley_block(th.data(), b, mix, host[t].data() + (size_t)c * b * b);
      if (st) return st;
    }
  }
  rot_status st = rot_plan_create(out, K, n_stages, radices, params.data(), nb.data(), perms, signs);
  if (st) return st;
  for (int t = 0; t < n_stages; ++t) {
    if (!expand[t]) continue;
    Stage& S = (*out)->stages[t];
    const int64_t n = nb[t];
    int8_t* dq = nullptr;
    cudaError_t e = cudaMalloc(&dq, (size_t)n);
    if (e == cudaSuccess) e = cudaMemcpy(dq, codes[t], (size_t)n, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
      const int64_t grid = std::min<int64_t>((n + 255) / 256, 4096);
      givens_expand_kernel<<<(unsigned)grid, 256>>>(dq, scales[t], n, S.d_blocks);
      e = cudaGetLastError();
      if (e == cudaSuccess) e = cudaDeviceSynchronize();
    }
    if (dq) cudaFree(dq);
    if (e != cudaSuccess) {
      rot_plan_destroy(*out);
      *out = nullptr;
      return cuda_error(e, "rot_plan_create_q8: expanding Givens blocks");
    }
  }
  return ROT_OK;
}

extern "C" rot_status rot_harp_qr_block(const double* g, int b, float* out) {
  if (b < 1 || !g || !out) return set_error(ROT_EINVAL, "rot_harp_qr_block: bad arguments");
  // Householder QR of the b x b matrix g: R = H_{b-1} ... H_0 g, Q = H_0 ... H_{b-1};
  // then the columns of Q are flipped so that diag(R) > 0.
  std::vector<double> R(g, g + (size_t)b * b), Q((size_t)b * b, 0.0), v(b);
  for (int i = 0; i < b; ++i) Q[i * b + i] = 1.0;
  for (int k = 0; k < b - 1; ++k) {
    double norm = 0.0;
    for (int i = k; i < b; ++i) norm += R[i * b + k] * R[i * b + k];
    norm = std::sqrt(norm);
    if (norm == 0.0) continue;
    const double alpha = R[k * b + k] > 0 ? -norm : norm;
    double vnorm2 = 0.0;
    for (int i = 0; i < b; ++i) v[i] = 0.0;
    for (int i = k; i < b; ++i) v[i] = R[i * b + k];
    v[k] -= alpha;
    for (int i = k; i < b; ++i) vnorm2 += v[i] * v[i];
    if (vnorm2 == 0.0) continue;
    // R <- (I - 2 v v^T / v^T v) R
    for (int c = 0; c < b; ++c) {
      double d = 0.0;
      for (int i = k; i < b; ++i) d += v[i] * R[i * b + c];
      d = 2.0 * d / vnorm2;
      for (int i = k; i < b; ++i) R[i * b + c] -= d * v[i];
    }
    // Q <- Q (I - 2 v v^T / v^T v)
    for (int r = 0; r < b; ++r) {
      double d = 0.0;
      for (int i = k; i < b; ++i) d += Q[r * b + i] * v[i];
      d = 2.0 * d / vnorm2;
      for (int i = k; i < b; ++i) Q[r * b + i] -= d * v[i];
    }
  }
  for (int c = 0; c < b; ++c) {
    const double sgn = R[c * b + c] < 0 ? -1.0 : 1.0;
    for (int r = 0; r < b; ++r) out[r * b + c] = (float)(Q[r * b + c] * sgn);
  }
  return ROT_OK;
}

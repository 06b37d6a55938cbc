// Dequantisation x_hat = q * s of packed int8 / int4 / int2 codes with binary16 group scales
// [Hadamard-Int4-Accuracy wiki, Method: q_dequant_vec quantise -> dequantise].
// One thread per 32-bit code word (4 int8, 8 int4 or 16 int2 codes); fp32 output rows.
#include "rot_internal.cuh"

namespace rotb {
namespace {

template <int BITS>
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ codes,
                                                      const uint16_t* __restrict__ scales,
                                                      int64_t n_words, int K, int G,
                                                      float* __restrict__ out) {
  constexpr int CPW = 32 / BITS;
  const int64_t words_per_row = K / CPW;
  const int64_t ngr = K / G;
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < n_words;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = w / words_per_row;
    const int64_t col = (w - row * words_per_row) * CPW;
    const float s = __half2float(__ushort_as_half(scales[row * ngr + col / G]));
    const uint32_t c = codes[w];
    float v[CPW];
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int q = ((int)(c << (32 - BITS * (j + 1)))) >> (32 - BITS);  // sign-extend field j
      v[j] = (float)q * s;
    }
    float4* dst = reinterpret_cast<float4*>(out + row * (int64_t)K + col);
#pragma unroll
    for (int j = 0; j < CPW / 4; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  }
}

}  // namespace

rot_status dequant_launch(const uint8_t* codes, const uint16_t* scales, int64_t M, int K, int bits,
                          int G, float* out, cudaStream_t s) {
  const int cpw = 32 / bits;
  const int64_t n_words = M * (K / cpw);
  if (n_words == 0) return ROT_OK;
  const int64_t grid = std::min<int64_t>((n_words + 255) / 256, (int64_t)sm_count() * 8);
  if (bits == 8)
    dequant_kernel<8><<<(unsigned)grid, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(codes), scales, n_words, K, G, out);
  else if (bits == 4)
    dequant_kernel<4><<<(unsigned)grid, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(codes), scales, n_words, K, G, out);
  else
    dequant_kernel<2><<<(unsigned)grid, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(codes), scales, n_words, K, G, out);
  ROT_CUDA_TRY(cudaGetLastError());
  return ROT_OK;
}

}  // namespace rotb

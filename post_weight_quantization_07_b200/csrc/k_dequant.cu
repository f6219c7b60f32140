// Dequantisation of packed GPTQ output: Q[i][j] = scale[i][g] * (q[i][j] - zero[i][g])
// with g = j / groupsize, codes read from each row's LSB-first bitstream of
// wbits-bit codes (the layout oc_gptq_quantize writes; a 3-bit code may
// straddle two words).  One thread per output element, HBM bound.
#include <cuda_bf16.h>

#include "oc_internal.cuh"

namespace oc {
namespace {

template <bool BF16>
__global__ void dequant_kernel(const uint32_t* __restrict__ codes, const float* __restrict__ scales,
                               const float* __restrict__ zeros, int64_t m, int64_t n, int wbits, int64_t G,
                               void* __restrict__ out) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= m * n) return;
  const int64_t i = e / n, j = e % n;
  const int64_t words = n * wbits / 32;
  const uint32_t* row = codes + i * words;
  const int64_t bit = j * wbits;
  const int64_t w = bit >> 5;
  const int s = static_cast<int>(bit & 31);
  uint32_t v = row[w] >> s;
  if (s + wbits > 32) v |= row[w + 1] << (32 - s);
  const float q = static_cast<float>(v & ((1u << wbits) - 1u));
  const int64_t g = j / G;
  const int64_t ng = n / G;
  const float x = scales[i * ng + g] * (q - zeros[i * ng + g]);
  if (BF16) static_cast<__nv_bfloat16*>(out)[e] = __float2bfloat16_rn(x);
  else static_cast<float*>(out)[e] = x;
}

}  // namespace

void launch_dequant(const Ctx& c, const uint32_t* codes, const float* scales, const float* zeros, int64_t m,
                    int64_t n, int wbits, int64_t G, void* out, bool bf16) {
  const int64_t total = m * n;
  const unsigned blocks = static_cast<unsigned>((total + 255) / 256);
  if (bf16) dequant_kernel<true><<<blocks, 256, 0, c.stream>>>(codes, scales, zeros, m, n, wbits, G, out);
  else dequant_kernel<false><<<blocks, 256, 0, c.stream>>>(codes, scales, zeros, m, n, wbits, G, out);
  check_launch("dequant_kernel");
}

}  // namespace oc

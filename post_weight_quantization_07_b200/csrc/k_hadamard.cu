// Block Hadamard rotation along the feature axis:  Y = X (I_{n/b} (x) H_b) / sqrt(b)
// with H_b the Sylvester Hadamard matrix of order b (a power of two, 2..4096),
// i.e. every contiguous segment of b features of every row goes through an
// orthonormal fast Walsh-Hadamard transform.  Rotating a layer's weight rows
// and its input rows by the same orthonormal matrix leaves W X^T unchanged.
//
// The array is processed flat (rows x n elements; n is a multiple of b, so
// segments never straddle rows) in chunks of 4096 elements per CTA of 256
// threads, 16 contiguous elements per thread: butterfly strides 1..8 run in
// registers, 16..256 across the lanes of a warp (shuffles), 512..2048 across
// the warps of the CTA (one transpose through shared memory and back).  fp32
// arithmetic; bf16 or fp32 in and out.  HBM bound.
#include <cuda_bf16.h>

#include "oc_internal.cuh"

namespace oc {
namespace {

constexpr int HT = 256;        // threads per CTA
constexpr int HE = 16;         // elements per thread
constexpr int HC = HT * HE;    // elements per chunk

template <bool BF16>
__device__ __forceinline__ void load16(const void* src, int64_t e, int64_t total, float (&v)[HE]) {
  if (e + HE <= total) {
    if (BF16) {
      const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src) + e);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint4 u = p[q];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[8 * q + 2 * k] = __uint_as_float(w[k] << 16);
          v[8 * q + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        }
      }
    } else {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + e);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 u = p[q];
        v[4 * q] = u.x;
        v[4 * q + 1] = u.y;
        v[4 * q + 2] = u.z;
        v[4 * q + 3] = u.w;
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < HE; ++k) {
      float x = 0.f;
      if (e + k < total)
        x = BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(src)[e + k]) : static_cast<const float*>(src)[e + k];
      v[k] = x;
    }
  }
}

template <bool BF16>
__device__ __forceinline__ void store16(void* dst, int64_t e, int64_t total, const float (&v)[HE]) {
  if (e + HE <= total) {
    if (BF16) {
      uint4* p = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + e);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * q + 2 * k], v[8 * q + 2 * k + 1]);
          w[k] = *reinterpret_cast<const uint32_t*>(&h);
        }
        p[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      float4* p = reinterpret_cast<float4*>(static_cast<float*>(dst) + e);
#pragma unroll
      for (int q = 0; q < 4; ++q) p[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < HE; ++k)
      if (e + k < total) {
        if (BF16) static_cast<__nv_bfloat16*>(dst)[e + k] = __float2bfloat16_rn(v[k]);
        else static_cast<float*>(dst)[e + k] = v[k];
      }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(HT) hadamard_kernel(const void* __restrict__ X, void* __restrict__ Y,
                                                      int64_t total, int log2b, float scale) {
  __shared__ float t[HE][HT + 1];  // transpose buffer: [element k][thread]
  const int tid = threadIdx.x, lane = tid & 31;
  for (int64_t chunk = blockIdx.x; chunk * HC < total; chunk += gridDim.x) {
    const int64_t e = chunk * HC + static_cast<int64_t>(tid) * HE;
    float v[HE];
    load16<BF16>(X, e, total, v);
    // strides 1, 2, 4, 8: inside the thread
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      if (s >= log2b) break;
      const int st = 1 << s;
#pragma unroll
      for (int k = 0; k < HE; ++k)
        if (!(k & st)) {
          const float a = v[k], b = v[k + st];
          v[k] = a + b;
          v[k + st] = a - b;
        }
    }
    // strides 16 .. 256: partner lane differs in bit (s - 4) of the lane index
#pragma unroll
    for (int s = 4; s < 9; ++s) {
      if (s >= log2b) break;
      const int lb = 1 << (s - 4);
      const bool upper = lane & lb;
#pragma unroll
      for (int k = 0; k < HE; ++k) {
        const float o = __shfl_xor_sync(0xffffffffu, v[k], lb);
        v[k] = upper ? (o - v[k]) : (v[k] + o);
      }
    }
    // strides 512, 1024, 2048: partner warp differs in bit (s - 9) of the warp
    // index; transpose so that each thread holds one element of every warp
    if (log2b > 9) {
      __syncthreads();
#pragma unroll
      for (int k = 0; k < HE; ++k) t[k][tid] = v[k];
      __syncthreads();
      // Element (k, lane) of every warp w sits at chunk position
      // 512 w + 16 lane + k.  The 16 x 32 = 512 (k, lane) pairs are shared out
      // two per thread; each thread gathers its pairs' 8 values (one per warp)
      // and applies the cross-warp butterflies in registers.
      float w8[2][8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int pair = tid * 2 + h;  // 0..511: (k, lane)
        const int k = pair >> 5, ln = pair & 31;
#pragma unroll
        for (int wv = 0; wv < 8; ++wv) w8[h][wv] = t[k][wv * 32 + ln];
      }
#pragma unroll
      for (int s = 9; s < 12; ++s) {
        if (s >= log2b) break;
        const int wb = 1 << (s - 9);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int wv = 0; wv < 8; ++wv)
            if (!(wv & wb)) {
              const float a = w8[h][wv], b = w8[h][wv + wb];
              w8[h][wv] = a + b;
              w8[h][wv + wb] = a - b;
            }
      }
      __syncthreads();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int pair = tid * 2 + h;
        const int k = pair >> 5, ln = pair & 31;
#pragma unroll
        for (int wv = 0; wv < 8; ++wv) t[k][wv * 32 + ln] = w8[h][wv];
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < HE; ++k) v[k] = t[k][tid];
    }
#pragma unroll
    for (int k = 0; k < HE; ++k) v[k] *= scale;
    store16<BF16>(Y, e, total, v);
  }
}

}  // namespace

void launch_hadamard(const Ctx& c, const void* X, void* Y, int64_t rows, int64_t n, int log2b, bool bf16) {
  const int64_t total = rows * n;
  const int64_t chunks = (total + HC - 1) / HC;
  const int grid = static_cast<int>(std::min<int64_t>(chunks, static_cast<int64_t>(c.sm_count) * 8));
  const float scale = 1.0f / sqrtf(static_cast<float>(int64_t(1) << log2b));
  if (bf16) hadamard_kernel<true><<<grid, HT, 0, c.stream>>>(X, Y, total, log2b, scale);
  else hadamard_kernel<false><<<grid, HT, 0, c.stream>>>(X, Y, total, log2b, scale);
  check_launch("hadamard_kernel");
}

}  // namespace oc

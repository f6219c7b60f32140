// y = x Q^T for a few bf16 activation rows over packed GPTQ codes, with Q
// dequantised on the fly: Q[i][j] = scale[i][g] * (q[i][j] - zero[i][g]),
// g = j / groupsize (the layout oc_gptq_quantize writes: per row an LSB-first
// bitstream of wbits-bit codes).  This is the quantised layer applied at
// decode time, where reading the codes is the cost.
//
// Each warp takes 4 output rows at a time (2 with 5..8 activation rows), 4
// warps per CTA, persistent grid.  Lane l takes the 32-column segments l,
// l + 32, ... of those rows: a segment's 32 codes fill exactly wbits
// consecutive words, so every code is extracted with compile-time shifts (a
// 3-bit code may straddle two words of the segment).  Segments are processed 8
// columns at a time: one 16-byte load of 8 bf16 activations per batch row,
// shared by the warp's rows, then per row 8 dequantised weights and 8 fused
// multiply-adds per batch row into fp32 accumulators; shuffle reductions end
// the rows.  The codes are read once from HBM; the activations, re-read for
// every group of rows, come from L1 (their traffic is what the rows per warp
// divide).
#include <cuda_bf16.h>

#include "oc_internal.cuh"

namespace oc {
namespace {

constexpr int GV_WARPS = 4;

template <int B>
__device__ __forceinline__ uint32_t seg_code(const uint32_t (&w)[B], int k) {
  const int p = k * B;
  const int wi = p >> 5, off = p & 31;
  uint32_t v = w[wi] >> off;
  if (off + B > 32) v |= w[wi + 1] << (32 - off);
  return v & ((1u << B) - 1u);
}

template <int B>
__device__ __forceinline__ void load_seg(const uint32_t* crow, int64_t seg, uint32_t (&w)[B]) {
  if constexpr (B == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(crow + seg * 4);
    w[0] = v.x;
    w[1] = v.y;
    w[2] = v.z;
    w[3] = v.w;
  } else if constexpr (B == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(crow + seg * 2);
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = crow[seg * B + k];
  }
}

// 2^23 + q as a float is the bit pattern 0x4B000000 | q (q < 2^23), so
// q - z = (that float) - (2^23 + z) exactly, without an integer conversion.
constexpr float kMagic = 8388608.f;

// Rows per warp: each 16-byte load of activations serves all of them (the
// activations, re-read for every row, would otherwise dominate L1 traffic).
template <int NB>
constexpr int rows_per_warp() { return NB >= 8 ? 2 : 4; }

template <int B, int NB>
__global__ void __launch_bounds__(GV_WARPS * 32, 3)
dequant_gemv_kernel(const uint32_t* __restrict__ codes, const float* __restrict__ scales,
                    const float* __restrict__ zeros, int64_t m, int64_t n, int64_t G,
                    const __nv_bfloat16* __restrict__ x, int nb, float* __restrict__ y) {
  constexpr int R = rows_per_warp<NB>();
  const int lane = threadIdx.x & 31;
  const int64_t words = n * B / 32;
  const int64_t nseg = n / 32;
  const int64_t ng = n / G;
  const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * GV_WARPS + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * GV_WARPS;
  for (int64_t row0 = warp0 * R; row0 < m; row0 += nwarps * R) {
    float acc[R][NB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
    for (int64_t seg = lane; seg < nseg; seg += 32) {
      // the R rows' code words of this segment (rows past m re-read the last row)
      uint32_t w[R][B];
#pragma unroll
      for (int r = 0; r < R; ++r) load_seg<B>(codes + ::min(row0 + r, m - 1) * words, seg, w[r]);
      const int64_t col0 = seg * 32;
      float s_seg[R], zz_seg[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        s_seg[r] = 0.f;
        zz_seg[r] = 0.f;
        if (G >= 32) {
          const int64_t rr = ::min(row0 + r, m - 1);
          s_seg[r] = scales[rr * ng + col0 / G];
          zz_seg[r] = kMagic + zeros[rr * ng + col0 / G];
        }
      }
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        uint4 xv[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b)
          if (b < nb) xv[b] = __ldg(reinterpret_cast<const uint4*>(x + b * n + col0 + c8 * 8));
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float q[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float f = __uint_as_float(0x4B000000u | seg_code<B>(w[r], c8 * 8 + k));
            float sc = s_seg[r], zz = zz_seg[r];
            if (G < 32) {
              const int64_t rr = ::min(row0 + r, m - 1);
              const int64_t g = (col0 + c8 * 8 + k) / G;
              sc = scales[rr * ng + g];
              zz = kMagic + zeros[rr * ng + g];
            }
            q[k] = sc * (f - zz);
          }
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b < nb) {
              const uint32_t xw[4] = {xv[b].x, xv[b].y, xv[b].z, xv[b].w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                acc[r][b] = fmaf(q[2 * k], __uint_as_float(xw[k] << 16), acc[r][b]);
                acc[r][b] = fmaf(q[2 * k + 1], __uint_as_float(xw[k] & 0xFFFF0000u), acc[r][b]);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float v = acc[r][b];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && b < nb && row0 + r < m) y[b * m + row0 + r] = v;
      }
    }
  }
}

template <int B, int NB>
void launch_gemv_shape(const Ctx& c, const uint32_t* codes, const float* scales, const float* zeros, int64_t m,
                       int64_t n, int64_t G, const __nv_bfloat16* x, int nb, float* y) {
  constexpr int R = rows_per_warp<NB>();
  const int64_t want = (m + GV_WARPS * R - 1) / (GV_WARPS * R);
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(c.sm_count) * 8));
  dequant_gemv_kernel<B, NB><<<grid, GV_WARPS * 32, 0, c.stream>>>(codes, scales, zeros, m, n, G, x, nb, y);
}

template <int B>
void launch_gemv_bits(const Ctx& c, const uint32_t* codes, const float* scales, const float* zeros, int64_t m,
                      int64_t n, int64_t G, const void* x, int nb, float* y) {
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  if (nb <= 1) launch_gemv_shape<B, 1>(c, codes, scales, zeros, m, n, G, xb, nb, y);
  else if (nb <= 2) launch_gemv_shape<B, 2>(c, codes, scales, zeros, m, n, G, xb, nb, y);
  else if (nb <= 4) launch_gemv_shape<B, 4>(c, codes, scales, zeros, m, n, G, xb, nb, y);
  else launch_gemv_shape<B, 8>(c, codes, scales, zeros, m, n, G, xb, nb, y);
  check_launch("dequant_gemv_kernel");
}

}  // namespace

void launch_dequant_gemv(const Ctx& c, const uint32_t* codes, const float* scales, const float* zeros, int64_t m,
                         int64_t n, int wbits, int64_t G, const void* x, int nb, float* y) {
  if (wbits == 4) launch_gemv_bits<4>(c, codes, scales, zeros, m, n, G, x, nb, y);
  else if (wbits == 3) launch_gemv_bits<3>(c, codes, scales, zeros, m, n, G, x, nb, y);
  else launch_gemv_bits<2>(c, codes, scales, zeros, m, n, G, x, nb, y);
}

}  // namespace oc

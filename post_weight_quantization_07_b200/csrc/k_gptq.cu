// GPTQ column sweep, grids and packing.
//
// Sweep of one block of 128 columns (processing order).  One warp owns one
// row of W at a time; lane l holds columns 4l..4l+3 of the block in registers
// and the block's 128x128 slice of U sits in shared memory.  For column j the
// owning lane rounds w_j on its group's grid, forms the scaled error
// e = (w_j - deq) / U_jj and broadcasts it; every lane then applies the
// rank-1 update w_k -= e U_jk to its columns (U_jk = 0 for k < j).  The
// errors of the block are written out for the trailing GEMM that updates all
// later columns.  Rows are independent, so the grid covers rows only.
#include <algorithm>

#include "oc_internal.cuh"

namespace oc {
namespace {

constexpr int SB = 128;          // sweep block width
constexpr int SWEEP_WARPS = 16;

__device__ __forceinline__ void grid_from_minmax(float xmin, float xmax, float maxq, float& s,
                                                 float& z) {
  if (xmax == xmin) {
    xmin -= 1.f;
    xmax += 1.f;
  }
  s = (xmax - xmin) / maxq;
  z = fminf(fmaxf(rintf(-xmin / s), 0.f), maxq);
}

// Wp[r][j] = dead[p(j)] ? 0 : W[r][p(j)], one block per row (row staged in shared memory).
__global__ void permute_w_kernel(const float* __restrict__ W, int64_t n, const int32_t* __restrict__ perm,
                                 const unsigned char* __restrict__ dead, float* __restrict__ Wp) {
  extern __shared__ float row[];
  const int64_t r = blockIdx.x;
  for (int64_t c = threadIdx.x; c < n; c += blockDim.x) row[c] = W[r * n + c];
  __syncthreads();
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const int64_t p = perm[j];
    Wp[r * n + j] = dead[p] ? 0.f : row[p];
  }
}

// act_order grid: one warp per (row, group) over the original column order.
__global__ void static_grid_kernel(const float* __restrict__ W, int64_t m, int64_t n, int G, float maxq,
                                   const unsigned char* __restrict__ dead, float* __restrict__ scales,
                                   float* __restrict__ zeros) {
  const int64_t ng = n / G;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= m * ng) return;
  const int64_t r = wid / ng, g = wid % ng;
  float xmin = INFINITY, xmax = -INFINITY;
  for (int64_t c = g * G + lane; c < (g + 1) * G; c += 32) {
    const float v = dead[c] ? 0.f : W[r * n + c];
    xmin = fminf(xmin, v);
    xmax = fmaxf(xmax, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    xmin = fminf(xmin, __shfl_xor_sync(0xffffffffu, xmin, o));
    xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, o));
  }
  if (lane == 0) {
    float s, z;
    grid_from_minmax(xmin, xmax, maxq, s, z);
    scales[r * ng + g] = s;
    zeros[r * ng + g] = z;
  }
}

__global__ void __launch_bounds__(SWEEP_WARPS * 32)
sweep_block_kernel(float* __restrict__ Wp, int64_t m, int64_t n, const float* __restrict__ U, int64_t j1, int G,
                   float maxq, int static_groups, const int32_t* __restrict__ perm, float* __restrict__ scales,
                   float* __restrict__ zeros, unsigned char* __restrict__ codes8, float* __restrict__ Err) {
  extern __shared__ __align__(16) float Ub[];  // [SB][SB]
  const int bw = static_cast<int>(::min((int64_t)SB, n - j1));
  for (int e = threadIdx.x; e < SB * SB; e += blockDim.x) {
    const int j = e / SB, k = e % SB;
    Ub[e] = (j < bw && k < bw) ? U[(j1 + j) * n + j1 + k] : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ng = n / G;
  const int64_t col0 = j1 + 4 * lane;  // first column of this lane
  // Group starts inside this block (all 32-bit, no division in the loop): a
  // group of at most one block (G divides 128) starts wherever j % G == 0; a
  // wider group can only start at the block's first column.
  const bool g_small = G <= SB;
  const bool block_starts_group = (j1 % G) == 0;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * SWEEP_WARPS + warp; r < m;
       r += static_cast<int64_t>(gridDim.x) * SWEEP_WARPS) {
    float* wrow = Wp + r * n;
    float w[4], s[4], z[4], ev[4];
    unsigned qv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      w[c] = (4 * lane + c < bw) ? wrow[col0 + c] : 0.f;
      s[c] = 1.f;
      z[c] = 0.f;
      ev[c] = 0.f;
      qv[c] = 0u;
      if (static_groups && 4 * lane + c < bw) {
        const int g = perm[col0 + c] / G;
        s[c] = scales[r * ng + g];
        z[c] = zeros[r * ng + g];
      }
    }
    if (!static_groups && !block_starts_group) {
      // a group wider than the block started in an earlier block: its grid
      // was written by that block's sweep
      const int64_t g = j1 / G;
      const float gs = scales[r * ng + g], gz = zeros[r * ng + g];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[c] = gs;
        z[c] = gz;
      }
    }
    for (int j = 0; j < bw; ++j) {
      if (!static_groups && (g_small ? ((j & (G - 1)) == 0) : (j == 0 && block_starts_group))) {
        // group [j1 + j, j1 + j + G): min/max of its current values
        float xmin = INFINITY, xmax = -INFINITY;
        if (g_small) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int k = 4 * lane + c;
            if (k >= j && k < j + G && k < bw) {
              xmin = fminf(xmin, w[c]);
              xmax = fmaxf(xmax, w[c]);
            }
          }
        } else {
          // the group starts at this block and extends beyond it; every column
          // of it is current (earlier blocks' updates are applied, this block's
          // have not started)
          for (int64_t k = j1 + lane; k < j1 + G; k += 32) {
            const float v = wrow[k];
            xmin = fminf(xmin, v);
            xmax = fmaxf(xmax, v);
          }
        }
        for (int o = 16; o > 0; o >>= 1) {
          xmin = fminf(xmin, __shfl_xor_sync(0xffffffffu, xmin, o));
          xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, o));
        }
        float gs, gz;
        grid_from_minmax(xmin, xmax, maxq, gs, gz);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int k = 4 * lane + c;
          if (!g_small || (k >= j && k < j + G)) {
            s[c] = gs;
            z[c] = gz;
          }
        }
        if (lane == 0) {
          const int64_t g = (j1 + j) / G;
          scales[r * ng + g] = gs;
          zeros[r * ng + g] = gz;
        }
      }
      const int owner = j >> 2, comp = j & 3;
      const float4 u = *reinterpret_cast<const float4*>(&Ub[j * SB + 4 * lane]);
      float e = 0.f;
      if (lane == owner) {
        float wj = w[0], sj = s[0], zj = z[0];
#pragma unroll
        for (int c = 1; c < 4; ++c)
          if (comp == c) {
            wj = w[c];
            sj = s[c];
            zj = z[c];
          }
        const float q = fminf(fmaxf(rintf(wj / sj) + zj, 0.f), maxq);
        const float dq = sj * (q - zj);
        e = (wj - dq) / Ub[j * SB + j];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (comp == c) {
            qv[c] = static_cast<unsigned>(q);
            ev[c] = e;
          }
      }
      e = __shfl_sync(0xffffffffu, e, owner);
      w[0] = fmaf(-e, u.x, w[0]);
      w[1] = fmaf(-e, u.y, w[1]);
      w[2] = fmaf(-e, u.z, w[2]);
      w[3] = fmaf(-e, u.w, w[3]);
    }
    if (4 * lane < bw) {
      // bw is a multiple of 4 (n % 64 == 0), so a lane's 4 columns are all valid
      const unsigned packed = qv[0] | (qv[1] << 8) | (qv[2] << 16) | (qv[3] << 24);
      *reinterpret_cast<unsigned*>(codes8 + r * n + col0) = packed;
      *reinterpret_cast<float4*>(Err + r * SB + 4 * lane) = make_float4(ev[0], ev[1], ev[2], ev[3]);
    }
  }
}

// inv[perm[j]] = j
__global__ void invert_perm_kernel(const int32_t* __restrict__ perm, int64_t n, int32_t* __restrict__ inv) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j < n) inv[perm[j]] = static_cast<int32_t>(j);
}

// One thread per packed word: stream bits [32w, 32w+32) of row r take the
// codes of original columns c with [c*b, c*b+b) overlapping them.
__global__ void pack_kernel(const unsigned char* __restrict__ codes8, int64_t m, int64_t n, int wbits,
                            const int32_t* __restrict__ inv, uint32_t* __restrict__ out) {
  const int64_t words = n * wbits / 32;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= m * words) return;
  const int64_t r = e / words, wi = e % words;
  const int64_t bit0 = wi * 32;
  const int64_t c_first = bit0 / wbits, c_last = (bit0 + 31) / wbits;
  uint32_t word = 0;
  for (int64_t c = c_first; c <= c_last && c < n; ++c) {
    const uint32_t code = codes8[r * n + inv[c]];
    const int64_t sh = c * wbits - bit0;
    if (sh >= 0) word |= code << sh;
    else word |= code >> (-sh);
  }
  out[e] = word;
}

__global__ void sub_half_kernel(float* __restrict__ D, const float* __restrict__ H, int64_t count) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e < count) D[e] = fmaf(-0.5f, H[e], D[e]);
}

__global__ void copy_kernel(const float* __restrict__ a, float* __restrict__ b, int64_t count) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e < count) b[e] = a[e];
}

__global__ void fill_kernel(float* __restrict__ a, int64_t count, float v) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e < count) a[e] = v;
}

__global__ void check_finite_kernel(const float* __restrict__ a, int64_t count, int* status) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e < count && !isfinite(a[e])) record_error(status, kDevNonfinite);
}

unsigned blocks_for(int64_t count, int bs) { return static_cast<unsigned>((count + bs - 1) / bs); }

}  // namespace

void launch_permute_w(const Ctx& c, const float* W, int64_t m, int64_t n, const int32_t* perm,
                      const unsigned char* dead, float* Wp) {
  static bool attr_done[64] = {false};
  if (!attr_done[c.device & 63]) {
    check_cuda(cudaFuncSetAttribute(permute_w_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 49152 * 4),
               "cudaFuncSetAttribute(permute_w)");
    attr_done[c.device & 63] = true;
  }
  permute_w_kernel<<<static_cast<unsigned>(m), 256, static_cast<size_t>(n) * 4, c.stream>>>(W, n, perm, dead, Wp);
  check_launch("permute_w_kernel");
}

void launch_static_grid(const Ctx& c, const float* W, int64_t m, int64_t n, int G, int wbits,
                        const unsigned char* dead, float* scales, float* zeros) {
  const int64_t warps = m * (n / G);
  static_grid_kernel<<<blocks_for(warps * 32, 256), 256, 0, c.stream>>>(
      W, m, n, G, static_cast<float>((1 << wbits) - 1), dead, scales, zeros);
  check_launch("static_grid_kernel");
}

void launch_sweep_block(const Ctx& c, float* Wp, int64_t m, int64_t n, const float* U, int64_t j1, int G,
                        int wbits, bool static_groups, const int32_t* perm, float* scales, float* zeros,
                        unsigned char* codes8, float* Err) {
  static bool attr_done[64] = {false};
  const int smem = SB * SB * 4;
  if (!attr_done[c.device & 63]) {
    check_cuda(cudaFuncSetAttribute(sweep_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
               "cudaFuncSetAttribute(sweep)");
    attr_done[c.device & 63] = true;
  }
  const int64_t rows_per_cta = SWEEP_WARPS;
  const int64_t want = (m + rows_per_cta - 1) / rows_per_cta;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(c.sm_count) * 3));
  // (16 warps and 64 KB of shared memory per CTA: three CTAs per SM, so 4096
  // rows run in a single wave)
  sweep_block_kernel<<<grid, SWEEP_WARPS * 32, smem, c.stream>>>(
      Wp, m, n, U, j1, G, static_cast<float>((1 << wbits) - 1), static_groups ? 1 : 0, perm, scales, zeros,
      codes8, Err);
  check_launch("sweep_block_kernel");
}

void launch_pack(const Ctx& c, const unsigned char* codes8, int64_t m, int64_t n, int wbits,
                 int32_t* perm2, uint32_t* codes) {
  // perm2 holds 2n entries: the processing order, then room for its inverse.
  int32_t* inv = perm2 + n;
  invert_perm_kernel<<<blocks_for(n, 256), 256, 0, c.stream>>>(perm2, n, inv);
  check_launch("invert_perm_kernel");
  const int64_t total = m * (n * wbits / 32);
  pack_kernel<<<blocks_for(total, 256), 256, 0, c.stream>>>(codes8, m, n, wbits, inv, codes);
  check_launch("pack_kernel");
}

void launch_invert_perm(const Ctx& c, int32_t* perm2, int64_t n) {
  invert_perm_kernel<<<blocks_for(n, 256), 256, 0, c.stream>>>(perm2, n, perm2 + n);
  check_launch("invert_perm_kernel");
}

void launch_sub_half(const Ctx& c, float* D, const float* H, int64_t n) {
  sub_half_kernel<<<blocks_for(n * n, 256), 256, 0, c.stream>>>(D, H, n * n);
  check_launch("sub_half_kernel");
}

void launch_copy_f32(const Ctx& c, const float* src, float* dst, int64_t count) {
  copy_kernel<<<blocks_for(count, 256), 256, 0, c.stream>>>(src, dst, count);
  check_launch("copy_kernel");
}

void launch_fill_f32(const Ctx& c, float* dst, int64_t count, float v) {
  fill_kernel<<<blocks_for(count, 256), 256, 0, c.stream>>>(dst, count, v);
  check_launch("fill_kernel");
}

void launch_check_finite(const Ctx& c, const float* x, int64_t count) {
  check_finite_kernel<<<blocks_for(count, 256), 256, 0, c.stream>>>(x, count, c.status);
  check_launch("check_finite_kernel");
}

}  // namespace oc

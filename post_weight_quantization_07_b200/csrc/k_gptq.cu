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
#include "ptx_sm100.cuh"

namespace oc {
namespace {

constexpr int SB = 128;          // sweep block width

__device__ __forceinline__ void grid_from_minmax(float xmin, float xmax, float maxq, float& s,
                                                 float& z) {
  if (xmax == xmin) {
    xmin -= 1.f;
    xmax += 1.f;
  }
  s = (xmax - xmin) / maxq;
  z = fminf(fmaxf(rintf(-xmin / s), 0.f), maxq);
}

// Wp[r][j] = dead[p(j)] ? 0 : W[r][p(j)] (dead may be null: no zeroing), one
// block per row (row staged in shared memory).
__global__ void permute_w_kernel(const float* __restrict__ W, int64_t n, const int32_t* __restrict__ perm,
                                 const unsigned char* __restrict__ dead, float* __restrict__ Wp) {
  extern __shared__ float row[];
  const int64_t r = blockIdx.x;
  for (int64_t c = threadIdx.x; c < n; c += blockDim.x) row[c] = W[r * n + c];
  __syncthreads();
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const int64_t p = perm[j];
    Wp[r * n + j] = (dead != nullptr && dead[p]) ? 0.f : row[p];
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

// LPR lanes per row (8, 16 or 32), CPL = 128 / LPR consecutive columns per
// lane (lane q of a row's group holds block columns CPL q .. CPL q + CPL - 1),
// 16 rows per CTA.  Step j of the block belongs to lane j / CPL (register
// j % CPL, a compile-time index inside the unrolled CPL-step chunk); its error
// reaches the other lanes of the row by a width-LPR shuffle.  Each lane then
// updates its own columns from the U row in shared memory.  The sweep is a
// chain of dependent steps per row, so it is bound by latency: more lanes per
// row give each SM more warps to interleave and shorter steps.  U rows are
// stored skewed (4 floats of padding every 256 / CPL columns) so that each
// 8-lane phase of a 16-byte shared-memory read falls in distinct banks.
// Groups of at least CPL columns start on chunk boundaries and are handled
// once per chunk (SMALLG: smaller groups, checked every step).
constexpr int SWEEP_ROWS = 16;            // rows per CTA

template <int LPR>
struct SweepShape {
  static constexpr int CPL = SB / LPR;                      // columns per lane
  static constexpr int SKEW = 256 / CPL;                    // columns between paddings
  static constexpr int UPAD = SB + SB / SKEW * 4;           // skewed U row length
  static constexpr int THREADS = SWEEP_ROWS * LPR;
  static constexpr int SMEM = (SB * UPAD + SB) * 4;
  __device__ static __forceinline__ int upos(int j, int k) { return j * UPAD + k + (k / SKEW) * 4; }
};

template <int LPR, bool SMALLG>
__device__ __forceinline__ void group_grid(float (&w)[SB / LPR], float (&sc)[SB / LPR], float (&zc)[SB / LPR],
                                           float (&rs)[SB / LPR], int j, int G, int bw, int q, bool g_small,
                                           const float* wrow, int64_t j1, float maxq, bool store, float* scales,
                                           float* zeros, int64_t srow) {
  constexpr int CPL = SB / LPR;
  float xmin = INFINITY, xmax = -INFINITY;
  if (g_small) {
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int k = CPL * q + i;
      if (k >= j && k < j + G && k < bw) {
        xmin = fminf(xmin, w[i]);
        xmax = fmaxf(xmax, w[i]);
      }
    }
  } else {
    // a group wider than the block starts at its first column: every column
    // of it is current (earlier blocks' updates are applied, this block's
    // have not started)
    for (int64_t k = j1 + q; k < j1 + G; k += LPR) {
      const float v = wrow[k];
      xmin = fminf(xmin, v);
      xmax = fmaxf(xmax, v);
    }
  }
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) {
    xmin = fminf(xmin, __shfl_xor_sync(0xffffffffu, xmin, o, LPR));
    xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, o, LPR));
  }
  float gs, gz;
  grid_from_minmax(xmin, xmax, maxq, gs, gz);
  const float grs = 1.f / gs;
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const int k = CPL * q + i;
    if (!g_small || (k >= j && k < j + G)) {
      sc[i] = gs;
      zc[i] = gz;
      rs[i] = grs;
    }
  }
  if (store) {
    const int64_t g = (j1 + j) / G;
    scales[srow + g] = gs;
    zeros[srow + g] = gz;
  }
}

template <int LPR, bool SMALLG>
__global__ void __launch_bounds__(SweepShape<LPR>::THREADS, 2)
sweep_block_kernel(float* __restrict__ Wp, int64_t m, int64_t n, const float* __restrict__ U, int64_t j1, int G,
                   float maxq, int static_groups, const int32_t* __restrict__ perm, float* __restrict__ scales,
                   float* __restrict__ zeros, unsigned char* __restrict__ codes8, float* __restrict__ Err,
                   float* __restrict__ Err_lo, int64_t err_ld) {
  using S = SweepShape<LPR>;
  constexpr int CPL = S::CPL;
  constexpr int NT = S::THREADS;
  extern __shared__ __align__(16) float Ub[];  // [SB][UPAD], skewed
  const int bw = static_cast<int>(::min((int64_t)SB, n - j1));
  {
    // 16-byte loads, all of a thread's in flight at once (U rows are 16-byte
    // aligned: n is a multiple of 64); only the upper triangle is non-zero.
    constexpr int PER = SB * SB / 4 / NT;
    float4 v[PER];
#pragma unroll
    for (int q4 = 0; q4 < PER; ++q4) {
      const int e4 = threadIdx.x + NT * q4;
      const int j = e4 / (SB / 4), k = (e4 % (SB / 4)) * 4;
      v[q4] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < bw && k < bw && k + 3 >= j) {
        v[q4] = *reinterpret_cast<const float4*>(U + (j1 + j) * n + j1 + k);
        // exact zeros left of the diagonal: the sweep's updates rely on them
        if (k < j) v[q4].x = 0.f;
        if (k + 1 < j) v[q4].y = 0.f;
        if (k + 2 < j) v[q4].z = 0.f;
      }
    }
#pragma unroll
    for (int q4 = 0; q4 < PER; ++q4) {
      const int e4 = threadIdx.x + NT * q4;
      const int j = e4 / (SB / 4), k = (e4 % (SB / 4)) * 4;
      *reinterpret_cast<float4*>(&Ub[S::upos(j, k)]) = v[q4];
    }
  }
  __syncthreads();
  // reciprocal pivots 1 / U_jj (the serial chain then multiplies instead of dividing)
  float* rU = Ub + SB * S::UPAD;
  if (threadIdx.x < SB) rU[threadIdx.x] = (threadIdx.x < bw) ? 1.f / Ub[S::upos(threadIdx.x, threadIdx.x)] : 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int q = lane & (LPR - 1);        // lane within the row's group
  const int64_t ng = n / G;
  const int64_t col0 = j1 + CPL * q;     // first column of this lane
  const bool lane_valid = CPL * q < bw;  // bw is 64 or 128
  const bool g_small = G <= SB;
  const bool block_starts_group = (j1 % G) == 0;
  for (int64_t rbase = static_cast<int64_t>(blockIdx.x) * SWEEP_ROWS; rbase < m;
       rbase += static_cast<int64_t>(gridDim.x) * SWEEP_ROWS) {
    const int64_t r = rbase + threadIdx.x / LPR;
    const bool row_valid = r < m;
    const int64_t rr = row_valid ? r : 0;  // inactive rows compute on row 0 and store nothing
    float* wrow = Wp + rr * n;
    float w[CPL], sc[CPL], zc[CPL], rs[CPL], ev[CPL], qf[CPL];
#pragma unroll
    for (int i = 0; i < CPL; i += 4) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (lane_valid) v = *reinterpret_cast<const float4*>(wrow + col0 + i);
      w[i] = v.x;
      w[i + 1] = v.y;
      w[i + 2] = v.z;
      w[i + 3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      sc[i] = 1.f;
      zc[i] = 0.f;
      ev[i] = 0.f;
      qf[i] = 0.f;
      if (static_groups && lane_valid) {
        const int g = perm[col0 + i] / G;
        sc[i] = scales[rr * ng + g];
        zc[i] = zeros[rr * ng + g];
      }
      rs[i] = 1.f / sc[i];
    }
    if (!static_groups && !block_starts_group) {
      // a group wider than the block started in an earlier block
      const int64_t g = j1 / G;
      const float gs = scales[rr * ng + g], gz = zeros[rr * ng + g];
      const float grs = 1.f / gs;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        sc[i] = gs;
        zc[i] = gz;
        rs[i] = grs;
      }
    }
    const int nchunks = bw / CPL;
    for (int c = 0; c < nchunks; ++c) {
      if (!SMALLG && !static_groups && (g_small ? (((c * CPL) & (G - 1)) == 0) : (c == 0 && block_starts_group)))
        group_grid<LPR, SMALLG>(w, sc, zc, rs, c * CPL, G, bw, q, g_small, wrow, j1, maxq, q == 0 && row_valid,
                                scales, zeros, rr * ng);
      const bool own = q == c;    // this lane owns the chunk
#pragma unroll
      for (int jj = 0; jj < CPL; ++jj) {
        const int j = c * CPL + jj;
        if (SMALLG && !static_groups && ((j & (G - 1)) == 0))
          group_grid<LPR, SMALLG>(w, sc, zc, rs, j, G, bw, q, true, wrow, j1, maxq, q == 0 && row_valid, scales,
                                  zeros, rr * ng);
        // Every lane rounds its own column jj (no divergence); only the chunk
        // owner's result is kept and broadcast.  q = clip(rint(w / scale) + zero)
        // with w / scale taken as w * (1 / scale), within an ulp of the quotient.
        const float wj = w[jj], sj = sc[jj], zj = zc[jj];
        const float qq = fminf(fmaxf(rintf(wj * rs[jj]) + zj, 0.f), maxq);
        const float dq = sj * (qq - zj);
        float e = (wj - dq) * rU[j];
        if (own) {
          qf[jj] = qq;
          ev[jj] = e;
        }
        e = __shfl_sync(0xffffffffu, e, c, LPR);
        // w_k -= e U_jk for all of this lane's columns: U_jk is exactly zero for
        // k < j, and column j itself is not read again, so no column needs a test.
        const float* urow = &Ub[S::upos(j, CPL * q)];  // CPL contiguous floats (one skew segment)
#pragma unroll
        for (int i = 0; i < CPL; i += 4) {
          const float4 u = *reinterpret_cast<const float4*>(urow + i);
          w[i] = fmaf(-e, u.x, w[i]);
          w[i + 1] = fmaf(-e, u.y, w[i + 1]);
          w[i + 2] = fmaf(-e, u.z, w[i + 2]);
          w[i + 3] = fmaf(-e, u.w, w[i + 3]);
        }
      }
    }
    if (row_valid && lane_valid) {
      uint32_t pk[CPL / 4];
#pragma unroll
      for (int i = 0; i < CPL / 4; ++i)
        pk[i] = static_cast<uint32_t>(qf[4 * i]) | (static_cast<uint32_t>(qf[4 * i + 1]) << 8) |
                (static_cast<uint32_t>(qf[4 * i + 2]) << 16) | (static_cast<uint32_t>(qf[4 * i + 3]) << 24);
      unsigned char* cdst = codes8 + r * n + col0;
      if constexpr (CPL == 16) {
        *reinterpret_cast<uint4*>(cdst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      } else if constexpr (CPL == 8) {
        *reinterpret_cast<uint2*>(cdst) = make_uint2(pk[0], pk[1]);
      } else {
        *reinterpret_cast<uint32_t*>(cdst) = pk[0];
      }
      if (Err_lo) {
        // the trailing product's operand, split for 3xTF32: hi = tf32(e), lo = tf32(e - hi)
#pragma unroll
        for (int i = 0; i < CPL; i += 4) {
          float h[4], l[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            h[k] = tf32_rna(ev[i + k]);
            l[k] = tf32_rna(ev[i + k] - h[k]);
          }
          *reinterpret_cast<float4*>(Err + r * err_ld + CPL * q + i) = make_float4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<float4*>(Err_lo + r * err_ld + CPL * q + i) = make_float4(l[0], l[1], l[2], l[3]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < CPL; i += 4)
          *reinterpret_cast<float4*>(Err + r * err_ld + CPL * q + i) = make_float4(ev[i], ev[i + 1], ev[i + 2], ev[i + 3]);
      }
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

namespace {

// Lanes per row.  Measured on the q_proj shapes (4096 x 4096, 32 blocks):
// 8, 16 and 32 lanes per row took 1.12, 0.91 and 0.81 ms for the whole sweep,
// with bit-identical results (every column sees the same operations).
constexpr int kSweepLPR = 32;

template <int LPR, bool SMALLG>
void launch_sweep_shape(const Ctx& c, float* Wp, int64_t m, int64_t n, const float* U, int64_t j1, int G,
                        float maxq, bool static_groups, const int32_t* perm, float* scales, float* zeros,
                        unsigned char* codes8, float* Err, float* Err_lo, int64_t err_ld) {
  using S = SweepShape<LPR>;
  static bool attr_done[64] = {false};
  if (!attr_done[c.device & 63]) {
    check_cuda(cudaFuncSetAttribute(sweep_block_kernel<LPR, SMALLG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    S::SMEM),
               "cudaFuncSetAttribute(sweep)");
    attr_done[c.device & 63] = true;
  }
  const int64_t want = (m + SWEEP_ROWS - 1) / SWEEP_ROWS;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(c.sm_count) * 2));
  sweep_block_kernel<LPR, SMALLG><<<grid, S::THREADS, S::SMEM, c.stream>>>(
      Wp, m, n, U, j1, G, maxq, static_groups ? 1 : 0, perm, scales, zeros, codes8, Err, Err_lo, err_ld);
  check_launch("sweep_block_kernel");
}

}  // namespace

void launch_sweep_block(const Ctx& c, float* Wp, int64_t m, int64_t n, const float* U, int64_t j1, int G,
                        int wbits, bool static_groups, const int32_t* perm, float* scales, float* zeros,
                        unsigned char* codes8, float* Err, float* Err_lo, int64_t err_ld) {
  constexpr int LPR = kSweepLPR;
  const float maxq = static_cast<float>((1 << wbits) - 1);
  if (err_ld < SB || err_ld % 4) fail(OC_ERR_INVALID_ARG, "sweep: error leading dimension");
  if (!static_groups && G < SB / LPR)
    launch_sweep_shape<LPR, true>(c, Wp, m, n, U, j1, G, maxq, static_groups, perm, scales, zeros, codes8, Err,
                                  Err_lo, err_ld);
  else
    launch_sweep_shape<LPR, false>(c, Wp, m, n, U, j1, G, maxq, static_groups, perm, scales, zeros, codes8, Err,
                                   Err_lo, err_ld);
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

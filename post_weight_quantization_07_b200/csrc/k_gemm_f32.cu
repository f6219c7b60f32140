// fp32 GEMM on the CUDA cores: C = beta*C + alpha*op(A)*op(B), row-major.
//
// Used where the quantisation needs full fp32 accuracy (the inverse-Hessian
// factor, the QEP apply and the GPTQ trailing update).  128x128 block tile,
// 8-deep k slices staged in shared memory, 8x8 outputs per thread.  When an
// operand is triangular (flags) the k range of each tile is clipped to the
// part that can be non-zero; tiles wholly above the diagonal are skipped when
// only the lower triangle of C is wanted.
#include <algorithm>

#include "oc_internal.cuh"

namespace oc {
namespace {

constexpr int TM = 128, TN = 128, TK = 8, NT = 256;

template <bool TA, bool TB>
__global__ void __launch_bounds__(NT) sgemm_kernel(int64_t M, int64_t N, int64_t K, float alpha,
                                                   const float* __restrict__ A, int64_t lda,
                                                   const float* __restrict__ B, int64_t ldb,
                                                   float beta, float* __restrict__ C, int64_t ldc,
                                                   unsigned flags) {
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * TM;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * TN;
  if ((flags & kCLowerOnly) && j0 > i0 + TM - 1) return;
  int64_t kb = 0, ke = K;
  if (flags & kAUpper) kb = max(kb, i0);
  if (flags & kALower) ke = min(ke, i0 + TM);
  if (flags & kBLower) kb = max(kb, j0);
  if (flags & kBUpper) ke = min(ke, j0 + TN);

  __shared__ __align__(16) float As[2][TK][TM];
  __shared__ __align__(16) float Bs[2][TK][TN];

  const int t = threadIdx.x;
  const int tx = t & 15, ty = t >> 4;

  // global -> register staging of one k slice
  float ra[4], rb[4];
  auto load_a = [&](int64_t k0) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int64_t i, k;
      if (TA) {  // A stored K x M: coalesced along i
        k = k0 + (t >> 5);
        i = i0 + (t & 31) * 4 + e;
        ra[e] = (i < M && k < ke) ? A[k * lda + i] : 0.f;
      } else {   // A stored M x K
        i = i0 + (t >> 1);
        k = k0 + (t & 1) * 4 + e;
        ra[e] = (i < M && k < ke) ? A[i * lda + k] : 0.f;
      }
    }
  };
  auto load_b = [&](int64_t k0) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int64_t j, k;
      if (TB) {  // B stored N x K
        j = j0 + (t >> 1);
        k = k0 + (t & 1) * 4 + e;
        rb[e] = (j < N && k < ke) ? B[j * ldb + k] : 0.f;
      } else {   // B stored K x N: coalesced along j
        k = k0 + (t >> 5);
        j = j0 + (t & 31) * 4 + e;
        rb[e] = (j < N && k < ke) ? B[k * ldb + j] : 0.f;
      }
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (TA) As[buf][t >> 5][(t & 31) * 4 + e] = ra[e];
      else As[buf][(t & 1) * 4 + e][t >> 1] = ra[e];
      if (TB) Bs[buf][(t & 1) * 4 + e][t >> 1] = rb[e];
      else Bs[buf][t >> 5][(t & 31) * 4 + e] = rb[e];
    }
  };

  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

  if (kb < ke) {
    load_a(kb);
    load_b(kb);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int64_t k0 = kb; k0 < ke; k0 += TK) {
      const bool more = k0 + TK < ke;
      if (more) {
        load_a(k0 + TK);
        load_b(k0 + TK);
      }
#pragma unroll
      for (int kk = 0; kk < TK; ++kk) {
        float a[8], b[8];
        const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
        a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
        a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
        b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
        b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
          for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
      }
      if (more) {
        store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }

#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const int64_t i = i0 + (x < 4 ? ty * 4 + x : 64 + ty * 4 + (x - 4));
    if (i >= M) continue;
#pragma unroll
    for (int y = 0; y < 8; ++y) {
      const int64_t j = j0 + (y < 4 ? tx * 4 + y : 64 + tx * 4 + (y - 4));
      if (j >= N) continue;
      float v = alpha * acc[x][y];
      if (beta != 0.f) v = fmaf(beta, C[i * ldc + j], v);
      C[i * ldc + j] = v;
    }
  }
}

// Small problems (a few tiles): 64x64 tiles for more CTAs and 32-deep k
// slices so that a product of depth 128-256 takes only a handful of global
// round trips; 256 threads, 4x4 outputs each.
constexpr int SM_T = 64, SM_K = 32;

template <bool TA, bool TB>
__global__ void __launch_bounds__(256) sgemm_small_kernel(int64_t M, int64_t N, int64_t K, float alpha,
                                                          const float* __restrict__ A, int64_t lda,
                                                          const float* __restrict__ B, int64_t ldb,
                                                          float beta, float* __restrict__ C, int64_t ldc,
                                                          unsigned flags) {
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * SM_T;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * SM_T;
  if ((flags & kCLowerOnly) && j0 > i0 + SM_T - 1) return;
  int64_t kb = 0, ke = K;
  if (flags & kAUpper) kb = max(kb, i0);
  if (flags & kALower) ke = min(ke, i0 + SM_T);
  if (flags & kBLower) kb = max(kb, j0);
  if (flags & kBUpper) ke = min(ke, j0 + SM_T);

  __shared__ __align__(16) float As[2][SM_K][SM_T + 4];
  __shared__ __align__(16) float Bs[2][SM_K][SM_T + 4];
  const int t = threadIdx.x;
  const int tx = t & 15, ty = t >> 4;
  float ra[8], rb[8];
  auto load = [&](int64_t k0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = t + 256 * e;  // 0..2047 over a 64 x 32 slice
      int64_t i, k, j;
      if (TA) {  // A stored K x M: rows k, contiguous i
        k = k0 + idx / SM_T;
        i = i0 + idx % SM_T;
        ra[e] = (i < M && k < ke) ? A[k * lda + i] : 0.f;
      } else {
        i = i0 + idx / SM_K;
        k = k0 + idx % SM_K;
        ra[e] = (i < M && k < ke) ? A[i * lda + k] : 0.f;
      }
      if (TB) {  // B stored N x K
        j = j0 + idx / SM_K;
        k = k0 + idx % SM_K;
        rb[e] = (j < N && k < ke) ? B[j * ldb + k] : 0.f;
      } else {
        k = k0 + idx / SM_T;
        j = j0 + idx % SM_T;
        rb[e] = (j < N && k < ke) ? B[k * ldb + j] : 0.f;
      }
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = t + 256 * e;
      if (TA) As[buf][idx / SM_T][idx % SM_T] = ra[e];
      else As[buf][idx % SM_K][idx / SM_K] = ra[e];
      if (TB) Bs[buf][idx % SM_K][idx / SM_K] = rb[e];
      else Bs[buf][idx / SM_T][idx % SM_T] = rb[e];
    }
  };
  float acc[4][4] = {};
  if (kb < ke) {
    load(kb);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int64_t k0 = kb; k0 < ke; k0 += SM_K) {
      const bool more = k0 + SM_K < ke;
      if (more) load(k0 + SM_K);
#pragma unroll 8
      for (int kk = 0; kk < SM_K; ++kk) {
        const float4 a4 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
        const float4 b4 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
      }
      if (more) {
        store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int64_t i = i0 + ty * 4 + x;
    if (i >= M) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int64_t j = j0 + tx * 4 + y;
      if (j >= N) continue;
      float v = alpha * acc[x][y];
      if (beta != 0.f) v = fmaf(beta, C[i * ldc + j], v);
      C[i * ldc + j] = v;
    }
  }
}

}  // namespace

void gemm_f32(const Ctx& c, bool tA, bool tB, int64_t M, int64_t N, int64_t K, float alpha,
              const float* A, int64_t lda, const float* B, int64_t ldb, float beta, float* C,
              int64_t ldc, unsigned flags) {
  if (M <= 0 || N <= 0) return;
  const int64_t big_tiles = ((M + TM - 1) / TM) * ((N + TN - 1) / TN);
  if (big_tiles < 2 * static_cast<int64_t>(c.sm_count)) {
    dim3 grid(static_cast<unsigned>((N + SM_T - 1) / SM_T), static_cast<unsigned>((M + SM_T - 1) / SM_T));
    if (grid.y > 65535u) fail(OC_ERR_INVALID_ARG, "gemm_f32: M too large");
    if (!tA && !tB)
      sgemm_small_kernel<false, false><<<grid, 256, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    else if (!tA && tB)
      sgemm_small_kernel<false, true><<<grid, 256, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    else if (tA && !tB)
      sgemm_small_kernel<true, false><<<grid, 256, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    else
      sgemm_small_kernel<true, true><<<grid, 256, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
    check_launch("sgemm_small_kernel");
    return;
  }
  dim3 grid(static_cast<unsigned>((N + TN - 1) / TN), static_cast<unsigned>((M + TM - 1) / TM));
  if (grid.y > 65535u) fail(OC_ERR_INVALID_ARG, "gemm_f32: M too large");
  if (!tA && !tB)
    sgemm_kernel<false, false><<<grid, NT, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
  else if (!tA && tB)
    sgemm_kernel<false, true><<<grid, NT, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
  else if (tA && !tB)
    sgemm_kernel<true, false><<<grid, NT, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
  else
    sgemm_kernel<true, true><<<grid, NT, 0, c.stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, flags);
  check_launch("sgemm_kernel");
}

}  // namespace oc

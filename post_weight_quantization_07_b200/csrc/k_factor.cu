// Dampening, act_order ordering and the inverse-Hessian factor U.
//
// GPTQ needs U, the upper Cholesky factor of H_d^-1 (U^T U = H_d^-1).  With J
// the index reversal, J H_d J = L L^T gives H_d = R R^T for the upper
// triangular R = J L J, hence H_d^-1 = (R^-1)^T R^-1 and, by uniqueness of the
// factor with positive diagonal, U = R^-1 = J L^-1 J.  So one Cholesky
// factorisation and one triangular inverse of the reversed matrix give U
// directly, with no explicit inverse of H_d.
//
// The factorisation is a recursive blocked Cholesky that also builds L^-1:
//   [A11  .  ]   L11 = chol(A11), X11 = L11^-1            (recurse)
//   [A21 A22 ]   L21 = A21 X11^T                           (GEMM)
//                A22' = A22 - L21 L21^T (lower tiles)       (GEMM)
//                Y = L21 X11                               (GEMM, before the next recursion)
//                L22 = chol(A22'), X22 = L22^-1            (recurse)
//                X21 = -X22 Y                              (GEMM)
// with 64x64 leaves factored and inverted inside one CTA.
#include <algorithm>
#include <cmath>

#include "oc_internal.cuh"

namespace oc {
namespace {

constexpr int LEAF = 64;

// ---------------------------------------------------------------- diag stats
// One block: dead mask, non-finite check and the dampening constant
// lam = damp * mean(diag(hscale * H)) (with dead entries counted as 1).
__global__ void diag_stats_kernel(const float* __restrict__ H, int64_t n, float damp, float hscale,
                                  int fix_dead, DiagStats* stats, unsigned char* dead, int* status) {
  __shared__ double ssum[32];
  __shared__ int sbad[32], sdead[32];
  double sum = 0.0;
  int bad = 0, nd = 0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    float d = H[j * n + j] * hscale;
    const bool is_dead = fix_dead && d == 0.f;
    if (dead) dead[j] = is_dead ? 1 : 0;
    if (is_dead) {
      d = 1.f;
      ++nd;
    }
    if (!isfinite(d)) ++bad;
    sum += static_cast<double>(d);
  }
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    bad += __shfl_xor_sync(0xffffffffu, bad, o);
    nd += __shfl_xor_sync(0xffffffffu, nd, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    ssum[w] = sum;
    sbad[w] = bad;
    sdead[w] = nd;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    int b = 0, dd = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) {
      s += ssum[i];
      b += sbad[i];
      dd += sdead[i];
    }
    const double mean = s / static_cast<double>(n);
    stats->mean_diag = static_cast<float>(mean);
    stats->lam = static_cast<float>(static_cast<double>(damp) * mean);
    stats->n_dead = dd;
    stats->nonfinite = b;
    if (b) record_error(status, kDevNonfinite);
  }
}

// ---------------------------------------------------------------- act_order
// perm[rank(j)] = j with rank(j) = #{k : d_k > d_j} + #{k < j : d_k == d_j},
// d the diagonal with dead entries set to 1: a stable descending sort.  NaN is
// ordered as -inf so that the ranks always form a permutation (a NaN diagonal
// is reported separately as a non-finite input).
__device__ __forceinline__ float sort_key(float d) {
  if (d == 0.f) return 1.f;
  return isnan(d) ? -INFINITY : d;
}

__global__ void act_order_rank_kernel(const float* __restrict__ H, int64_t n, int32_t* perm) {
  extern __shared__ float sd[];
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const float dj = (j < n) ? sort_key(H[j * n + j]) : 0.f;
  int64_t rank = 0;
  for (int64_t k0 = 0; k0 < n; k0 += blockDim.x) {
    const int64_t k = k0 + threadIdx.x;
    sd[threadIdx.x] = (k < n) ? sort_key(H[k * n + k]) : 0.f;
    __syncthreads();
    const int64_t kn = ::min((int64_t)static_cast<int64_t>(blockDim.x), n - k0);
    if (j < n) {
      for (int64_t q = 0; q < kn; ++q) {
        const float v = sd[q];
        const int64_t kk = k0 + q;
        rank += (v > dj) || (v == dj && kk < j);
      }
    }
    __syncthreads();
  }
  if (j < n) perm[rank] = static_cast<int32_t>(j);
}

__global__ void identity_perm_kernel(int64_t n, int32_t* perm) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j < n) perm[j] = static_cast<int32_t>(j);
}

// ---------------------------------------------------------------- build M
// M[a][b] = hscale * Hfix[p(n-1-a)][p(n-1-b)] + lam [a == b]; one block per
// output row, the source row staged in shared memory for the column gather.
__global__ void build_reversed_kernel(const float* __restrict__ H, int64_t n,
                                      const int32_t* __restrict__ perm, const DiagStats* stats,
                                      float hscale, int fix_dead, float* __restrict__ M) {
  extern __shared__ float row[];
  const int64_t a = blockIdx.x;
  const int64_t src = perm ? perm[n - 1 - a] : (n - 1 - a);
  for (int64_t c = threadIdx.x; c < n; c += blockDim.x) row[c] = H[src * n + c];
  __syncthreads();
  const float lam = stats->lam;
  for (int64_t b = threadIdx.x; b < n; b += blockDim.x) {
    const int64_t col = perm ? perm[n - 1 - b] : (n - 1 - b);
    float v = row[col] * hscale;
    if (a == b) {
      if (fix_dead && v == 0.f) v = 1.f;
      v += lam;
    }
    M[a * n + b] = v;
  }
}

// ---------------------------------------------------------------- leaf
// Cholesky of the s x s diagonal block at M (lower part read) and the inverse
// of its factor, written to X (lower, explicit zeros above the diagonal).
// Right-looking elimination without normalising the pivot column:
//   A[i][j] -= A[i][k] A[j][k] / A[k][k]   for k < j <= i,
// so that afterwards L[i][k] = A[i][k] / sqrt(A[k][k]); one barrier per column.
__global__ void __launch_bounds__(256) leaf_chol_inv_kernel(const float* __restrict__ M, float* __restrict__ X,
                                                            int64_t ld, int s, int* status) {
  __shared__ float A[LEAF][LEAF + 1];
  __shared__ float B[LEAF][LEAF + 1];
  const int t = threadIdx.x;
  for (int e = t; e < LEAF * LEAF; e += blockDim.x) {
    const int i = e / LEAF, j = e % LEAF;
    float v = 0.f;
    if (i < s && j <= i) v = M[static_cast<int64_t>(i) * ld + j];
    else if (i == j) v = 1.f;  // padding rows beyond s: identity
    A[i][j] = v;
    B[i][j] = (i == j) ? 1.f : 0.f;
  }
  __syncthreads();
  for (int k = 0; k < LEAF - 1; ++k) {
    const float inv_piv = 1.f / A[k][k];
    for (int e = t; e < (LEAF - 1 - k) * (LEAF - 1 - k); e += blockDim.x) {
      const int i = k + 1 + e / (LEAF - 1 - k);
      const int j = k + 1 + e % (LEAF - 1 - k);
      if (j <= i) A[i][j] -= A[i][k] * A[j][k] * inv_piv;
    }
    __syncthreads();
  }
  // pivots, then normalise: L[i][k] = A[i][k] / sqrt(A[k][k])
  __shared__ float rs[LEAF];
  if (t < LEAF) {
    const float piv = A[t][t];
    if (!(piv > 0.f) || !isfinite(piv)) {
      record_error(status, kDevNotSpd);
      rs[t] = 0.f;
    } else {
      rs[t] = rsqrtf(piv);
    }
  }
  __syncthreads();
  for (int e = t; e < LEAF * LEAF; e += blockDim.x) {
    const int i = e / LEAF, k = e % LEAF;
    A[i][k] = (k <= i) ? A[i][k] * rs[k] : 0.f;
  }
  __syncthreads();
  // Forward substitution L Y = I for all columns: at step k, rows i > k take
  // B[i][j] -= L[i][k] * B[k][j] / L[k][k] for j <= k; then X = B / diag(L).
  for (int k = 0; k < LEAF - 1; ++k) {
    const float inv_lkk = 1.f / A[k][k];
    for (int e = t; e < (LEAF - 1 - k) * (k + 1); e += blockDim.x) {
      const int i = k + 1 + e / (k + 1);
      const int j = e % (k + 1);
      B[i][j] -= A[i][k] * B[k][j] * inv_lkk;
    }
    __syncthreads();
  }
  for (int e = t; e < s * s; e += blockDim.x) {
    const int i = e / s, j = e % s;
    X[static_cast<int64_t>(i) * ld + j] = (j <= i) ? B[i][j] / A[i][i] : 0.f;
  }
}

// U[i][j] = X[n-1-i][n-1-j]
__global__ void reverse_kernel(const float* __restrict__ X, float* __restrict__ U, int64_t n) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n * n) return;
  const int64_t i = e / n, j = e % n;
  U[e] = X[(n - 1 - i) * n + (n - 1 - j)];
}

void chol_inv_rec(const Ctx& c, float* M, float* X, int64_t ld, int64_t off, int64_t s,
                  float* scratch) {
  float* Md = M + off * ld + off;
  float* Xd = X + off * ld + off;
  if (s <= LEAF) {
    leaf_chol_inv_kernel<<<1, 256, 0, c.stream>>>(Md, Xd, ld, static_cast<int>(s), c.status);
    check_launch("leaf_chol_inv_kernel");
    return;
  }
  const int64_t nblk = (s + LEAF - 1) / LEAF;
  const int64_t h = std::max<int64_t>(1, nblk / 2) * LEAF;
  const int64_t r = s - h;
  chol_inv_rec(c, M, X, ld, off, h, scratch);
  float* Y = scratch;
  float* T = scratch + r * h;
  const float* M21 = M + (off + h) * ld + off;
  float* M22 = M + (off + h) * ld + (off + h);
  const float* X11 = Xd;
  // L21 = A21 X11^T
  gemm_f32(c, false, true, r, h, h, 1.f, M21, ld, X11, ld, 0.f, T, h, kBUpper);
  // A22 -= L21 L21^T (lower tiles only)
  gemm_f32(c, false, true, r, r, h, -1.f, T, h, T, h, 1.f, M22, ld, kCLowerOnly);
  // Y = L21 X11
  gemm_f32(c, false, false, r, h, h, 1.f, T, h, X11, ld, 0.f, Y, h, kBLower);
  chol_inv_rec(c, M, X, ld, off + h, r, scratch + r * h);
  // X21 = -X22 Y
  const float* X22 = X + (off + h) * ld + (off + h);
  float* X21 = X + (off + h) * ld + off;
  gemm_f32(c, false, false, r, h, r, -1.f, X22, ld, Y, h, 0.f, X21, ld, kALower);
}

}  // namespace

void launch_diag_stats(const Ctx& c, const float* H, int64_t n, float damp, float hscale,
                       bool fix_dead, DiagStats* stats, unsigned char* dead) {
  diag_stats_kernel<<<1, 1024, 0, c.stream>>>(H, n, damp, hscale, fix_dead ? 1 : 0, stats, dead,
                                              c.status);
  check_launch("diag_stats_kernel");
}

void launch_act_order_perm(const Ctx& c, const float* H, int64_t n, int32_t* perm) {
  const int bs = 256;
  act_order_rank_kernel<<<static_cast<unsigned>((n + bs - 1) / bs), bs, bs * sizeof(float), c.stream>>>(H, n, perm);
  check_launch("act_order_rank_kernel");
}

void launch_identity_perm(const Ctx& c, int64_t n, int32_t* perm) {
  identity_perm_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, c.stream>>>(n, perm);
  check_launch("identity_perm_kernel");
}

void launch_build_reversed(const Ctx& c, const float* H, int64_t n, const int32_t* perm,
                           const DiagStats* stats, float hscale, bool fix_dead, float* M) {
  const size_t smem = static_cast<size_t>(n) * sizeof(float);
  static bool attr_done[64] = {false};
  if (!attr_done[c.device & 63]) {
    check_cuda(cudaFuncSetAttribute(build_reversed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    49152 * 4),
               "cudaFuncSetAttribute(build_reversed)");
    attr_done[c.device & 63] = true;
  }
  build_reversed_kernel<<<static_cast<unsigned>(n), 256, smem, c.stream>>>(H, n, perm, stats, hscale,
                                                                          fix_dead ? 1 : 0, M);
  check_launch("build_reversed_kernel");
}

void factor_inverse_upper(const Ctx& c, float* M, float* X, float* scratch, float* U, int64_t n) {
  check_cuda(cudaMemsetAsync(X, 0, static_cast<size_t>(n) * n * sizeof(float), c.stream), "memset X");
  chol_inv_rec(c, M, X, n, 0, n, scratch);
  const int64_t total = n * n;
  reverse_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, c.stream>>>(X, U, n);
  check_launch("reverse_kernel");
}

}  // namespace oc

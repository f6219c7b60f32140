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
// with 128x128 leaves that go straight to X = L^-1 inside one CTA.
#include <algorithm>
#include <cmath>
#include <vector>

#include "oc_internal.cuh"

namespace oc {
namespace {

constexpr int LEAF = 128;

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
// Cholesky of an s x s (s <= 128) diagonal block at M (lower part read) and
// the inverse of its factor, written to X (lower, explicit zeros above), in
// one CTA with the block in shared memory.  Rows and columns beyond s are
// padded with the identity.
//
// One array S holds both: before step K its columns < K hold rows of
// X = L^-1 and its columns >= K the Cholesky trailing matrix.  Step K takes
// the 4 x 4 pivot block P = S[K:K+4, K:K+4], factors it, P = L_p L_p^T, and
// inverts the factor, Z = L_p^-1 (every thread, in registers), then forms one
// 4-vector per index j:
//   v_j = Z S[K:K+4, j]   (j < K: the final rows K..K+3 of X at column j),
//   v_j = Z[:, j - K]     (K <= j < K+4: the pivot block of X),
//   v_j = Z S[j, K:K+4]   (j >= K+4: row j of L's column block),
// stores the first two kinds as rows K..K+3 of X (final from here on), clears
// the column block below the pivot, and applies
//   S_ij -= v_i . v_j   for every i >= K+4 and j <= i,
// which is at once the trailing update A_ij -= L_i,K:K+4 L_j,K:K+4 (j >= K+4),
// the new columns X_i,K:K+4 = -L_i,K:K+4 Z (K <= j < K+4) and the row
// operation that applies the inverse of step K's elementary factor to the
// rows of X (j < K).  So the leaf is 32 rank-4 steps, each two barriers apart,
// with all threads sharing the update of the rows below the pivot: a warp per
// row, and each lane keeps the same four columns (and their 4-vectors, loaded
// once per step) for every row, so a row costs one broadcast load and one
// load and store per 32 columns of shared memory.
constexpr int LDS = LEAF + 1;      // padded row (bank spread for the column reads)
constexpr int LEAF_THREADS = 512;
constexpr int PB = 4;              // pivot block
constexpr size_t LEAF_SMEM = static_cast<size_t>(LEAF) * LDS * sizeof(float) + LEAF * sizeof(float4);

__global__ void __launch_bounds__(LEAF_THREADS) leaf_chol_inv_kernel(const float* __restrict__ M,
                                                                     float* __restrict__ X, int64_t ld, int s,
                                                                     int* status) {
  extern __shared__ __align__(16) float leaf_smem[];
  float4* V = reinterpret_cast<float4*>(leaf_smem);              // [LEAF]
  float* S = leaf_smem + 4 * LEAF;                               // [LEAF][LDS]
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  // Load: 16-byte loads (rows of M are 16-byte aligned: ld is a multiple of
  // 64 and the block starts at a multiple of 128), lower part only.
  for (int e4 = t; e4 < LEAF * LEAF / 4; e4 += LEAF_THREADS) {
    const int i = e4 / (LEAF / 4), j = (e4 % (LEAF / 4)) * 4;
    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < s && j <= i && j < s) q = *reinterpret_cast<const float4*>(M + static_cast<int64_t>(i) * ld + j);
    const float qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float x = (j + c <= i && j + c < s) ? qq[c] : 0.f;
      if (i >= s && i == j + c) x = 1.f;  // identity padding beyond s
      S[i * LDS + j + c] = x;
    }
  }
  __syncthreads();
  bool bad = false;
  for (int K = 0; K < LEAF; K += PB) {
    if (t < LEAF) {
      // P = L_p L_p^T and Z = L_p^-1 (lower 4 x 4), redundantly per thread
      const float* P = S + K * LDS + K;
      const float p00 = P[0];
      const float p10 = P[LDS], p11 = P[LDS + 1];
      const float p20 = P[2 * LDS], p21 = P[2 * LDS + 1], p22 = P[2 * LDS + 2];
      const float p30 = P[3 * LDS], p31 = P[3 * LDS + 1], p32 = P[3 * LDS + 2], p33 = P[3 * LDS + 3];
      const float r0 = rsqrtf(p00);
      const float l10 = p10 * r0, l20 = p20 * r0, l30 = p30 * r0;
      const float d1 = fmaf(-l10, l10, p11);
      const float r1 = rsqrtf(d1);
      const float l21 = fmaf(-l20, l10, p21) * r1, l31 = fmaf(-l30, l10, p31) * r1;
      const float d2 = fmaf(-l21, l21, fmaf(-l20, l20, p22));
      const float r2 = rsqrtf(d2);
      const float l32 = fmaf(-l31, l21, fmaf(-l30, l20, p32)) * r2;
      const float d3 = fmaf(-l32, l32, fmaf(-l31, l31, fmaf(-l30, l30, p33)));
      const float r3 = rsqrtf(d3);
      if (!(p00 > 0.f) || !(d1 > 0.f) || !(d2 > 0.f) || !(d3 > 0.f) || !isfinite(p00 + d1 + d2 + d3)) bad = true;
      // Z = L_p^-1 by forward substitution (z_ii = r_i)
      const float z00 = r0;
      const float z10 = -l10 * r0 * r1, z11 = r1;
      const float z20 = -fmaf(l21, z10, l20 * z00) * r2, z21 = -l21 * z11 * r2, z22 = r2;
      const float z30 = -fmaf(l32, z20, fmaf(l31, z10, l30 * z00)) * r3;
      const float z31 = -fmaf(l32, z21, l31 * z11) * r3, z32 = -l32 * z22 * r3, z33 = r3;
      const int j = t;
      float4 w;
      if (j < K || j >= K + PB) {
        float a0, a1, a2, a3;
        if (j < K) {
          a0 = S[K * LDS + j]; a1 = S[(K + 1) * LDS + j]; a2 = S[(K + 2) * LDS + j]; a3 = S[(K + 3) * LDS + j];
        } else {
          a0 = S[j * LDS + K]; a1 = S[j * LDS + K + 1]; a2 = S[j * LDS + K + 2]; a3 = S[j * LDS + K + 3];
        }
        w.x = z00 * a0;
        w.y = fmaf(z11, a1, z10 * a0);
        w.z = fmaf(z22, a2, fmaf(z21, a1, z20 * a0));
        w.w = fmaf(z33, a3, fmaf(z32, a2, fmaf(z31, a1, z30 * a0)));
        if (j < K) {
          S[K * LDS + j] = w.x; S[(K + 1) * LDS + j] = w.y; S[(K + 2) * LDS + j] = w.z; S[(K + 3) * LDS + j] = w.w;
        } else {
          S[j * LDS + K] = 0.f; S[j * LDS + K + 1] = 0.f; S[j * LDS + K + 2] = 0.f; S[j * LDS + K + 3] = 0.f;
        }
      } else {
        // column c = j - K of Z; rows K + c .. K + 3 of S take its lower part
        // after the barrier below (every thread is still reading the pivot
        // block here)
        const int c = j - K;
        w = (c == 0) ? make_float4(z00, z10, z20, z30)
          : (c == 1) ? make_float4(0.f, z11, z21, z31)
          : (c == 2) ? make_float4(0.f, 0.f, z22, z32) : make_float4(0.f, 0.f, 0.f, z33);
      }
      V[j] = w;
    }
    __syncthreads();
    if (t >= K && t < K + PB) {
      // the pivot rows are not read again in this step
      const float4 w = V[t];
      const float wc[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int r = 0; r < PB; ++r)
        if (r >= t - K) S[(K + r) * LDS + t] = wc[r];
    }
    {
      // lane keeps columns j = lane + 32 q and their 4-vectors for the step
      float4 vj[LEAF / 32];
#pragma unroll
      for (int q = 0; q < LEAF / 32; ++q) vj[q] = V[lane + 32 * q];
      for (int i = K + PB + warp; i < LEAF; i += LEAF_THREADS / 32) {
        const float4 vi = V[i];
        float* row = S + i * LDS;
        float x[LEAF / 32];
#pragma unroll
        for (int q = 0; q < LEAF / 32; ++q)
          if (lane + 32 * q <= i) x[q] = row[lane + 32 * q];
#pragma unroll
        for (int q = 0; q < LEAF / 32; ++q)
          if (lane + 32 * q <= i)
            row[lane + 32 * q] =
                fmaf(-vi.w, vj[q].w, fmaf(-vi.z, vj[q].z, fmaf(-vi.y, vj[q].y, fmaf(-vi.x, vj[q].x, x[q]))));
      }
    }
    __syncthreads();
  }
  if (t == 0 && bad) record_error(status, kDevNotSpd);
  for (int e4 = t; e4 < LEAF * LEAF / 4; e4 += LEAF_THREADS) {
    const int i = e4 / (LEAF / 4), j = (e4 % (LEAF / 4)) * 4;
    if (i < s && j < s) {
      float4 o;
      o.x = (j + 0 <= i) ? S[i * LDS + j + 0] : 0.f;
      o.y = (j + 1 <= i) ? S[i * LDS + j + 1] : 0.f;
      o.z = (j + 2 <= i) ? S[i * LDS + j + 2] : 0.f;
      o.w = (j + 3 <= i) ? S[i * LDS + j + 3] : 0.f;
      *reinterpret_cast<float4*>(X + static_cast<int64_t>(i) * ld + j) = o;
    }
  }
}

// U[i][j] = X[n-1-i][n-1-j]
__global__ void reverse_kernel(const float* __restrict__ X, float* __restrict__ U, int64_t n) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n * n) return;
  const int64_t i = e / n, j = e % n;
  U[e] = X[(n - 1 - i) * n + (n - 1 - j)];
}

// Nodes whose halves are at least this wide run their four products on the
// tensor cores (3xTF32 from split copies); smaller ones are latency bound and
// stay on the CUDA cores.
constexpr int64_t kTensorNode = 512;

// Split of a node of width s into halves h + r (h a multiple of the leaf).
inline int64_t node_half(int64_t s) {
  const int64_t nblk = (s + LEAF - 1) / LEAF;
  return std::max<int64_t>(1, nblk / 2) * LEAF;
}

// Largest split-copy area any tensor-core node of the recursion needs.
size_t split_need(int64_t s) {
  if (s <= LEAF) return 0;
  const int64_t h = node_half(s), r = s - h;
  size_t here = 0;
  if (h >= kTensorNode) {
    const size_t before = 2 * static_cast<size_t>(r * h + h * h + h * h + r * h);
    const size_t after = 2 * static_cast<size_t>(h * r + r * r);
    here = std::max(before, after);
  }
  return std::max(here, std::max(split_need(h), split_need(r)));
}

void chol_inv_rec(const Ctx& c, float* M, float* X, int64_t ld, int64_t off, int64_t s, float* scratch,
                  float* split) {
  float* Md = M + off * ld + off;
  float* Xd = X + off * ld + off;
  if (s <= LEAF) {
    static bool attr_done[64] = {false};
    if (!attr_done[c.device & 63]) {
      check_cuda(cudaFuncSetAttribute(leaf_chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(LEAF_SMEM)),
                 "cudaFuncSetAttribute(leaf)");
      attr_done[c.device & 63] = true;
    }
    leaf_chol_inv_kernel<<<1, LEAF_THREADS, LEAF_SMEM, c.stream>>>(Md, Xd, ld, static_cast<int>(s), c.status);
    check_launch("leaf_chol_inv_kernel");
    return;
  }
  const int64_t h = node_half(s);
  const int64_t r = s - h;
  chol_inv_rec(c, M, X, ld, off, h, scratch, split);
  float* Y = scratch;
  float* T = scratch + r * h;
  const float* M21 = M + (off + h) * ld + off;
  float* M22 = M + (off + h) * ld + (off + h);
  const float* X11 = Xd;
  const float* X22 = X + (off + h) * ld + (off + h);
  float* X21 = X + (off + h) * ld + off;
  const bool tensor = split != nullptr && h >= kTensorNode;
  if (tensor) {
    // split copies (hi, lo) in `split`: [M21 | X11 | X11^T | T], then [Y^T | X22]
    float* m21h = split;
    float* m21l = m21h + r * h;
    float* x11h = m21l + r * h;
    float* x11l = x11h + h * h;
    float* x11th = x11l + h * h;
    float* x11tl = x11th + h * h;
    float* th = x11tl + h * h;
    float* tl = th + r * h;
    split_tf32(c, M21, r, h, ld, m21h, m21l, h);
    split_tf32(c, X11, h, h, ld, x11h, x11l, h);
    split_tf32(c, X11, h, h, ld, x11th, x11tl, h, true);
    // L21 = A21 X11^T  (B stored = X11, op(B) = X11^T upper)
    gemm_tf32x3(c, r, h, h, 1.f, m21h, m21l, h, x11h, x11l, h, false, T, h, kBUpper);
    split_tf32(c, T, r, h, h, th, tl, h);
    // A22 -= L21 L21^T  (lower tiles)
    gemm_tf32x3(c, r, r, h, -1.f, th, tl, h, th, tl, h, true, M22, ld, kCLowerOnly);
    // Y = L21 X11  (B stored = X11^T, op(B) = X11 lower)
    gemm_tf32x3(c, r, h, h, 1.f, th, tl, h, x11th, x11tl, h, false, Y, h, kBLower);
  } else {
    // L21 = A21 X11^T
    gemm_f32(c, false, true, r, h, h, 1.f, M21, ld, X11, ld, 0.f, T, h, kBUpper);
    // A22 -= L21 L21^T (lower tiles only)
    gemm_f32(c, false, true, r, r, h, -1.f, T, h, T, h, 1.f, M22, ld, kCLowerOnly);
    // Y = L21 X11
    gemm_f32(c, false, false, r, h, h, 1.f, T, h, X11, ld, 0.f, Y, h, kBLower);
  }
  chol_inv_rec(c, M, X, ld, off + h, r, scratch + r * h, split);
  if (tensor) {
    float* yth = split;
    float* ytl = yth + h * r;
    float* x22h = ytl + h * r;
    float* x22l = x22h + r * r;
    split_tf32(c, Y, r, h, h, yth, ytl, r, true);
    split_tf32(c, X22, r, r, ld, x22h, x22l, r);
    // X21 = -X22 Y  (A = X22 lower; B stored = Y^T)
    gemm_tf32x3(c, r, h, r, -1.f, x22h, x22l, r, yth, ytl, r, false, X21, ld, kALower);
  } else {
    // X21 = -X22 Y
    gemm_f32(c, false, false, r, h, r, -1.f, X22, ld, Y, h, 0.f, X21, ld, kALower);
  }
}

}  // namespace

size_t factor_split_floats(int64_t n) { return split_need(n) + 4096; }

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

namespace {

void factor_direct(const Ctx& c, float* M, float* X, float* scratch, float* U, int64_t n, float* split) {
  check_cuda(cudaMemsetAsync(X, 0, static_cast<size_t>(n) * n * sizeof(float), c.stream), "memset X");
  chol_inv_rec(c, M, X, n, 0, n, scratch, split);
  const int64_t total = n * n;
  reverse_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, c.stream>>>(X, U, n);
  check_launch("reverse_kernel");
}

// The factorisation is a fixed sequence of a few hundred small launches for a
// given n and buffers; it is recorded once into a CUDA graph and replayed.
struct FactorGraph {
  int device;
  int64_t n;
  const void *M, *X, *scratch, *U, *status, *split;
  cudaGraphExec_t exec;
  int64_t launches;
};
std::vector<FactorGraph> g_factor_graphs;

}  // namespace

void factor_inverse_upper(const Ctx& c, float* M, float* X, float* scratch, float* U, int64_t n,
                          bool use_graph, float* split) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (c.stream != nullptr) check_cuda(cudaStreamIsCapturing(c.stream, &cs), "cudaStreamIsCapturing");
  if (!use_graph || cs != cudaStreamCaptureStatusNone) {
    factor_direct(c, M, X, scratch, U, n, split);
    return;
  }
  for (const FactorGraph& g : g_factor_graphs) {
    if (g.device == c.device && g.n == n && g.M == M && g.X == X && g.scratch == scratch && g.U == U &&
        g.status == c.status && g.split == split) {
      check_cuda(cudaGraphLaunch(g.exec, c.stream), "cudaGraphLaunch(factor)");
      count_launches(g.launches);
      return;
    }
  }
  // Record on a private stream (recording runs nothing), replay on the caller's.
  static cudaStream_t capture_stream[64] = {};
  if (capture_stream[c.device & 63] == nullptr)
    check_cuda(cudaStreamCreateWithFlags(&capture_stream[c.device & 63], cudaStreamNonBlocking),
               "cudaStreamCreate(capture)");
  Ctx cc = c;
  cc.stream = capture_stream[c.device & 63];
  const int64_t l0 = launch_count();
  check_cuda(cudaStreamBeginCapture(cc.stream, cudaStreamCaptureModeThreadLocal), "cudaStreamBeginCapture");
  cudaGraph_t graph = nullptr;
  try {
    factor_direct(cc, M, X, scratch, U, n, split);
  } catch (...) {
    cudaStreamEndCapture(cc.stream, &graph);
    if (graph) cudaGraphDestroy(graph);
    throw;
  }
  check_cuda(cudaStreamEndCapture(cc.stream, &graph), "cudaStreamEndCapture");
  cudaGraphExec_t exec = nullptr;
  const cudaError_t e = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  check_cuda(e, "cudaGraphInstantiate(factor)");
  const int64_t recorded = launch_count() - l0;
  if (g_factor_graphs.size() >= 8) {
    cudaGraphExecDestroy(g_factor_graphs.front().exec);
    g_factor_graphs.erase(g_factor_graphs.begin());
  }
  g_factor_graphs.push_back({c.device, n, M, X, scratch, U, c.status, split, exec, recorded});
  check_cuda(cudaGraphLaunch(exec, c.stream), "cudaGraphLaunch(factor)");
}

namespace {

// Sets the graph's condition: 1 when GPTQ's preparation found dead columns.
__global__ void set_dead_condition_kernel(cudaGraphConditionalHandle h, const DiagStats* stats) {
  cudaGraphSetConditional(h, stats->n_dead > 0 ? 1u : 0u);
}

struct SelectGraph {
  int device;
  int64_t n;
  const void *H, *perm, *stats_g, *stats_q, *Ug, *Uq, *X, *scratch, *split, *status;
  cudaGraphExec_t exec;
};
std::vector<SelectGraph> g_select_graphs;

}  // namespace

void qep_factor_select(const Ctx& c, const float* H, int64_t n, const int32_t* perm, const DiagStats* stats_g,
                       const DiagStats* stats_q, const float* Ug, float* Uq, float* X, float* scratch, float* split) {
  for (const SelectGraph& g : g_select_graphs) {
    if (g.device == c.device && g.n == n && g.H == H && g.perm == perm && g.stats_g == stats_g &&
        g.stats_q == stats_q && g.Ug == Ug && g.Uq == Uq && g.X == X && g.scratch == scratch && g.split == split &&
        g.status == c.status) {
      check_cuda(cudaGraphLaunch(g.exec, c.stream), "cudaGraphLaunch(select)");
      count_launches(1);
      return;
    }
  }
  // One graph: a kernel that reads the dead-column count on the device, then
  // an if/else node.  If: QEP's own matrix H + lam I (no dead-column fix, lam
  // from stats_q) in processing order, factored into Uq.  Else: Uq = Ug.
  cudaGraph_t graph = nullptr;
  check_cuda(cudaGraphCreate(&graph, 0), "cudaGraphCreate(select)");
  cudaGraphExec_t exec = nullptr;
  static cudaStream_t capture_stream[64] = {};
  try {
    cudaGraphConditionalHandle h;
    check_cuda(cudaGraphConditionalHandleCreate(&h, graph, 0, cudaGraphCondAssignDefault),
               "cudaGraphConditionalHandleCreate");
    cudaKernelNodeParams kp = {};
    void* args[2] = {&h, const_cast<DiagStats**>(&stats_g)};
    kp.func = reinterpret_cast<void*>(set_dead_condition_kernel);
    kp.gridDim = dim3(1);
    kp.blockDim = dim3(1);
    kp.kernelParams = args;
    cudaGraphNode_t setter = nullptr;
    check_cuda(cudaGraphAddKernelNode(&setter, graph, nullptr, 0, &kp), "cudaGraphAddKernelNode(select)");
    cudaGraphNodeParams cp = {};
    cp.type = cudaGraphNodeTypeConditional;
    cp.conditional.handle = h;
    cp.conditional.type = cudaGraphCondTypeIf;
    cp.conditional.size = 2;
    cudaGraphNode_t cond = nullptr;
    check_cuda(cudaGraphAddNode(&cond, graph, &setter, 1, &cp), "cudaGraphAddNode(conditional)");
    cudaGraph_t body_dead = cp.conditional.phGraph_out[0];
    cudaGraph_t body_live = cp.conditional.phGraph_out[1];
    if (capture_stream[c.device & 63] == nullptr)
      check_cuda(cudaStreamCreateWithFlags(&capture_stream[c.device & 63], cudaStreamNonBlocking),
                 "cudaStreamCreate(capture)");
    Ctx cc = c;
    cc.stream = capture_stream[c.device & 63];
    check_cuda(cudaStreamBeginCaptureToGraph(cc.stream, body_dead, nullptr, nullptr, 0,
                                             cudaStreamCaptureModeThreadLocal),
               "cudaStreamBeginCaptureToGraph(dead)");
    try {
      launch_build_reversed(cc, H, n, perm, stats_q, 1.0f, false, Uq);
      factor_direct(cc, Uq, X, scratch, Uq, n, split);
    } catch (...) {
      cudaStreamEndCapture(cc.stream, &body_dead);
      throw;
    }
    check_cuda(cudaStreamEndCapture(cc.stream, &body_dead), "cudaStreamEndCapture(dead)");
    check_cuda(cudaStreamBeginCaptureToGraph(cc.stream, body_live, nullptr, nullptr, 0,
                                             cudaStreamCaptureModeThreadLocal),
               "cudaStreamBeginCaptureToGraph(live)");
    const cudaError_t e = cudaMemcpyAsync(Uq, Ug, static_cast<size_t>(n) * n * sizeof(float),
                                          cudaMemcpyDeviceToDevice, cc.stream);
    check_cuda(cudaStreamEndCapture(cc.stream, &body_live), "cudaStreamEndCapture(live)");
    check_cuda(e, "copy factor");
    check_cuda(cudaGraphInstantiate(&exec, graph, 0), "cudaGraphInstantiate(select)");
  } catch (...) {
    cudaGraphDestroy(graph);
    throw;
  }
  cudaGraphDestroy(graph);
  if (g_select_graphs.size() >= 8) {
    cudaGraphExecDestroy(g_select_graphs.front().exec);
    g_select_graphs.erase(g_select_graphs.begin());
  }
  g_select_graphs.push_back({c.device, n, H, perm, stats_g, stats_q, Ug, Uq, X, scratch, split, c.status, exec});
  check_cuda(cudaGraphLaunch(exec, c.stream), "cudaGraphLaunch(select)");
  count_launches(1);
}

}  // namespace oc

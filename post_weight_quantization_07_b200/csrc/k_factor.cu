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
// with 128x128 leaves factored and inverted inside one CTA.
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
// one CTA with the whole block in shared memory.  The block is split
// recursively, 128 -> 64 -> 32, with the same four products as the outer
// recursion:
//   X11 = L11^-1 (recurse);  T = A21 X11^T (= L21);  A22 -= T T^T;
//   Y = T X11;  X22 = L22^-1 (recurse);  X21 = -X22 Y.
// A 32x32 block is factored and inverted by one warp: lane i holds row i in
// registers; column k of L reaches the other lanes by shuffles; the inverse is
// forward substitution per column (lane j owns column j of X) reading L from
// shared memory.  Rows and columns beyond s are padded with the identity.
constexpr int LDA = LEAF + 1;      // padded leading dimensions (bank spread)
constexpr int LDT = LEAF / 2 + 1;

struct LeafSmem {
  float4 col4[32];                 // 4 columns of the current 32 block, one row per lane
  float4 blk[4];                   // the current 4x4 pivot block
  float A[LEAF * LDA];
  float X[LEAF * LDA];
  float T[(LEAF / 2) * LDT];       // L21 of the 128 level; temporaries of the 64 level
  float Y[(LEAF / 2) * LDT];       // Y of the 128 level (lives across the right half)
  float L32[32 * 33];              // factor of the current 32 block
  float R32[32];                   // reciprocals of its diagonal
};

// One step of the 32x32 factor: columns K..K+3.  The 4x4 pivot block is
// factored redundantly by every lane in registers; each lane then finishes its
// own row's four entries, and the four columns reach the other lanes as one
// float4 per row through shared memory.
template <int K>
__device__ __forceinline__ void chol32_step(LeafSmem& sm, float (&a)[32], int lane, bool& bad) {
  if (lane >= K && lane < K + 4) sm.blk[lane - K] = make_float4(a[K], a[K + 1], a[K + 2], a[K + 3]);
  __syncwarp();
  const float4 q0 = sm.blk[0], q1 = sm.blk[1], q2 = sm.blk[2], q3 = sm.blk[3];
  const float r0 = rsqrtf(q0.x);
  const float l10 = q1.x * r0, l20 = q2.x * r0, l30 = q3.x * r0;
  const float d1 = fmaf(-l10, l10, q1.y);
  const float r1 = rsqrtf(d1);
  const float l21 = fmaf(-l20, l10, q2.y) * r1, l31 = fmaf(-l30, l10, q3.y) * r1;
  const float d2 = fmaf(-l21, l21, fmaf(-l20, l20, q2.z));
  const float r2 = rsqrtf(d2);
  const float l32 = fmaf(-l31, l21, fmaf(-l30, l20, q3.z)) * r2;
  const float d3 = fmaf(-l32, l32, fmaf(-l31, l31, fmaf(-l30, l30, q3.w)));
  const float r3 = rsqrtf(d3);
  if (!(q0.x > 0.f) || !(d1 > 0.f) || !(d2 > 0.f) || !(d3 > 0.f) || !isfinite(q0.x + d1 + d2 + d3)) bad = true;
  const float x0 = a[K] * r0;
  const float x1 = fmaf(-x0, l10, a[K + 1]) * r1;
  const float x2 = fmaf(-x1, l21, fmaf(-x0, l20, a[K + 2])) * r2;
  const float x3 = fmaf(-x2, l32, fmaf(-x1, l31, fmaf(-x0, l30, a[K + 3]))) * r3;
  const int rr = lane - K;  // rows of the pivot block keep zeros above the diagonal
  a[K] = x0;
  a[K + 1] = (rr >= 0 && rr < 1) ? 0.f : x1;
  a[K + 2] = (rr >= 0 && rr < 2) ? 0.f : x2;
  a[K + 3] = (rr >= 0 && rr < 3) ? 0.f : x3;
  if constexpr (K + 4 < 32) {
    sm.col4[lane] = make_float4(a[K], a[K + 1], a[K + 2], a[K + 3]);
    __syncwarp();
#pragma unroll
    for (int j = K + 4; j < 32; ++j) {
      const float4 v = sm.col4[j];
      if (lane >= j)
        a[j] = fmaf(-a[K + 3], v.w, fmaf(-a[K + 2], v.z, fmaf(-a[K + 1], v.y, fmaf(-a[K], v.x, a[j]))));
    }
    chol32_step<K + 4>(sm, a, lane, bad);
  }
}

__device__ __noinline__ void warp_chol_inv32(LeafSmem& sm, int off, int* status) {
  const int lane = threadIdx.x & 31;
  float a[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) a[j] = (j <= lane) ? sm.A[(off + lane) * LDA + off + j] : 0.f;
  bool bad = false;
  chol32_step<0>(sm, a, lane, bad);
  if (bad && lane == 0) record_error(status, kDevNotSpd);
  float dl = 1.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    sm.L32[lane * 33 + j] = a[j];
    if (j == lane) dl = a[j];
  }
  sm.R32[lane] = 1.f / dl;
  __syncwarp();
  // Column `lane` of X = L^-1 by right-looking forward substitution: at step k
  // x_k = b_k / L_kk, then every later row takes b_i -= L_ik x_k (independent
  // updates: the dependent chain is one multiply and one FMA per step).
  float b[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) b[i] = (i == lane) ? 1.f : 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float xk = b[k] * sm.R32[k];
    b[k] = xk;
#pragma unroll
    for (int i = k + 1; i < 32; ++i) b[i] = fmaf(-sm.L32[i * 33 + k], xk, b[i]);
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) sm.X[(off + i) * LDA + off + lane] = b[i];
}

// The four products of one recursion node of half width H inside the CTA
// (256 threads, each a TR x TC register tile of the H x H outputs).
template <int H>
__device__ __forceinline__ void node_pre(LeafSmem& sm, int off, float* T, int ldt, float* Y, int ldy) {
  constexpr int TR = (H == 64) ? 4 : 2, TC = TR;
  constexpr int NTC = H / TC;
  const int t = threadIdx.x;
  const int i0 = (t / NTC) * TR, j0 = (t % NTC) * TC;
  const float* A21 = &sm.A[(off + H) * LDA + off];
  float* A22 = &sm.A[(off + H) * LDA + off + H];
  const float* X11 = &sm.X[off * LDA + off];
  // T = A21 X11^T: T[i][j] = sum_{k <= j} A21[i][k] X11[j][k]
  {
    float acc[TR][TC] = {};
    for (int k = 0; k < j0 + TC; ++k) {
      float av[TR], bv[TC];
#pragma unroll
      for (int r = 0; r < TR; ++r) av[r] = A21[(i0 + r) * LDA + k];
#pragma unroll
      for (int c = 0; c < TC; ++c) bv[c] = X11[(j0 + c) * LDA + k];
#pragma unroll
      for (int r = 0; r < TR; ++r)
#pragma unroll
        for (int c = 0; c < TC; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int c = 0; c < TC; ++c) T[(i0 + r) * ldt + j0 + c] = acc[r][c];
  }
  __syncthreads();
  // A22 -= T T^T (tiles touching the lower triangle)
  if (j0 <= i0 + TR - 1) {
    float acc[TR][TC] = {};
    for (int k = 0; k < H; ++k) {
      float av[TR], bv[TC];
#pragma unroll
      for (int r = 0; r < TR; ++r) av[r] = T[(i0 + r) * ldt + k];
#pragma unroll
      for (int c = 0; c < TC; ++c) bv[c] = T[(j0 + c) * ldt + k];
#pragma unroll
      for (int r = 0; r < TR; ++r)
#pragma unroll
        for (int c = 0; c < TC; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int c = 0; c < TC; ++c) A22[(i0 + r) * LDA + j0 + c] -= acc[r][c];
  }
  // Y = T X11: Y[i][j] = sum_{k >= j} T[i][k] X11[k][j]
  {
    float acc[TR][TC] = {};
    for (int k = j0; k < H; ++k) {
      float av[TR], bv[TC];
#pragma unroll
      for (int r = 0; r < TR; ++r) av[r] = T[(i0 + r) * ldt + k];
#pragma unroll
      for (int c = 0; c < TC; ++c) bv[c] = X11[k * LDA + j0 + c];
#pragma unroll
      for (int r = 0; r < TR; ++r)
#pragma unroll
        for (int c = 0; c < TC; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int c = 0; c < TC; ++c) Y[(i0 + r) * ldy + j0 + c] = acc[r][c];
  }
  __syncthreads();
}

template <int H>
__device__ __forceinline__ void node_post(LeafSmem& sm, int off, const float* Y, int ldy) {
  constexpr int TR = (H == 64) ? 4 : 2, TC = TR;
  constexpr int NTC = H / TC;
  const int t = threadIdx.x;
  const int i0 = (t / NTC) * TR, j0 = (t % NTC) * TC;
  const float* X22 = &sm.X[(off + H) * LDA + off + H];
  float* X21 = &sm.X[(off + H) * LDA + off];
  // X21 = -X22 Y: X21[i][j] = -sum_{k <= i} X22[i][k] Y[k][j]
  float acc[TR][TC] = {};
  for (int k = 0; k < i0 + TR; ++k) {
    float av[TR], bv[TC];
#pragma unroll
    for (int r = 0; r < TR; ++r) av[r] = X22[(i0 + r) * LDA + k];
#pragma unroll
    for (int c = 0; c < TC; ++c) bv[c] = Y[k * ldy + j0 + c];
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int c = 0; c < TC; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
  }
#pragma unroll
  for (int r = 0; r < TR; ++r)
#pragma unroll
    for (int c = 0; c < TC; ++c) X21[(i0 + r) * LDA + j0 + c] = -acc[r][c];
  __syncthreads();
}

__device__ __forceinline__ void leaf32(LeafSmem& sm, int off, int* status) {
  if ((threadIdx.x >> 5) == 0) warp_chol_inv32(sm, off, status);
  __syncthreads();
}

// 64 block at `off`; its temporaries live in sm.T (T at 0, Y at 32 rows on).
__device__ __forceinline__ void leaf64(LeafSmem& sm, int off, int* status) {
  float* T = sm.T;
  float* Y = sm.T + 32 * 33;
  leaf32(sm, off, status);
  node_pre<32>(sm, off, T, 33, Y, 33);
  leaf32(sm, off + 32, status);
  node_post<32>(sm, off, Y, 33);
}

__global__ void __launch_bounds__(256) leaf_chol_inv_kernel(const float* __restrict__ M, float* __restrict__ X,
                                                            int64_t ld, int s, int* status) {
  extern __shared__ __align__(16) float leaf_smem[];
  LeafSmem& sm = *reinterpret_cast<LeafSmem*>(leaf_smem);
  const int t = threadIdx.x;
  // Load the block with 16 independent 16-byte loads per thread in flight
  // (rows of M are 16-byte aligned: n is a multiple of 64).
  float4 v[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int e4 = t + 256 * q;          // float4 index in the 128 x 128 block
    const int i = e4 >> 5, j = (e4 & 31) * 4;
    v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < s && j <= i && j < s) v[q] = *reinterpret_cast<const float4*>(M + static_cast<int64_t>(i) * ld + j);
  }
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int e4 = t + 256 * q;
    const int i = e4 >> 5, j = (e4 & 31) * 4;
    const float vv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float x = (j + c <= i && j + c < s) ? vv[c] : 0.f;
      if (i >= s && i == j + c) x = 1.f;  // identity padding beyond s
      sm.A[i * LDA + j + c] = x;
      sm.X[i * LDA + j + c] = 0.f;
    }
  }
  __syncthreads();
  leaf64(sm, 0, status);
  node_pre<64>(sm, 0, sm.T, LDT, sm.Y, LDT);
  leaf64(sm, 64, status);
  node_post<64>(sm, 0, sm.Y, LDT);
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int e4 = t + 256 * q;
    const int i = e4 >> 5, j = (e4 & 31) * 4;
    if (i < s && j < s) {
      float4 o;
      o.x = (j + 0 <= i) ? sm.X[i * LDA + j + 0] : 0.f;
      o.y = (j + 1 <= i) ? sm.X[i * LDA + j + 1] : 0.f;
      o.z = (j + 2 <= i) ? sm.X[i * LDA + j + 2] : 0.f;
      o.w = (j + 3 <= i) ? sm.X[i * LDA + j + 3] : 0.f;
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
                                      static_cast<int>(sizeof(LeafSmem))),
                 "cudaFuncSetAttribute(leaf)");
      attr_done[c.device & 63] = true;
    }
    leaf_chol_inv_kernel<<<1, 256, sizeof(LeafSmem), c.stream>>>(Md, Xd, ld, static_cast<int>(s), c.status);
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

// Internal declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/oc.h"

namespace oc {

// Device-side error codes recorded in the status word (same values as oc_status).
enum DevErr : int {
  kDevOk = 0,
  kDevNotSpd = OC_ERR_NOT_SPD,
  kDevNonfinite = OC_ERR_NONFINITE,
  kDevTimeout = OC_ERR_TIMEOUT,
};

// Record the first device-side error (later ones are dropped).
__device__ __forceinline__ void record_error(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Per-call context handed to the internal launchers.
struct Ctx {
  cudaStream_t stream;
  int* status;      // device status word
  int sm_count;
  int device;
};

// Host-side failure carrying a status and a message (converted to the C ABI
// return value at the boundary).
struct Failure {
  int status;
  char msg[512];
};
[[noreturn]] void fail(int status, const char* fmt, ...);
void check_cuda(cudaError_t e, const char* what);
void set_last_error(const char* msg);  // text returned by oc_last_error() on this thread
// The lock every entry point holds while it sets up and enqueues its work
// (launch helpers share host-side state such as one-time attribute flags).
std::mutex& library_mutex();
void check_launch(const char* kernel);

// ------------------------------------------------------------------ profiling
enum Phase : int {
  kPhHessian = 0,   // the tensor-core SYRK launch of the Hessian (one launch)
  kPhQepCross,      // the tensor-core X^T Xhat launch (one launch)
  kPhQepSyrk,       // Xhat^T Xhat when no H is supplied
  kPhQepWDelta,     // G = W d
  kPhFactor,        // dampening, reversal, blocked Cholesky + inverse, reversal
  kPhQepApply,      // W + 2 alpha (G U^T) U
  kPhGptqPrep,      // act_order order, permutation of W, static grid
  kPhGptqSweep,     // 128-column block sweeps
  kPhGptqTrailing,  // trailing updates of later columns
  kPhGptqPack,      // inverse permutation + bit packing
  kPhHessianFix,    // clearing H, mirroring its upper triangle
  kPhQepCrossFix,   // clearing d before the cross product accumulates into it
  kPhRotate,        // Hadamard rotation
  kPhLpcdLeft,      // LPCD's relaxed layer-1 step (products, factorisation, solve)
  kPhGemv,          // dequantising GEMV over packed codes
  kPhQepDiff,       // cross-product operands when no Hessian launch carries them
  kNumPhases
};

void count_launch();
void count_launches(int64_t k);  // launches replayed from a recorded graph
int64_t launch_count();
void profile_enable(bool on);
int profile_read(double* ms, int64_t* launches, int max_phases);
const char* phase_name(int p);

// Records a CUDA event pair around its lifetime on the call's stream when
// profiling is enabled (no-op otherwise).
class PhaseScope {
 public:
  PhaseScope(const struct Ctx& c, Phase p);
  ~PhaseScope();
  PhaseScope(const PhaseScope&) = delete;
  PhaseScope& operator=(const PhaseScope&) = delete;

 private:
  cudaStream_t stream_;
  Phase phase_;
  cudaEvent_t a_ = nullptr;
  int64_t l0_ = 0;
  bool active_ = false;
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// TMA descriptor for a row-major 2-D array [rows x cols] of `elem_bytes`
// elements with leading dimension `ld` (elements), box [box_rows x box_cols].
enum class Swz { None, B128 };
CUtensorMap make_tmap_2d(const void* base, CUtensorMapDataType dt, int elem_bytes,
                         uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
                         uint32_t box_cols, Swz swz);

// ------------------------------------------------------------------ kernels

// C[i][j] += alpha * sum_t A[t][i] * B[t][j] with A, B bf16 token-major
// [n_tok x M] and [n_tok x N]; C fp32 [M x N] (ldc).  upper_only: A == B and
// only tiles touching the upper triangle are computed (the caller mirrors).
// max_ctas > 0 caps the persistent grid (leaving SMs free for concurrent work).
void launch_atb16(const Ctx& c, const void* A, const void* B, int64_t n_tok, int64_t M, int64_t N, float alpha,
                  float* C, int64_t ldc, bool upper_only, int max_ctas = 0);

// How a persistent tensor-core product over tokens cuts its work: units of
// (output tile, token chunk of kc_stages 128-token stages, n_kc chunks),
// taken round-robin by `clusters` CTA pairs; units [0, full_units) are whole
// chunks, the rest split_k parts of the leftover chunks (units in all).
struct UnitPlan {
  int64_t kc_stages, n_kc, full_units, units;
  int split_k;
};
UnitPlan plan_units(int64_t n_tok, int64_t n_tiles, int64_t clusters);

// The next launch_atb16 / launch_cross_product launch of the tensor-core
// product stalls on a barrier nothing releases (test of the failure path).
void request_test_stall();

// QEP's cross term d = (X - Xhat)^T Xhat (n x n, fp32, overwritten) from the
// bf16 token-major pair X, Xhat [n_tok x n] and H = 2 Xhat^T Xhat of the same
// tokens (its diagonal sets per-feature fp16 scales).  Runs as `parts` token
// slices on at most max_ctas SMs (0: all), each slice's operands prepared
// while the previous slice runs.  `scratch`: cross_scratch_bytes(n_tok, n)
// bytes of device memory, 256-byte aligned.
size_t cross_scratch_bytes(int64_t n_tok, int64_t n);
void launch_cross_product(const Ctx& c, const void* X, const void* Xhat, int64_t n_tok, int64_t n, const float* H,
                          float* d, void* scratch, int parts, int max_ctas);

// Per-device side stream and fork/join events for running the (latency
// bound) factorisation beside a tensor-core product on the call's stream.
struct SideStream {
  cudaStream_t stream;
  cudaEvent_t fork, join;
};
SideStream& side_stream(int device);
// SMs left to the side stream while the main stream's product runs.
constexpr int kSideSMs = 8;
// Most layers one oc_quantize_layer_group call takes.
constexpr int kMaxGroup = 16;
// The cross product beside it runs as up to kCrossParts launches over token
// ranges of at least kCrossPartMinTokens tokens each: each boundary lets the
// factorisation's pending products take the whole GPU.
constexpr int64_t kCrossParts = 32;
constexpr int64_t kCrossPartMinTokens = 8192;

// Mirror the upper triangle of an n x n matrix into its lower triangle.
void launch_mirror_upper(const Ctx& c, float* H, int64_t n);

// Flags for gemm_f32: triangular structure of op(A)/op(B) (zeros skipped) and
// C tiles wholly above the diagonal skipped.
enum GemmFlags : unsigned {
  kANone = 0,
  kALower = 1u << 0,
  kAUpper = 1u << 1,
  kBLower = 1u << 2,
  kBUpper = 1u << 3,
  kCLowerOnly = 1u << 4,
};

// C = beta*C + alpha*op(A)*op(B), fp32, row-major, op = transpose when tX.
void gemm_f32(const Ctx& c, bool tA, bool tB, int64_t M, int64_t N, int64_t K, float alpha,
              const float* A, int64_t lda, const float* B, int64_t ldb, float beta, float* C,
              int64_t ldc, unsigned flags);

// x_hi = tf32(x), x_lo = tf32(x - x_hi) of a rows x cols block of src
// (leading dimension lds); written untransposed (ldd) or, with transpose,
// as the cols x rows transpose (ldd = leading dimension of the transpose).
// lo_nz (untransposed, 16-byte aligned rows only): a device flag set to 1 if
// any lo is non-zero, else 0 (x exact in tf32).
void split_tf32(const Ctx& c, const float* src, int64_t rows, int64_t cols, int64_t lds, float* hi,
                float* lo, int64_t ldd, bool transpose = false, int* lo_nz = nullptr);

// fp32-accurate tensor-core GEMM from split operands: C (+)= alpha A B^T with
// A [M x K] (lda) and B [N x K] (ldb) row-major; accumulate selects C += over
// C =.  Flags describe the triangles of A and of op(B) = B^T.  Pointers and
// leading dimensions must allow 16-byte aligned TMA rows.
// a_lo_nz, b_lo_nz: optional device flags from split_tf32; when one reads 0
// that operand's lo half is all zero and its correction product is skipped.
void gemm_tf32x3(const Ctx& c, int64_t M, int64_t N, int64_t K, float alpha, const float* A_hi,
                 const float* A_lo, int64_t lda, const float* B_hi, const float* B_lo, int64_t ldb,
                 bool accumulate, float* C, int64_t ldc, unsigned flags, const int* a_lo_nz = nullptr,
                 const int* b_lo_nz = nullptr);

// U = upper Cholesky factor of (H_prepared)^-1, where H_prepared is formed by
// `launch_build_reversed` into M (consumed).  Scratch must hold n*n/2 + 4096
// floats.  X receives L^-1 of the reversed matrix (lower), U its reversal.
// use_graph: record the launch sequence once per (n, buffers) into a CUDA
// graph and replay it (instantiating a graph allocates; pass false to run the
// launches directly).  split: NULL, or room for factor_split_floats(n) floats,
// which lets the large products run on the tensor cores (3xTF32).
void factor_inverse_upper(const Ctx& c, float* M, float* X, float* scratch, float* U,
                          int64_t n, bool use_graph = true, float* split = nullptr);
size_t factor_split_floats(int64_t n);

// M[a][b] = Hfix[p(n-1-a)][p(n-1-b)] + lam*[a==b] where Hfix has dead
// diagonal entries set to 1 (when fix_dead), p = perm (identity if null) and
// lam = damp * mean(diag Hfix) (computed on device into stats).
struct DiagStats {
  float lam;
  float mean_diag;
  int n_dead;
  int nonfinite;
};
void launch_diag_stats(const Ctx& c, const float* H, int64_t n, float damp, float hscale,
                       bool fix_dead, DiagStats* stats, unsigned char* dead);
void launch_act_order_perm(const Ctx& c, const float* H, int64_t n, int32_t* perm);
void launch_identity_perm(const Ctx& c, int64_t n, int32_t* perm);
void launch_build_reversed(const Ctx& c, const float* H, int64_t n, const int32_t* perm,
                           const DiagStats* stats, float hscale, bool fix_dead, float* M);

// QEP's inverse factor in GPTQ's processing order, decided on the device:
// when GPTQ's preparation (stats_g) found dead columns, QEP's own matrix
// H + lam I (lam = stats_q->lam, no dead-column fix) permuted by perm is
// factored into Uq (X, scratch, split: the factorisation's scratch);
// otherwise the two dampened matrices are the same and Uq = Ug.  Recorded
// once per (n, buffers) as a graph with a conditional node; no host read.
void qep_factor_select(const Ctx& c, const float* H, int64_t n, const int32_t* perm, const DiagStats* stats_g,
                       const DiagStats* stats_q, const float* Ug, float* Uq, float* X, float* scratch, float* split);

// GPTQ pieces.
void launch_permute_w(const Ctx& c, const float* W, int64_t m, int64_t n, const int32_t* perm,
                      const unsigned char* dead, float* Wp);
void launch_static_grid(const Ctx& c, const float* W, int64_t m, int64_t n, int G, int wbits,
                        const unsigned char* dead, float* scales, float* zeros);
// Err (and Err_lo) rows have err_ld floats (>= 128); the block's errors go to
// their first 128 columns.
void launch_sweep_block(const Ctx& c, float* Wp, int64_t m, int64_t n, const float* U,
                        int64_t j1, int G, int wbits, bool static_groups, const int32_t* perm,
                        float* scales, float* zeros, unsigned char* codes8, float* Err,
                        float* Err_lo = nullptr, int64_t err_ld = 128);
// GPTQ's lazy updates: superblocks of this many columns (four sweep blocks).
constexpr int64_t kSuperBlock = 512;
// Packs codes8 (processing order) into the original-order bitstream; perm2
// holds the processing order in its first n entries and receives the inverse
// permutation in the next n.
// Y = X (I (x) H_b) / sqrt(b) along rows of n features, b = 2^log2b <= 4096.
void launch_hadamard(const Ctx& c, const void* X, void* Y, int64_t rows, int64_t n, int log2b, bool bf16);
// out[i][j] = scale * (code - zero), fp32 or bf16, original column order.
// y[b][i] = sum_j x[b][j] Q[i][j] over packed codes (nb <= 8 bf16 rows of x, fp32 y).
void launch_dequant_gemv(const Ctx& c, const uint32_t* codes, const float* scales, const float* zeros, int64_t m,
                         int64_t n, int wbits, int64_t G, const void* x, int nb, float* y);
void launch_dequant(const Ctx& c, const uint32_t* codes, const float* scales, const float* zeros, int64_t m,
                    int64_t n, int wbits, int64_t G, void* out, bool bf16);
void launch_pack(const Ctx& c, const unsigned char* codes8, int64_t m, int64_t n, int wbits,
                 int32_t* perm2, uint32_t* codes);

// perm2[n .. 2n) := inverse of the permutation in perm2[0 .. n).
void launch_invert_perm(const Ctx& c, int32_t* perm2, int64_t n);

// QEP pieces.
void launch_copy_f32(const Ctx& c, const float* src, float* dst, int64_t count);
void launch_fill_f32(const Ctx& c, float* dst, int64_t count, float v);
void launch_check_finite(const Ctx& c, const float* x, int64_t count);

}  // namespace oc

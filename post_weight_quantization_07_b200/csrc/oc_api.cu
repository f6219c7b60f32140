// C ABI entry points (include/oc.h): argument checks, per-device workspace and
// status word, and the sequencing of the kernels of each call.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include "oc_internal.cuh"

namespace oc {

namespace {

thread_local char g_last_error[768] = "";
int g_sync_mode = 1;
std::mutex g_mu;

struct DeviceState {
  bool init = false;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  int* status = nullptr;  // device status word
  void* ws = nullptr;
  size_t ws_bytes = 0;
};
DeviceState g_dev[64];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    check_cuda(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q),
               "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
    if (q != cudaDriverEntryPointSuccess || p == nullptr)
      fail(OC_ERR_UNSUPPORTED, "driver does not provide cuTensorMapEncodeTiled");
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

DeviceState& device_state(int dev) {
  if (dev < 0 || dev >= 64) fail(OC_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  DeviceState& d = g_dev[dev];
  if (!d.init) {
    check_cuda(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev), "sm count");
    check_cuda(cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev), "cc major");
    check_cuda(cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev), "cc minor");
    check_cuda(cudaMalloc(&d.status, 256), "cudaMalloc(status)");
    check_cuda(cudaMemset(d.status, 0, 256), "cudaMemset(status)");
    d.init = true;
  }
  if (d.cc_major != 10 || d.cc_minor != 0)
    fail(OC_ERR_UNSUPPORTED, "liboc is built for sm_100a; device %d is sm_%d%d", dev, d.cc_major, d.cc_minor);
  return d;
}

Ctx make_ctx(void* stream) {
  int dev = 0;
  check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  DeviceState& d = device_state(dev);
  Ctx c{};
  c.stream = static_cast<cudaStream_t>(stream);
  c.status = d.status;
  c.sm_count = d.sm_count;
  c.device = dev;
  return c;
}

// Bump allocator over the device workspace (256-byte aligned pieces).
struct Carve {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

char* workspace(const Ctx& c, size_t bytes) {
  DeviceState& d = g_dev[c.device];
  if (d.ws_bytes < bytes) {
    if (d.ws) {
      check_cuda(cudaDeviceSynchronize(), "cudaDeviceSynchronize (workspace grow)");
      check_cuda(cudaFree(d.ws), "cudaFree(workspace)");
      d.ws = nullptr;
      d.ws_bytes = 0;
    }
    const size_t want = bytes + (bytes >> 4);
    if (cudaMalloc(&d.ws, want) != cudaSuccess) {
      cudaGetLastError();
      d.ws = nullptr;
      fail(OC_ERR_OOM, "could not allocate a %zu-byte workspace", want);
    }
    d.ws_bytes = want;
  }
  return static_cast<char*>(d.ws);
}

int finish(const Ctx& c) {
  if (!g_sync_mode) return OC_OK;
  check_cuda(cudaStreamSynchronize(c.stream), "cudaStreamSynchronize");
  int st = 0;
  check_cuda(cudaMemcpy(&st, c.status, sizeof(int), cudaMemcpyDeviceToHost), "read status");
  if (st != 0) {
    check_cuda(cudaMemset(c.status, 0, sizeof(int)), "reset status");
    snprintf(g_last_error, sizeof(g_last_error), "device reported %s", oc_status_string(st));
  }
  return st;
}

template <class F>
int guarded(F&& f) {
  try {
    g_last_error[0] = '\0';
    std::lock_guard<std::mutex> lock(g_mu);
    return f();
  } catch (const Failure& e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", e.msg);
    return e.status;
  } catch (const std::bad_alloc&) {
    snprintf(g_last_error, sizeof(g_last_error), "host allocation failed");
    return OC_ERR_OOM;
  }
}

}  // namespace

void fail(int status, const char* fmt, ...) {
  Failure f{};
  f.status = status;
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(f.msg, sizeof(f.msg), fmt, ap);
  va_end(ap);
  throw f;
}

void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

std::mutex& library_mutex() { return g_mu; }

void check_cuda(cudaError_t e, const char* what) {
  if (e != cudaSuccess) fail(OC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

void check_launch(const char* kernel) {
  count_launch();
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) fail(OC_ERR_CUDA, "launch of %s failed: %s", kernel, cudaGetErrorString(e));
}

SideStream& side_stream(int device) {
  static SideStream ss[64] = {};
  SideStream& s = ss[device & 63];
  if (s.stream == nullptr) {
    // Highest priority: when SMs free up, the factorisation's kernels are
    // placed before the next piece of the cross product.
    int least = 0, greatest = 0;
    check_cuda(cudaDeviceGetStreamPriorityRange(&least, &greatest), "cudaDeviceGetStreamPriorityRange");
    check_cuda(cudaStreamCreateWithPriority(&s.stream, cudaStreamNonBlocking, greatest), "cudaStreamCreate(side)");
    check_cuda(cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming), "cudaEventCreate(fork)");
    check_cuda(cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming), "cudaEventCreate(join)");
  }
  return s;
}

CUtensorMap make_tmap_2d(const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t rows, uint64_t cols,
                         uint64_t ld, uint32_t box_rows, uint32_t box_cols, Swz swz) {
  if (!aligned16(base)) fail(OC_ERR_INVALID_ARG, "TMA base address must be 16-byte aligned");
  if ((ld * elem_bytes) % 16) fail(OC_ERR_INVALID_ARG, "TMA row pitch must be a multiple of 16 bytes");
  CUtensorMap m;
  std::memset(&m, 0, sizeof(m));
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode_fn()(&m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 swz == Swz::B128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) fail(OC_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return m;
}

}  // namespace oc

namespace oc {
namespace {

void check_gptq_args(const float* W, int64_t m, int64_t n, int wbits, int groupsize, float damp, int act_order,
                     const uint32_t* codes, const float* scales, const float* zeros) {
  if (!W || !codes || !scales || !zeros) fail(OC_ERR_INVALID_ARG, "W, codes, scales, zeros must be non-null");
  if (n < 64 || n % 64) fail(OC_ERR_INVALID_ARG, "n must be a positive multiple of 64");
  if (n > 49152) fail(OC_ERR_INVALID_ARG, "n above 49152 is not supported");
  if (m < 1) fail(OC_ERR_INVALID_ARG, "m must be >= 1");
  if (wbits < 2 || wbits > 4) fail(OC_ERR_INVALID_ARG, "wbits must be 2, 3 or 4");
  if (act_order != 0 && act_order != 1) fail(OC_ERR_INVALID_ARG, "act_order must be 0 or 1");
  if (!(damp >= 0.f) || damp > 3.4e38f) fail(OC_ERR_INVALID_ARG, "damp must be finite and >= 0");
  const int64_t G = (groupsize == -1) ? n : groupsize;
  if (G < 4 || n % G) fail(OC_ERR_INVALID_ARG, "groupsize must divide n (or be -1)");
  const bool pow2_small = G <= 128 && (G & (G - 1)) == 0;
  if (!(G == n || pow2_small || G % 128 == 0))
    fail(OC_ERR_INVALID_ARG, "groupsize must be a power of two <= 128, a multiple of 128, or -1");
  if (!aligned16(codes) || !aligned16(W)) fail(OC_ERR_INVALID_ARG, "W and codes must be 16-byte aligned");
}

// GPTQ after the factor: blocked sweep over the permuted working copy Wp with
// tensor-core trailing updates, then packing (and the processing order out).
// Lazy updates on two levels: the errors of each 128-column block update the
// rest of its 512-column superblock at once (k = 128); at the end of a
// superblock, its 512 columns of errors update every later column in one
// product (k = 512), so the wide updates pass over W a quarter as often.
// Errh, Errl: m x kSuperBlock each.
void gptq_sweep_and_pack(const Ctx& c, float* Wp, int64_t m, int64_t n, const float* U, const float* UTh,
                         const float* UTl, int G, int wbits, bool act_order, int32_t* perm, float* scales,
                         float* zeros, unsigned char* codes8, float* Errh, float* Errl, uint32_t* codes,
                         int32_t* perm_out) {
  constexpr int64_t SBW = kSuperBlock;
  for (int64_t s1 = 0, s2 = 0; s1 < n; s1 = s2) {
    s2 = std::min(n, s1 + SBW);
    // A grid taken at a group's first column reads every column of the group,
    // and only the columns up to the superblock's end have seen all earlier
    // blocks' errors.  A group wider than a block that does not tile the
    // superblock (384, 640, 768 ...) therefore starts a superblock of its own.
    if (!act_order && G > 128 && SBW % G != 0) s2 = std::min(s2, (s1 / G + 1) * G);
    for (int64_t j1 = s1; j1 < s2; j1 += 128) {
      const int64_t bw = std::min<int64_t>(128, s2 - j1);
      const int64_t j2 = j1 + bw;
      float* eh = Errh + (j1 - s1);
      float* el = Errl + (j1 - s1);
      {
        // the sweep writes the block's errors already split for 3xTF32
        PhaseScope ps(c, kPhGptqSweep);
        launch_sweep_block(c, Wp, m, n, U, j1, G, wbits, act_order, perm, scales, zeros, codes8, eh, el, SBW);
      }
      if (j2 < s2) {
        // W[:, j2:s2] -= Err U[j1:j2, j2:s2] on the tensor cores (3xTF32); B
        // stored = U^T[j2:s2, j1:j2] (rows j2.., columns j1..j2 of the transpose)
        PhaseScope ps(c, kPhGptqTrailing);
        gemm_tf32x3(c, m, s2 - j2, bw, -1.f, eh, el, SBW, UTh + j2 * n + j1, UTl + j2 * n + j1, n, true, Wp + j2,
                    n, kANone);
      }
    }
    if (s2 < n) {
      // W[:, s2:] -= ErrS U[s1:s2, s2:] (k = s2 - s1)
      PhaseScope ps(c, kPhGptqTrailing);
      gemm_tf32x3(c, m, n - s2, s2 - s1, -1.f, Errh, Errl, SBW, UTh + s2 * n + s1, UTl + s2 * n + s1, n, true,
                  Wp + s2, n, kANone);
    }
  }
  {
    PhaseScope ps(c, kPhGptqPack);
    launch_pack(c, codes8, m, n, wbits, perm, codes);
  }
  if (perm_out)
    check_cuda(cudaMemcpyAsync(perm_out, perm, static_cast<size_t>(n) * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                               c.stream),
               "copy perm");
}

// Hessian + QEP + GPTQ of `count` layers that read the same inputs X, Xhat
// (q/k/v of one attention block, gate/up of one MLP): H, d and the inverse
// factor U depend only on the inputs and are made once; W d, the QEP apply
// and GPTQ run per layer.  W[l], W_out[l], codes[l], scales[l], zeros[l] are
// the l-th layer's device buffers (m[l] rows each).
int quantize_group(int count, const float* const* W, const int64_t* m, int64_t n, const void* X, const void* Xhat,
                   int64_t n_tok, float alpha, float damp, int wbits, int groupsize, int act_order, float* H,
                   float* const* W_out, uint32_t* const* codes, float* const* scales, float* const* zeros,
                   int32_t* perm_out, void* stream, const float* D_in = nullptr) {
  // D_in non-null: H (read only) and D_in = d are the layer's global terms,
  // already summed over all tokens (e.g. over the ranks of a token-sharded
  // layer); X, Xhat and n_tok are then not used.
  const bool terms_given = D_in != nullptr;
  if (count < 1 || count > kMaxGroup) fail(OC_ERR_INVALID_ARG, "count must be 1..%d", kMaxGroup);
  if (!W || !m || !W_out || !codes || !scales || !zeros) fail(OC_ERR_INVALID_ARG, "layer arrays must be non-null");
  int64_t m_max = 0;
  for (int l = 0; l < count; ++l) {
    check_gptq_args(W[l], m[l], n, wbits, groupsize, damp, act_order, codes[l], scales[l], zeros[l]);
    if (!W_out[l]) fail(OC_ERR_INVALID_ARG, "W_out[%d] must be non-null", l);
    if (!aligned16(W_out[l])) fail(OC_ERR_INVALID_ARG, "W_out[%d] must be 16-byte aligned", l);
    for (int k = 0; k < count; ++k)
      if (W_out[l] == W[k]) fail(OC_ERR_INVALID_ARG, "W_out[%d] must not alias an input weight", l);
    m_max = std::max(m_max, m[l]);
  }
  if (!H) fail(OC_ERR_INVALID_ARG, "H must be non-null");
  if (!terms_given) {
    if (!X || !Xhat) fail(OC_ERR_INVALID_ARG, "X, Xhat must be non-null");
    if (n_tok < 1 || n_tok > (int64_t(1) << 31) - 64) fail(OC_ERR_INVALID_ARG, "n_tok out of range");
    if (!aligned16(X) || !aligned16(Xhat)) fail(OC_ERR_INVALID_ARG, "X, Xhat must be 16-byte aligned");
  }
  if (!(alpha == alpha) || alpha > 3.4e38f || alpha < -3.4e38f) fail(OC_ERR_INVALID_ARG, "alpha must be finite");
  if (!aligned16(H)) fail(OC_ERR_INVALID_ARG, "H must be 16-byte aligned");
  const int64_t G = (groupsize == -1) ? n : groupsize;
  Ctx c = make_ctx(stream);
  const size_t nn = static_cast<size_t>(n) * n, mn = static_cast<size_t>(m_max) * n;
  Carve sizing{nullptr};
  sizing.take<float>(nn);                 // d -> U
  sizing.take<float>(nn);                 // d^T hi -> U hi
  sizing.take<float>(nn + 4096);          // d^T lo -> U lo
  sizing.take<float>(nn);                 // factor input -> U -> U^T hi
  sizing.take<float>(nn);                 // inverse factor -> U^T lo
  sizing.take<float>(nn + 4096);          // factor recursion scratch
  sizing.take<float>(mn);                 // hi halves (W, G, T)
  sizing.take<float>(mn);                 // lo halves
  sizing.take<float>(mn * count);         // G -> T, one per layer
  sizing.take<float>(mn);                 // permuted working copy of W
  sizing.take<unsigned char>(mn);         // codes, processing order
  sizing.take<float>(2 * static_cast<size_t>(m_max) * kSuperBlock);  // superblock errors, hi and lo halves
  sizing.take<int32_t>(2 * static_cast<size_t>(n));          // order | inverse
  sizing.take<unsigned char>(n);          // dead-column mask
  sizing.take<float>(factor_split_floats(n));
  sizing.take<DiagStats>(2);              // GPTQ's and QEP's dampening
  sizing.take<int>(1);                    // W's tf32 lo-half flag
  const size_t cross_bytes = terms_given ? 0 : cross_scratch_bytes(n_tok, n);
  sizing.take<unsigned char>(cross_bytes);  // the cross product's operands
  Carve cv{workspace(c, sizing.off + 256)};
  float* D = cv.take<float>(nn);
  float* Xi = cv.take<float>(nn);
  float* scratch = cv.take<float>(nn + 4096);
  float* UTh = cv.take<float>(nn);
  float* UTl = cv.take<float>(nn);
  float* Fs = cv.take<float>(nn + 4096);
  float* Ph = cv.take<float>(mn);
  float* Pl = cv.take<float>(mn);
  float* Gs = cv.take<float>(mn * count);
  float* Wp = cv.take<float>(mn);
  unsigned char* codes8 = cv.take<unsigned char>(mn);
  float* Errh = cv.take<float>(2 * static_cast<size_t>(m_max) * kSuperBlock);
  float* Errl = Errh + static_cast<size_t>(m_max) * kSuperBlock;
  int32_t* perm = cv.take<int32_t>(2 * static_cast<size_t>(n));
  unsigned char* dead = cv.take<unsigned char>(n);
  float* fsplit = cv.take<float>(factor_split_floats(n));
  DiagStats* stats = cv.take<DiagStats>(2);
  DiagStats* stats_q = stats + 1;
  int* lo_flag = cv.take<int>(1);
  unsigned char* cross_scratch = cv.take<unsigned char>(cross_bytes);
  auto Gl = [&](int l) { return Gs + static_cast<size_t>(l) * mn; };
  const size_t nn_bytes = nn * sizeof(float);

  if (!terms_given) {
    {
      PhaseScope ps(c, kPhHessianFix);
      check_cuda(cudaMemsetAsync(H, 0, nn_bytes, c.stream), "memset H");
    }
    {
      PhaseScope ps(c, kPhHessian);
      launch_atb16(c, Xhat, Xhat, n_tok, n, n, 2.0f, H, n, true);
    }
    {
      PhaseScope ps(c, kPhHessianFix);
      launch_mirror_upper(c, H, n);
    }
  }
  // GPTQ's preparation: dead-column mask and dampening constant (device only;
  // a non-finite diagonal is recorded in the status word and the call runs
  // to its end on the bad values).
  launch_diag_stats(c, H, n, damp, 1.0f, true, stats, dead);
  // GPTQ's inverse factor needs only H: it runs on a side stream, on a few
  // SMs, while the cross product X^T Xhat occupies the rest; it factors into
  // UTh (input reversed and dampened, output U) with UTl, Fs and fsplit as
  // its scratch.
  SideStream& ss = side_stream(c.device);
  Ctx cs = c;
  cs.stream = ss.stream;
  check_cuda(cudaEventRecord(ss.fork, c.stream), "cudaEventRecord(fork)");
  check_cuda(cudaStreamWaitEvent(cs.stream, ss.fork, 0), "cudaStreamWaitEvent(fork)");
  {
    PhaseScope ps(cs, kPhFactor);
    if (act_order) launch_act_order_perm(cs, H, n, perm);
    else launch_identity_perm(cs, n, perm);
    launch_build_reversed(cs, H, n, perm, stats, 1.0f, true, UTh);
    factor_inverse_upper(cs, UTh, UTl, Fs, UTh, n, true, fsplit);
  }
  check_cuda(cudaEventRecord(ss.join, cs.stream), "cudaEventRecord(join)");
  if (terms_given) {
    check_cuda(cudaMemcpyAsync(D, D_in, nn_bytes, cudaMemcpyDeviceToDevice, c.stream), "copy d");
  } else {
    // d = (X - Xhat)^T Xhat in token ranges: between two launches the
    // high-priority factorisation can take the freed SMs for its wide
    // tensor-core products
    PhaseScope ps(c, kPhQepCross);
    const int parts = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kCrossParts, n_tok / kCrossPartMinTokens)));
    launch_cross_product(c, X, Xhat, n_tok, n, H, D, cross_scratch, parts, c.sm_count - kSideSMs);
  }
  {
    // G = W d for every layer while the split copies of d^T are live
    PhaseScope ps(c, kPhQepWDelta);
    split_tf32(c, D, n, n, n, Xi, scratch, n, true);
    for (int l = 0; l < count; ++l) {
      // bf16-valued weights are exact in tf32: W_lo = 0 skips a third of the MMAs
      split_tf32(c, W[l], m[l], n, n, Ph, Pl, n, false, lo_flag);
      gemm_tf32x3(c, m[l], n, n, 1.f, Ph, Pl, n, Xi, scratch, n, false, Gl(l), n, kANone, lo_flag);
    }
  }
  check_cuda(cudaStreamWaitEvent(c.stream, ss.join, 0), "cudaStreamWaitEvent(join)");
  {
    // QEP's factor Uq into D: GPTQ's when no column is dead (its dampened
    // Hessian then equals QEP's 2A), else QEP's own in the same processing
    // order (the two dampening constants differ): decided on the device.
    PhaseScope ps(c, kPhFactor);
    launch_diag_stats(c, H, n, damp, 1.0f, false, stats_q, nullptr);
    qep_factor_select(c, H, n, perm, stats, stats_q, UTh, D, Xi, scratch, fsplit);
  }
  {
    PhaseScope ps(c, kPhQepApply);
    split_tf32(c, D, n, n, n, Xi, scratch, n);            // Uq hi, lo
    split_tf32(c, D, n, n, n, UTl, Fs, n, true);          // Uq^T hi, lo
    launch_invert_perm(c, perm, n);
  }
  for (int l = 0; l < count; ++l) {
    // QEP applied in processing order: W'P = WP + 2 alpha ((G P) Uq^T) Uq.
    // QEP makes no dead-column fix: a dead column's correction is zero (its
    // column of d is), so W' keeps W there; GPTQ zeroes it below.
    PhaseScope ps(c, kPhQepApply);
    if (act_order) {
      launch_permute_w(c, Gl(l), m[l], n, perm, nullptr, Wp);        // G P
      split_tf32(c, Wp, m[l], n, n, Ph, Pl, n);
    } else {
      split_tf32(c, Gl(l), m[l], n, n, Ph, Pl, n);                   // P = I
    }
    gemm_tf32x3(c, m[l], n, n, 1.f, Ph, Pl, n, Xi, scratch, n, false, Gl(l), n, kBLower);  // T = (G P) Uq^T
    split_tf32(c, Gl(l), m[l], n, n, Ph, Pl, n);
    if (act_order) {
      launch_permute_w(c, W[l], m[l], n, perm, nullptr, Wp);         // W P
      gemm_tf32x3(c, m[l], n, n, 2.f * alpha, Ph, Pl, n, UTl, Fs, n, true, Wp, n, kBUpper);
      launch_permute_w(c, Wp, m[l], n, perm + n, nullptr, W_out[l]); // back to original order
    } else {
      check_cuda(cudaMemcpyAsync(W_out[l], W[l], static_cast<size_t>(m[l]) * n * sizeof(float),
                                 cudaMemcpyDeviceToDevice, c.stream),
                 "copy W");
      gemm_tf32x3(c, m[l], n, n, 2.f * alpha, Ph, Pl, n, UTl, Fs, n, true, W_out[l], n, kBUpper);
    }
  }
  {
    // GPTQ with its own factor U (in UTh): U^T split for the trailing updates
    PhaseScope ps(c, kPhGptqPrep);
    split_tf32(c, UTh, n, n, n, Xi, scratch, n, true);
  }
  for (int l = 0; l < count; ++l) {
    {
      // GPTQ's working copy: W' in processing order, dead columns zeroed
      PhaseScope ps(c, kPhGptqPrep);
      launch_permute_w(c, W_out[l], m[l], n, perm, dead, Wp);
    }
    if (act_order) {
      PhaseScope ps(c, kPhGptqPrep);
      launch_static_grid(c, W_out[l], m[l], n, static_cast<int>(G), wbits, dead, scales[l], zeros[l]);
    }
    gptq_sweep_and_pack(c, Wp, m[l], n, UTh, Xi, scratch, static_cast<int>(G), wbits, act_order != 0, perm,
                        scales[l], zeros[l], codes8, Errh, Errl, codes[l], l == 0 ? perm_out : nullptr);
  }
  return finish(c);
}

}  // namespace
}  // namespace oc

using namespace oc;

extern "C" {

const char* oc_status_string(int status) {
  switch (status) {
    case OC_OK: return "OC_OK";
    case OC_ERR_INVALID_ARG: return "OC_ERR_INVALID_ARG";
    case OC_ERR_UNSUPPORTED: return "OC_ERR_UNSUPPORTED";
    case OC_ERR_NOT_SPD: return "OC_ERR_NOT_SPD";
    case OC_ERR_NONFINITE: return "OC_ERR_NONFINITE";
    case OC_ERR_TIMEOUT: return "OC_ERR_TIMEOUT";
    case OC_ERR_CUDA: return "OC_ERR_CUDA";
    case OC_ERR_OOM: return "OC_ERR_OOM";
    default: return "OC_ERR_UNKNOWN";
  }
}

const char* oc_last_error(void) { return g_last_error; }

int oc_version(void) { return 100; }

void oc_set_sync(int sync) { g_sync_mode = sync ? 1 : 0; }

int oc_stream_status(void* stream) {
  return guarded([&]() -> int {
    Ctx c = make_ctx(stream);
    check_cuda(cudaStreamSynchronize(c.stream), "cudaStreamSynchronize");
    int st = 0;
    check_cuda(cudaMemcpy(&st, c.status, sizeof(int), cudaMemcpyDeviceToHost), "read status");
    if (st != 0) check_cuda(cudaMemset(c.status, 0, sizeof(int)), "reset status");
    return st;
  });
}

int oc_profile_enable(int on) {
  return guarded([&]() -> int {
    profile_enable(on != 0);
    return OC_OK;
  });
}

int oc_profile_read(double* ms, int64_t* launches, int max_phases) {
  return guarded([&]() -> int { return profile_read(ms, launches, max_phases); });
}

const char* oc_profile_phase_name(int phase) { return phase_name(phase); }

int64_t oc_launch_count(void) { return launch_count(); }

int oc_test_inject_stall(void) {
  return guarded([&]() -> int {
    request_test_stall();
    return OC_OK;
  });
}

int oc_test_unit_plan(int64_t n_tok, int64_t n_tiles, int64_t clusters, int64_t* out) {
  return guarded([&]() -> int {
    if (n_tok <= 0 || n_tiles <= 0 || clusters <= 0 || out == nullptr)
      fail(OC_ERR_INVALID_ARG, "unit plan: n_tok, n_tiles and clusters must be positive, out non-null");
    const UnitPlan u = plan_units(n_tok, n_tiles, clusters);
    out[0] = u.kc_stages;
    out[1] = u.n_kc;
    out[2] = u.split_k;
    out[3] = u.full_units;
    out[4] = u.units;
    return OC_OK;
  });
}

int oc_workspace_release(void) {
  return guarded([&]() -> int {
    int dev = 0;
    check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev >= 0 && dev < 64 && g_dev[dev].ws) {
      check_cuda(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
      check_cuda(cudaFree(g_dev[dev].ws), "cudaFree(workspace)");
      g_dev[dev].ws = nullptr;
      g_dev[dev].ws_bytes = 0;
    }
    return OC_OK;
  });
}

int oc_hessian_accumulate(const void* X, int64_t n_tok, int64_t n, float* H, void* stream) {
  return guarded([&]() -> int {
    if (!H) fail(OC_ERR_INVALID_ARG, "H must be non-null");
    if (n < 64 || n % 64) fail(OC_ERR_INVALID_ARG, "n must be a positive multiple of 64 (got %lld)", (long long)n);
    if (n_tok < 0) fail(OC_ERR_INVALID_ARG, "n_tok must be >= 0");
    if (n_tok == 0) return OC_OK;  // nothing to add (X may be NULL)
    if (!X) fail(OC_ERR_INVALID_ARG, "X must be non-null");
    if (n_tok > (int64_t(1) << 31) - 64) fail(OC_ERR_INVALID_ARG, "n_tok too large for one call; split it");
    if (!aligned16(X) || !aligned16(H)) fail(OC_ERR_INVALID_ARG, "X and H must be 16-byte aligned");
    Ctx c = make_ctx(stream);
    {
      PhaseScope ps(c, kPhHessian);
      launch_atb16(c, X, X, n_tok, n, n, 2.0f, H, n, true);
    }
    {
      PhaseScope ps(c, kPhHessianFix);
      launch_mirror_upper(c, H, n);
    }
    return finish(c);
  });
}

int oc_qep_correct(const float* W, int64_t m, int64_t n, const void* X, const void* Xhat, int64_t n_tok,
                   float alpha, float damp, const float* H_opt, float* W_out, void* stream) {
  return guarded([&]() -> int {
    if (!W || !X || !Xhat || !W_out) fail(OC_ERR_INVALID_ARG, "W, X, Xhat, W_out must be non-null");
    if (n < 64 || n % 64) fail(OC_ERR_INVALID_ARG, "n must be a positive multiple of 64");
    if (n > 49152) fail(OC_ERR_INVALID_ARG, "n above 49152 is not supported");
    if (m < 1) fail(OC_ERR_INVALID_ARG, "m must be >= 1");
    if (n_tok < 1 || n_tok > (int64_t(1) << 31) - 64) fail(OC_ERR_INVALID_ARG, "n_tok out of range");
    if (!(alpha == alpha) || alpha > 3.4e38f || alpha < -3.4e38f) fail(OC_ERR_INVALID_ARG, "alpha must be finite");
    if (!(damp >= 0.f) || damp > 3.4e38f) fail(OC_ERR_INVALID_ARG, "damp must be finite and >= 0");
    if (!aligned16(X) || !aligned16(Xhat) || (H_opt && !aligned16(H_opt)))
      fail(OC_ERR_INVALID_ARG, "X, Xhat, H_opt must be 16-byte aligned");
    Ctx c = make_ctx(stream);
    const size_t nn = static_cast<size_t>(n) * n, mn = static_cast<size_t>(m) * n;
    if (alpha == 0.f) {
      if (W_out != W) launch_copy_f32(c, W, W_out, static_cast<int64_t>(mn));
      return finish(c);
    }
    Carve sizing{nullptr};
    sizing.take<float>(nn);                       // d -> M -> U
    if (!H_opt) sizing.take<float>(nn);           // Hs
    sizing.take<float>(nn);                       // d_hi -> inverse factor -> U_hi
    sizing.take<float>(nn + 4096);                // d_lo -> recursion scratch -> U_lo
    sizing.take<float>(nn);                       // (U^T)_hi
    sizing.take<float>(nn);                       // (U^T)_lo
    sizing.take<float>(mn);                       // W_hi -> G_hi -> T_hi
    sizing.take<float>(mn);                       // W_lo -> G_lo -> T_lo
    sizing.take<float>(mn);                       // G -> T
    sizing.take<float>(nn + 4096);                // recursion scratch of the side-stream factorisation
    sizing.take<float>(factor_split_floats(n));   // split copies inside the factorisation
    sizing.take<DiagStats>(1);
    sizing.take<int>(1);                          // W's tf32 lo-half flag
    const size_t cross_bytes = cross_scratch_bytes(n_tok, n);
    sizing.take<unsigned char>(cross_bytes);      // the cross product's operands
    Carve cv{workspace(c, sizing.off + 256)};
    float* D = cv.take<float>(nn);
    float* Hs = H_opt ? nullptr : cv.take<float>(nn);
    float* Xi = cv.take<float>(nn);
    float* scratch = cv.take<float>(nn + 4096);
    float* UTh = cv.take<float>(nn);
    float* UTl = cv.take<float>(nn);
    float* Ph = cv.take<float>(mn);
    float* Pl = cv.take<float>(mn);
    float* G = cv.take<float>(mn);
    float* Fs = cv.take<float>(nn + 4096);
    float* fsplit = cv.take<float>(factor_split_floats(n));
    DiagStats* stats = cv.take<DiagStats>(1);
    int* lo_flag = cv.take<int>(1);
    unsigned char* cross_scratch = cv.take<unsigned char>(cross_bytes);

    const float* Hp = H_opt;
    if (!H_opt) {
      PhaseScope ps(c, kPhQepSyrk);
      check_cuda(cudaMemsetAsync(Hs, 0, nn * sizeof(float), c.stream), "memset Hs");
      launch_atb16(c, Xhat, Xhat, n_tok, n, n, 2.0f, Hs, n, true);
      launch_mirror_upper(c, Hs, n);
      Hp = Hs;
    }
    // 2A = Hp + damp mean(diag Hp) I = R R^T;  U = R^-1 upper, A^-1 = 2 U^T U.
    // The factorisation needs only H: it runs on the high-priority side stream
    // (into UTh, with UTl and Fs as scratch) beside the cross product, which
    // runs in token ranges so that the factorisation's wide products can take
    // SMs between its launches.
    SideStream& ss = side_stream(c.device);
    Ctx cs = c;
    cs.stream = ss.stream;
    check_cuda(cudaEventRecord(ss.fork, c.stream), "cudaEventRecord(fork)");
    check_cuda(cudaStreamWaitEvent(cs.stream, ss.fork, 0), "cudaStreamWaitEvent(fork)");
    {
      PhaseScope ps(cs, kPhFactor);
      launch_diag_stats(cs, Hp, n, damp, 1.0f, false, stats, nullptr);
      launch_build_reversed(cs, Hp, n, nullptr, stats, 1.0f, false, UTh);
      factor_inverse_upper(cs, UTh, UTl, Fs, UTh, n, true, fsplit);
    }
    check_cuda(cudaEventRecord(ss.join, cs.stream), "cudaEventRecord(join)");
    {
      // d = (X - Xhat)^T Xhat, in token ranges beside the factorisation
      PhaseScope ps(c, kPhQepCross);
      const int parts = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kCrossParts, n_tok / kCrossPartMinTokens)));
      launch_cross_product(c, X, Xhat, n_tok, n, Hp, D, cross_scratch, parts, c.sm_count - kSideSMs);
    }
    {
      // G = W d on the tensor cores (3xTF32 from split operands)
      PhaseScope ps(c, kPhQepWDelta);
      split_tf32(c, D, n, n, n, Xi, scratch, n, true);  // d^T: B operands are stored [N x K]
      split_tf32(c, W, m, n, n, Ph, Pl, n, false, lo_flag);
      gemm_tf32x3(c, m, n, n, 1.f, Ph, Pl, n, Xi, scratch, n, false, G, n, kANone, lo_flag);
    }
    check_cuda(cudaStreamWaitEvent(c.stream, ss.join, 0), "cudaStreamWaitEvent(join)");
    {
      // W_out = W + alpha G A^-1 = W + 2 alpha (G U^T) U
      PhaseScope ps(c, kPhQepApply);
      check_cuda(cudaMemcpyAsync(D, UTh, nn * sizeof(float), cudaMemcpyDeviceToDevice, c.stream), "copy U");
      const float* U = D;
      float* Uh = Xi;
      float* Ul = scratch;
      split_tf32(c, U, n, n, n, Uh, Ul, n);
      split_tf32(c, U, n, n, n, UTh, UTl, n, true);
      split_tf32(c, G, m, n, n, Ph, Pl, n);
      float* T = G;
      // T = G U^T (B stored = U; op(B) = U^T is lower triangular)
      gemm_tf32x3(c, m, n, n, 1.f, Ph, Pl, n, Uh, Ul, n, false, T, n, kBLower);
      split_tf32(c, T, m, n, n, Ph, Pl, n);
      if (W_out != W) launch_copy_f32(c, W, W_out, static_cast<int64_t>(mn));
      // W_out += 2 alpha T U (B stored = U^T; op(B) = U is upper triangular)
      gemm_tf32x3(c, m, n, n, 2.f * alpha, Ph, Pl, n, UTh, UTl, n, true, W_out, n, kBUpper);
    }
    return finish(c);
  });
}

int oc_gptq_quantize(const float* W, int64_t m, int64_t n, const float* H, int wbits, int groupsize, float damp,
                     int act_order, uint32_t* codes, float* scales, float* zeros, int32_t* perm_out,
                     void* stream) {
  return guarded([&]() -> int {
    check_gptq_args(W, m, n, wbits, groupsize, damp, act_order, codes, scales, zeros);
    if (!H) fail(OC_ERR_INVALID_ARG, "H must be non-null");
    const int64_t G = (groupsize == -1) ? n : groupsize;
    Ctx c = make_ctx(stream);
    const size_t nn = static_cast<size_t>(n) * n, mn = static_cast<size_t>(m) * n;
    Carve sizing{nullptr};
    sizing.take<float>(nn);            // M -> U
    sizing.take<float>(nn);            // inverse factor -> U_hi
    sizing.take<float>(nn + 4096);     // recursion scratch -> U_lo
    sizing.take<float>(mn);            // Wp
    sizing.take<unsigned char>(mn);    // codes8
    sizing.take<float>(static_cast<size_t>(m) * kSuperBlock);  // superblock errors, hi
    sizing.take<float>(static_cast<size_t>(m) * kSuperBlock);  // and lo
    sizing.take<int32_t>(2 * static_cast<size_t>(n));  // perm | inverse
    sizing.take<unsigned char>(n);     // dead
    sizing.take<float>(factor_split_floats(n));  // split copies inside the factorisation
    sizing.take<DiagStats>(1);
    Carve cv{workspace(c, sizing.off + 256)};
    float* M = cv.take<float>(nn);
    float* Xi = cv.take<float>(nn);
    float* scratch = cv.take<float>(nn + 4096);
    float* Wp = cv.take<float>(mn);
    unsigned char* codes8 = cv.take<unsigned char>(mn);
    float* Errh = cv.take<float>(static_cast<size_t>(m) * kSuperBlock);
    float* Errl = cv.take<float>(static_cast<size_t>(m) * kSuperBlock);
    int32_t* perm = cv.take<int32_t>(2 * static_cast<size_t>(n));
    unsigned char* dead = cv.take<unsigned char>(n);
    float* fsplit = cv.take<float>(factor_split_floats(n));
    DiagStats* stats = cv.take<DiagStats>(1);

    {
      PhaseScope ps(c, kPhFactor);
      launch_diag_stats(c, H, n, damp, 1.0f, true, stats, dead);
      if (act_order) launch_act_order_perm(c, H, n, perm);
      else launch_identity_perm(c, n, perm);
      launch_build_reversed(c, H, n, perm, stats, 1.0f, true, M);
      factor_inverse_upper(c, M, Xi, scratch, M, n, true, fsplit);
    }
    const float* U = M;
    float* UTh = Xi;
    float* UTl = scratch;
    {
      PhaseScope ps(c, kPhGptqPrep);
      split_tf32(c, U, n, n, n, UTh, UTl, n, true);
      launch_permute_w(c, W, m, n, perm, dead, Wp);
      if (act_order) launch_static_grid(c, W, m, n, static_cast<int>(G), wbits, dead, scales, zeros);
    }
    gptq_sweep_and_pack(c, Wp, m, n, U, UTh, UTl, static_cast<int>(G), wbits, act_order != 0, perm, scales, zeros,
                        codes8, Errh, Errl, codes, perm_out);
    return finish(c);
  });
}

int oc_hadamard_rotate(const void* X, int64_t rows, int64_t n, int block, void* Y, int bf16, void* stream) {
  return guarded([&]() -> int {
    if (rows < 0 || n < 1) fail(OC_ERR_INVALID_ARG, "rows must be >= 0 and n >= 1");
    if (rows == 0) return OC_OK;
    if (!X || !Y) fail(OC_ERR_INVALID_ARG, "X and Y must be non-null");
    if (block < 2 || block > 4096 || (block & (block - 1))) fail(OC_ERR_INVALID_ARG, "block must be a power of two in 2..4096");
    if (n % block) fail(OC_ERR_INVALID_ARG, "block must divide n");
    if (bf16 != 0 && bf16 != 1) fail(OC_ERR_INVALID_ARG, "bf16 must be 0 or 1");
    if (!aligned16(X) || !aligned16(Y)) fail(OC_ERR_INVALID_ARG, "X and Y must be 16-byte aligned");
    int log2b = 0;
    while ((1 << log2b) < block) ++log2b;
    Ctx c = make_ctx(stream);
    {
      PhaseScope ps(c, kPhRotate);
      launch_hadamard(c, X, Y, rows, n, log2b, bf16 != 0);
    }
    return finish(c);
  });
}

int oc_lpcd_left_project(const float* B, const float* W2, int64_t m, int64_t d, const float* V, int64_t n,
                         float damp, float* W_out, void* stream) {
  return guarded([&]() -> int {
    if (!B || !W2 || !V || !W_out) fail(OC_ERR_INVALID_ARG, "B, W2, V, W_out must be non-null");
    if (d < 64 || d % 64) fail(OC_ERR_INVALID_ARG, "d must be a positive multiple of 64");
    if (d > 49152) fail(OC_ERR_INVALID_ARG, "d above 49152 is not supported");
    if (m < 4 || m % 4 || n < 4 || n % 4) fail(OC_ERR_INVALID_ARG, "m and n must be positive multiples of 4");
    if (m > (int64_t(1) << 30) || n > (int64_t(1) << 30)) fail(OC_ERR_INVALID_ARG, "m or n too large");
    if (!(damp >= 0.f) || damp > 3.4e38f) fail(OC_ERR_INVALID_ARG, "damp must be finite and >= 0");
    if (!aligned16(B) || !aligned16(W2) || !aligned16(V) || !aligned16(W_out))
      fail(OC_ERR_INVALID_ARG, "B, W2, V, W_out must be 16-byte aligned");
    Ctx c = make_ctx(stream);
    const size_t dd = static_cast<size_t>(d) * d, dm = static_cast<size_t>(d) * m, dn = static_cast<size_t>(d) * n;
    Carve sizing{nullptr};
    sizing.take<float>(dm);                       // B^T hi
    sizing.take<float>(dm);                       // B^T lo
    sizing.take<float>(dm);                       // W2^T hi
    sizing.take<float>(dm);                       // W2^T lo
    sizing.take<float>(dd);                       // B^T B -> (U^T) hi
    sizing.take<float>(dd);                       // B^T W2 -> (U^T) lo
    sizing.take<float>(dd);                       // P hi -> U hi
    sizing.take<float>(dd);                       // P lo -> U lo
    sizing.take<float>(dn);                       // V^T hi -> T^T hi -> S^T hi
    sizing.take<float>(dn);                       // V^T lo -> T^T lo -> S^T lo
    sizing.take<float>(dn);                       // T -> S
    sizing.take<float>(dd);                       // factor input -> U
    sizing.take<float>(dd);                       // inverse factor
    sizing.take<float>(dd + 4096);                // recursion scratch
    sizing.take<float>(factor_split_floats(d));   // split copies inside the factorisation
    sizing.take<DiagStats>(1);
    Carve cv{workspace(c, sizing.off + 256)};
    float* Bth = cv.take<float>(dm);
    float* Btl = cv.take<float>(dm);
    float* Wth = cv.take<float>(dm);
    float* Wtl = cv.take<float>(dm);
    float* Mm = cv.take<float>(dd);
    float* P = cv.take<float>(dd);
    float* Ph = cv.take<float>(dd);
    float* Pl = cv.take<float>(dd);
    float* Qh = cv.take<float>(dn);
    float* Ql = cv.take<float>(dn);
    float* T = cv.take<float>(dn);
    float* F = cv.take<float>(dd);
    float* Fx = cv.take<float>(dd);
    float* Fs = cv.take<float>(dd + 4096);
    float* fsplit = cv.take<float>(factor_split_floats(d));
    DiagStats* stats = cv.take<DiagStats>(1);
    PhaseScope ps(c, kPhLpcdLeft);
    // M = B^T B and P = B^T W2 (d x d, contraction over the m rows)
    split_tf32(c, B, m, d, d, Bth, Btl, m, true);
    split_tf32(c, W2, m, d, d, Wth, Wtl, m, true);
    gemm_tf32x3(c, d, d, m, 1.f, Bth, Btl, m, Bth, Btl, m, false, Mm, d, kANone);
    gemm_tf32x3(c, d, d, m, 1.f, Bth, Btl, m, Wth, Wtl, m, false, P, d, kANone);
    // (M + mu I)^-1 = U^T U, mu = damp mean(diag M)
    launch_diag_stats(c, Mm, d, damp, 1.0f, false, stats, nullptr);
    launch_build_reversed(c, Mm, d, nullptr, stats, 1.0f, false, F);
    factor_inverse_upper(c, F, Fx, Fs, F, d, true, fsplit);
    // T = P V
    split_tf32(c, P, d, d, d, Ph, Pl, d);
    split_tf32(c, V, d, n, n, Qh, Ql, d, true);
    gemm_tf32x3(c, d, n, d, 1.f, Ph, Pl, d, Qh, Ql, d, false, T, n, kANone);
    // S = U T (U upper), then W_out = U^T S (U^T lower)
    split_tf32(c, F, d, d, d, Ph, Pl, d);
    split_tf32(c, F, d, d, d, Mm, P, d, true);
    split_tf32(c, T, d, n, n, Qh, Ql, d, true);
    gemm_tf32x3(c, d, n, d, 1.f, Ph, Pl, d, Qh, Ql, d, false, T, n, kAUpper);
    split_tf32(c, T, d, n, n, Qh, Ql, d, true);
    gemm_tf32x3(c, d, n, d, 1.f, Mm, P, d, Qh, Ql, d, false, W_out, n, kALower);
    return finish(c);
  });
}

int oc_dequant_gemv(const uint32_t* codes, const float* scales, const float* zeros, int64_t m, int64_t n, int wbits,
                    int groupsize, const void* x, int64_t batch, float* y, void* stream) {
  return guarded([&]() -> int {
    if (!codes || !scales || !zeros || !x || !y) fail(OC_ERR_INVALID_ARG, "codes, scales, zeros, x, y must be non-null");
    if (m < 1 || n < 32 || n % 32) fail(OC_ERR_INVALID_ARG, "m must be >= 1 and n a positive multiple of 32");
    if (wbits < 2 || wbits > 4) fail(OC_ERR_INVALID_ARG, "wbits must be 2, 3 or 4");
    if (batch < 1 || batch > 8) fail(OC_ERR_INVALID_ARG, "batch must be 1..8");
    const int64_t G = (groupsize == -1) ? n : groupsize;
    if (G < 1 || n % G) fail(OC_ERR_INVALID_ARG, "groupsize must divide n (or be -1)");
    if (G < 32 ? (32 % G != 0) : (G % 32 != 0))
      fail(OC_ERR_INVALID_ARG, "groupsize must divide 32 or be a multiple of 32");
    if (!aligned16(codes) || !aligned16(x)) fail(OC_ERR_INVALID_ARG, "codes and x must be 16-byte aligned");
    Ctx c = make_ctx(stream);
    {
      PhaseScope ps(c, kPhGemv);
      launch_dequant_gemv(c, codes, scales, zeros, m, n, wbits, G, x, static_cast<int>(batch), y);
    }
    return finish(c);
  });
}

int oc_dequantize(const uint32_t* codes, const float* scales, const float* zeros, int64_t m, int64_t n, int wbits,
                  int groupsize, void* out, int out_bf16, void* stream) {
  return guarded([&]() -> int {
    if (!codes || !scales || !zeros || !out) fail(OC_ERR_INVALID_ARG, "codes, scales, zeros, out must be non-null");
    if (m < 1 || n < 1) fail(OC_ERR_INVALID_ARG, "m and n must be >= 1");
    if (wbits < 2 || wbits > 4) fail(OC_ERR_INVALID_ARG, "wbits must be 2, 3 or 4");
    if ((n * wbits) % 32) fail(OC_ERR_INVALID_ARG, "n * wbits must be a multiple of 32");
    const int64_t G = (groupsize == -1) ? n : groupsize;
    if (G < 1 || n % G) fail(OC_ERR_INVALID_ARG, "groupsize must divide n (or be -1)");
    if (out_bf16 != 0 && out_bf16 != 1) fail(OC_ERR_INVALID_ARG, "out_bf16 must be 0 or 1");
    Ctx c = make_ctx(stream);
    launch_dequant(c, codes, scales, zeros, m, n, wbits, G, out, out_bf16 != 0);
    return finish(c);
  });
}

int oc_quantize_layer(const float* W, int64_t m, int64_t n, const void* X, const void* Xhat, int64_t n_tok,
                      float alpha, float damp, int wbits, int groupsize, int act_order, float* H, float* W_out,
                      uint32_t* codes, float* scales, float* zeros, int32_t* perm_out, void* stream) {
  return guarded([&]() -> int {
    return quantize_group(1, &W, &m, n, X, Xhat, n_tok, alpha, damp, wbits, groupsize, act_order, H, &W_out, &codes,
                          &scales, &zeros, perm_out, stream);
  });
}

int oc_qep_terms(const void* X, const void* Xhat, int64_t n_tok, int64_t n, float* H_part, float* D_part,
                 void* stream) {
  return guarded([&]() -> int {
    if (!H_part || !D_part) fail(OC_ERR_INVALID_ARG, "H_part, D_part must be non-null");
    if (n < 64 || n % 64) fail(OC_ERR_INVALID_ARG, "n must be a positive multiple of 64");
    if (n_tok < 0 || n_tok > (int64_t(1) << 31) - 64) fail(OC_ERR_INVALID_ARG, "n_tok out of range");
    if (n_tok > 0 && (!X || !Xhat)) fail(OC_ERR_INVALID_ARG, "X, Xhat must be non-null");
    if ((n_tok > 0 && (!aligned16(X) || !aligned16(Xhat))) || !aligned16(H_part) || !aligned16(D_part))
      fail(OC_ERR_INVALID_ARG, "X, Xhat, H_part, D_part must be 16-byte aligned");
    Ctx c = make_ctx(stream);
    const size_t nn_bytes = static_cast<size_t>(n) * n * sizeof(float);
    {
      PhaseScope ps(c, kPhHessianFix);
      check_cuda(cudaMemsetAsync(H_part, 0, nn_bytes, c.stream), "memset H_part");
      if (n_tok == 0) check_cuda(cudaMemsetAsync(D_part, 0, nn_bytes, c.stream), "memset D_part");
    }
    if (n_tok == 0) return finish(c);
    unsigned char* cross_scratch = reinterpret_cast<unsigned char*>(workspace(c, cross_scratch_bytes(n_tok, n) + 256));
    {
      PhaseScope ps(c, kPhHessian);
      launch_atb16(c, Xhat, Xhat, n_tok, n, n, 2.0f, H_part, n, true);
    }
    {
      PhaseScope ps(c, kPhHessianFix);
      launch_mirror_upper(c, H_part, n);
    }
    {
      // D_part = (X - Xhat)^T Xhat
      PhaseScope ps(c, kPhQepCross);
      const int parts = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kCrossParts, n_tok / kCrossPartMinTokens)));
      launch_cross_product(c, X, Xhat, n_tok, n, H_part, D_part, cross_scratch, parts, 0);
    }
    return finish(c);
  });
}

int oc_quantize_from_terms(const float* W, int64_t m, int64_t n, const float* H, const float* D, float alpha,
                           float damp, int wbits, int groupsize, int act_order, float* W_out, uint32_t* codes,
                           float* scales, float* zeros, int32_t* perm_out, void* stream) {
  return guarded([&]() -> int {
    if (!D) fail(OC_ERR_INVALID_ARG, "D must be non-null");
    if (!aligned16(D)) fail(OC_ERR_INVALID_ARG, "D must be 16-byte aligned");
    return quantize_group(1, &W, &m, n, nullptr, nullptr, 0, alpha, damp, wbits, groupsize, act_order,
                          const_cast<float*>(H), &W_out, &codes, &scales, &zeros, perm_out, stream, D);
  });
}

int oc_quantize_layer_group(int count, const float* const* W, const int64_t* m, int64_t n, const void* X,
                            const void* Xhat, int64_t n_tok, float alpha, float damp, int wbits, int groupsize,
                            int act_order, float* H, float* const* W_out, uint32_t* const* codes,
                            float* const* scales, float* const* zeros, int32_t* perm_out, void* stream) {
  return guarded([&]() -> int {
    return quantize_group(count, W, m, n, X, Xhat, n_tok, alpha, damp, wbits, groupsize, act_order, H, W_out, codes,
                          scales, zeros, perm_out, stream);
  });
}

}  // extern "C"

// Allocation-free variant of the GPTQ entry point.
//
// Some callers cannot let a library allocate device memory on its own: a
// process that hands the whole GPU to its own caching allocator at start-up,
// a service that runs under a fixed, pre-reserved memory budget, or any host
// code where a cudaMalloc (and the device-wide synchronisation a cudaFree
// brings) at an arbitrary point is not acceptable.  oc_gptq_quantize_noalloc
// serves them: it takes the same steps as oc_gptq_quantize (its trailing
// updates run on the CUDA cores in fp32, which needs no split copies of the
// factor), but takes all of its scratch memory from one fixed array that is part of the library image
// (g_noalloc_scratch below), so it never calls cudaMalloc, cudaFree or any
// other allocating routine.  The price is a size limit (kNoallocBytes of
// scratch, enough for d_in = 512 with up to 1024 output rows) and the memory
// that every GPU which loads the library keeps for the array until exit.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include <cuda.h>

#include "oc_internal.cuh"

namespace oc {
namespace {

constexpr size_t kNoallocBytes = size_t(6) << 20;  // 6 MiB

// The scratch shared by every call on a device.  It keeps whatever the last
// call left in it; each call clears what has to start at zero.  In host code
// this name is only a stand-in for the array, never a device address: the
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

// Device address of g_noalloc_scratch per device, with the id of the context
// it was looked up in: a process that destroys a device's primary context
// (cudaDeviceReset) and creates a new one gets the array at a new address.
struct ScratchAddr {
  unsigned long long ctx_id = 0;
  void* addr = nullptr;
};
ScratchAddr g_scratch_addr[64];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <class Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q{};
  check_cuda(cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q), "cudaGetDriverEntryPoint");
  if (q != cudaDriverEntryPointSuccess || p == nullptr) fail(OC_ERR_UNSUPPORTED, "driver does not provide %s", name);
  return reinterpret_cast<Fn>(p);
}

// Id of the context current on this thread (the device's primary context,
// made current by the runtime's cudaGetDevice/cudaFree-free calls before).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) fail(OC_ERR_CUDA, "no current CUDA context");
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) fail(OC_ERR_CUDA, "cuCtxGetId failed");
  return id;
}

// Device address of g_noalloc_scratch on `dev` (which must be current),
// looked up on the first call there and again only if the context changed.
unsigned char* scratch_address(int dev) {
  // the runtime makes the device's primary context current (no allocation)
  check_cuda(cudaSetDevice(dev), "cudaSetDevice");
  const unsigned long long id = current_context_id();
  ScratchAddr& s = g_scratch_addr[dev];
  if (s.addr == nullptr || s.ctx_id != id) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      fail(OC_ERR_CUDA, "cudaGetSymbolAddress(g_noalloc_scratch) failed: %s", cudaGetErrorString(e));
    s.addr = p;
    s.ctx_id = id;
  }
  return static_cast<unsigned char*>(s.addr);
}

// Same 256-byte-aligned carving as the allocating entry point, over a fixed base.
struct Carve {
  unsigned char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

int run(const float* W, int64_t m, int64_t n, const float* H, int wbits, int groupsize, float damp,
        int act_order, uint32_t* codes, float* scales, float* zeros, int32_t* perm_out, void* stream) {
  if (!W || !H || !codes || !scales || !zeros) fail(OC_ERR_INVALID_ARG, "W, H, codes, scales, zeros must be non-null");
  if (n < 64 || n % 64) fail(OC_ERR_INVALID_ARG, "n must be a positive multiple of 64");
  if (m < 1) fail(OC_ERR_INVALID_ARG, "m must be >= 1");
  if (wbits < 2 || wbits > 4) fail(OC_ERR_INVALID_ARG, "wbits must be 2, 3 or 4");
  if (act_order != 0 && act_order != 1) fail(OC_ERR_INVALID_ARG, "act_order must be 0 or 1");
  if (!(damp >= 0.f) || damp > 3.4e38f) fail(OC_ERR_INVALID_ARG, "damp must be finite and >= 0");
  const int64_t G = (groupsize == -1) ? n : groupsize;
  if (G < 4 || n % G) fail(OC_ERR_INVALID_ARG, "groupsize must divide n (or be -1)");
  const bool pow2_small = G <= 128 && (G & (G - 1)) == 0;
  if (!(G == n || pow2_small || G % 128 == 0))
    fail(OC_ERR_INVALID_ARG, "groupsize must be a power of two <= 128, a multiple of 128, or -1");
  if ((reinterpret_cast<uintptr_t>(codes) | reinterpret_cast<uintptr_t>(W)) & 15u)
    fail(OC_ERR_INVALID_ARG, "W and codes must be 16-byte aligned");

  const size_t nn = static_cast<size_t>(n) * n, mn = static_cast<size_t>(m) * n;
  Carve sizing{nullptr};
  sizing.take<int>(1);               // status word
  sizing.take<float>(nn);            // M -> U
  sizing.take<float>(nn);            // inverse factor of the reversed matrix
  sizing.take<float>(nn / 2 + 4096); // recursion scratch
  sizing.take<float>(mn);            // permuted working copy of W
  sizing.take<unsigned char>(mn);    // codes, processing order
  sizing.take<float>(static_cast<size_t>(m) * 128);  // block errors
  sizing.take<int32_t>(2 * static_cast<size_t>(n));  // order | inverse
  sizing.take<unsigned char>(n);     // dead-column mask
  sizing.take<DiagStats>(1);
  if (sizing.off > kNoallocBytes)
    fail(OC_ERR_INVALID_ARG,
         "oc_gptq_quantize_noalloc: m=%lld, n=%lld need %zu bytes of scratch but the built-in array holds "
         "%zu (e.g. n=512 fits up to m=1024); use oc_gptq_quantize for larger layers",
         static_cast<long long>(m), static_cast<long long>(n), sizing.off, kNoallocBytes);

  int dev = 0;
  check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) fail(OC_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  int major = 0, minor = 0, sms = 0;
  check_cuda(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "cc major");
  check_cuda(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "cc minor");
  check_cuda(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "sm count");
  if (major != 10 || minor != 0)
    fail(OC_ERR_UNSUPPORTED, "liboc is built for sm_100a; device %d is sm_%d%d", dev, major, minor);

  Carve cv{scratch_address(dev)};
  int* status = cv.take<int>(1);
  float* M = cv.take<float>(nn);
  float* Xi = cv.take<float>(nn);
  float* scratch = cv.take<float>(nn / 2 + 4096);
  float* Wp = cv.take<float>(mn);
  unsigned char* codes8 = cv.take<unsigned char>(mn);
  float* Err = cv.take<float>(static_cast<size_t>(m) * 128);
  int32_t* perm = cv.take<int32_t>(2 * static_cast<size_t>(n));
  unsigned char* dead = cv.take<unsigned char>(n);
  DiagStats* stats = cv.take<DiagStats>(1);

  Ctx c{};
  c.stream = static_cast<cudaStream_t>(stream);
  c.status = status;
  c.sm_count = sms;
  c.device = dev;
  // the only state that must start at zero: the status word (the inverse
  // factor is cleared by factor_inverse_upper itself)
  check_cuda(cudaMemsetAsync(status, 0, sizeof(int), c.stream), "clear status");

  launch_diag_stats(c, H, n, damp, 1.0f, true, stats, dead);
  if (act_order) launch_act_order_perm(c, H, n, perm);
  else launch_identity_perm(c, n, perm);
  launch_build_reversed(c, H, n, perm, stats, 1.0f, true, M);
  factor_inverse_upper(c, M, Xi, scratch, M, n, /*use_graph=*/false);  // no graph: it would allocate
  const float* U = M;
  launch_permute_w(c, W, m, n, perm, dead, Wp);
  if (act_order) launch_static_grid(c, W, m, n, static_cast<int>(G), wbits, dead, scales, zeros);
  for (int64_t j1 = 0; j1 < n; j1 += 128) {
    const int64_t bw = std::min<int64_t>(128, n - j1);
    const int64_t j2 = j1 + bw;
    launch_sweep_block(c, Wp, m, n, U, j1, static_cast<int>(G), wbits, act_order != 0, perm, scales, zeros,
                       codes8, Err);
    if (j2 < n)
      gemm_f32(c, false, false, m, n - j2, bw, -1.f, Err, 128, U + j1 * n + j2, n, 1.f, Wp + j2, n, kANone);
  }
  launch_pack(c, codes8, m, n, wbits, perm, codes);
  if (perm_out)
    check_cuda(cudaMemcpyAsync(perm_out, perm, static_cast<size_t>(n) * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                               c.stream),
               "copy perm");
  check_cuda(cudaStreamSynchronize(c.stream), "cudaStreamSynchronize");
  int st = 0;
  check_cuda(cudaMemcpy(&st, status, sizeof(int), cudaMemcpyDeviceToHost), "read status");
  if (st != 0) {
    char msg[128];
    snprintf(msg, sizeof(msg), "device reported %s", oc_status_string(st));
    set_last_error(msg);
  }
  return st;
}

}  // namespace
}  // namespace oc

extern "C" int oc_gptq_quantize_noalloc(const float* W, int64_t m, int64_t n, const float* H, int wbits,
                                        int groupsize, float damp, int act_order, uint32_t* codes,
                                        float* scales, float* zeros, int32_t* perm_out, void* stream) {
  try {
    oc::set_last_error("");
    // the same lock as every other entry point: the launch helpers share
    // host-side state (one-time kernel attribute flags, the launch counter)
    std::lock_guard<std::mutex> lock(oc::library_mutex());
    return oc::run(W, m, n, H, wbits, groupsize, damp, act_order, codes, scales, zeros, perm_out, stream);
  } catch (const oc::Failure& e) {
    oc::set_last_error(e.msg);
    return e.status;
  }
}

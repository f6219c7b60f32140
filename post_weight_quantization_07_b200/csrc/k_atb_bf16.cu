// C += alpha * A^T B over calibration tokens on the 5th-generation tensor cores.
//
// A and B are token-major bf16 activations ([n_tok x M], [n_tok x N]); the
// contraction runs over tokens, so both operands are MN-major in shared
// memory (features contiguous).  This is the Hessian accumulation
// H += 2 Xhat^T Xhat (A == B, upper tiles only) and QEP's cross product
// X^T Xhat (all tiles).
//
// Design: persistent clusters of two CTAs (one per SM) that share each MMA
// (tcgen05 cta_group::2).  A pair owns a 256 x 256 output tile: CTA r holds
// features [128r, 128r + 128) of the tile's A columns and of its B columns in
// its shared memory and rows [128r, 128r + 128) of the fp32 accumulator in its
// TMEM, so each SM loads 64 KB per 128-token stage for a 128 x 256 x 128 share
// of the MMA work (a lone CTA would need 96 KB).  256 threads per CTA:
//   warp 0       TMA producer: 2 + 2 boxes of 64 features x 128 tokens per
//                stage, 128-byte swizzle, 3-stage ring; both CTAs' bytes are
//                counted on the leader's "full" barrier, which each producer
//                arms with its own 64 KB.  Long stages matter more than a deep
//                ring here: each stage costs a fixed handshake (barrier waits,
//                TMA issue, commit), and with the same 192 KB in flight,
//                32-, 64- and 128-token stages ran at about 0.39, 0.56 and
//                0.65 TFLOP/s per MHz.
//   warp 1       TMEM owner (both CTAs allocate 512 columns together = two
//                accumulators) and, in the leader CTA only, MMA issuer:
//                M=256 N=256 K=16, eight per stage, committed to the stage's
//                "empty" barrier in both CTAs; a unit's last commit signals
//                both CTAs' epilogues.
//   warps 4..7   epilogue (both CTAs): tcgen05.ld 32 lanes x 32 columns, scale,
//                stage a 32x32 fp32 box in swizzled shared memory and TMA
//                reduce-add it into C (fp32 add at L2), then release the
//                accumulator on the leader's barrier.  Double-buffered TMEM lets
//                the next unit's MMAs run while this drains.
// Work units are (output tile, token chunk); chunks are the outer index so
// that the clusters of one wave stream the same token window through L2.
// Every wait is bounded; a wait that gives up records OC_ERR_TIMEOUT and the
// kernel winds down (both CTAs still meet at the final cluster barrier).
#include <algorithm>
#include <cstdio>

#include "oc_internal.cuh"
#include "ptx_sm100.cuh"

namespace oc {
namespace {

constexpr int TM = 256;          // pair tile rows (A features)
constexpr int TN = 256;          // pair tile cols (B features) = TMEM columns per accumulator
constexpr int HM = TM / 2;       // rows per CTA = TMEM lanes
constexpr int HN = TN / 2;       // B features held per CTA
constexpr int BK = 128;          // tokens per stage
constexpr int STAGES = 3;
constexpr int A_BYTES = HM * BK * 2;              // 32 KB
constexpr int B_BYTES = HN * BK * 2;              // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // 64 KB per CTA
constexpr int BOX_BYTES = 64 * BK * 2;            // one 64-feature x 128-token box, 16 KB
constexpr int EPI_WARPS = 4;
constexpr int EPI_BOX_BYTES = 32 * 32 * 4;        // 32x32 fp32 staging box
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BOX_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 /*barriers*/ + 1024 /*align*/;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
constexpr uint32_t TMEM_COLS = 512;
constexpr int THREADS = 256;
constexpr uint16_t kBothCtas = 0x3;

struct Params {
  int64_t n_tok;
  int tiles_i, tiles_j, n_tiles;
  int kc_stages, n_kc;
  int64_t units;
  int upper_only;
  float alpha;
  int* status;
};

__device__ __forceinline__ void decode_tile(const Params& p, int tile, int& ti, int& tj) {
  if (!p.upper_only) {
    ti = tile % p.tiles_i;
    tj = tile / p.tiles_i;
    return;
  }
  // upper tiles: for column block tj, row blocks ti <= tj
  int t = tile;
  for (tj = 0; tj < p.tiles_j; ++tj) {
    const int cnt = min(p.tiles_i, tj + 1);
    if (t < cnt) break;
    t -= cnt;
  }
  ti = t;
}

__global__ void __launch_bounds__(THREADS, 1)
atb_bf16_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                const __grid_constant__ CUtensorMap mapC, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stage_base = smem;
  unsigned char* epi_base = smem + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_base + EPI_BYTES);
  uint64_t* full = bars;                 // [STAGES], used in the leader: both CTAs' loads
  uint64_t* empty = bars + STAGES;       // [STAGES], this CTA's ring slots
  uint64_t* tfull = bars + 2 * STAGES;   // [2], accumulator ready (this CTA's TMEM half)
  uint64_t* tempty = tfull + 2;          // [2], used in the leader: both epilogues done
  uint64_t* drain = tempty + 2;          // [1], all MMAs finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int64_t cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mapA);
    prefetch_tensormap(&mapB);
    prefetch_tensormap(&mapC);
  }
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before anything arrives on them
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t stages_total = (p.n_tok + BK - 1) / BK;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    uint64_t issued = 0;
    bool ok = true;
    for (int64_t u = cid; u < p.units && ok; u += ncl) {
      const int kc = static_cast<int>(u / p.n_tiles);
      int ti, tj;
      decode_tile(p, static_cast<int>(u % p.n_tiles), ti, tj);
      const int64_t ks0 = static_cast<int64_t>(kc) * p.kc_stages;
      const int64_t ks1 = ::min((int64_t)stages_total, ks0 + p.kc_stages);
      for (int64_t ks = ks0; ks < ks1; ++ks) {
        const int s = static_cast<int>(issued % STAGES);
        const uint32_t ph = static_cast<uint32_t>((issued / STAGES) & 1);
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty[s], ph ^ 1) && !*abort_flag;
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        if (lane == 0) {
          unsigned char* sa = stage_base + s * STAGE_BYTES;
          unsigned char* sb = sa + A_BYTES;
          mbar_arrive_expect_tx_cluster(mapa_shared(smem_u32(&full[s]), 0), STAGE_BYTES);
          const int32_t t0 = static_cast<int32_t>(ks * BK);
          const int32_t i0 = ti * TM + HM * static_cast<int32_t>(rank);
          const int32_t j0 = tj * TN + HN * static_cast<int32_t>(rank);
          const CUtensorMap* mb = p.upper_only ? &mapA : &mapB;
          tma_load_2d_pair(&mapA, &full[s], sa, i0, t0);
          tma_load_2d_pair(&mapA, &full[s], sa + BOX_BYTES, i0 + 64, t0);
          tma_load_2d_pair(mb, &full[s], sb, j0, t0);
          tma_load_2d_pair(mb, &full[s], sb + BOX_BYTES, j0 + 64, t0);
        }
        __syncwarp();
        ++issued;
      }
    }
    if (lane == 0) {
      if (!ok) {
        record_error(p.status, kDevTimeout);
        *abort_flag = 1;
      }
      // Drain (leader): the last issued stages, counted with both CTAs' bytes,
      // must have landed before either CTA lets its shared memory go.
      if (leader) {
        const uint64_t first = issued > STAGES ? issued - STAGES : 0;
        for (uint64_t q = first; q < issued; ++q) {
          if (!mbar_wait(&full[q % STAGES], static_cast<uint32_t>((q / STAGES) & 1))) {
            record_error(p.status, kDevTimeout);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader) {
      // ---------------------------------------------------------------- MMA issuer (leader)
      constexpr uint32_t idesc = instr_desc(1, 1, true, true, TM, TN);
      uint64_t consumed = 0;
      int it = 0;
      bool ok = true;
      for (int64_t u = cid; u < p.units && ok; u += ncl, ++it) {
        const int kc = static_cast<int>(u / p.n_tiles);
        const int64_t ks0 = static_cast<int64_t>(kc) * p.kc_stages;
        const int64_t ks1 = ::min((int64_t)stages_total, ks0 + p.kc_stages);
        const int acc = it & 1;
        int w = 1;
        if (lane == 0) w = mbar_wait(&tempty[acc], static_cast<uint32_t>(((it >> 1) & 1) ^ 1));
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        tc_fence_after();
        const uint32_t dcol = tmem_base + static_cast<uint32_t>(acc * TN);
        for (int64_t ks = ks0; ks < ks1; ++ks) {
          const int s = static_cast<int>(consumed % STAGES);
          const uint32_t ph = static_cast<uint32_t>((consumed / STAGES) & 1);
          w = 1;
          if (lane == 0) w = mbar_wait(&full[s], ph) && !*abort_flag;
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t sa = smem_u32(stage_base + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(sa + kk * 2048, BOX_BYTES, 1024);
              const uint64_t bdesc = smem_desc_sw128(sb + kk * 2048, BOX_BYTES, 1024);
              mma_bf16_ss_pair(dcol, adesc, bdesc, idesc, (ks > ks0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_pair(&empty[s], kBothCtas);
          }
          __syncwarp();
          ++consumed;
        }
        if (!ok) break;
        if (lane == 0) mma_commit_pair(&tfull[acc], kBothCtas);
        __syncwarp();
      }
      if (lane == 0) {
        if (!ok) {
          record_error(p.status, kDevTimeout);
          *abort_flag = 1;
        }
        // Every issued MMA must be done before TMEM and shared memory are
        // released, in both CTAs: the commit reaches both drain barriers.
        mma_commit_pair(drain, kBothCtas);
        if (!mbar_wait(drain, 0)) record_error(p.status, kDevTimeout);
      }
    } else {
      // peer: no MMA reads this CTA's shared memory or writes its TMEM after this
      if (lane == 0 && !mbar_wait(drain, 0)) record_error(p.status, kDevTimeout);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp - 4;  // TMEM lanes 32q .. 32q+31
    unsigned char* stage_buf = epi_base + q * 2 * EPI_BOX_BYTES;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int it = 0;
    int nbuf = 0;
    bool ok = true;
    for (int64_t u = cid; u < p.units; u += ncl, ++it) {
      int ti, tj;
      decode_tile(p, static_cast<int>(u % p.n_tiles), ti, tj);
      const int acc = it & 1;
      int w = 1;
      if (lane == 0) w = mbar_wait(&tfull[acc], static_cast<uint32_t>((it >> 1) & 1)) && !*abort_flag;
      w = __shfl_sync(0xffffffffu, w, 0);
      if (!w) { ok = false; break; }
      tc_fence_after();
      const int row0 = ti * TM + HM * static_cast<int>(rank) + 32 * q;
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t r[32];
        const uint32_t taddr =
            tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * TN + c * 32);
        tmem_ld_32x32b_x32(taddr, r);
        tmem_ld_wait();
        unsigned char* buf = stage_buf + (nbuf & 1) * EPI_BOX_BYTES;
        // the reduce that last read this buffer (two boxes ago) must be done reading
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        // row `lane` of the box: 8 chunks of 16 bytes, chunk k stored at (k ^ (lane & 7))
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float4 v;
          v.x = __uint_as_float(r[4 * k + 0]) * p.alpha;
          v.y = __uint_as_float(r[4 * k + 1]) * p.alpha;
          v.z = __uint_as_float(r[4 * k + 2]) * p.alpha;
          v.w = __uint_as_float(r[4 * k + 3]) * p.alpha;
          *reinterpret_cast<float4*>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&mapC, buf, tj * TN + c * 32, row0);
          bulk_commit_group();
        }
        ++nbuf;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
    if (!ok && lane == 0) {
      record_error(p.status, kDevTimeout);
      *abort_flag = 1;
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  // Both CTAs meet here before TMEM is released (a collective over the pair)
  // and before either CTA's shared memory goes away.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

__global__ void mirror_upper_kernel(float* H, int64_t n) {
  // One 32x32 tile of the strictly lower block triangle per block: lower(bi, bj)
  // with bi > bj takes the transpose of upper(bj, bi); diagonal tiles copy their
  // own upper half.
  __shared__ float t[32][33];
  const int64_t bi = blockIdx.y, bj = blockIdx.x;
  if (bj > bi) return;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int r = ty; r < 32; r += 8) {
    const int64_t row = bj * 32 + r, col = bi * 32 + tx;  // source: upper tile (bj, bi)
    if (row < n && col < n) t[r][tx] = H[row * n + col];
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int64_t row = bi * 32 + r, col = bj * 32 + tx;  // destination: lower tile (bi, bj)
    if (row < n && col < n && row > col) H[row * n + col] = t[tx][r];
  }
}

}  // namespace

void launch_atb_bf16(const Ctx& c, const void* A, const void* B, int64_t n_tok, int64_t M,
                     int64_t N, float alpha, float* C, int64_t ldc, bool upper_only, int max_ctas) {
  if (n_tok <= 0 || M <= 0 || N <= 0) return;
  if ((M % 64) || (N % 64) || (ldc % 4)) fail(OC_ERR_INVALID_ARG, "atb_bf16: bad sizes");
  const CUtensorMap mA = make_tmap_2d(A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_tok, M, M, BK, 64, Swz::B128);
  const CUtensorMap mB = make_tmap_2d(upper_only ? A : B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_tok, N, N,
                                      BK, 64, Swz::B128);
  const CUtensorMap mC = make_tmap_2d(C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, M, N, ldc, 32, 32, Swz::B128);
  Params p{};
  p.n_tok = n_tok;
  p.tiles_i = static_cast<int>((M + TM - 1) / TM);
  p.tiles_j = static_cast<int>((N + TN - 1) / TN);
  p.upper_only = upper_only ? 1 : 0;
  if (upper_only) {
    int cnt = 0;
    for (int tj = 0; tj < p.tiles_j; ++tj) cnt += std::min(p.tiles_i, tj + 1);
    p.n_tiles = cnt;
  } else {
    p.n_tiles = p.tiles_i * p.tiles_j;
  }

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = c.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Clusters that can be resident at once (one CTA per SM; pairs sit in one GPC).
  static int max_clusters[64] = {0};
  const int dv = c.device & 63;
  if (max_clusters[dv] == 0) {
    check_cuda(cudaFuncSetAttribute(atb_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
               "cudaFuncSetAttribute(atb_bf16)");
    cfg.gridDim = dim3(static_cast<unsigned>(2 * (c.sm_count / 2)), 1, 1);
    int ncl = 0;
    check_cuda(cudaOccupancyMaxActiveClusters(&ncl, atb_bf16_kernel, &cfg), "cudaOccupancyMaxActiveClusters");
    if (ncl < 1) fail(OC_ERR_UNSUPPORTED, "atb_bf16: no CTA pair fits on this device");
    max_clusters[dv] = ncl;
  }
  const int ctas = (max_ctas > 0 && max_ctas < c.sm_count) ? max_ctas : c.sm_count;
  const int64_t clusters_avail = std::max(1, std::min(ctas / 2, max_clusters[dv]));

  const int64_t stages_total = (n_tok + BK - 1) / BK;
  // Token chunk per unit: long enough to amortise the epilogue, and enough
  // units (about four per cluster) to balance the clusters.
  const int64_t want_chunks = std::max<int64_t>(1, (4 * clusters_avail + p.n_tiles - 1) / p.n_tiles);
  int64_t kcs = (stages_total + want_chunks - 1) / want_chunks;
  kcs = std::max<int64_t>(1024 / BK, std::min<int64_t>(8192 / BK, kcs));
  kcs = std::min(kcs, stages_total);
  p.kc_stages = static_cast<int>(kcs);
  p.n_kc = static_cast<int>((stages_total + kcs - 1) / kcs);
  p.units = static_cast<int64_t>(p.n_kc) * p.n_tiles;
  p.alpha = alpha;
  p.status = c.status;
  const int64_t clusters = std::min<int64_t>(p.units, clusters_avail);
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  check_cuda(cudaLaunchKernelEx(&cfg, atb_bf16_kernel, mA, mB, mC, p), "cudaLaunchKernelEx(atb_bf16)");
  check_launch("atb_bf16_kernel");
}

void launch_mirror_upper(const Ctx& c, float* H, int64_t n) {
  const int64_t nb = (n + 31) / 32;
  dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>(nb));
  mirror_upper_kernel<<<grid, dim3(32, 8), 0, c.stream>>>(H, n);
  check_launch("mirror_upper_kernel");
}

}  // namespace oc

// fp32-accurate GEMM on the 5th-generation tensor cores (3xTF32):
//   C  = alpha * A op(B)        (store)        or
//   C += alpha * A op(B)        (accumulate: TMA reduce-add)
// with A [M x K] and B [N x K] both row-major (op(B) = B^T), i.e. both operands
// K-major in shared memory.  A product whose B is stored [K x N] passes the
// transposed split copy instead (split_tf32 with transpose writes it).
//
// Every operand x is split once, outside this kernel, into x_hi = tf32(x) and
// x_lo = tf32(x - x_hi); the product is accumulated as
//   a_hi b_hi + a_hi b_lo + a_lo b_hi
// in fp32 TMEM (the dropped a_lo b_lo term is ~2^-22 of a b).  The tensor
// cores read both halves exactly, so the result carries about 21 bits.
//
// One persistent CTA per SM, 256 threads: warp 0 issues TMA loads (4 boxes of
// 16 KB per 32-deep k slice: A_hi, A_lo, B_hi, B_lo, 128-byte swizzle,
// 3-stage ring), warp 1 owns TMEM (two 128x128 fp32 accumulators) and issues
// tcgen05.mma kind::tf32 M128 N128 K8 (12 per slice), warps 4..7 drain the
// accumulator through swizzled 32x32 shared-memory boxes into TMA stores or
// reduce-adds.  Triangular operands clip the k range of each tile.
//
// Segmented accumulation.  Adding an MMA's products into a TMEM accumulator
// is not rounded to nearest: the sum is truncated, which biases every
// addition towards zero by about half an ulp.  A chain of one accumulator
// over a long k range (3 MMAs per 8-deep step) piles the bias up in
// proportion to its length: measured against float64, the products with
// k = 28672 came out about 6e-4 too small.  So each tile's k range is cut into
// segments of KSEG; every segment restarts its accumulator (double-buffered in
// TMEM, so the next segment's MMAs overlap), and the epilogue adds the
// segments in fp32 registers, rounded to nearest, before the one store of
// the tile.  The bias is then that of KSEG / 8 * 3 = 96 additions.
#include <algorithm>

#include "oc_internal.cuh"
#include "ptx_sm100.cuh"

namespace oc {
namespace {

constexpr int BM = 128, BN = 128, BK = 32;  // BK fp32 = 128 bytes = one swizzle row
constexpr int KSEG = 256;                   // k per accumulator chain (a multiple of BK)
constexpr int STAGES = 3;
constexpr int TILE_BYTES = BM * BK * 4;      // 16 KB (A or B, one half)
constexpr int STAGE_BYTES = 4 * TILE_BYTES;  // A_hi, A_lo, B_hi, B_lo
constexpr int EPI_WARPS = 4;
constexpr int EPI_BOX_BYTES = 32 * 32 * 4;
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BOX_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 1024;
constexpr uint32_t TMEM_COLS = 256;
constexpr int THREADS = 256;

struct Params {
  int M, N, K;
  int tiles_m, tiles_n;
  unsigned flags;
  float alpha;
  int accumulate;
  int* status;
  // optional device flags, zero when the operand's lo half is all zero (the
  // operand is exact in tf32, e.g. bf16-valued weights): its correction MMA
  // adds nothing and is skipped
  const int* a_lo_nz;
  const int* b_lo_nz;
};

// Tiles wholly above the diagonal are skipped when only the lower triangle of
// C is wanted (every role applies the same test, so the pipelines stay aligned).
__device__ __forceinline__ bool tile_skipped(const Params& p, int i0, int j0) {
  return (p.flags & kCLowerOnly) && j0 > i0 + BM - 1;
}

__device__ __forceinline__ void k_range(const Params& p, int i0, int j0, int& kb, int& ke) {
  kb = 0;
  ke = p.K;
  if (p.flags & kAUpper) kb = max(kb, i0);
  if (p.flags & kALower) ke = min(ke, i0 + BM);
  if (p.flags & kBLower) kb = max(kb, j0);
  if (p.flags & kBUpper) ke = min(ke, j0 + BN);
  kb = (kb / BK) * BK;
}

// Segments of one tile's k range [kb, ke) (one, with no MMAs, when it is empty).
__device__ __forceinline__ int n_segments(int kb, int ke) { return ke > kb ? (ke - kb + KSEG - 1) / KSEG : 1; }

__global__ void __launch_bounds__(THREADS, 1)
gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
                   const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl,
                   const __grid_constant__ CUtensorMap mC, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stage_base = smem;
  unsigned char* epi_base = smem + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_base + EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mAh);
    prefetch_tensormap(&mAl);
    prefetch_tensormap(&mBh);
    prefetch_tensormap(&mBl);
    prefetch_tensormap(&mC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    uint64_t issued = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const int i0 = (t % p.tiles_m) * BM, j0 = (t / p.tiles_m) * BN;
      if (tile_skipped(p, i0, j0)) continue;
      int kb, ke;
      k_range(p, i0, j0, kb, ke);
      for (int k0 = kb; k0 < ke; k0 += BK) {
        const int s = static_cast<int>(issued % STAGES);
        const uint32_t ph = static_cast<uint32_t>((issued / STAGES) & 1);
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty[s], ph ^ 1) && !*abort_flag;
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        if (lane == 0) {
          unsigned char* st = stage_base + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(&mAh, &full[s], st, k0, i0);
          tma_load_2d(&mAl, &full[s], st + TILE_BYTES, k0, i0);
          tma_load_2d(&mBh, &full[s], st + 2 * TILE_BYTES, k0, j0);
          tma_load_2d(&mBl, &full[s], st + 3 * TILE_BYTES, k0, j0);
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
      const uint64_t first = issued > STAGES ? issued - STAGES : 0;
      for (uint64_t q = first; q < issued; ++q) {
        if (!mbar_wait(&full[q % STAGES], static_cast<uint32_t>((q / STAGES) & 1))) {
          record_error(p.status, kDevTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = instr_desc(2, 2, false, false, BM, BN);
    const bool use_al = p.a_lo_nz == nullptr || *p.a_lo_nz != 0;
    const bool use_bl = p.b_lo_nz == nullptr || *p.b_lo_nz != 0;
    uint64_t consumed = 0;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const int i0 = (t % p.tiles_m) * BM, j0 = (t / p.tiles_m) * BN;
      if (tile_skipped(p, i0, j0)) continue;
      int kb, ke;
      k_range(p, i0, j0, kb, ke);
      const int nseg = n_segments(kb, ke);
      for (int sg = 0; sg < nseg && ok; ++sg) {
        const int acc = it & 1;
        int w = 1;
        if (lane == 0) w = mbar_wait(&tempty[acc], static_cast<uint32_t>(((it >> 1) & 1) ^ 1));
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        tc_fence_after();
        const uint32_t dcol = tmem_base + static_cast<uint32_t>(acc * BN);
        const int s0 = kb + sg * KSEG, s1 = min(ke, s0 + KSEG);
        for (int k0 = s0; k0 < s1; k0 += BK) {
          const int s = static_cast<int>(consumed % STAGES);
          const uint32_t ph = static_cast<uint32_t>((consumed / STAGES) & 1);
          w = 1;
          if (lane == 0) w = mbar_wait(&full[s], ph) && !*abort_flag;
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t sa = smem_u32(stage_base + s * STAGE_BYTES);
            const uint32_t sah = sa, sal = sa + TILE_BYTES, sbh = sa + 2 * TILE_BYTES, sbl = sa + 3 * TILE_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 8; ++kk) {
              const uint64_t ah = smem_desc_sw128(sah + kk * 32, 16, 1024);
              const uint64_t al = smem_desc_sw128(sal + kk * 32, 16, 1024);
              const uint64_t bh = smem_desc_sw128(sbh + kk * 32, 16, 1024);
              const uint64_t bl = smem_desc_sw128(sbl + kk * 32, 16, 1024);
              uint32_t accf = (k0 == s0 && kk == 0) ? 0u : 1u;
              if (use_al) { mma_tf32_ss(dcol, al, bh, idesc, accf); accf = 1u; }
              if (use_bl) { mma_tf32_ss(dcol, ah, bl, idesc, accf); accf = 1u; }
              mma_tf32_ss(dcol, ah, bh, idesc, accf);
            }
            mma_commit(&empty[s]);
          }
          __syncwarp();
          ++consumed;
        }
        if (!ok) break;
        if (lane == 0) mma_commit(&tfull[acc]);
        __syncwarp();
        ++it;
      }
    }
    if (lane == 0) {
      if (!ok) {
        record_error(p.status, kDevTimeout);
        *abort_flag = 1;
      }
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) record_error(p.status, kDevTimeout);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp - 4;
    unsigned char* stage_buf = epi_base + q * 2 * EPI_BOX_BYTES;
    int it = 0, nbuf = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const int i0 = (t % p.tiles_m) * BM, j0 = (t / p.tiles_m) * BN;
      if (tile_skipped(p, i0, j0)) continue;
      int kb, ke;
      k_range(p, i0, j0, kb, ke);
      const bool empty_k = kb >= ke;
      const int nseg = n_segments(kb, ke);
      // row `lane` of this warp's 32 rows, all BN columns: the tile's sum
      float sum[BN];
#pragma unroll
      for (int e = 0; e < BN; ++e) sum[e] = 0.f;
      for (int sg = 0; sg < nseg; ++sg) {
        const int acc = it & 1;
        int w = 1;
        if (lane == 0) w = mbar_wait(&tfull[acc], static_cast<uint32_t>((it >> 1) & 1)) && !*abort_flag;
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        tc_fence_after();
        if (!empty_k) {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t r[32];
            const uint32_t taddr =
                tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * BN + c * 32);
            tmem_ld_32x32b_x32(taddr, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) sum[32 * c + e] += __uint_as_float(r[e]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        ++it;
      }
      if (!ok) break;
      if (!(empty_k && p.accumulate)) {
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          unsigned char* buf = stage_buf + (nbuf & 1) * EPI_BOX_BYTES;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float4 v;
            v.x = sum[32 * c + 4 * k + 0] * p.alpha;
            v.y = sum[32 * c + 4 * k + 1] * p.alpha;
            v.z = sum[32 * c + 4 * k + 2] * p.alpha;
            v.w = sum[32 * c + 4 * k + 3] * p.alpha;
            *reinterpret_cast<float4*>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) = v;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (p.accumulate) tma_reduce_add_2d(&mC, buf, j0 + c * 32, i0 + 32 * q);
            else tma_store_2d(&mC, buf, j0 + c * 32, i0 + 32 * q);
            bulk_commit_group();
          }
          ++nbuf;
        }
      }
    }
    if (!ok && lane == 0) {
      record_error(p.status, kDevTimeout);
      *abort_flag = 1;
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------- CTA-pair variant
// Same product on clusters of two CTAs sharing each MMA (tcgen05 cta_group::2):
// a pair owns a 256 x 256 tile of C; CTA r loads rows [128r, 128r + 128) of the
// tile's A and of its B (hi and lo halves, 64 KB per 32-deep k slice) and
// holds rows [128r, 128r + 128) of the accumulator (two 128 x 256 fp32
// accumulators = all 512 TMEM columns).  Each SM thus loads the same bytes
// per slice as the single-CTA kernel for twice the MMA work.  Both producers
// arm the leader's "full" barrier with their own bytes; the leader issues
// M=256 N=256 K=8 kind::tf32 MMAs (3 per k step) and commits to both CTAs.
// Segmented accumulation as above; the tile's running sum (256 columns per
// row) is held by eight epilogue warps, 128 columns each: warps 4..11, warp w
// reading TMEM lanes 32 (w % 4) .. + 31 and column half (w - 4) / 4.
constexpr int PM = 256, PN = 256;              // pair tile
constexpr int P_STAGES = 3;
constexpr int P_STAGE_BYTES = 4 * TILE_BYTES;  // A_hi, A_lo, B_hi, B_lo (128 rows each)
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + EPI_BYTES + 1024 + 1024;
static_assert(P_SMEM_BYTES <= 232448, "shared memory per CTA");
constexpr uint32_t P_TMEM_COLS = 512;
constexpr uint16_t kPairMask = 0x3;
constexpr int P_THREADS = 384;
constexpr int P_EPI_WARPS = 8;      // one 4 KB staging box each: P_EPI_WARPS * EPI_BOX_BYTES == EPI_BYTES
static_assert(P_EPI_WARPS * EPI_BOX_BYTES == EPI_BYTES, "pair staging boxes");

__device__ __forceinline__ bool pair_tile_skipped(const Params& p, int i0, int j0) {
  return (p.flags & kCLowerOnly) && j0 > i0 + PM - 1;
}

__device__ __forceinline__ void pair_k_range(const Params& p, int i0, int j0, int& kb, int& ke) {
  kb = 0;
  ke = p.K;
  if (p.flags & kAUpper) kb = max(kb, i0);
  if (p.flags & kALower) ke = min(ke, i0 + PM);
  if (p.flags & kBLower) kb = max(kb, j0);
  if (p.flags & kBUpper) ke = min(ke, j0 + PN);
  kb = (kb / BK) * BK;
}

__global__ void __launch_bounds__(P_THREADS, 1)
gemm_tf32x3_pair_kernel(const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
                        const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl,
                        const __grid_constant__ CUtensorMap mC, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stage_base = smem;
  unsigned char* epi_base = smem + P_STAGES * P_STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_base + EPI_BYTES);
  uint64_t* full = bars;                   // leader: both CTAs' loads
  uint64_t* empty = bars + P_STAGES;       // this CTA's ring slots
  uint64_t* tfull = bars + 2 * P_STAGES;   // this CTA's accumulator half ready
  uint64_t* tempty = tfull + 2;            // leader: both epilogues done
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const int n_tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * P_EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mAh);
    prefetch_tensormap(&mAl);
    prefetch_tensormap(&mBh);
    prefetch_tensormap(&mBl);
    prefetch_tensormap(&mC);
  }
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, P_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int half = BM * static_cast<int>(rank);  // this CTA's rows of the pair tile

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    uint64_t issued = 0;
    bool ok = true;
    for (int t = cid; t < n_tiles && ok; t += ncl) {
      const int i0 = (t % p.tiles_m) * PM, j0 = (t / p.tiles_m) * PN;
      if (pair_tile_skipped(p, i0, j0)) continue;
      int kb, ke;
      pair_k_range(p, i0, j0, kb, ke);
      for (int k0 = kb; k0 < ke; k0 += BK) {
        const int s = static_cast<int>(issued % P_STAGES);
        const uint32_t ph = static_cast<uint32_t>((issued / P_STAGES) & 1);
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty[s], ph ^ 1) && !*abort_flag;
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        if (lane == 0) {
          unsigned char* st = stage_base + s * P_STAGE_BYTES;
          mbar_arrive_expect_tx_cluster(mapa_shared(smem_u32(&full[s]), 0), P_STAGE_BYTES);
          tma_load_2d_pair(&mAh, &full[s], st, k0, i0 + half);
          tma_load_2d_pair(&mAl, &full[s], st + TILE_BYTES, k0, i0 + half);
          tma_load_2d_pair(&mBh, &full[s], st + 2 * TILE_BYTES, k0, j0 + half);
          tma_load_2d_pair(&mBl, &full[s], st + 3 * TILE_BYTES, k0, j0 + half);
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
      if (leader) {
        const uint64_t first = issued > P_STAGES ? issued - P_STAGES : 0;
        for (uint64_t q = first; q < issued; ++q) {
          if (!mbar_wait(&full[q % P_STAGES], static_cast<uint32_t>((q / P_STAGES) & 1))) {
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
      constexpr uint32_t idesc = instr_desc(2, 2, false, false, PM, PN);
      const bool use_al = p.a_lo_nz == nullptr || *p.a_lo_nz != 0;
      const bool use_bl = p.b_lo_nz == nullptr || *p.b_lo_nz != 0;
      uint64_t consumed = 0;
      int it = 0;
      bool ok = true;
      for (int t = cid; t < n_tiles && ok; t += ncl) {
        const int i0 = (t % p.tiles_m) * PM, j0 = (t / p.tiles_m) * PN;
        if (pair_tile_skipped(p, i0, j0)) continue;
        int kb, ke;
        pair_k_range(p, i0, j0, kb, ke);
        const int nseg = n_segments(kb, ke);
        for (int sg = 0; sg < nseg && ok; ++sg) {
          const int acc = it & 1;
          int w = 1;
          if (lane == 0) w = mbar_wait(&tempty[acc], static_cast<uint32_t>(((it >> 1) & 1) ^ 1));
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) { ok = false; break; }
          tc_fence_after();
          const uint32_t dcol = tmem_base + static_cast<uint32_t>(acc * PN);
          const int s0 = kb + sg * KSEG, s1 = min(ke, s0 + KSEG);
          for (int k0 = s0; k0 < s1; k0 += BK) {
            const int s = static_cast<int>(consumed % P_STAGES);
            const uint32_t ph = static_cast<uint32_t>((consumed / P_STAGES) & 1);
            w = 1;
            if (lane == 0) w = mbar_wait(&full[s], ph) && !*abort_flag;
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
              const uint32_t sa = smem_u32(stage_base + s * P_STAGE_BYTES);
              const uint32_t sah = sa, sal = sa + TILE_BYTES, sbh = sa + 2 * TILE_BYTES, sbl = sa + 3 * TILE_BYTES;
#pragma unroll
              for (int kk = 0; kk < BK / 8; ++kk) {
                const uint64_t ah = smem_desc_sw128(sah + kk * 32, 16, 1024);
                const uint64_t al = smem_desc_sw128(sal + kk * 32, 16, 1024);
                const uint64_t bh = smem_desc_sw128(sbh + kk * 32, 16, 1024);
                const uint64_t bl = smem_desc_sw128(sbl + kk * 32, 16, 1024);
                uint32_t accf = (k0 == s0 && kk == 0) ? 0u : 1u;
                if (use_al) { mma_tf32_ss_pair(dcol, al, bh, idesc, accf); accf = 1u; }
                if (use_bl) { mma_tf32_ss_pair(dcol, ah, bl, idesc, accf); accf = 1u; }
                mma_tf32_ss_pair(dcol, ah, bh, idesc, accf);
              }
              mma_commit_pair(&empty[s], kPairMask);
            }
            __syncwarp();
            ++consumed;
          }
          if (!ok) break;
          if (lane == 0) mma_commit_pair(&tfull[acc], kPairMask);
          __syncwarp();
          ++it;
        }
      }
      if (lane == 0) {
        if (!ok) {
          record_error(p.status, kDevTimeout);
          *abort_flag = 1;
        }
        mma_commit_pair(drain, kPairMask);
        if (!mbar_wait(drain, 0)) record_error(p.status, kDevTimeout);
      }
    } else {
      if (lane == 0 && !mbar_wait(drain, 0)) record_error(p.status, kDevTimeout);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;                 // TMEM lanes 32q .. 32q + 31
    const int hc = (warp - 4) >> 2;         // columns 128 hc .. 128 hc + 127 of the tile
    unsigned char* buf = epi_base + (warp - 4) * EPI_BOX_BYTES;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int it = 0;
    bool ok = true;
    for (int t = cid; t < n_tiles && ok; t += ncl) {
      const int i0 = (t % p.tiles_m) * PM, j0 = (t / p.tiles_m) * PN;
      if (pair_tile_skipped(p, i0, j0)) continue;
      int kb, ke;
      pair_k_range(p, i0, j0, kb, ke);
      const bool empty_k = kb >= ke;
      const int nseg = n_segments(kb, ke);
      float sum[128];
#pragma unroll
      for (int e = 0; e < 128; ++e) sum[e] = 0.f;
      for (int sg = 0; sg < nseg; ++sg) {
        const int acc = it & 1;
        int w = 1;
        if (lane == 0) w = mbar_wait(&tfull[acc], static_cast<uint32_t>((it >> 1) & 1)) && !*abort_flag;
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        tc_fence_after();
        if (!empty_k) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                   static_cast<uint32_t>(acc * PN + hc * 128 + c * 32);
            tmem_ld_32x32b_x32(taddr, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) sum[32 * c + e] += __uint_as_float(r[e]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        ++it;
      }
      if (!ok) break;
      if (!(empty_k && p.accumulate)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          // the store that last read the box must be done reading it
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float4 v;
            v.x = sum[32 * c + 4 * k + 0] * p.alpha;
            v.y = sum[32 * c + 4 * k + 1] * p.alpha;
            v.z = sum[32 * c + 4 * k + 2] * p.alpha;
            v.w = sum[32 * c + 4 * k + 3] * p.alpha;
            *reinterpret_cast<float4*>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) = v;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int col = j0 + hc * 128 + c * 32, row = i0 + half + 32 * q;
            if (p.accumulate) tma_reduce_add_2d(&mC, buf, col, row);
            else tma_store_2d(&mC, buf, col, row);
            bulk_commit_group();
          }
        }
      }
    }
    if (!ok && lane == 0) {
      record_error(p.status, kDevTimeout);
      *abort_flag = 1;
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, P_TMEM_COLS);
}

// x_hi = tf32(x), x_lo = tf32(x - x_hi), both rounded to nearest (ties away).
__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__global__ void split_tf32_kernel(const float* __restrict__ src, int64_t rows, int64_t cols, int64_t lds,
                                  float* __restrict__ hi, float* __restrict__ lo, int64_t ldd) {
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < cols;
         c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const float x = src[r * lds + c];
      const float h = to_tf32(x);
      hi[r * ldd + c] = h;
      lo[r * ldd + c] = to_tf32(x - h);
    }
  }
}

// Transposing split: hi[c][r], lo[c][r] from src[r][c], through 32x32 tiles.
__global__ void split_tf32_t_kernel(const float* __restrict__ src, int64_t rows, int64_t cols, int64_t lds,
                                    float* __restrict__ hi, float* __restrict__ lo, int64_t ldd) {
  __shared__ float t[32][33];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32, c0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int k = ty; k < 32; k += 8) {
    const int64_t r = r0 + k, c = c0 + tx;
    t[k][tx] = (r < rows && c < cols) ? src[r * lds + c] : 0.f;
  }
  __syncthreads();
  for (int k = ty; k < 32; k += 8) {
    const int64_t c = c0 + k, r = r0 + tx;  // output row c, column r
    if (c < cols && r < rows) {
      const float x = t[tx][k];
      const float h = to_tf32(x);
      hi[c * ldd + r] = h;
      lo[c * ldd + r] = to_tf32(x - h);
    }
  }
}

// Vectorised split of a matrix whose rows are 16-byte aligned and a multiple
// of 4 floats long: 4 independent float4 per thread in flight, grid-stride.
__device__ __forceinline__ void split4(const float4 x, float4& h, float4& l) {
  h = make_float4(to_tf32(x.x), to_tf32(x.y), to_tf32(x.z), to_tf32(x.w));
  l = make_float4(to_tf32(x.x - h.x), to_tf32(x.y - h.y), to_tf32(x.z - h.z), to_tf32(x.w - h.w));
}

__global__ void __launch_bounds__(256) split_tf32_v4_kernel(const float4* __restrict__ src, int64_t rows,
                                                            int64_t cols4, int64_t lds4, float4* __restrict__ hi,
                                                            float4* __restrict__ lo, int64_t ldd4, int* lo_nz) {
  const int64_t total = rows * cols4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  bool nz = false;
  for (int64_t e0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e0 < total; e0 += 4 * stride) {
    float4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = e0 + u * stride;
      if (e < total) x[u] = src[(e / cols4) * lds4 + e % cols4];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = e0 + u * stride;
      if (e < total) {
        float4 h, l;
        split4(x[u], h, l);
        const int64_t d = (e / cols4) * ldd4 + e % cols4;
        hi[d] = h;
        lo[d] = l;
        nz |= (l.x != 0.f) | (l.y != 0.f) | (l.z != 0.f) | (l.w != 0.f);
      }
    }
  }
  if (lo_nz != nullptr && nz) *lo_nz = 1;
}

// Vectorised transposing split through 64 x 64 tiles (rows and cols multiples
// of 4, 16-byte aligned rows): float4 reads along the source rows, float4
// writes along the destination rows.
constexpr int TT = 64;
__global__ void __launch_bounds__(256) split_tf32_t64_kernel(const float* __restrict__ src, int64_t rows,
                                                             int64_t cols, int64_t lds, float* __restrict__ hi,
                                                             float* __restrict__ lo, int64_t ldd) {
  __shared__ float t[TT][TT + 1];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * TT, c0 = static_cast<int64_t>(blockIdx.x) * TT;
  const int tid = threadIdx.x;
  const int cq = tid & 15, rq = tid >> 4;  // 16 float4 columns x 16 rows per pass
#pragma unroll
  for (int p = 0; p < TT / 16; ++p) {
    const int rl = rq + 16 * p;
    const int64_t r = r0 + rl, c = c0 + 4 * cq;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows && c < cols) x = *reinterpret_cast<const float4*>(src + r * lds + c);
    t[rl][4 * cq] = x.x;
    t[rl][4 * cq + 1] = x.y;
    t[rl][4 * cq + 2] = x.z;
    t[rl][4 * cq + 3] = x.w;
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < TT / 16; ++p) {
    const int cl = rq + 16 * p;            // destination row = source column c0 + cl
    const int64_t c = c0 + cl, r = r0 + 4 * cq;
    if (c < cols && r < rows) {
      const float4 x = make_float4(t[4 * cq][cl], t[4 * cq + 1][cl], t[4 * cq + 2][cl], t[4 * cq + 3][cl]);
      float4 h, l;
      split4(x, h, l);
      *reinterpret_cast<float4*>(hi + c * ldd + r) = h;
      *reinterpret_cast<float4*>(lo + c * ldd + r) = l;
    }
  }
}

void set_attr_once(int device) {
  static bool done[64] = {false};
  if (!done[device & 63]) {
    check_cuda(cudaFuncSetAttribute(gemm_tf32x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
               "cudaFuncSetAttribute(gemm_tf32x3)");
    done[device & 63] = true;
  }
}

}  // namespace

void split_tf32(const Ctx& c, const float* src, int64_t rows, int64_t cols, int64_t lds, float* hi, float* lo,
                int64_t ldd, bool transpose, int* lo_nz) {
  if (rows <= 0 || cols <= 0) return;
  if (lo_nz != nullptr) {
    if (transpose || !(aligned16(src) && aligned16(hi) && aligned16(lo) && lds % 4 == 0 && ldd % 4 == 0 && cols % 4 == 0))
      fail(OC_ERR_INVALID_ARG, "split_tf32: the lo flag needs the vectorised untransposed split");
    check_cuda(cudaMemsetAsync(lo_nz, 0, sizeof(int), c.stream), "clear lo flag");
  }
  const bool vec = aligned16(src) && aligned16(hi) && aligned16(lo) && lds % 4 == 0 && ldd % 4 == 0 &&
                   cols % 4 == 0 && (!transpose || rows % 4 == 0);
  if (vec && transpose && (rows + TT - 1) / TT <= 65535) {
    dim3 grid(static_cast<unsigned>((cols + TT - 1) / TT), static_cast<unsigned>((rows + TT - 1) / TT));
    split_tf32_t64_kernel<<<grid, 256, 0, c.stream>>>(src, rows, cols, lds, hi, lo, ldd);
    check_launch("split_tf32_t64_kernel");
    return;
  }
  if (vec && !transpose) {
    const int64_t total = rows * (cols / 4);
    const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(c.sm_count) * 8));
    split_tf32_v4_kernel<<<grid, 256, 0, c.stream>>>(reinterpret_cast<const float4*>(src), rows, cols / 4, lds / 4,
                                                     reinterpret_cast<float4*>(hi), reinterpret_cast<float4*>(lo),
                                                     ldd / 4, lo_nz);
    check_launch("split_tf32_v4_kernel");
    return;
  }
  if (transpose) {
    if ((rows + 31) / 32 > 65535) fail(OC_ERR_INVALID_ARG, "split_tf32: too many rows");
    dim3 grid(static_cast<unsigned>((cols + 31) / 32), static_cast<unsigned>((rows + 31) / 32));
    split_tf32_t_kernel<<<grid, dim3(32, 8), 0, c.stream>>>(src, rows, cols, lds, hi, lo, ldd);
    check_launch("split_tf32_t_kernel");
    return;
  }
  dim3 grid(static_cast<unsigned>(std::min<int64_t>((cols + 255) / 256, 64)),
            static_cast<unsigned>(std::min<int64_t>(rows, 8192)));
  split_tf32_kernel<<<grid, 256, 0, c.stream>>>(src, rows, cols, lds, hi, lo, ldd);
  check_launch("split_tf32_kernel");
}

void gemm_tf32x3(const Ctx& c, int64_t M, int64_t N, int64_t K, float alpha, const float* A_hi,
                 const float* A_lo, int64_t lda, const float* B_hi, const float* B_lo, int64_t ldb,
                 bool accumulate, float* C, int64_t ldc, unsigned flags, const int* a_lo_nz, const int* b_lo_nz) {
  if (M <= 0 || N <= 0) return;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30))
    fail(OC_ERR_INVALID_ARG, "gemm_tf32x3: size too large");
  const CUtensorMap mAh = make_tmap_2d(A_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, M, K, lda, BM, BK, Swz::B128);
  const CUtensorMap mAl = make_tmap_2d(A_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, M, K, lda, BM, BK, Swz::B128);
  const CUtensorMap mBh = make_tmap_2d(B_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, K, ldb, BN, BK, Swz::B128);
  const CUtensorMap mBl = make_tmap_2d(B_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, K, ldb, BN, BK, Swz::B128);
  const CUtensorMap mC = make_tmap_2d(C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, M, N, ldc, 32, 32, Swz::B128);
  Params p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.tiles_m = static_cast<int>((M + BM - 1) / BM);
  p.tiles_n = static_cast<int>((N + BN - 1) / BN);
  p.flags = flags;
  p.alpha = alpha;
  p.accumulate = accumulate ? 1 : 0;
  p.status = c.status;
  p.a_lo_nz = a_lo_nz;
  p.b_lo_nz = b_lo_nz;
  // A product with at least a wave of 256 x 256 tiles runs on CTA pairs (half
  // the operand traffic per SM); smaller ones keep more, smaller tiles.
  const int64_t pair_tiles = ((M + PM - 1) / PM) * ((N + PN - 1) / PN);
  if (pair_tiles >= c.sm_count / 2) {
    static int max_clusters[64] = {0};
    const int dv = c.device & 63;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(P_THREADS, 1, 1);
    cfg.dynamicSmemBytes = P_SMEM_BYTES;
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (max_clusters[dv] == 0) {
      check_cuda(cudaFuncSetAttribute(gemm_tf32x3_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      P_SMEM_BYTES),
                 "cudaFuncSetAttribute(gemm_tf32x3_pair)");
      cfg.gridDim = dim3(static_cast<unsigned>(2 * (c.sm_count / 2)), 1, 1);
      int ncl = 0;
      check_cuda(cudaOccupancyMaxActiveClusters(&ncl, gemm_tf32x3_pair_kernel, &cfg),
                 "cudaOccupancyMaxActiveClusters(gemm_tf32x3_pair)");
      if (ncl < 1) fail(OC_ERR_UNSUPPORTED, "gemm_tf32x3: no CTA pair fits on this device");
      max_clusters[dv] = ncl;
    }
    Params q = p;
    q.tiles_m = static_cast<int>((M + PM - 1) / PM);
    q.tiles_n = static_cast<int>((N + PN - 1) / PN);
    const int64_t clusters = std::min<int64_t>(pair_tiles, max_clusters[dv]);
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
    check_cuda(cudaLaunchKernelEx(&cfg, gemm_tf32x3_pair_kernel, mAh, mAl, mBh, mBl, mC, q),
               "cudaLaunchKernelEx(gemm_tf32x3_pair)");
    check_launch("gemm_tf32x3_pair_kernel");
    return;
  }
  const int64_t n_tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  const int grid = static_cast<int>(std::min<int64_t>(n_tiles, c.sm_count));
  set_attr_once(c.device);
  gemm_tf32x3_kernel<<<grid, THREADS, SMEM_BYTES, c.stream>>>(mAh, mAl, mBh, mBl, mC, p);
  check_launch("gemm_tf32x3_kernel");
}

}  // namespace oc

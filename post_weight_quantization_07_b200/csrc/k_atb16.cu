// C += alpha * A^T B over calibration tokens on the 5th-generation tensor cores.
//
// A and B are token-major 16-bit activations ([n_tok x M], [n_tok x N], both
// bf16 or both fp16); the contraction runs over tokens, so both operands are
// MN-major in shared memory (features contiguous).  This is the Hessian
// accumulation H += 2 Xhat^T Xhat (A == B, upper tiles only, bf16) and QEP's
// cross product d = (X - Xhat)^T Xhat (all tiles, on the operands the pass
// described at the end of this comment prepares).
//
// Design: persistent clusters of two CTAs (one per SM) that share each MMA
// (tcgen05 cta_group::2).  A pair owns a 256 x 256 output tile: CTA r holds
// features [128r, 128r + 128) of the tile's A columns and of its B columns in
// its shared memory and rows [128r, 128r + 128) of the fp32 accumulator in its
// TMEM, so each SM loads 64 KB per 128-token stage for a 128 x 256 x 128 share
// of the MMA work (a lone CTA would need 96 KB).  384 threads per CTA:
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
//   warps 2, 3, 8..11  (optional) an elementwise pass beside the product:
//                the operands of the next token slice of QEP's cross product,
//                from X and Xhat.  The product is bound by the tensor cores
//                and leaves most of the memory bandwidth free; these warps use
//                it with plain 16-byte loads and stores (no shared memory,
//                which the ring fills).
// Work units are (output tile, token chunk); chunks are the outer index so
// that the clusters of one wave stream the same token window through L2, and
// the chunks of a last, partly filled round are cut into equal parts so that
// it spreads over every cluster (plan_units).
// Every wait is bounded; a wait that gives up records OC_ERR_TIMEOUT and the
// kernel winds down (both CTAs still meet at the final cluster barrier).
//
// Cross-product operands.  d = (X - Xhat)^T Xhat is formed from D = X - Xhat
// directly, not as X^T Xhat - Xhat^T Xhat (which cancels about 50 times when
// Xhat is X plus 2% noise).  D and Xhat enter the MMA as fp16 with one
// power-of-two scale s_j per feature: with H = 2 Xhat^T Xhat already formed,
// |Xhat[t][j]| <= sqrt(H_jj / 2), and s_j brings that bound below 2^14, so the
// scaled Xhat cannot overflow fp16 and its values keep fp16's 11 significant
// bits down to 2^-28 of the column's bound (bf16 values convert exactly there).
// Each difference is computed in fp32 (exact unless the two values differ in
// magnitude by more than 2^16), scaled by s_j (exact) and rounded once to
// fp16.  The epilogue multiplies d[i][j] by 1 / (s_i s_j), exactly.  D itself
// has no bound from H; should a scaled difference overflow fp16 (X far from
// Xhat), the pass raises a device flag, and three launches that do nothing
// unless it is raised clear d and redo the product on bf16 operands
// (D = bf16(X - Xhat), Xhat itself).  No host round trip decides it.

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
constexpr int THREADS = 384;
constexpr int DIFF_WARPS = 6;      // warps 2, 3 and 8..11
constexpr int DIFF_UNROLL = 8;     // 16-byte chunks of each input in flight per lane
constexpr uint16_t kBothCtas = 0x3;

// What a launch computes.
constexpr int kPlainBf16 = 0;    // A, B bf16, C += alpha A^T B
constexpr int kScaledF16 = 1;    // A, B fp16 scaled per feature, C[i][j] += alpha (A^T B)[i][j] / (s_i s_j)
constexpr int kBf16IfFlag = 2;   // as kPlainBf16, but only when *flag != 0 (else the launch returns at once)

struct Params {
  int64_t n_tok;
  int tiles_i, tiles_j, n_tiles;
  int kc_stages, n_kc;
  int64_t units;
  int64_t full_units;    // units [0, full_units) are whole chunks
  int split_k;           // each later unit is one of split_k parts of a chunk
  int upper_only;
  float alpha;
  int* status;
  int mode;
  const int* flag;       // kBf16IfFlag
  int stall;             // test of the failure path: stall on a barrier nothing releases
  const float* isc;      // kScaledF16: 1 / s_j, isc_n entries
  int64_t isc_n;
  // operand pass of the next token slice (xcount = 0: none): xcount 16-byte
  // chunks of 8 values, row_chunks per token row, column scales psc
  const uint4* px;
  const uint4* pxh;
  uint4* pd;
  uint4* ph16;
  const float* psc;
  int* ovf;
  int64_t xcount;
  int64_t row_chunks;
};

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two fp32 values rounded to fp16 (to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t f16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Either half an infinity or NaN (exponent field all ones).
__device__ __forceinline__ bool f16x2_nonfinite(uint32_t h) {
  return ((h & 0x7C00u) == 0x7C00u) || ((h & 0x7C000000u) == 0x7C000000u);
}

// Scaled fp16 operands from one pair of bf16 words (features 2k, 2k+1 with
// scales s0, s1): d = fp16((x - xh) s), h = fp16(xh s).
__device__ __forceinline__ void f16_pair(uint32_t x, uint32_t xh, float s0, float s1, uint32_t& d, uint32_t& h,
                                         bool& bad) {
  d = f16x2_rn((bf16_lo(x) - bf16_lo(xh)) * s0, (bf16_hi(x) - bf16_hi(xh)) * s1);
  h = f16x2_rn(bf16_lo(xh) * s0, bf16_hi(xh) * s1);
  bad |= f16x2_nonfinite(d) | f16x2_nonfinite(h);
}

// Two bf16 differences a - b, each the exact difference rounded once to bf16.
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The scaled fp16 operands of a token range: thread `tid` of `nthreads` keeps
// one 8-feature column chunk for the whole pass (its 8 scales in registers)
// and walks the token rows, DIFF_UNROLL rows in flight; threads beyond the
// last whole sweep of a row stay idle.  Raises *ovf if a value does not fit.
// X and Xhat are read once (streaming); the outputs are read by the next
// launch (a token slice later), after L2 has seen the rest of this one.
__device__ __forceinline__ void scaled_f16_pass(const uint4* __restrict__ x, const uint4* __restrict__ xh,
                                                uint4* __restrict__ d, uint4* __restrict__ h16,
                                                const float* __restrict__ sc, int* ovf, int64_t count,
                                                int64_t row_chunks, int64_t tid, int64_t nthreads) {
  const int64_t R = nthreads / row_chunks;   // rows per sweep
  if (tid >= R * row_chunks) return;
  const int64_t cc = tid % row_chunks;
  const int64_t rows = count / row_chunks;
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(sc) + 2 * cc);
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(sc) + 2 * cc + 1);
  bool bad = false;
  for (int64_t r0 = tid / row_chunks; r0 < rows; r0 += DIFF_UNROLL * R) {
    uint4 a[DIFF_UNROLL], b[DIFF_UNROLL];
#pragma unroll
    for (int u = 0; u < DIFF_UNROLL; ++u) {
      const int64_t r = r0 + u * R;
      if (r < rows) {
        a[u] = __ldcs(x + r * row_chunks + cc);
        b[u] = __ldcs(xh + r * row_chunks + cc);
      }
    }
#pragma unroll
    for (int u = 0; u < DIFF_UNROLL; ++u) {
      const int64_t r = r0 + u * R;
      if (r < rows) {
        uint4 dv, hv;
        f16_pair(a[u].x, b[u].x, s0.x, s0.y, dv.x, hv.x, bad);
        f16_pair(a[u].y, b[u].y, s0.z, s0.w, dv.y, hv.y, bad);
        f16_pair(a[u].z, b[u].z, s1.x, s1.y, dv.z, hv.z, bad);
        f16_pair(a[u].w, b[u].w, s1.z, s1.w, dv.w, hv.w, bad);
        d[r * row_chunks + cc] = dv;
        h16[r * row_chunks + cc] = hv;
      }
    }
  }
  if (bad) *ovf = 1;
}

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

// Unit u -> output tile and token stages [ks0, ks1).  Units are chunk-major
// (the clusters of one round stream the same token window through L2).  The
// chunks that would form a last, partly filled round are cut into split_k
// parts, so that the last round spreads over every cluster.
__device__ __forceinline__ void decode_unit(const Params& p, int64_t u, int64_t stages_total, int& tile,
                                            int64_t& ks0, int64_t& ks1) {
  int64_t b = u, part = 0, k = 1;
  if (u >= p.full_units) {
    k = p.split_k;
    b = p.full_units + (u - p.full_units) / k;
    part = (u - p.full_units) % k;
  }
  tile = static_cast<int>(b % p.n_tiles);
  const int64_t c0 = (b / p.n_tiles) * p.kc_stages;
  const int64_t len = ::min(stages_total, c0 + p.kc_stages) - c0;
  ks0 = c0 + len * part / k;
  ks1 = c0 + len * (part + 1) / k;
}

__global__ void __launch_bounds__(THREADS, 1)
atb16_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
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
  uint64_t* stall_bar = drain + 1;       // [1], never arrived on (the test stall)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stall_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // the same decision in every thread of every CTA, before any barrier
  if (p.mode == kBf16IfFlag && *p.flag == 0) return;

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
    mbar_init(stall_bar, 1);
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

  if (p.stall) {
    // Test of the failure path: one thread waits on a barrier that nothing
    // arrives on.  The bounded wait gives up, records OC_ERR_TIMEOUT and
    // raises the abort flag before any copy or MMA is issued, so every role
    // below stops at its first wait and the kernel winds down normally.
    if (threadIdx.x == 0 && !mbar_wait(stall_bar, 0)) {
      record_error(p.status, kDevTimeout);
      *abort_flag = 1;
    }
    __syncthreads();
  }

  const int64_t stages_total = (p.n_tok + BK - 1) / BK;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    uint64_t issued = 0;
    bool ok = true;
    for (int64_t u = cid; u < p.units && ok; u += ncl) {
      int tile, ti, tj;
      int64_t ks0, ks1;
      decode_unit(p, u, stages_total, tile, ks0, ks1);
      decode_tile(p, tile, ti, tj);
      for (int64_t ks = ks0; ks < ks1; ++ks) {
        const int s = static_cast<int>(issued % STAGES);
        const uint32_t ph = static_cast<uint32_t>((issued / STAGES) & 1);
        int w = 1;
        if (lane == 0) w = mbar_wait_or_abort(&empty[s], ph ^ 1, abort_flag) && !*abort_flag;
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
      const uint32_t fmt = (p.mode == kScaledF16) ? 0u : 1u;  // 0 fp16, 1 bf16
      const uint32_t idesc = instr_desc(fmt, fmt, true, true, TM, TN);
      uint64_t consumed = 0;
      int it = 0;
      bool ok = true;
      for (int64_t u = cid; u < p.units && ok; u += ncl, ++it) {
        int tile;
        int64_t ks0, ks1;
        decode_unit(p, u, stages_total, tile, ks0, ks1);
        const int acc = it & 1;
        int w = 1;
        if (lane == 0) w = mbar_wait_or_abort(&tempty[acc], static_cast<uint32_t>(((it >> 1) & 1) ^ 1), abort_flag);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        tc_fence_after();
        const uint32_t dcol = tmem_base + static_cast<uint32_t>(acc * TN);
        for (int64_t ks = ks0; ks < ks1; ++ks) {
          const int s = static_cast<int>(consumed % STAGES);
          const uint32_t ph = static_cast<uint32_t>((consumed / STAGES) & 1);
          w = 1;
          if (lane == 0) w = mbar_wait_or_abort(&full[s], ph, abort_flag) && !*abort_flag;
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
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp - 4;  // TMEM lanes 32q .. 32q+31
    unsigned char* stage_buf = epi_base + q * 2 * EPI_BOX_BYTES;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int it = 0;
    int nbuf = 0;
    bool ok = true;
    for (int64_t u = cid; u < p.units; u += ncl, ++it) {
      int tile, ti, tj;
      int64_t ks0, ks1;
      decode_unit(p, u, stages_total, tile, ks0, ks1);
      decode_tile(p, tile, ti, tj);
      const int acc = it & 1;
      int w = 1;
      if (lane == 0) w = mbar_wait_or_abort(&tfull[acc], static_cast<uint32_t>((it >> 1) & 1), abort_flag) && !*abort_flag;
      w = __shfl_sync(0xffffffffu, w, 0);
      if (!w) { ok = false; break; }
      tc_fence_after();
      const int row0 = ti * TM + HM * static_cast<int>(rank) + 32 * q;
      // kScaledF16: row scale of this lane's row, column scales by shuffle
      const bool scaled = p.mode == kScaledF16;
      const float rs = scaled ? p.alpha * p.isc[::min(static_cast<int64_t>(row0 + lane), p.isc_n - 1)] : p.alpha;
      for (int c = 0; c < TN / 32; ++c) {
        const float cs = scaled ? p.isc[::min(static_cast<int64_t>(tj * TN + c * 32 + lane), p.isc_n - 1)] : 1.f;
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
          v.x = __uint_as_float(r[4 * k + 0]) * rs * __shfl_sync(0xffffffffu, cs, 4 * k + 0);
          v.y = __uint_as_float(r[4 * k + 1]) * rs * __shfl_sync(0xffffffffu, cs, 4 * k + 1);
          v.z = __uint_as_float(r[4 * k + 2]) * rs * __shfl_sync(0xffffffffu, cs, 4 * k + 2);
          v.w = __uint_as_float(r[4 * k + 3]) * rs * __shfl_sync(0xffffffffu, cs, 4 * k + 3);
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
  } else if (p.xcount > 0) {
    // ------------------------------------------------------------------ next slice's operands
    const int dw = (warp < 4) ? (warp - 2) : (warp - 6);  // 0 .. DIFF_WARPS-1
    const int64_t per_cta = DIFF_WARPS * 32;
    scaled_f16_pass(p.px, p.pxh, p.pd, p.ph16, p.psc, p.ovf, p.xcount, p.row_chunks,
                    static_cast<int64_t>(blockIdx.x) * per_cta + dw * 32 + lane,
                    static_cast<int64_t>(gridDim.x) * per_cta);
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

__global__ void __launch_bounds__(256) scaled_f16_kernel(const uint4* __restrict__ x, const uint4* __restrict__ xh,
                                                         uint4* __restrict__ d, uint4* __restrict__ h16,
                                                         const float* __restrict__ sc, int* ovf, int64_t count,
                                                         int64_t row_chunks) {
  scaled_f16_pass(x, xh, d, h16, sc, ovf, count, row_chunks, static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x,
                  static_cast<int64_t>(gridDim.x) * blockDim.x);
}

// The bf16 operands, written only when a pass raised the flag:
// D = bf16(X - Xhat) (each difference exact, rounded once) and Xhat copied.
__global__ void __launch_bounds__(256) bf16_operands_kernel(const uint4* __restrict__ x, const uint4* __restrict__ xh,
                                                            uint4* __restrict__ d, uint4* __restrict__ h16,
                                                            const int* flag, int64_t count) {
  if (*flag == 0) return;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
    const uint4 a = x[i], b = xh[i];
    d[i] = make_uint4(bf16x2_sub(a.x, b.x), bf16x2_sub(a.y, b.y), bf16x2_sub(a.z, b.z), bf16x2_sub(a.w, b.w));
    h16[i] = b;
  }
}

// d = 0 when the flag is raised (the fp16 products are then redone in bf16).
__global__ void zero_if_flag_kernel(float4* __restrict__ d, int64_t count4, const int* flag) {
  if (*flag == 0) return;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count4; i += stride)
    d[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Per-feature scales from the Hessian diagonal: s_j = 2^(14 - e_j) with
// sqrt(H_jj / 2) < 2^e_j (frexp), so s_j |Xhat[t][j]| < 2^14; sc[j] = s_j,
// sc[n + j] = 1 / s_j.  Exponents are kept within +-120 (both factors finite
// and exact); a zero or non-finite diagonal gives s_j = 1.
__global__ void column_scales_kernel(const float* __restrict__ H, int64_t n, float* __restrict__ sc) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const float h = H[j * n + j];
  int e = 14;
  if (h > 0.f && isfinite(h)) {
    int ex = 0;
    frexpf(sqrtf(0.5f * h) * 1.000001f, &ex);   // a hair above the bound: its own rounding cannot reach 2^14
    e = ::max(-120, ::min(120, 14 - ex));
  } else {
    e = 0;
  }
  sc[j] = ldexpf(1.f, e);
  sc[n + j] = ldexpf(1.f, -e);
}

}  // namespace

namespace {

bool g_stall_request = false;  // guarded by the library lock, like every launch

bool take_stall_request() {
  const bool r = g_stall_request;
  g_stall_request = false;
  return r;
}

// One token slice's operand pass for the fused launch (or a standalone one).
struct SlicePass {
  const void* X;
  const void* Xhat;
  void* D;
  void* Xh16;
  const float* sc;
  int* ovf;
  int64_t elems;
  int64_t n;
};

void launch_scaled_pass(const Ctx& c, const SlicePass& sp) {
  const int64_t count = sp.elems / 8, rc = sp.n / 8;
  if (count <= 0) return;
  const int64_t want = std::max<int64_t>(rc, (count + DIFF_UNROLL - 1) / DIFF_UNROLL);
  const int grid = static_cast<int>(std::max<int64_t>(
      (rc + 255) / 256, std::min<int64_t>((want + 255) / 256, static_cast<int64_t>(c.sm_count) * 4)));
  scaled_f16_kernel<<<grid, 256, 0, c.stream>>>(static_cast<const uint4*>(sp.X), static_cast<const uint4*>(sp.Xhat),
                                               static_cast<uint4*>(sp.D), static_cast<uint4*>(sp.Xh16), sp.sc, sp.ovf,
                                               count, rc);
  check_launch("scaled_f16_kernel");
}

void launch_atb16_ex(const Ctx& c, const void* A, const void* B, int64_t n_tok, int64_t M, int64_t N, float alpha,
                     float* C, int64_t ldc, bool upper_only, int max_ctas, int mode, const int* flag,
                     const float* isc, const SlicePass* pass) {
  if (n_tok <= 0 || M <= 0 || N <= 0) {
    if (pass) launch_scaled_pass(c, *pass);
    return;
  }
  if ((M % 64) || (N % 64) || (ldc % 4)) fail(OC_ERR_INVALID_ARG, "atb16: bad sizes");
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
    check_cuda(cudaFuncSetAttribute(atb16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
               "cudaFuncSetAttribute(atb16)");
    cfg.gridDim = dim3(static_cast<unsigned>(2 * (c.sm_count / 2)), 1, 1);
    int ncl = 0;
    check_cuda(cudaOccupancyMaxActiveClusters(&ncl, atb16_kernel, &cfg), "cudaOccupancyMaxActiveClusters");
    if (ncl < 1) fail(OC_ERR_UNSUPPORTED, "atb16: no CTA pair fits on this device");
    max_clusters[dv] = ncl;
  }
  const int ctas = (max_ctas > 0 && max_ctas < c.sm_count) ? max_ctas : c.sm_count;
  const int64_t clusters_avail = std::max(1, std::min(ctas / 2, max_clusters[dv]));

  const UnitPlan plan = plan_units(n_tok, p.n_tiles, clusters_avail);
  p.kc_stages = static_cast<int>(plan.kc_stages);
  p.n_kc = static_cast<int>(plan.n_kc);
  p.split_k = plan.split_k;
  p.full_units = plan.full_units;
  p.units = plan.units;
  p.alpha = alpha;
  p.status = c.status;
  p.mode = mode;
  p.flag = flag;
  p.stall = take_stall_request() ? 1 : 0;
  p.isc = isc;
  p.isc_n = std::max(M, N);
  const int64_t clusters = std::min<int64_t>(p.units, clusters_avail);
  if (pass && pass->elems > 0) {
    // the pass needs every thread to keep one column chunk: at least a row's
    // worth of pass threads, else it runs as a launch of its own
    if (2 * clusters * DIFF_WARPS * 32 >= pass->n / 8) {
      p.px = static_cast<const uint4*>(pass->X);
      p.pxh = static_cast<const uint4*>(pass->Xhat);
      p.pd = static_cast<uint4*>(pass->D);
      p.ph16 = static_cast<uint4*>(pass->Xh16);
      p.psc = pass->sc;
      p.ovf = pass->ovf;
      p.xcount = pass->elems / 8;
      p.row_chunks = pass->n / 8;
    } else {
      launch_scaled_pass(c, *pass);
    }
  }
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  check_cuda(cudaLaunchKernelEx(&cfg, atb16_kernel, mA, mB, mC, p), "cudaLaunchKernelEx(atb16)");
  check_launch("atb16_kernel");
}

}  // namespace

UnitPlan plan_units(int64_t n_tok, int64_t n_tiles, int64_t clusters) {
  UnitPlan u{};
  const int64_t stages_total = (n_tok + BK - 1) / BK;
  // Token chunk per unit: long enough to amortise the epilogue (at most 8192
  // tokens, so that the clusters of a round share an L2-sized token window),
  // and at least one unit per cluster.
  const int64_t want_chunks = std::max<int64_t>(1, (clusters + n_tiles - 1) / n_tiles);
  int64_t kcs = (stages_total + want_chunks - 1) / want_chunks;
  kcs = std::max<int64_t>(1024 / BK, std::min<int64_t>(8192 / BK, kcs));
  kcs = std::min(kcs, stages_total);
  u.kc_stages = kcs;
  u.n_kc = (stages_total + kcs - 1) / kcs;
  const int64_t chunks = u.n_kc * n_tiles;
  // The units go round the clusters in order.  When the chunks do not fill
  // the last round, the leftover ones are cut into k parts: a cluster then
  // ends with ceil(left k / clusters) parts of 1/k chunk instead of one whole
  // chunk or none (the 256 tiles of a 4096-feature cross product over 70
  // clusters: 3 chunks + 2 thirds each, in place of 3 or 4 chunks).  Parts
  // keep at least 8 stages.
  const int64_t left = chunks % clusters;
  const int64_t last_len = stages_total - (u.n_kc - 1) * kcs;
  const int64_t min_len = left <= n_tiles ? last_len : std::min(kcs, last_len);
  int best_k = 1;
  if (left > 0) {
    double best = 1.0;
    for (int k = 2; k <= 8 && min_len / k >= 8; ++k) {
      const double load = static_cast<double>((left * k + clusters - 1) / clusters) / k;
      if (load < best - 1e-9) {
        best = load;
        best_k = k;
      }
    }
  }
  u.split_k = best_k;
  u.full_units = chunks - (best_k > 1 ? left : 0);
  u.units = u.full_units + (chunks - u.full_units) * best_k;
  return u;
}

void request_test_stall() { g_stall_request = true; }

void launch_atb16(const Ctx& c, const void* A, const void* B, int64_t n_tok, int64_t M, int64_t N, float alpha,
                  float* C, int64_t ldc, bool upper_only, int max_ctas) {
  launch_atb16_ex(c, A, B, n_tok, M, N, alpha, C, ldc, upper_only, max_ctas, kPlainBf16, nullptr, nullptr, nullptr);
}

size_t cross_scratch_bytes(int64_t n_tok, int64_t n) {
  // D and Xhat as 16-bit values, 2n column scales, the overflow flag
  return 2 * (static_cast<size_t>(n_tok) * n * 2 + 256) + (2 * static_cast<size_t>(n) * 4 + 256) + 256;
}

void launch_cross_product(const Ctx& c, const void* X, const void* Xhat, int64_t n_tok, int64_t n, const float* H,
                          float* d, void* scratch, int parts, int max_ctas) {
  if (n % 64) fail(OC_ERR_INVALID_ARG, "cross product: n must be a multiple of 64");
  check_cuda(cudaMemsetAsync(d, 0, static_cast<size_t>(n) * n * sizeof(float), c.stream), "memset d");
  if (n_tok <= 0) return;
  if (!aligned16(X) || !aligned16(Xhat) || !aligned16(scratch))
    fail(OC_ERR_INVALID_ARG, "cross product: X, Xhat and the scratch must be 16-byte aligned");
  // carve the scratch: D, Xh16, scales, flag (256-byte aligned pieces)
  const size_t tok_bytes = static_cast<size_t>(n_tok) * n * 2;
  unsigned char* base = static_cast<unsigned char*>(scratch);
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  unsigned char* Dp = base;
  unsigned char* Hp = base + up(tok_bytes);
  float* sc = reinterpret_cast<float*>(Hp + up(tok_bytes));
  int* flag = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(sc) + up(2 * static_cast<size_t>(n) * 4));
  check_cuda(cudaMemsetAsync(flag, 0, sizeof(int), c.stream), "clear flag");
  column_scales_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, c.stream>>>(H, n, sc);
  check_launch("column_scales_kernel");

  const unsigned char* xb = static_cast<const unsigned char*>(X);
  const unsigned char* hb = static_cast<const unsigned char*>(Xhat);
  const int64_t k = std::max<int64_t>(1, std::min<int64_t>(parts, n_tok / 64));
  const int64_t per = ((n_tok + k - 1) / k + 63) / 64 * 64;
  auto slice = [&](int64_t t0) {
    const int64_t len = std::min(per, n_tok - t0);
    const size_t off = static_cast<size_t>(t0) * n * 2;
    return SlicePass{xb + off, hb + off, Dp + off, Hp + off, sc, flag, len * n, n};
  };
  // slice 0 alone; then slice s on the tensor cores while the launch's idle
  // warps prepare slice s + 1
  const SlicePass first = slice(0);
  launch_scaled_pass(c, first);
  for (int64_t t0 = 0; t0 < n_tok; t0 += per) {
    const int64_t len = std::min(per, n_tok - t0);
    const size_t off = static_cast<size_t>(t0) * n * 2;
    const bool more = t0 + per < n_tok;
    const SlicePass next = more ? slice(t0 + per) : SlicePass{};
    launch_atb16_ex(c, Dp + off, Hp + off, len, n, n, 1.0f, d, n, false, max_ctas, kScaledF16, nullptr, sc + n,
                    more ? &next : nullptr);
  }
  // a difference that did not fit fp16: redo the product on bf16 operands
  // (each of these launches returns at once unless the flag is raised)
  const int64_t count = n_tok * n / 8;
  const int grid = static_cast<int>(std::min<int64_t>((count + 255) / 256, static_cast<int64_t>(c.sm_count) * 4));
  zero_if_flag_kernel<<<grid, 256, 0, c.stream>>>(reinterpret_cast<float4*>(d), n * n / 4, flag);
  check_launch("zero_if_flag_kernel");
  bf16_operands_kernel<<<grid, 256, 0, c.stream>>>(reinterpret_cast<const uint4*>(X), reinterpret_cast<const uint4*>(Xhat),
                                                  reinterpret_cast<uint4*>(Dp), reinterpret_cast<uint4*>(Hp), flag, count);
  check_launch("bf16_operands_kernel");
  launch_atb16_ex(c, Dp, Hp, n_tok, n, n, 1.0f, d, n, false, 0, kBf16IfFlag, flag, nullptr, nullptr);
}

void launch_mirror_upper(const Ctx& c, float* H, int64_t n) {
  const int64_t nb = (n + 31) / 32;
  dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>(nb));
  mirror_upper_kernel<<<grid, dim3(32, 8), 0, c.stream>>>(H, n);
  check_launch("mirror_upper_kernel");
}

}  // namespace oc

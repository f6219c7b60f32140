/*
 * oc.h -- C ABI of liboc.so: layer-wise GPTQ + QEP weight quantisation on one
 * NVIDIA B200 (sm_100a).
 *
 * The operations follow the quantisation pipeline of the OneComp pages:
 *   - the OneComp v1.1.0 release summary (easyvibecoding.app/curated/1062),
 *     section "量化錯誤傳播 (QEP)": Quantization Error Propagation corrects a
 *     layer's weights for the quantisation error of the layers before it;
 *     section "v1.1.0全新量化方法": group quantisation, e.g. 4-bit, groupsize 128;
 *   - the One Compression hub page (pomoai.com/hubs/FujitsuResearch/OneCompression),
 *     section "核心功能拆解", quantiser table: GPTQ, 2-4 bit Hessian-optimal
 *     rounding; API GPTQ(wbits, groupsize) with qep=True.
 * The pages print no equations; each call below states what it computes.
 *
 * Conventions shared by every call
 *   - All array arguments are DEVICE pointers on the current CUDA device,
 *     owned by the caller, row-major, densely packed (leading dimension = the
 *     number of columns).  The library never frees or retains them.
 *   - Calibration activations are token-major bf16 (the PyTorch activation
 *     layout): X[t * n + c] is channel c of token t.
 *   - W is d_out x d_in = m x n fp32.  n must be a positive multiple of 64
 *     (at most 49152 for QEP and GPTQ); m >= 1.  Pointers handed to the
 *     tensor-memory-access (TMA) paths (X, Xhat, H, W, codes) must be 16-byte aligned.
 *   - The stream argument is a cudaStream_t (NULL = legacy default stream).
 *     All work of a call is ordered on that stream.
 *   - The library owns one scratch workspace per device, grown on demand with
 *     cudaMalloc (which synchronises the device when it grows) and released by
 *     oc_workspace_release().  Calls that share a device must not overlap in
 *     time (they share the workspace and the device status word).
 *   - Return value: an oc_status.  Argument errors are detected on the host
 *     before anything is launched.  Errors found on the device (a non-positive
 *     pivot, a non-finite value, a bounded wait that ran out) are recorded in a
 *     device status word; in synchronous mode (the default) each call
 *     synchronises its stream and returns that status.  In asynchronous mode
 *     (oc_set_sync(0)) calls return OC_OK after launching and
 *     oc_stream_status() synchronises and reports the first recorded error.
 *   - oc_last_error() gives a human-readable detail of the last failure on the
 *     calling thread.
 */
#ifndef OC_H
#define OC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  OC_OK = 0,
  OC_ERR_INVALID_ARG = 1,  /* null pointer, bad size, unsupported combination of arguments */
  OC_ERR_UNSUPPORTED = 2,  /* valid request this build does not handle (e.g. not sm_100) */
  OC_ERR_NOT_SPD = 3,      /* a Cholesky pivot was <= 0: the (dampened) Hessian is not SPD */
  OC_ERR_NONFINITE = 4,    /* a NaN or Inf was met in an input or an intermediate */
  OC_ERR_TIMEOUT = 5,      /* a bounded on-device wait ran out (kernel gave up cleanly) */
  OC_ERR_CUDA = 6,         /* a CUDA runtime call failed; see oc_last_error() */
  OC_ERR_OOM = 7           /* the workspace could not be grown */
} oc_status;

/* Name of a status code ("OC_OK", ...). Never NULL. */
const char* oc_status_string(int status);

/* Detail text of the last failure on the calling thread ("" if none). */
const char* oc_last_error(void);

/* ABI version of this library (major * 100 + minor). */
int oc_version(void);

/* 1 (default): every call synchronises its stream and returns the device status.
 * 0: calls return after launching; use oc_stream_status() to collect errors. */
void oc_set_sync(int sync);

/* Synchronise `stream`, return the first device-side error recorded since the
 * last collection, and clear it. */
int oc_stream_status(void* stream);

/* Free this device's workspace (synchronises the device). */
int oc_workspace_release(void);

/* Per-phase device timing, for benchmarking.  When enabled, every phase of a
 * call (see oc_profile_phase_name) records a pair of CUDA events on the call's
 * stream around its kernels.  Off by default. */
int oc_profile_enable(int on);

/* Wait for the recorded events and write, per phase, the milliseconds and the
 * kernel launches accumulated since the last read into ms[0..max_phases) and
 * launches[0..max_phases) (either may be NULL); clears the record.  Returns
 * the number of phases. */
int oc_profile_read(double* ms, int64_t* launches, int max_phases);

/* Name of phase `phase` ("" when out of range). */
const char* oc_profile_phase_name(int phase);

/* Kernel launches made by this library since it was loaded. */
int64_t oc_launch_count(void);

/* Test of the failure path (no counterpart in the method).  The next launch of
 * the tensor-core product behind oc_hessian_accumulate, oc_qep_correct,
 * oc_qep_terms and the fused calls has one thread per CTA wait on an
 * on-device barrier that nothing releases.  That bounded wait gives up after
 * its limit (2 s), records OC_ERR_TIMEOUT in the status word and stops the
 * kernel before it issues any copy or MMA, so the call returns
 * OC_ERR_TIMEOUT (synchronous mode) with its outputs not computed, and the
 * device stays usable for the next call.  One-shot. */
int oc_test_inject_stall(void);

/* Test of host logic (no counterpart in the method; touches no device).  How
 * the tensor-core product over calibration tokens behind the Hessian and the
 * QEP cross product cuts its work for n_tok tokens, n_tiles output tiles and
 * `clusters` persistent CTA pairs: units of (tile, token chunk), chunks of
 * out[0] stages of 128 tokens, out[1] chunks; the units go round the clusters
 * in order, units [0, out[3]) are whole chunks and each later one is one of
 * out[2] equal parts of a leftover chunk, out[4] units in all.
 *   out  int64 [5], host memory, written.
 * Returns OC_ERR_INVALID_ARG unless n_tok, n_tiles and clusters are positive
 * and out is non-null. */
int oc_test_unit_plan(int64_t n_tok, int64_t n_tiles, int64_t clusters, int64_t* out);

/*
 * Hessian accumulation:  H += 2 * X^T X   (n x n, fp32)
 *
 * The Hessian of the layer-wise loss ||(W - Q) X^T||_F^2 with respect to a
 * row of the weights -- the matrix behind GPTQ's "Hessian-optimal rounding"
 * (One Compression hub page, section "核心功能拆解", quantiser table, GPTQ row).
 * Pass the inputs the quantised layer will see (X-hat); repeated calls over
 * token chunks accumulate (chunked calibration).
 *
 *   X      bf16 [n_tok x n], token-major (device).  Read only.
 *   n_tok  number of tokens, 0 <= n_tok < 2^31 - 64 (0 leaves H unchanged and X may be NULL).
 *   n      number of input channels (d_in), positive multiple of 64.
 *   H      fp32 [n x n] (device), read-modify-write.  Must be symmetric on entry
 *          (e.g. zeros, or the output of a previous call): the update is
 *          computed for the upper triangle, added in place, and the lower
 *          triangle is then overwritten with the mirror of the upper one.
 * Products are exact (bf16 x bf16 in fp32) and accumulated in fp32 on the
 * tensor cores (tcgen05, TMEM accumulators), split over token chunks whose
 * partial sums are added into H in fp32 (summation order not fixed).
 */
int oc_hessian_accumulate(const void* X, int64_t n_tok, int64_t n, float* H, void* stream);

/*
 * QEP weight correction (OneComp release summary, section "量化錯誤傳播 (QEP)"):
 *
 *   W_out = W + alpha * W d A^-1,   d = (X - Xhat)^T Xhat,
 *   A = Xhat^T Xhat + lam I,        lam = damp * mean(diag(Xhat^T Xhat)).
 *
 * W + W d A^-1 is the minimiser of ||W X^T - W' Xhat^T||_F^2 + lam ||W' - W||_F^2:
 * the weight that, fed the perturbed inputs Xhat, best reproduces the
 * full-precision output; alpha in [0, 1] moves that fraction of the way.
 * alpha == 0 returns W unchanged, bit for bit.
 *
 *   W      fp32 [m x n] (device), read only.
 *   X      bf16 [n_tok x n] full-precision inputs (device).
 *   Xhat   bf16 [n_tok x n] inputs the quantised layer sees (device).
 *   n_tok  >= 1.
 *   alpha  finite.   damp  >= 0 (damp == 0 requires Xhat^T Xhat to be SPD).
 *   H_opt  NULL, or fp32 [n x n] = 2 Xhat^T Xhat over the same tokens (from
 *          oc_hessian_accumulate); it then replaces the recomputation.
 *   W_out  fp32 [m x n] (device); may equal W (in place).
 * Errors: OC_ERR_NOT_SPD if A is not positive definite.
 */
int oc_qep_correct(const float* W, int64_t m, int64_t n, const void* X, const void* Xhat,
                   int64_t n_tok, float alpha, float damp, const float* H_opt,
                   float* W_out, void* stream);

/*
 * GPTQ quantisation with a per-group asymmetric min/max grid (One Compression
 * hub page, section "核心功能拆解": GPTQ 2-4 bit Hessian-optimal rounding,
 * GPTQ(wbits, groupsize); OneComp release summary, section "v1.1.0全新量化方法":
 * 4-bit, groupsize 128).  Steps:
 *   1. dead columns (H_jj == 0): H_jj := 1 and W[:, j] := 0;
 *   2. act_order: process columns by a stable descending sort of diag(H);
 *   3. H_d = H + damp * mean(diag H) * I;  U = upper Cholesky factor of H_d^-1;
 *   4. sweep columns in processing order: q = clip(rint(w/scale) + zero, 0, 2^b-1),
 *      e = (w - scale (q - zero)) / U_jj, later columns w_k -= e U_jk
 *      (inside blocks of 128 columns; a tensor-core GEMM applies each block's
 *      errors to all later columns);
 *   5. grid: scale = (max - min) / (2^b - 1), zero = clip(rint(-min/scale), 0, 2^b-1)
 *      over the group's values (min = max widens to [min-1, max+1]); without
 *      act_order taken at the group's first column from its current values,
 *      with act_order taken up front from W (after step 1); groups are
 *      contiguous in original column order;
 *   6. codes are packed per row as an LSB-first bitstream of wbits-bit codes
 *      along d_in in original column order (wbits = 3 crosses word boundaries).
 *
 *   W          fp32 [m x n] (device), read only (the library works on a copy).
 *   H          fp32 [n x n] symmetric (device), read only.
 *   wbits      2, 3 or 4.
 *   groupsize  -1 (one group per row), or a power of two 4..128 dividing n, or a
 *              multiple of 128 dividing n.
 *   damp       >= 0.   act_order  0 or 1.
 *   codes      uint32 [m x (n * wbits / 32)] (device), written.
 *   scales     fp32 [m x n/G] (device), written.   zeros  fp32 [m x n/G], integer
 *              valued, written.  (G = n when groupsize == -1.)
 *   perm_out   NULL, or int32 [n] (device): the processing order as original
 *              column indices (identity without act_order).
 * Errors: OC_ERR_NOT_SPD if H_d is not positive definite, OC_ERR_NONFINITE for
 * non-finite entries of diag(H).
 */
int oc_gptq_quantize(const float* W, int64_t m, int64_t n, const float* H, int wbits,
                     int groupsize, float damp, int act_order, uint32_t* codes,
                     float* scales, float* zeros, int32_t* perm_out, void* stream);

/*
 * One layer end to end (the OneComp pipeline's GPTQ + QEP step for one linear
 * layer, OneComp release summary section "量化錯誤傳播 (QEP)" and One
 * Compression hub page section "核心功能拆解"):
 *   H      = 2 Xhat^T Xhat                                (overwritten),
 *   W_out  = W + alpha W d A^-1  as oc_qep_correct with H_opt = H,
 *   codes, scales, zeros, perm_out = GPTQ of W_out with H as oc_gptq_quantize.
 * Same results as the three calls in sequence (within rounding), with less
 * work: GPTQ's dampened Hessian H + damp mean(diag H) I equals QEP's 2A when
 * no column is dead, so one factorisation serves both (QEP is applied in
 * GPTQ's processing order).  With dead columns the two dampening constants
 * differ and two factorisations are made.  The call reads the dead-column
 * count back to the host once (a short synchronisation of its stream).
 *   W         fp32 [m x n], read only.    X, Xhat  bf16 [n_tok x n].
 *   H         fp32 [n x n], written.      W_out    fp32 [m x n], written; must not alias W.
 *   wbits, groupsize, damp, act_order, codes, scales, zeros, perm_out:
 *             as oc_gptq_quantize.        alpha: as oc_qep_correct.
 */
int oc_quantize_layer(const float* W, int64_t m, int64_t n, const void* X, const void* Xhat,
                      int64_t n_tok, float alpha, float damp, int wbits, int groupsize,
                      int act_order, float* H, float* W_out, uint32_t* codes, float* scales,
                      float* zeros, int32_t* perm_out, void* stream);

/*
 * The layer's data-dependent terms over one shard of the calibration tokens:
 *   H_part = 2 Xhat^T Xhat,   D_part = X^T Xhat - Xhat^T Xhat  (= (X - Xhat)^T Xhat)
 * Both are sums over tokens, so the terms of a layer whose tokens are split
 * over several GPUs are the element-wise sums of every shard's terms (one
 * all-reduce); oc_quantize_from_terms then finishes the layer.  Same
 * arithmetic as the first stages of oc_quantize_layer.
 *   X, Xhat  bf16 [n_tok x n] (this shard);  n_tok >= 0 (0 gives zeros).
 *   H_part, D_part  fp32 [n x n], overwritten.
 */
int oc_qep_terms(const void* X, const void* Xhat, int64_t n_tok, int64_t n, float* H_part, float* D_part,
                 void* stream);

/*
 * oc_quantize_layer from the layer's global terms H = 2 Xhat^T Xhat and
 * D = (X - Xhat)^T Xhat (e.g. all-reduced oc_qep_terms of the token shards):
 * the QEP correction of W, then GPTQ of W_out with H.  Rows of W are
 * independent in both steps, so a layer whose rows are split over GPUs runs
 * this per shard of rows with the same H and D.
 *   W, W_out  fp32 [m x n] (W_out must not alias W).   H, D fp32 [n x n], read only.
 *   Other arguments and errors as oc_quantize_layer.
 */
int oc_quantize_from_terms(const float* W, int64_t m, int64_t n, const float* H, const float* D, float alpha,
                           float damp, int wbits, int groupsize, int act_order, float* W_out, uint32_t* codes,
                           float* scales, float* zeros, int32_t* perm_out, void* stream);

/*
 * Block Hadamard rotation along the features of each row:
 *   Y = X (I_{n/block} (x) H_block) / sqrt(block),
 * H_block the Sylvester Hadamard matrix (H_1 = [1], H_2k = [[H_k, H_k], [H_k, -H_k]]).
 * The rotation is orthonormal and symmetric, so rotating a layer's weight
 * rows (W H) and its input rows (X H, Xhat H) by the same matrix leaves its
 * output W X^T unchanged while spreading outlier channels over their block
 * before the Hessian is formed (OneComp release summary, section
 * "進階預處理與後處理": rotation preprocessing with online Hadamard transforms).
 *   X, Y    [rows x n] bf16 (bf16 = 1) or fp32 (bf16 = 0), row-major; Y may be X.
 *   block   a power of two in 2..4096 dividing n.
 * Sums in fp32, one rounding to the output type.
 */
int oc_hadamard_rotate(const void* X, int64_t rows, int64_t n, int block, void* Y, int bf16, void* stream);

/*
 * The relaxed layer-1 step of LPCD (layer-projected coordinate descent) for a
 * two-layer linear submodule y = x W1^T W2^T (OneComp release summary, LPCD
 * bullet of section "v1.1.0全新量化方法" and section "量化錯誤傳播 (QEP)"; One
 * Compression hub page, section "3. LPCD：子模块联合优化": related layers are
 * optimised together on a relaxed objective and each layer's solution is
 * projected with the layer-wise quantiser).  With the second layer held at
 * its quantised value B, the minimiser over the first layer of
 * ||x W1^T W2^T - xh W^T B^T||^2 (ridge-regularised on both sides) is
 *   W_out = (B^T B + mu I)^-1 B^T W2 V,   mu = damp * mean(diag(B^T B)),
 * where V is W1 corrected by QEP with alpha = 1 (oc_qep_correct); GPTQ of
 * W_out with the first layer's Hessian is the projection.
 *   B, W2   fp32 [m x d] row-major (quantised and full-precision second layer).
 *   V       fp32 [d x n] row-major.   W_out fp32 [d x n]; may alias V.
 *   d       a positive multiple of 64, at most 49152; m, n positive multiples of 4.
 * Arithmetic: 3xTF32 products on the tensor cores and the library's
 * inverse-Cholesky factorisation of B^T B + mu I.
 * Errors: OC_ERR_INVALID_ARG for null or unaligned pointers, bad sizes or a
 * negative damp; OC_ERR_NOT_SPD when B^T B + mu I is not positive definite
 * (a zero damp with B of rank below d).
 */
int oc_lpcd_left_project(const float* B, const float* W2, int64_t m, int64_t d, const float* V, int64_t n,
                         float damp, float* W_out, void* stream);

/*
 * Dequantise packed GPTQ output: out[i][j] = scales[i][g] * (q[i][j] - zeros[i][g]),
 * g = j / groupsize, q read from row i's LSB-first bitstream of wbits-bit codes
 * (the layout oc_gptq_quantize writes).  This is the weight the quantised
 * layer applies (One Compression hub page, section "核心功能拆解": the
 * quantised model's layers); it feeds the next layer's calibration inputs when
 * quantisation error is propagated through a chain of layers.
 *   codes   uint32 [m x n*wbits/32];  scales, zeros fp32 [m x n/groupsize].
 *   out     [m x n], fp32 (out_bf16 = 0) or bf16 rounded to nearest even (1).
 * Errors: OC_ERR_INVALID_ARG for null pointers, wbits outside 2..4, n*wbits
 * not a multiple of 32, or a groupsize that does not divide n.
 */
int oc_dequantize(const uint32_t* codes, const float* scales, const float* zeros, int64_t m, int64_t n,
                  int wbits, int groupsize, void* out, int out_bf16, void* stream);

/*
 * The quantised layer applied to a few activation rows straight from its
 * packed codes: y[b][i] = sum_j x[b][j] * scales[i][g] * (q[i][j] - zeros[i][g]),
 * g = j / groupsize (One Compression hub page, section "4. vLLM 插件：量化模型直接
 * 推理": quantised GPTQ models are served by inference from their codes; at
 * decode time a layer is a matrix-vector product whose cost is reading them).
 *   codes   uint32 [m x n*wbits/32], the layout oc_gptq_quantize writes.
 *   scales, zeros fp32 [m x n/groupsize].
 *   x       bf16 [batch x n] row-major, batch 1..8.    y fp32 [batch x m].
 *   n       a positive multiple of 32; groupsize dividing both n and 32, a
 *           multiple of 32 dividing n, or -1 (= n).
 * fp32 products and sums; each warp takes four output rows (two with more than
 * four activation rows) and reads their codes once.
 * Errors: OC_ERR_INVALID_ARG for null or unaligned codes/x, bad sizes or groups.
 */
int oc_dequant_gemv(const uint32_t* codes, const float* scales, const float* zeros, int64_t m, int64_t n,
                    int wbits, int groupsize, const void* x, int64_t batch, float* y, void* stream);

/*
 * Several layers that read the same calibration inputs, e.g. the q, k and v
 * projections of one attention block or gate and up of one MLP (the One
 * Compression hub page, section "核心功能拆解", quantises a model layer by
 * layer; layers fed the same activations have the same Hessian).  For each
 * layer l the results are those of oc_quantize_layer(W[l], m[l], ...) with
 * the shared n, X, Xhat and settings; H, the cross term d and the
 * inverse-Hessian factor depend only on the inputs and are computed once.
 *   count     1..16 layers.
 *   W, W_out, codes, scales, zeros: host arrays of `count` device pointers,
 *             each as in oc_quantize_layer for a layer of m[l] rows
 *             (m: host array of `count` row counts).  No W_out[l] may alias
 *             any W[k].
 *   H         fp32 [n x n], written once.   perm_out: the shared processing
 *             order (optional).
 * Errors are those of oc_quantize_layer; a bad argument of any layer fails
 * the call before any launch.
 */
int oc_quantize_layer_group(int count, const float* const* W, const int64_t* m, int64_t n,
                            const void* X, const void* Xhat, int64_t n_tok, float alpha, float damp,
                            int wbits, int groupsize, int act_order, float* H,
                            float* const* W_out, uint32_t* const* codes, float* const* scales,
                            float* const* zeros, int32_t* perm_out, void* stream);

/*
 * Allocation-free GPTQ (no counterpart in the paper: an addition for callers of
 * this library).  Some callers cannot have a library allocate device memory on
 * its own -- e.g. a process whose memory is entirely reserved for its own
 * caching allocator at start-up, or a service held to a fixed, pre-reserved
 * budget -- because the workspace that oc_gptq_quantize grows with cudaMalloc
 * (and the device-wide synchronisation of the cudaFree before a regrowth)
 * would fail or stall there.  This entry point takes the same steps as
 * oc_gptq_quantize, with the same arguments (its trailing updates run on the
 * CUDA cores in fp32, so results agree within rounding), but takes every byte of
 * scratch from one array built into the library (6 MiB per GPU, held by every
 * GPU that loads the library until the process exits) and never calls
 * cudaMalloc, cudaFree or any other allocating routine.  The caller still
 * passes all inputs and outputs.
 *   - Size limit: the layer must fit the 6 MiB scratch (about
 *     10 n^2 + m (5 n + 512) bytes), e.g. n = 512 with m <= 1024, or n = 256
 *     with m <= 3072; larger requests return OC_ERR_INVALID_ARG with the bytes
 *     needed in oc_last_error().
 *   - The first call on a device looks up the array's device address on that
 *     device (the device must be current); make that first call before any
 *     stream capture begins.  The address is looked up again only if the
 *     device's context was destroyed and re-created in between.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents (each call clears what must start at zero).  Calls that
 *     overlap on the GPU -- on different streams, or issued from different
 *     threads without waiting for the previous call's stream -- race on it and
 *     must not be issued.  On the host the call holds the same lock as every
 *     other entry point while it enqueues its work.
 *   - Always synchronous: the call waits for its stream and returns the
 *     device-side status (OC_ERR_NOT_SPD, OC_ERR_NONFINITE, ...), whatever
 *     oc_set_sync() says.
 */
int oc_gptq_quantize_noalloc(const float* W, int64_t m, int64_t n, const float* H, int wbits,
                             int groupsize, float damp, int act_order, uint32_t* codes,
                             float* scales, float* zeros, int32_t* perm_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* OC_H */

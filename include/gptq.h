/*
 * gptq.h — C ABI of the B200 (sm_100a) GPTQ layer-quantization library (libgptq_b200.so).
 *
 * The library computes GPTQ's per-layer hot path: the Hessian H = 2 X X^T / N of the
 * calibration activations, its damped inverse in upper-Cholesky form R (R^T R = H_λ^{-1}),
 * the column-by-column quantization of W to a fixed affine grid with lazy block error
 * feedback, and the dense bit-packing of the integer codes.
 *
 * Sources, cited by page title and section / equation:
 *   [T] "GPTQ 从零推导：4-bit 权重量化为什么能‘量化一列，补偿一列’" (hbblog.cn derivation tutorial)
 *   [W] "GPTQ 完全拆解：二阶信息驱动的权重量化，如何把 175B 模型塞进一张 A100" (pinghaoyang.com.cn)
 *
 * Conventions shared by every entry point
 *   - Every array argument is a DEVICE pointer owned by the caller, unless the parameter
 *     says "host".  The library never frees caller memory.
 *   - Matrices are dense and row-major with the row stride equal to their column count.
 *   - Work is enqueued asynchronously on the context's CUDA stream.  Only
 *     gptq_prepare_hinv and gptq_sync_status synchronize that stream.
 *   - Argument errors return GPTQ_ERR_ARG before anything is enqueued.  Errors found on
 *     the device (non-finite input, non-positive-definite matrix, a bounded wait that ran
 *     out) are recorded in a device status word and returned by the next
 *     gptq_sync_status (or by gptq_prepare_hinv, which synchronizes).
 *   - Scratch memory comes from the workspace given to gptq_create; a call whose needs
 *     exceed it returns GPTQ_ERR_NOMEM without enqueuing work.
 *   - gptq_last_error(ctx) describes the most recent host-side failure.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gptq_ctx gptq_ctx;

/* Status codes. */
enum {
  GPTQ_OK = 0,
  GPTQ_ERR_ARG = 1,        /* invalid argument (nothing enqueued) */
  GPTQ_ERR_CUDA = 2,       /* a CUDA runtime call or launch failed */
  GPTQ_ERR_NOT_PD = 3,     /* H_λ not positive definite after the damping retries */
  GPTQ_ERR_NONFINITE = 4,  /* NaN/Inf in X, H or W */
  GPTQ_ERR_TIMEOUT = 5,    /* a bounded on-device wait gave up */
  GPTQ_ERR_NOMEM = 6       /* workspace too small */
};

/* Element types of X and W. */
enum { GPTQ_BF16 = 0, GPTQ_F16 = 1, GPTQ_F32 = 2 };

/* Workspace bytes that gptq_prepare_hinv and gptq_quantize_layer need for a layer with m
 * output rows and d input columns (the larger of the two, plus the status block).  Pure
 * host function. */
size_t gptq_workspace_bytes(int64_t m, int64_t d, int act_order);

/* Creates a context bound to the current CUDA device and to `cuda_stream` (a cudaStream_t;
 * NULL = legacy default stream).  `workspace` is a caller-owned device buffer of
 * `workspace_bytes` bytes (>= 256); if `workspace` is NULL the library allocates
 * `workspace_bytes` itself and frees them in gptq_destroy.  The first 256 bytes hold the
 * device status word.  Returns GPTQ_OK, GPTQ_ERR_ARG or GPTQ_ERR_CUDA. */
int gptq_create(gptq_ctx** ctx, void* cuda_stream, void* workspace, size_t workspace_bytes);

/* Releases the context (and the workspace if the library allocated it). */
int gptq_destroy(gptq_ctx* ctx);

/* Text of the most recent host-side error on this context ("" if none).  Owned by ctx. */
const char* gptq_last_error(const gptq_ctx* ctx);

/* Number of kernels this context has launched so far (a host-side counter; no sync). */
uint64_t gptq_kernel_launches(const gptq_ctx* ctx);

/* Sets how long a pipelined kernel launched through this context waits for its next stage,
 * buffer or partial before it gives up (GPU clock cycles; 0 restores the default, 4e9 cycles,
 * about 2 s at the B200's clock).  A wait that runs out records GPTQ_ERR_TIMEOUT in the device
 * status word, and its CTA waits for the copies and tensor-core operations it has already issued
 * (a separate, fixed budget), frees its tensor memory and exits; the context stays usable.
 * Kernels that run on CTA pairs keep the default budget.  The pages have no counterpart: this is
 * the failure path of the library's own bounded waits, for callers that need a hang turned into an
 * error quickly and for testing that path.  Errors: ARG (cycles < 0). */
int gptq_set_wait_budget(gptq_ctx* ctx, int64_t cycles);

/* Stages that gptq_timing_read reports; every kernel launch counts under one of them.  The
 * a-numbers are the steps of the hot path: a1 Hessian, a2 preconditioning, a3 factorization
 * (base blocks, recursion GEMMs, copies), a4 grid fit, a5 column loop (working copy, column
 * blocks), a6 lazy trailing updates, a7 outputs in original order, a8 packing; then the W4A16
 * product and two-sided rounding. */
enum {
  GPTQ_STAGE_HESSIAN = 0, GPTQ_STAGE_PREPARE = 1, GPTQ_STAGE_FACTOR_BASE = 2,
  GPTQ_STAGE_FACTOR_GEMM = 3, GPTQ_STAGE_FACTOR_COPY = 4, GPTQ_STAGE_GRID = 5,
  GPTQ_STAGE_COLUMN = 6, GPTQ_STAGE_UPDATE = 7, GPTQ_STAGE_OUTPUT = 8, GPTQ_STAGE_PACK = 9,
  GPTQ_STAGE_DEQUANT = 10, GPTQ_STAGE_TWOSIDED = 11, GPTQ_STAGE_OTHER = 12,
  GPTQ_NUM_STAGES = 13
};

/* Per-stage kernel timing, for measurement.  on != 0: from now on every kernel this context
 * launches is bracketed by two CUDA events on its stream (which serializes it with its
 * neighbours: programmatic dependent launch no longer overlaps their set-up), the factorization
 * runs all its launches on the context stream (no second stream, so no two timed launches
 * overlap), and the records kept so far are dropped; on == 0: launches are no longer timed.
 * Errors: ARG. */
int gptq_timing_enable(gptq_ctx* ctx, int on);

/* Synchronizes on the last timed launch and adds up, per stage, the time between each timed
 * launch's two events (ms, host double[GPTQ_NUM_STAGES]) and the number of timed launches (host
 * int64_t[GPTQ_NUM_STAGES]); then drops the records.  Errors: ARG, CUDA. */
int gptq_timing_read(gptq_ctx* ctx, double* ms, int64_t* launches);

/* Synchronizes the context stream, returns and clears the device status word
 * (GPTQ_OK, GPTQ_ERR_NONFINITE, GPTQ_ERR_NOT_PD or GPTQ_ERR_TIMEOUT), or GPTQ_ERR_CUDA. */
int gptq_sync_status(gptq_ctx* ctx);

/* Hessian statistic, [T] §2.1 eq.(5) and §2.4 eq.(9); accumulated in batches as [T] §9.4
 * allows.  Computes S += Xc^T Xc for one token chunk:
 *   Xc      [n_chunk, d] token-major activations (row t = token t's input vector), of type
 *           `dtype` (GPTQ_BF16 / GPTQ_F16: tensor-core path, products exact in fp32;
 *           GPTQ_F32: CUDA-core fp32 path).
 *   S       [d, d] fp32.  Only the lower triangle (i >= j) is defined on return.
 *   n_total host int64: tokens accumulated so far.  If *n_total == 0, S is overwritten
 *           (not read); afterwards *n_total += n_chunk.
 * Then H = 2 S / n_total.  Errors: ARG (d < 1, n_chunk < 1, bad dtype, NULL pointers). */
int gptq_hessian_accumulate(gptq_ctx* ctx, const void* Xc, int dtype, int64_t n_chunk,
                            int64_t d, float* S, int64_t* n_total);

/* Preconditioning and inverse factor, [T] §10 (order: dead features, act-order permutation,
 * damping), eq.(12), §8.3 eq.(34), §9.1 eq.(37)-(40).
 *   S        [d, d] fp32, lower triangle read: the unnormalised statistic with
 *            H = 2 S / n_total when n_total > 0, or H itself when n_total <= 0.
 *            Overwritten with the permuted, normalised, undamped H' = Π H Π^T.
 *   percdamp damping ratio: λ = max(percdamp * mean(diag H'), 2^-23).
 *   act_order 0: π = identity; 1: π = stable argsort of diag(H) descending.
 *   R        [d, d] fp32 out: upper-triangular factor with R^T R = H_λ^{-1} and a positive
 *            diagonal, in processing order (strictly lower part set to 0).
 *   perm     [d] int32 out: perm[j] = original column processed at position j.
 *   dead     [d] uint8 out: 1 where diag(H) == 0 (original column order); such diagonal
 *            entries are replaced by 1 before damping.
 *   damp_used host float* (may be NULL): the λ finally used.
 *   retries  host int* (may be NULL): how many times percdamp was multiplied by 10 after a
 *            failed factorization ([T] §10 remark; at most 3).
 * Synchronizes the stream.  Errors: ARG, NOMEM, NONFINITE (non-finite diag of S),
 * NOT_PD (still not positive definite after 3 retries), CUDA. */
int gptq_prepare_hinv(gptq_ctx* ctx, float* S, int64_t n_total, int64_t d, float percdamp,
                      int act_order, float* R, int32_t* perm, uint8_t* dead,
                      float* damp_used, int* retries);

/* Column-by-column quantization with lazy block updates, [W] Algorithm 1, [T] §9.2-9.3
 * eq.(42)-(46) and §10; quantizer [T] eq.(36); static and dynamic groups [T] §8.3.
 *   W        [m, d] weights of type w_dtype (GPTQ_F16 / GPTQ_BF16 / GPTQ_F32), ORIGINAL
 *            column order; not modified.
 *   R, perm, dead  as produced by gptq_prepare_hinv for this layer's H.
 *   bits     1..8 (2, 3, 4 are the pages' cases); codes lie in 0 .. 2^bits - 1.
 *   group    -1 (one grid per row) or > 0 (one grid per `group` original columns; the last
 *            group may be shorter).  n_g = 1 or ceil(d / group).
 *   block    lazy block size B >= 1.  Blocks of up to 128 columns are run as given; a larger
 *            B is run as 128-column blocks, which gives the same result in exact arithmetic
 *            ([T] eq.(47)-(49)).
 *   grid_given 0: static groups: fit a min-max grid on the original W (range extended to
 *            contain 0, Δ = (max - min) / (2^b - 1), z = clip(rint(-min / Δ)); all-zero range
 *            -> Δ = 1) and write it to scales/zeros; 1: read scales/zeros as the fixed grid;
 *            2: dynamic groups ([T] §8.3): group k holds PROCESSING positions k g .. k g + g - 1
 *            and its grid is fitted by the same rule, per row, at the group's start from the
 *            current working weights (all earlier columns' compensation applied); scales/zeros
 *            are written and indexed by processing group, and original column π_j belongs to
 *            group j / g (the deployment metadata group_id[π_j] = j / g, from perm).  Needs
 *            group == 32 (with min(block, 128) a multiple of 32) or group == 128 (with
 *            block >= 128); otherwise ARG.
 *            3: static groups with a symmetric grid (the pages name symmetric grids beside the
 *            min-max fit, [T] §1.1): per (row, group) M = max |w| over the original columns,
 *            Δ = 2M / (2^b - 1) (M = 0 -> Δ = 1), z = 2^(b-1); written to scales/zeros.
 *            4: static groups with the ternary grid {-Δ, 0, +Δ} of the pages' extreme case
 *            ([W] section "extreme quantization: 2-bit and ternary", used there with g = 8):
 *            bits must be 2;
 *            Δ = M (M = 0 -> Δ = 1), z = 1, and codes lie in 0..2 (2 bits each when packed).
 *   scales   [m, n_g] fp32, zeros [m, n_g] int32 (in or out, see grid_given).
 *   codes    [m, d] uint8 out, W_hat [m, d] fp32 out (= Δ (c - z)), col_loss [d] fp32 out
 *            (Σ_rows ρ² / (2 R_jj²), [T] eq.(43)); all in ORIGINAL column order.
 * Asynchronous.  Errors: ARG, NOMEM; NONFINITE (W) via gptq_sync_status. */
int gptq_quantize_layer(gptq_ctx* ctx, const void* W, int w_dtype, int64_t m, int64_t d,
                        const float* R, const int32_t* perm, const uint8_t* dead, int bits,
                        int group, int block, int grid_given, float* scales, int32_t* zeros,
                        uint8_t* codes, float* W_hat, float* col_loss);

/* Size of the fixed device scratch used by gptq_quantize_layer_noalloc. */
#define GPTQ_NOALLOC_SCRATCH_BYTES (16u << 20)

/* gptq_quantize_layer for callers that cannot allocate device memory — for example code that
 * runs inside another allocator's hooks, or a process whose device memory is fully committed
 * before it loads this library.  It takes no context and no workspace: its scratch is one
 * file-scope device array of GPTQ_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU loading the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree or allocating
 * library routine.  The pages have no counterpart; the arithmetic is that of
 * gptq_quantize_layer.
 *   cuda_stream  the cudaStream_t to enqueue on (NULL = legacy default stream), current device.
 *   other arguments exactly as for gptq_quantize_layer.
 * The scratch must hold about 4 m (1024 + d / 48) + 12 d bytes, plus 5 m d bytes when perm is
 * not NULL; a layer that needs more returns GPTQ_ERR_ARG (the only work enqueued then clears
 * the scratch's status word).
 * Device memory: under CUDA's lazy module loading the array is reserved on a device when the
 * library's module is first loaded there, i.e. at the first call of this entry point on that
 * device (or at any earlier library call there).  A caller with a fixed device budget should make
 * that first call before committing the rest of the device's memory; if the module cannot be
 * loaded the call returns GPTQ_ERR_CUDA.  Every call looks up the array's device address on the
 * current device (cudaGetSymbolAddress, which allocates nothing); the first call on a device
 * should come before any stream capture.
 * `cuda_stream` must belong to the current device, else GPTQ_ERR_ARG.
 * The call synchronizes `cuda_stream` and returns the device status (GPTQ_OK or
 * GPTQ_ERR_NONFINITE) like gptq_sync_status.  If a launch fails after earlier kernels were
 * enqueued it synchronizes the stream too and returns GPTQ_ERR_CUDA.  Every call shares the one
 * array and it keeps the last call's contents: calls whose work overlaps on the GPU (other
 * streams or host threads) race and must be serialized by the caller. */
int gptq_quantize_layer_noalloc(void* cuda_stream, const void* W, int w_dtype, int64_t m,
                                int64_t d, const float* R, const int32_t* perm,
                                const uint8_t* dead, int bits, int group, int block,
                                int grid_given, float* scales, int32_t* zeros, uint8_t* codes,
                                float* W_hat, float* col_loss);

/* Dense packing of the codes ([T] §3.1 output table, §9.4: about m d b / 8 bytes, stored as
 * 32-bit words).  Layout: per row a little-endian bitstream in which code k occupies bits
 * [b k, b k + b); word w of the row holds stream bits [32 w, 32 w + 32); every row starts on
 * a new word.  codes [m, d] uint8 (values < 2^bits) -> packed [m, ceil(d bits / 32)] uint32.
 * Asynchronous.  Errors: ARG. */
int gptq_pack(gptq_ctx* ctx, const uint8_t* codes, int64_t m, int64_t d, int bits,
              uint32_t* packed);

/* Inverse of gptq_pack. */
int gptq_unpack(gptq_ctx* ctx, const uint32_t* packed, int64_t m, int64_t d, int bits,
                uint8_t* codes);

/* The consumer of the packed format: Y = X Ŵᵀ, the product of a W4A16 linear layer at inference
 * ([T] §1.2: codes stored, activations kept in FP16/BF16; [A] "how it works": the codes are
 * dequantized on the fly inside the fused kernel), with Ŵ[r, k] = Δ[r, g(k)] (c[r, k] - z[r, g(k)])
 * exactly as gptq_quantize_layer defines W_hat.
 *   X        [T, d] of type x_dtype (GPTQ_BF16 / GPTQ_F16 / GPTQ_F32), token-major, device.
 *   packed   [m, ceil(d bits / 32)] uint32 in gptq_pack's layout, device; bits 1..8.
 *   group    -1 or > 0; group_id [d] int32 device or NULL.  NULL: column k uses grid column
 *            k / group (0 for group -1), as static groups do; otherwise group_id[k] (dynamic
 *            groups under act-order: group_id[π_j] = j / g).
 *   n_g      grid columns per row (the row stride of scales / zeros); with group_id NULL it
 *            must be at least ceil(d / group) (1 for group -1).
 *   scales   [m, n_g] fp32, zeros [m, n_g] int32, device; on the tensor path the zeros
 *            must lie in 0..15 (any 4-bit grid does), else ARG via gptq_sync_status.
 *   Y        [T, m] fp32 out (token-major), device.  T <= 524280.
 * 4-bit codes with 16-bit X (d % 32 == 0, X and packed 16-byte aligned, group -1 or a multiple
 * of 128, group_id NULL) run on the tensor cores: (c - z) is exact in X's 16-bit type and each
 * 128-column partial sum is scaled by its Δ in fp32.  Every other case runs on CUDA cores.
 * Split-K partials use the context workspace (T m per split, fp32); with too little workspace
 * the product runs unsplit.  Asynchronous.  Errors: ARG (also a group_id entry outside
 * [0, n_g), reported via gptq_sync_status), CUDA, TIMEOUT via gptq_sync_status. */
int gptq_dequant_matmul(gptq_ctx* ctx, const void* X, int x_dtype, int64_t T, int64_t d,
                        const uint32_t* packed, int64_t m, int bits, int group,
                        const int32_t* group_id, int64_t n_g, const float* scales,
                        const int32_t* zeros, float* Y);

/* A tile-contiguous copy of 4-bit packed codes for gptq_dequant_matmul_tiled: the codes of
 * 128 rows x 256 columns form one 16 KB tile (row blocks of 128, then column blocks of 256, in
 * row-major order of tiles); inside a tile row r takes 128 bytes, and its 16-byte chunk c (32
 * codes) is stored at position c XOR (r mod 8) of the row.  Rows and columns past the matrix are
 * zero.  The pages fix no layout for the deployed codes; this one lets the product read each
 * tile with one contiguous copy.
 *   packed   [m, d / 8] uint32 in gptq_pack's layout for 4-bit codes, d % 32 == 0, 16-byte
 *            aligned, device.
 *   tiled    gptq_tiled_words(m, d) uint32 out, 16-byte aligned, device.
 * Asynchronous.  Errors: ARG. */
long long gptq_tiled_words(int64_t m, int64_t d);
int gptq_retile_codes(gptq_ctx* ctx, const uint32_t* packed, int64_t m, int64_t d,
                      uint32_t* tiled);

/* gptq_dequant_matmul over the tile-contiguous codes, on the tensor path only: 4-bit codes, X
 * bf16 / f16 with d % 32 == 0 and 16-byte aligned, group -1 or a multiple of 128; the other
 * arguments as for gptq_dequant_matmul.  Asynchronous.  Errors: ARG, CUDA; ARG or TIMEOUT via
 * gptq_sync_status. */
int gptq_dequant_matmul_tiled(gptq_ctx* ctx, const void* X, int x_dtype, int64_t T, int64_t d,
                              const uint32_t* tiled, int64_t m, int group, int64_t n_g,
                              const float* scales, const int32_t* zeros, float* Y);

/* Two-sided rounding (GPTQ-2D, [D] "GPTQ-2D：把一个"四次方"难题压回"三次方"的故事"): X [m, n] is
 * rounded to an integer matrix Z for the metric ||A (Z - X) B||^2, given the metric factors
 * G_A = A^T A (m x m) and G_B = B B^T (n x n).  First each factor is turned in place into the
 * upper-triangular R with R^T R = G^{-1} (the reverse Cholesky and triangular inverse of
 * gptq_prepare_hinv, without damping):
 *   G        [k, k] fp32 symmetric positive definite, device; on return its upper triangle is R
 *            and its strict lower triangle is zero.
 * Synchronizes the stream.  Errors: ARG, NOMEM (workspace), NOT_PD, CUDA. */
int gptq_twosided_factor(gptq_ctx* ctx, float* G, int64_t k);

/* Then the rounding: the buffered row / column push of [D] (its Algorithm 3) over anti-diagonal
 * wavefronts (its Theorem 1), equal in exact arithmetic to one-dimensional GPTQ on the
 * vectorized problem with the Kronecker metric G_A ⊗ G_B:
 *   X        [m, n] fp32 row-major, device, not modified.
 *   RA       [m, m] and RB [n, n] from gptq_twosided_factor (row-major), device.
 *   Z        [m, n] fp32 out: the integers (round half to even of the compensated value).
 *   eta      [m, n] fp32 out: the scaled residuals η = (y - z) / (RA_ii RB_jj), whose squares
 *            sum to ||A (Z - X) B||^2.
 * Runs as a wavefront of 64 x 64 tiles: the cells of a tile in shared memory, the effects
 * between tiles as GEMMs.  Workspace: 3 m n + m^2 fp32.  Asynchronous.  Errors: ARG, NOMEM,
 * CUDA. */
int gptq_twosided_round(gptq_ctx* ctx, const float* X, int64_t m, int64_t n, const float* RA,
                        const float* RB, float* Z, float* eta);

#ifdef __cplusplus
}
#endif
#endif /* GPTQ_B200_H */

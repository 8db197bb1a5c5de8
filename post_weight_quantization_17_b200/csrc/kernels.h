// Host-side launchers of the library's kernels (internal; the C ABI is in include/gptq.h).
#pragma once
#include "common.cuh"

namespace gptq {

// ---- a1 Hessian statistic
int syrk_accumulate(Ctx* c, const void* X, int dtype, long long n, int d, float* S, bool overwrite);

// ---- a2 preconditioning
int prep_diag(Ctx* c, const float* S, int d, float scale, float* diagv, uint8_t* dead);
int prep_mean(Ctx* c, const float* diagv, int d);
int prep_perm(Ctx* c, const float* diagv, int d, int act_order, int32_t* perm);
// H' into Hp; with the identity order also into S itself (*wrote_S), else S is left as it was.
int prep_build(Ctx* c, float* S, int d, float scale, const float* diagv, const int32_t* perm,
               bool identity, float* Hp, bool* wrote_S);
int prep_copy(Ctx* c, const float* src, float* dst, size_t count);
int prep_damp(Ctx* c, float* Hl, int d, float percdamp);

// ---- a3 factorization: M (ld) holds H_λ (symmetric); on return its upper triangle is R with
// R^T R = H_λ^{-1} and its strict lower triangle is zero.  tmp: factor_tmp_floats(d) floats.
size_t factor_tmp_floats(int d);
int factor_inverse(Ctx* c, float* M, int d, float* tmp);

// ---- a4-a7 quantization
int grid_fit(Ctx* c, const void* W, int w_dtype, int m, int d, int maxq, bool symmetric,
             int group, float* scales, int32_t* zeros);
// grid index of each processing position: static groups floor(π_j / g), dynamic groups j / g
int make_gcol(Ctx* c, const int32_t* perm, int d, int group, bool dynamic, int32_t* gcol,
              int32_t* inv);
int init_work(Ctx* c, const void* W, int w_dtype, int m, int d, const int32_t* perm,
              const uint8_t* dead, bool identity, float* Wk);
// E (and, if not null, its tf32 halves Ehi / Elo) receive the block's scaled residuals.
// dyn = 32 or 128: dynamic groups of that many processing positions, whose grid the kernel
// fits and writes to scales/zeros; 0: the grid is read from scales/zeros.
int column_block(Ctx* c, float* Wk, int m, int d, int i, int nb, const float* R,
                 float* scales, int32_t* zeros, int ng, const int32_t* gcol,
                 bool uniform_grid, int dyn, int maxq, float* E, float* Ehi, float* Elo, int ldE,
                 uint8_t* codes, float* loss_part);
// Tail update on CTA pairs with operands split into tf32 halves (k_gemm_pair.cu):
// C = alpha A B + beta C, A [M, K] (lda), B [K, N] (ldb), both row-major.
bool gemm_pair_applies(int M, int N, int K, const float* Ah, long long lda, const float* Bh,
                       long long ldb, int num_sms);
int gemm_pair(Ctx* c, int M, int N, int K, const float* Ah, const float* Al, long long lda,
              const float* Bh, const float* Bl, long long ldb, float* C, long long ldc, float alpha,
              float beta);
// The general form: B either N-major ([K, N] row-major, ldb) or K-major (B(k, j) = Bh[j ldb + k]);
// structure flags of gemm_simt.cuh (kAUpper, kALower, kBUpper, kBLower restrict each tile's k
// range, kCUpper computes only tiles touching the upper triangle); with Ch / Cl set (and
// beta = 0) the result alpha A B is written as its tf32 halves there (row stride ldc), not to C.
struct GemmPairArgs {
  int M, N, K;
  const float *Ah, *Al;
  long long lda;
  const float *Bh, *Bl;
  long long ldb;
  bool b_kmajor;
  float* C;
  float *Ch, *Cl;
  long long ldc;
  float alpha, beta;
  int flags;
  // k-elements per TMEM partial (a multiple of 32; 0: 128).  The tensor core rounds its fp32
  // accumulator toward zero at every MMA, so a partial's error grows with the MMAs it sums;
  // products whose errors the factorization amplifies take short partials.
  int partial_k;
};
int gemm_pair(Ctx* c, const GemmPairArgs& g);
// k-elements per TMEM partial in the factorization's products (k_gemm_pair and k_gemm_tc)
constexpr int kFactorPartialK = 32;
// (hi, lo) halves of a rows x cols block; upper: the block's strict lower triangle as zeros
int split_tf32(Ctx* c, const float* src, long long lds, int rows, int cols, float* hi, float* lo,
               long long ldd, bool upper = false);
int trailing_update(Ctx* c, float* Wk, int m, int d, int i, int k, int c0, int c1,
                    const float* E, int ldE, const float* R);
int loss_reduce(Ctx* c, const float* loss_part, int parts, int d, float* loss_p);
int unpermute(Ctx* c, int m, int d, const int32_t* inv, const uint8_t* codes_p,
              const float* Wk, const float* loss_p, uint8_t* codes, float* W_hat,
              float* col_loss);

// ---- a8 packing
int pack_codes(Ctx* c, const uint8_t* codes, int m, int d, int bits, uint32_t* packed);
int unpack_codes(Ctx* c, const uint32_t* packed, int m, int d, int bits, uint8_t* codes);

// ---- the W4A16 consumer of the packed codes (k_dqmm.cu): Y [T, m] = X [T, d] Ŵᵀ
bool dequant_matmul_tc_applies(const void* X, int x_dtype, int d, const uint32_t* packed,
                               int bits, int group, const int32_t* group_id);
int dequant_matmul(Ctx* c, const void* X, int x_dtype, int T, int d, const uint32_t* packed,
                   int m, int bits, int group, const int32_t* group_id, int ng,
                   const float* scales, const int32_t* zeros, float* Y, float* part_ws,
                   size_t part_floats);
// the tile-contiguous layout of 4-bit codes (16 KB tiles of 128 rows x 256 codes, swizzled as the
// tensor kernel reads them) and the product over it
long long retile_words(long long m, long long d);
int retile_codes(Ctx* c, const uint32_t* packed, int m, int d, uint32_t* tiled);
int dequant_matmul_tiled(Ctx* c, const void* X, int x_dtype, int T, int d,
                         const uint32_t* tiled, int m, int group, int ng, const float* scales,
                         const int32_t* zeros, float* Y, float* part_ws, size_t part_floats);

// ---- two-sided rounding (GPTQ-2D, k_twosided.cu); workspace: Y, C, etas (m n floats each) and
// RAT (m m floats)
int twosided_round(Ctx* c, const float* X, int m, int n, const float* RA, const float* RB,
                   float* Z, float* eta, float* Y, float* C, float* etas, float* RAT);

constexpr int kColRows = 48;      // rows per column-block CTA (12 warps, 8 lanes per row)
constexpr int kColMax = 128;      // columns per kernel block
constexpr int kSuperCols = 1024;  // columns per super-block of the two-level lazy update

}  // namespace gptq

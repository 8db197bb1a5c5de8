// C ABI of the library (declared and documented in include/gptq.h).
#include <algorithm>
#include <new>

#include "kernels.h"

struct gptq_ctx {
  gptq::Ctx c;
};

using gptq::Carver;
using gptq::Ctx;

namespace {

inline bool valid_dtype(int t) { return t == GPTQ_BF16 || t == GPTQ_F16 || t == GPTQ_F32; }

size_t prep_bytes(int64_t d) {
  size_t b = gptq::kStatusBytes + 256 * 4;
  b += d * sizeof(float);
  b += gptq::factor_tmp_floats((int)d) * sizeof(float);
  return b;
}

// tf32 halves of E and of one super-block's slice of R for the pair tail GEMM (optional: a
// workspace without room for them runs the tail update on the single-CTA GEMM)
size_t pair_bytes(int64_t m, int64_t d) {
  return 256 * 4 + 2 * (size_t)m * gptq::kSuperCols * sizeof(float) +
         2 * (size_t)gptq::kSuperCols * (size_t)((d + 3) / 4 * 4) * sizeof(float);
}

size_t quant_bytes(int64_t m, int64_t d, bool general_perm) {
  size_t b = gptq::kStatusBytes + 256 * 10;
  b += 2 * d * sizeof(int32_t);                                  // gcol, inv
  b += (size_t)m * gptq::kSuperCols * sizeof(float);             // E of a super-block
  b += (size_t)((m + gptq::kColRows - 1) / gptq::kColRows) * d * sizeof(float);  // loss parts
  b += d * sizeof(float);                                        // loss in processing order
  if (general_perm) b += (size_t)m * d * (sizeof(float) + 1);    // W_work, codes (permuted)
  b += pair_bytes(m, d);                                         // optional: pair tail GEMM
  return b;
}

int read_status(Ctx* c, gptq::DeviceStatus* out) {
  GPTQ_CUDA_CHECK(c, cudaMemcpyAsync(out, c->status, sizeof(*out), cudaMemcpyDeviceToHost,
                                     c->stream));
  GPTQ_CUDA_CHECK(c, cudaStreamSynchronize(c->stream));
  return GPTQ_OK;
}

// Clears the error code and its location only; the cached reductions (mean diagonal, λ)
// survive so that a damping retry can reuse them.
int clear_status(Ctx* c) {
  GPTQ_CUDA_CHECK(c, cudaMemsetAsync(c->status, 0, 2 * sizeof(int), c->stream));
  return GPTQ_OK;
}

}  // namespace

extern "C" {

size_t gptq_workspace_bytes(int64_t m, int64_t d, int act_order) {
  if (m < 1 || d < 1) return gptq::kStatusBytes;
  return std::max(prep_bytes(d), quant_bytes(m, d, act_order != 0));
}

int gptq_create(gptq_ctx** out, void* stream, void* workspace, size_t workspace_bytes) {
  if (!out || workspace_bytes < gptq::kStatusBytes) return GPTQ_ERR_ARG;
  *out = nullptr;
  gptq_ctx* h = new (std::nothrow) gptq_ctx();
  if (!h) return GPTQ_ERR_NOMEM;
  Ctx* c = &h->c;
  c->stream = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaGetDevice(&c->device);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  if (e == cudaSuccess && !workspace) {
    void* p = nullptr;
    e = cudaMalloc(&p, workspace_bytes);
    workspace = p;
    c->owns_ws = (e == cudaSuccess);
  }
  if (e != cudaSuccess) {
    delete h;
    return GPTQ_ERR_CUDA;
  }
  c->ws = reinterpret_cast<char*>(workspace);
  c->ws_bytes = workspace_bytes;
  c->status = reinterpret_cast<gptq::DeviceStatus*>(c->ws);
  if (cudaMemsetAsync(c->ws, 0, gptq::kStatusBytes, c->stream) != cudaSuccess ||
      cudaStreamSynchronize(c->stream) != cudaSuccess) {
    if (c->owns_ws) cudaFree(c->ws);
    delete h;
    return GPTQ_ERR_CUDA;
  }
  *out = h;
  return GPTQ_OK;
}

int gptq_destroy(gptq_ctx* h) {
  if (!h) return GPTQ_ERR_ARG;
  for (cudaEvent_t e : h->c.event_pool) cudaEventDestroy(e);
  if (h->c.side) {
    cudaStreamSynchronize(h->c.side);
    for (int k = 0; k < 2 * 64; ++k)
      if (h->c.ev[k]) cudaEventDestroy(h->c.ev[k]);
    cudaStreamDestroy(h->c.side);
  }
  if (h->c.owns_ws) cudaFree(h->c.ws);
  delete h;
  return GPTQ_OK;
}

const char* gptq_last_error(const gptq_ctx* h) { return h ? h->c.last_error.c_str() : ""; }

uint64_t gptq_kernel_launches(const gptq_ctx* h) { return h ? h->c.launches : 0; }

int gptq_set_wait_budget(gptq_ctx* h, int64_t cycles) {
  if (!h) return GPTQ_ERR_ARG;
  if (cycles < 0) GPTQ_SET_ERR(&h->c, GPTQ_ERR_ARG, "set_wait_budget: cycles < 0");
  h->c.timeout_cycles = cycles == 0 ? gptq::kDefaultWaitCycles : (long long)cycles;
  return GPTQ_OK;
}

int gptq_timing_enable(gptq_ctx* h, int on) {
  if (!h) return GPTQ_ERR_ARG;
  h->c.timing = on != 0;
  if (on) {
    h->c.timed.clear();
    h->c.pool_used = 0;
  }
  return GPTQ_OK;
}

int gptq_timing_read(gptq_ctx* h, double* ms, int64_t* launches) {
  if (!h || !ms || !launches) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  for (int k = 0; k < GPTQ_NUM_STAGES; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  if (!c->timed.empty()) GPTQ_CUDA_CHECK(c, cudaEventSynchronize(c->timed.back().stop));
  for (const gptq::TimedLaunch& t : c->timed) {
    // a launch on the factorization's second stream may finish after the last one recorded
    GPTQ_CUDA_CHECK(c, cudaEventSynchronize(t.stop));
    float e = 0.f;
    GPTQ_CUDA_CHECK(c, cudaEventElapsedTime(&e, t.start, t.stop));
    const int k = (t.stage >= 0 && t.stage < GPTQ_NUM_STAGES) ? t.stage : GPTQ_STAGE_OTHER;
    ms[k] += e;
    launches[k] += 1;
  }
  c->timed.clear();
  c->pool_used = 0;
  return GPTQ_OK;
}

int gptq_sync_status(gptq_ctx* h) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  gptq::DeviceStatus st{};
  int rc = read_status(c, &st);
  if (rc) return rc;
  if (st.code) {
    c->last_error = "device status " + std::to_string(st.code) + " at " + std::to_string(st.where);
    if ((rc = clear_status(c))) return rc;
    return st.code;
  }
  return GPTQ_OK;
}

int gptq_hessian_accumulate(gptq_ctx* h, const void* Xc, int dtype, int64_t n_chunk, int64_t d,
                            float* S, int64_t* n_total) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!Xc || !S || !n_total || !valid_dtype(dtype) || d < 1 || d > (1 << 20) || n_chunk < 1 ||
      n_chunk > INT32_MAX || *n_total < 0)
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "hessian_accumulate: bad argument (d=%lld n_chunk=%lld)",
                 (long long)d, (long long)n_chunk);
  gptq::StageScope stage(c, GPTQ_STAGE_HESSIAN);
  int rc = gptq::syrk_accumulate(c, Xc, dtype, n_chunk, (int)d, S, *n_total == 0);
  if (rc) return rc;
  *n_total += n_chunk;
  return GPTQ_OK;
}

int gptq_prepare_hinv(gptq_ctx* h, float* S, int64_t n_total, int64_t d, float percdamp,
                      int act_order, float* R, int32_t* perm, uint8_t* dead, float* damp_used,
                      int* retries) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!S || !R || !perm || !dead || d < 1 || d > 65535 || !(percdamp >= 0.f) || S == R)
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "prepare_hinv: bad argument (d=%lld)", (long long)d);
  Carver cv(c);
  float* diagv = cv.take<float>(d);
  float* tmp = cv.take<float>(gptq::factor_tmp_floats((int)d));
  if (!cv.ok())
    GPTQ_SET_ERR(c, GPTQ_ERR_NOMEM, "prepare_hinv: workspace %zu < %zu bytes", c->ws_bytes, cv.off);
  const int di = (int)d;
  const float scale = n_total > 0 ? (float)(2.0 / (double)n_total) : 1.f;
  const size_t dd = (size_t)d * d;
  gptq::StageScope stage(c, GPTQ_STAGE_PREPARE);
  int rc;
  if ((rc = gptq::prep_diag(c, S, di, scale, diagv, dead))) return rc;
  if ((rc = gptq::prep_mean(c, diagv, di))) return rc;
  if ((rc = gptq::prep_perm(c, diagv, di, act_order, perm))) return rc;
  bool wrote_S = false;
  if ((rc = gptq::prep_build(c, S, di, scale, diagv, perm, !act_order, R, &wrote_S))) return rc;
  if (!wrote_S && (rc = gptq::prep_copy(c, R, S, dd))) return rc;
  float pd = percdamp;
  for (int attempt = 0; attempt <= 3; ++attempt) {
    if (attempt > 0 && (rc = gptq::prep_copy(c, S, R, dd))) return rc;
    if ((rc = gptq::prep_damp(c, R, di, pd))) return rc;
    if ((rc = gptq::factor_inverse(c, R, di, tmp))) return rc;
    gptq::DeviceStatus st{};
    if ((rc = read_status(c, &st))) return rc;
    if (st.code == 0) {
      if (damp_used) *damp_used = st.lam;
      if (retries) *retries = attempt;
      return GPTQ_OK;
    }
    if ((rc = clear_status(c))) return rc;
    if (st.code != GPTQ_ERR_NOT_PD) {
      c->last_error = "prepare_hinv: device status " + std::to_string(st.code) + " at " +
                      std::to_string(st.where);
      return st.code;
    }
    pd *= 10.f;
  }
  if (retries) *retries = 3;
  GPTQ_SET_ERR(c, GPTQ_ERR_NOT_PD, "prepare_hinv: H not positive definite after 3 retries");
}

int gptq_quantize_layer(gptq_ctx* h, const void* W, int w_dtype, int64_t m, int64_t d,
                        const float* R, const int32_t* perm, const uint8_t* dead, int bits,
                        int group, int block, int grid_given, float* scales, int32_t* zeros,
                        uint8_t* codes, float* W_hat, float* col_loss) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!W || !R || !scales || !zeros || !codes || !W_hat || !col_loss || !valid_dtype(w_dtype) ||
      m < 1 || d < 1 || m > INT32_MAX || d > INT32_MAX || (long long)m * d > (1LL << 40) ||
      bits < 1 || bits > 8 || !(group == -1 || group > 0) || block < 1 || grid_given < 0 ||
      grid_given > 4 || (grid_given == 4 && bits != 2))
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "quantize_layer: bad argument (m=%lld d=%lld bits=%d group=%d block=%d)",
                 (long long)m, (long long)d, bits, group, block);
  // dynamic groups: a group is one 32-column sub-block or one 128-column block of the column
  // kernel, so that the grid is fitted on columns that are all current at its start
  const int dyn = (grid_given == 2) ? group : 0;
  if (dyn && !((dyn == 32 && std::min(block, gptq::kColMax) % 32 == 0) ||
               (dyn == 128 && block >= gptq::kColMax)))
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "quantize_layer: dynamic groups need group 32 (block a multiple of 32) or 128 (block >= 128), got group=%d block=%d",
                 group, block);
  const int mi = (int)m, di = (int)d;
  const bool general = perm != nullptr;
  const int g = (group == -1) ? di : group;
  const int ng = (di + g - 1) / g;
  const int parts = (mi + gptq::kColRows - 1) / gptq::kColRows;
  Carver cv(c);
  int32_t* gcol = cv.take<int32_t>(d);
  int32_t* inv = cv.take<int32_t>(d);
  float* E = cv.take<float>((size_t)m * gptq::kSuperCols);
  float* loss_part = cv.take<float>((size_t)parts * d);
  float* loss_p = cv.take<float>(d);
  float* Wk = W_hat;
  uint8_t* codes_p = codes;
  if (general) {
    Wk = cv.take<float>((size_t)m * d);
    codes_p = cv.take<uint8_t>((size_t)m * d);
  }
  if (!cv.ok())
    GPTQ_SET_ERR(c, GPTQ_ERR_NOMEM, "quantize_layer: workspace %zu < %zu bytes", c->ws_bytes, cv.off);
  const int ldr = (di + 3) / 4 * 4;
  float* Ehi = cv.take<float>((size_t)m * gptq::kSuperCols);
  float* Elo = cv.take<float>((size_t)m * gptq::kSuperCols);
  float* Rhi = cv.take<float>((size_t)gptq::kSuperCols * ldr);
  float* Rlo = cv.take<float>((size_t)gptq::kSuperCols * ldr);
  const bool pair_ws = cv.ok();
  if (!pair_ws) Ehi = Elo = Rhi = Rlo = nullptr;
  int rc;
  gptq::StageScope stage(c, GPTQ_STAGE_GRID);  // restores the caller's stage on return
  // largest code: 2^b - 1, or 2 for the ternary grid
  const int maxq = (grid_given == 4) ? 2 : (1 << bits) - 1;
  c->stage = GPTQ_STAGE_GRID;
  if ((grid_given == 0 || grid_given >= 3) &&
      (rc = gptq::grid_fit(c, W, w_dtype, mi, di, maxq, grid_given >= 3, group, scales, zeros)))
    return rc;
  c->stage = GPTQ_STAGE_COLUMN;
  if ((rc = gptq::make_gcol(c, perm, di, group, dyn != 0, gcol, general ? inv : nullptr))) return rc;
  if ((rc = gptq::init_work(c, W, w_dtype, mi, di, perm, dead, !general, Wk))) return rc;
  // Two-level lazy blocks ([T] eq.(46); exact in exact arithmetic by eq.(47)-(49)): columns
  // are quantized in tiles of bk <= 128; after a tile only the rest of its super-block of
  // sb = 8 bk columns is updated, and after a super-block one GEMM with K = sb updates the
  // remaining tail (a long K, so that the tail GEMM's read-modify-write of W is small beside
  // its products).
  const int bk = std::min(block, gptq::kColMax);
  const int sb = bk * (gptq::kSuperCols / gptq::kColMax);
  for (int s0 = 0; s0 < di; s0 += sb) {
    const int s1 = std::min(di, s0 + sb);
    for (int i = s0; i < s1; i += bk) {
      const int nb = std::min(bk, s1 - i);
      const bool uniform = dyn || (group == -1) || (!general && (i / g) == ((i + nb - 1) / g));
      float* Et = E + (i - s0);
      c->stage = GPTQ_STAGE_COLUMN;
      if ((rc = gptq::column_block(c, Wk, mi, di, i, nb, R, scales, zeros, ng, gcol, uniform,
                                   dyn, maxq, Et, Ehi ? Ehi + (i - s0) : nullptr,
                                   Elo ? Elo + (i - s0) : nullptr, gptq::kSuperCols, codes_p,
                                   loss_part)))
        return rc;
      c->stage = GPTQ_STAGE_UPDATE;
      if ((rc = gptq::trailing_update(c, Wk, mi, di, i, nb, i + nb, s1, Et, gptq::kSuperCols, R)))
        return rc;
    }
    // tail: W[:, s1:] -= E R[s0:s1, s1:], on CTA pairs with split operands where it applies
    const int tn = di - s1, tk = s1 - s0;
    c->stage = GPTQ_STAGE_UPDATE;
    if (tn > 0 && pair_ws && gptq::gemm_pair_applies(mi, tn, tk, Ehi, gptq::kSuperCols, Rhi, ldr,
                                                     c->num_sms)) {
      if ((rc = gptq::split_tf32(c, R + (long long)s0 * di + s1, di, tk, tn, Rhi, Rlo, ldr)))
        return rc;
      if ((rc = gptq::gemm_pair(c, mi, tn, tk, Ehi, Elo, gptq::kSuperCols, Rhi, Rlo, ldr, Wk + s1,
                                di, -1.f, 1.f)))
        return rc;
    } else if ((rc = gptq::trailing_update(c, Wk, mi, di, s0, tk, s1, di, E, gptq::kSuperCols, R))) {
      return rc;
    }
  }
  c->stage = GPTQ_STAGE_OUTPUT;
  if ((rc = gptq::loss_reduce(c, loss_part, parts, di, general ? loss_p : col_loss))) return rc;
  if (general &&
      (rc = gptq::unpermute(c, mi, di, inv, codes_p, Wk, loss_p, codes, W_hat, col_loss)))
    return rc;
  return GPTQ_OK;
}

int gptq_pack(gptq_ctx* h, const uint8_t* codes, int64_t m, int64_t d, int bits,
              uint32_t* packed) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!codes || !packed || m < 1 || d < 1 || m > INT32_MAX || d > INT32_MAX || bits < 1 || bits > 8)
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "pack: bad argument");
  gptq::StageScope stage(c, GPTQ_STAGE_PACK);
  return gptq::pack_codes(c, codes, (int)m, (int)d, bits, packed);
}

int gptq_unpack(gptq_ctx* h, const uint32_t* packed, int64_t m, int64_t d, int bits,
                uint8_t* codes) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!codes || !packed || m < 1 || d < 1 || m > INT32_MAX || d > INT32_MAX || bits < 1 || bits > 8)
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "unpack: bad argument");
  gptq::StageScope stage(c, GPTQ_STAGE_PACK);
  return gptq::unpack_codes(c, packed, (int)m, (int)d, bits, codes);
}

int gptq_dequant_matmul(gptq_ctx* h, const void* X, int x_dtype, int64_t T, int64_t d,
                        const uint32_t* packed, int64_t m, int bits, int group,
                        const int32_t* group_id, int64_t n_g, const float* scales,
                        const int32_t* zeros, float* Y) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!X || !packed || !scales || !zeros || !Y || !valid_dtype(x_dtype) || T < 1 || d < 1 ||
      m < 1 || T > 65535LL * 8 || d > INT32_MAX || m > INT32_MAX || bits < 1 || bits > 8 ||
      !(group == -1 || group > 0) || n_g < 1 || n_g > INT32_MAX ||
      (!group_id && n_g < (group == -1 ? 1 : (d + group - 1) / group)))
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "dequant_matmul: bad argument (T=%lld d=%lld m=%lld bits=%d group=%d n_g=%lld)",
                 (long long)T, (long long)d, (long long)m, bits, group, (long long)n_g);
  Carver cv(c);
  const size_t avail = (c->ws_bytes > gptq::kStatusBytes + 256)
                            ? (c->ws_bytes - gptq::kStatusBytes - 256) / 4
                            : 0;
  float* part = cv.take<float>(0);
  gptq::StageScope stage(c, GPTQ_STAGE_DEQUANT);
  return gptq::dequant_matmul(c, X, x_dtype, (int)T, (int)d, packed, (int)m, bits, group,
                              group_id, (int)n_g, scales, zeros, Y, part, avail);
}

long long gptq_tiled_words(int64_t m, int64_t d) {
  if (m < 1 || d < 1) return 0;
  return gptq::retile_words(m, d);
}

int gptq_retile_codes(gptq_ctx* h, const uint32_t* packed, int64_t m, int64_t d,
                      uint32_t* tiled) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  if (!packed || !tiled || m < 1 || d < 1 || m > INT32_MAX || d > INT32_MAX || d % 32 != 0 ||
      !al(packed) || !al(tiled))
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "retile_codes: bad argument (m=%lld d=%lld)", (long long)m,
                 (long long)d);
  gptq::StageScope stage(c, GPTQ_STAGE_DEQUANT);
  return gptq::retile_codes(c, packed, (int)m, (int)d, tiled);
}

int gptq_dequant_matmul_tiled(gptq_ctx* h, const void* X, int x_dtype, int64_t T, int64_t d,
                              const uint32_t* tiled, int64_t m, int group, int64_t n_g,
                              const float* scales, const int32_t* zeros, float* Y) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  if (!X || !tiled || !scales || !zeros || !Y || !(x_dtype == GPTQ_BF16 || x_dtype == GPTQ_F16) ||
      T < 1 || d < 1 || m < 1 || T > 65535LL * 8 || d > INT32_MAX || m > INT32_MAX ||
      d % 32 != 0 || !al(X) || !al(tiled) || !(group == -1 || (group > 0 && group % 128 == 0)) ||
      n_g < (group == -1 ? 1 : (d + group - 1) / group) || n_g > INT32_MAX)
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "dequant_matmul_tiled: bad argument (T=%lld d=%lld m=%lld group=%d)",
                 (long long)T, (long long)d, (long long)m, group);
  Carver cv(c);
  const size_t avail = (c->ws_bytes > gptq::kStatusBytes + 256)
                            ? (c->ws_bytes - gptq::kStatusBytes - 256) / 4
                            : 0;
  float* part = cv.take<float>(0);
  gptq::StageScope stage(c, GPTQ_STAGE_DEQUANT);
  return gptq::dequant_matmul_tiled(c, X, x_dtype, (int)T, (int)d, tiled, (int)m, group,
                                    (int)n_g, scales, zeros, Y, part, avail);
}

int gptq_twosided_factor(gptq_ctx* h, float* G, int64_t k) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!G || k < 1 || k > 65535)
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "twosided_factor: bad argument (k=%lld)", (long long)k);
  Carver cv(c);
  float* tmp = cv.take<float>(gptq::factor_tmp_floats((int)k));
  if (!cv.ok())
    GPTQ_SET_ERR(c, GPTQ_ERR_NOMEM, "twosided_factor: workspace %zu < %zu bytes", c->ws_bytes, cv.off);
  int rc;
  {
    gptq::StageScope stage(c, GPTQ_STAGE_TWOSIDED);
    if ((rc = gptq::factor_inverse(c, G, (int)k, tmp))) return rc;
  }
  gptq::DeviceStatus st{};
  if ((rc = read_status(c, &st))) return rc;
  if (st.code == 0) return GPTQ_OK;
  if ((rc = clear_status(c))) return rc;
  if (st.code == GPTQ_ERR_NOT_PD)
    GPTQ_SET_ERR(c, GPTQ_ERR_NOT_PD, "twosided_factor: G not positive definite");
  c->last_error = "twosided_factor: device status " + std::to_string(st.code);
  return st.code;
}

int gptq_twosided_round(gptq_ctx* h, const float* X, int64_t m, int64_t n, const float* RA,
                        const float* RB, float* Z, float* eta) {
  if (!h) return GPTQ_ERR_ARG;
  Ctx* c = &h->c;
  if (!X || !RA || !RB || !Z || !eta || m < 1 || n < 1 || m > 65535 || n > 65535)
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "twosided_round: bad argument (m=%lld n=%lld)", (long long)m,
                 (long long)n);
  Carver cv(c);
  float* Y = cv.take<float>((size_t)m * n);
  float* C = cv.take<float>((size_t)m * n);
  float* etas = cv.take<float>((size_t)m * n);
  float* RAT = cv.take<float>((size_t)m * m);
  if (!cv.ok())
    GPTQ_SET_ERR(c, GPTQ_ERR_NOMEM, "twosided_round: workspace %zu < %zu bytes", c->ws_bytes, cv.off);
  gptq::StageScope stage(c, GPTQ_STAGE_TWOSIDED);
  return gptq::twosided_round(c, X, (int)m, (int)n, RA, RB, Z, eta, Y, C, etas, RAT);
}

}  // extern "C"

// api.cu -- C ABI entry points: argument checks, parameter block, codebook,
// launch sequencing.  See include/isoquant.h for the contract of each call.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "isoquant_internal.cuh"
#include "trace.cuh"

namespace isoquant {

// Lloyd's conditions for the 2^bits-level minimum-MSE quantizer of N(0,1):
// each decision threshold is the midpoint of its neighbouring levels and
// each level is the mean of the standard normal restricted to its cell,
// (pdf(a) - pdf(b)) / (cdf(b) - cdf(a)).  Iterated from evenly spaced levels;
// the levels are then rounded to fp16 (the stored decode values) and the
// thresholds taken as midpoints of the rounded levels.  Unused entries (past
// 2^bits) are zero.
int build_codebook(Codebook *cb, int bits) {
  const double inv_sqrt2pi = 0.39894228040143267794;
  auto pdf = [&](double z) { return inv_sqrt2pi * std::exp(-0.5 * z * z); };
  auto cdf = [](double z) { return 0.5 * std::erfc(-z * 0.70710678118654752440); };
  const int n = 1 << bits;
  *cb = Codebook{};
  cb->bits = bits;
  double lv[kMaxLevels], th[kMaxLevels - 1];
  for (int i = 0; i < n; ++i) lv[i] = 3.0 * (2.0 * i + 1.0 - n) / n;
  for (int iter = 0; iter < 200000; ++iter) {
    for (int k = 0; k < n - 1; ++k) th[k] = 0.5 * (lv[k] + lv[k + 1]);
    double moved = 0.0;
    for (int i = 0; i < n; ++i) {
      const double pa = i == 0 ? 0.0 : pdf(th[i - 1]);
      const double pb = i == n - 1 ? 0.0 : pdf(th[i]);
      const double ca = i == 0 ? 0.0 : cdf(th[i - 1]);
      const double cbv = i == n - 1 ? 1.0 : cdf(th[i]);
      const double c = (pa - pb) / (cbv - ca);
      moved = std::fmax(moved, std::fabs(c - lv[i]));
      lv[i] = c;
    }
    if (moved < 1e-15) break;
  }
  for (int i = 0; i < n; ++i) {
    const __half h = __double2half(lv[i]);
    cb->level16[i] = __half_as_ushort(h);
    cb->level[i] = __half2float(h);
  }
  for (int k = 0; k < n - 1; ++k) {
    cb->threshold64[k] = 0.5 * (static_cast<double>(cb->level[k]) + cb->level[k + 1]);
    cb->threshold[k] = static_cast<float>(cb->threshold64[k]);
  }
  return 0;
}

namespace {

// left multiplication by a: a (x) v = L(a) v;  right multiplication by c:
// v (x) c = Rm(c) v  (Hamilton product, quaternions as (w, x, y, z)).
void left_matrix(const double a[4], double m[16]) {
  const double t[16] = {a[0], -a[1], -a[2], -a[3], a[1], a[0], -a[3], a[2],
                        a[2], a[3],  a[0], -a[1], a[3], -a[2], a[1], a[0]};
  std::memcpy(m, t, sizeof(t));
}
void right_matrix(const double c[4], double m[16]) {
  const double t[16] = {c[0], -c[1], -c[2], -c[3], c[1], c[0], c[3], -c[2],
                        c[2], -c[3], c[0],  c[1], c[3], c[2], -c[1], c[0]};
  std::memcpy(m, t, sizeof(t));
}

bool build_head(const int8_t *signs, const float *quats, HeadParams *hp) {
  std::memset(hp, 0, sizeof(*hp));
  for (int j = 0; j < kD; ++j) {
    if (signs[j] != 1 && signs[j] != -1) return false;
    if (signs[j] < 0) hp->sign_bits[j >> 5] |= 1u << (j & 31);
  }
  for (int b = 0; b < kBlocks; ++b) {
    double ql[4], qr[4];
    for (int s = 0; s < 2; ++s) {
      const float *q = quats + (b * 2 + s) * 4;
      double n2 = 0.0;
      for (int c = 0; c < 4; ++c) {
        if (!std::isfinite(q[c])) return false;
        n2 += static_cast<double>(q[c]) * q[c];
      }
      if (!(n2 > 0.0)) return false;
      const double inv = 1.0 / std::sqrt(n2);
      double *dst = s == 0 ? ql : qr;
      for (int c = 0; c < 4; ++c) dst[c] = q[c] * inv;
    }
    // block b: v -> qL (x) v (x) conj(qR) = L(qL) Rm(conj qR) v
    const double cr[4] = {qr[0], -qr[1], -qr[2], -qr[3]};
    double Lm[16], Rm[16];
    left_matrix(ql, Lm);
    right_matrix(cr, Rm);
    for (int r = 0; r < 4; ++r)
      for (int c = 0; c < 4; ++c) {
        double acc = 0.0;
        for (int k = 0; k < 4; ++k) acc += Lm[4 * r + k] * Rm[4 * k + c];
        hp->m64[b][4 * r + c] = acc;
        hp->m32[b][4 * r + c] = static_cast<float>(acc);
      }
  }
  return true;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool valid_page_size(int ps) { return ps == 32 || ps == 64 || ps == 128 || ps == 256; }

int make_shape(const isoquant_ctx *ctx, int batch, int nq, int num_q_heads, int page_size, int causal,
               AttendShape *s) {
  if (batch < 0 || nq < 1 || num_q_heads < 1) return ISOQUANT_ERR_INVALID_ARG;
  if (num_q_heads % ctx->num_kv_heads != 0) return ISOQUANT_ERR_INVALID_ARG;
  // the kernels index rows, row groups x sequences and output rows in 32
  // bits: refuse shapes that would overflow them
  const int64_t rows = static_cast<int64_t>(nq) * (num_q_heads / ctx->num_kv_heads);
  const int64_t units = ((rows + 7) / 8) * static_cast<int64_t>(batch);
  const int64_t out_rows = static_cast<int64_t>(batch) * nq * num_q_heads;
  if (rows >= INT32_MAX || units >= INT32_MAX || units * ctx->num_kv_heads >= INT32_MAX || out_rows >= INT32_MAX)
    return ISOQUANT_ERR_INVALID_ARG;
  s->batch = batch;
  s->nq = nq;
  s->q_heads = num_q_heads;
  s->kv_heads = ctx->num_kv_heads;
  s->group = num_q_heads / ctx->num_kv_heads;
  s->rows = nq * s->group;
  s->row_groups = (s->rows + 7) / 8;
  s->page_size = page_size;
  s->causal = causal ? 1 : 0;
  s->bits = ctx->codebook.bits;
  s->n_cta = ctx->num_sms * attend_ctas_per_sm();
  s->slots = static_cast<size_t>(s->n_cta) +
             static_cast<size_t>(s->row_groups) * static_cast<size_t>(batch) * ctx->num_kv_heads;
  return ISOQUANT_OK;
}

}  // namespace

int attend_workspace_min(const isoquant_ctx *ctx, int batch, int nq, int num_q_heads, size_t *bytes) {
  AttendShape s;
  int st = make_shape(ctx, batch, nq, num_q_heads, 256, 0, &s);
  if (st != ISOQUANT_OK) return st;
  *bytes = attend_workspace_min_bytes(s);
  return ISOQUANT_OK;
}

namespace {

// The library launches on the device that is current; it must be the one
// the context's parameters live on.
int check_device(const isoquant_ctx *ctx) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ISOQUANT_ERR_CUDA;
  return dev == ctx->device ? ISOQUANT_OK : ISOQUANT_ERR_INVALID_ARG;
}

int check_cache(const isoquant_cache *cache) {
  if (cache == nullptr || cache->codes == nullptr || cache->norms == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  if (cache->num_pages < 1) return ISOQUANT_ERR_INVALID_ARG;
  if (!valid_page_size(cache->page_size)) return ISOQUANT_ERR_UNSUPPORTED;
  if (!aligned(cache->codes, 16) || !aligned(cache->norms, 16)) return ISOQUANT_ERR_ALIGNMENT;
  return ISOQUANT_OK;
}

int dtype_bytes(int dtype) {
  switch (dtype) {
    case ISOQUANT_F32: return 4;
    case ISOQUANT_BF16: return 2;
    case ISOQUANT_F16: return 2;
    default: return 0;
  }
}

}  // namespace
}  // namespace isoquant

using namespace isoquant;

// longest wait isoquant_selftest_wait accepts (10 s)
static constexpr uint64_t kSelftestMaxNs = 10000000000ull;

extern "C" {

const char *isoquant_strerror(int status) {
  switch (status) {
    case ISOQUANT_OK: return "ok";
    case ISOQUANT_ERR_INVALID_ARG: return "invalid argument";
    case ISOQUANT_ERR_UNSUPPORTED: return "unsupported (head_dim must be 128; dtype F32/BF16/F16; page size 32/64/128/256)";
    case ISOQUANT_ERR_OUT_OF_RANGE: return "index or length out of range";
    case ISOQUANT_ERR_WORKSPACE: return "workspace too small";
    case ISOQUANT_ERR_CUDA: return "CUDA runtime error";
    case ISOQUANT_ERR_ALIGNMENT: return "pointer not aligned (16 bytes required)";
    default: return "unknown status";
  }
}

int isoquant_codebook(float levels[8], float thresholds[7]) {
  return isoquant_codebook_bits(3, levels, thresholds);
}

int isoquant_codebook_bits(int bits, float *levels, float *thresholds) {
  if (levels == nullptr || thresholds == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  if (bits < 2 || bits > 4) return ISOQUANT_ERR_UNSUPPORTED;
  Codebook cb;
  build_codebook(&cb, bits);
  for (int i = 0; i < (1 << bits); ++i) levels[i] = cb.level[i];
  for (int k = 0; k < (1 << bits) - 1; ++k) thresholds[k] = cb.threshold[k];
  return ISOQUANT_OK;
}

int isoquant_init(isoquant_ctx **out, int num_kv_heads, int head_dim, const int8_t *signs, const float *quats) {
  return isoquant_init_bits(out, num_kv_heads, head_dim, signs, quats, 3);
}

int isoquant_init_bits(isoquant_ctx **out, int num_kv_heads, int head_dim, const int8_t *signs, const float *quats,
                       int bits) {
  ISOQUANT_TRACE("isoquant_init_bits");
  if (out == nullptr || signs == nullptr || quats == nullptr || num_kv_heads < 1) return ISOQUANT_ERR_INVALID_ARG;
  *out = nullptr;
  if (head_dim != kD || bits < 2 || bits > 4) return ISOQUANT_ERR_UNSUPPORTED;
  std::vector<HeadParams> host(static_cast<size_t>(num_kv_heads));
  for (int h = 0; h < num_kv_heads; ++h)
    if (!build_head(signs + static_cast<size_t>(h) * kD, quats + static_cast<size_t>(h) * kBlocks * 8, &host[h]))
      return ISOQUANT_ERR_INVALID_ARG;
  isoquant_ctx *ctx = new (std::nothrow) isoquant_ctx();
  if (ctx == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  build_codebook(&ctx->codebook, bits);
  ctx->num_kv_heads = num_kv_heads;
  if (cudaGetDevice(&ctx->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device) != cudaSuccess ||
      cudaMalloc(&ctx->params, sizeof(HeadParams) * num_kv_heads) != cudaSuccess ||
      cudaMalloc(&ctx->status, 16) != cudaSuccess ||
      cudaMemcpy(ctx->params, host.data(), sizeof(HeadParams) * num_kv_heads, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemset(ctx->status, 0, 16) != cudaSuccess) {
    if (ctx->params) cudaFree(ctx->params);
    if (ctx->status) cudaFree(ctx->status);
    delete ctx;
    return ISOQUANT_ERR_CUDA;
  }
  *out = ctx;
  return ISOQUANT_OK;
}

void isoquant_destroy(isoquant_ctx *ctx) {
  ISOQUANT_TRACE("isoquant_destroy");
  if (ctx == nullptr) return;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(ctx->device);
  cudaDeviceSynchronize();
  cudaFree(ctx->params);
  cudaFree(ctx->status);
  if (prev >= 0) cudaSetDevice(prev);
  delete ctx;
}

int isoquant_cache_bytes(const isoquant_ctx *ctx, int num_pages, int page_size, size_t *code_bytes,
                         size_t *norm_bytes) {
  if (ctx == nullptr || code_bytes == nullptr || norm_bytes == nullptr || num_pages < 0) return ISOQUANT_ERR_INVALID_ARG;
  if (!valid_page_size(page_size)) return ISOQUANT_ERR_UNSUPPORTED;
  const size_t vecs = static_cast<size_t>(num_pages) * 2 * ctx->num_kv_heads * page_size;
  *code_bytes = vecs * words_for(ctx->codebook.bits) * sizeof(uint32_t);
  *norm_bytes = vecs * sizeof(uint16_t);
  return ISOQUANT_OK;
}

int isoquant_compress_kv(isoquant_ctx *ctx, const isoquant_cache *cache, const void *k, const void *v, int dtype,
                         int n_tok, const int64_t *slot_mapping, void *stream) {
  ISOQUANT_TRACE("isoquant_compress_kv");
  if (ctx == nullptr || n_tok < 0) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  int st = check_cache(cache);
  if (st != ISOQUANT_OK) return st;
  const int eb = dtype_bytes(dtype);
  if (eb == 0) return ISOQUANT_ERR_UNSUPPORTED;
  if (n_tok == 0) return ISOQUANT_OK;
  if (k == nullptr || v == nullptr || slot_mapping == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  const uintptr_t need = eb == 4 ? 16 : 8;
  if (!aligned(k, need) || !aligned(v, need) || !aligned(slot_mapping, 8)) return ISOQUANT_ERR_ALIGNMENT;
  st = check_device(ctx);
  if (st != ISOQUANT_OK) return st;
  cudaError_t e = launch_compress(ctx, cache, k, v, dtype, n_tok, slot_mapping, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return ISOQUANT_ERR_CUDA;
  ctx->last_launches = 1;
  return ISOQUANT_OK;
}

int isoquant_rotate_q(isoquant_ctx *ctx, const void *q, int dtype, int n_rows, int num_q_heads, float *q_rot,
                      void *stream) {
  ISOQUANT_TRACE("isoquant_rotate_q");
  if (ctx == nullptr || n_rows < 0 || num_q_heads < 1) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  if (num_q_heads % ctx->num_kv_heads != 0) return ISOQUANT_ERR_INVALID_ARG;
  const int eb = dtype_bytes(dtype);
  if (eb == 0) return ISOQUANT_ERR_UNSUPPORTED;
  if (n_rows == 0) return ISOQUANT_OK;
  if (q == nullptr || q_rot == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  if (!aligned(q, eb == 4 ? 16 : 8) || !aligned(q_rot, 16)) return ISOQUANT_ERR_ALIGNMENT;
  const int dst = check_device(ctx);
  if (dst != ISOQUANT_OK) return dst;
  cudaError_t e = launch_rotate_q(ctx, q, dtype, n_rows, num_q_heads, q_rot, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return ISOQUANT_ERR_CUDA;
  ctx->last_launches = 1;
  return ISOQUANT_OK;
}

int isoquant_debug_export_z(isoquant_ctx *ctx, const void *x, int dtype, int n_tok, float *z, void *stream) {
  ISOQUANT_TRACE("isoquant_debug_export_z");
  if (ctx == nullptr || n_tok < 0) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  if (dtype_bytes(dtype) == 0) return ISOQUANT_ERR_UNSUPPORTED;
  if (n_tok == 0) return ISOQUANT_OK;
  if (x == nullptr || z == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(z, 16)) return ISOQUANT_ERR_ALIGNMENT;
  const int st = check_device(ctx);
  if (st != ISOQUANT_OK) return st;
  if (launch_export_z(ctx, x, dtype, n_tok, z, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ISOQUANT_ERR_CUDA;
  ctx->last_launches = 1;
  return ISOQUANT_OK;
}

int isoquant_decode_prep(isoquant_ctx *ctx, const isoquant_cache *cache, const void *k, const void *v, int n_tok,
                         const int64_t *slot_mapping, const void *q, int dtype, int n_rows, int num_q_heads,
                         float *q_rot, void *stream) {
  ISOQUANT_TRACE("isoquant_decode_prep");
  if (ctx == nullptr || n_tok < 0 || n_rows < 0 || num_q_heads < 1) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  int st = check_cache(cache);
  if (st != ISOQUANT_OK) return st;
  if (num_q_heads % ctx->num_kv_heads != 0) return ISOQUANT_ERR_INVALID_ARG;
  const int eb = dtype_bytes(dtype);
  if (eb == 0) return ISOQUANT_ERR_UNSUPPORTED;
  const uintptr_t need = eb == 4 ? 16 : 8;
  if (n_tok > 0) {
    if (k == nullptr || v == nullptr || slot_mapping == nullptr) return ISOQUANT_ERR_INVALID_ARG;
    if (!aligned(k, need) || !aligned(v, need) || !aligned(slot_mapping, 8)) return ISOQUANT_ERR_ALIGNMENT;
  }
  if (n_rows > 0) {
    if (q == nullptr || q_rot == nullptr) return ISOQUANT_ERR_INVALID_ARG;
    if (!aligned(q, need) || !aligned(q_rot, 16)) return ISOQUANT_ERR_ALIGNMENT;
  }
  if (n_tok == 0 && n_rows == 0) return ISOQUANT_OK;
  st = check_device(ctx);
  if (st != ISOQUANT_OK) return st;
  cudaError_t e = launch_decode_prep(ctx, cache, k, v, n_tok, slot_mapping, q, dtype, n_rows, num_q_heads, q_rot,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return ISOQUANT_ERR_CUDA;
  ctx->last_launches = 1;
  return ISOQUANT_OK;
}

namespace {
size_t round_up_256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }
}  // namespace

int isoquant_step_workspace_size(const isoquant_ctx *ctx, int batch, int nq, int num_q_heads, size_t *bytes) {
  if (ctx == nullptr || bytes == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  AttendShape s;
  int st = make_shape(ctx, batch, nq, num_q_heads, 256, 0, &s);
  if (st != ISOQUANT_OK) return st;
  *bytes = round_up_256(attend_workspace_bytes(s)) +
           static_cast<size_t>(batch) * nq * num_q_heads * kD * sizeof(float);
  return ISOQUANT_OK;
}

int isoquant_decode_step(isoquant_ctx *ctx, const isoquant_cache *cache, const void *k, const void *v, int n_tok,
                         const int64_t *slot_mapping, const void *q, int dtype, int batch, int nq, int num_q_heads,
                         const int32_t *page_table, int max_pages, const int32_t *seq_lens, int causal,
                         float scale, void *workspace, size_t ws_bytes, float *out, void *stream) {
  ISOQUANT_TRACE("isoquant_decode_step");
  if (ctx == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  size_t need = 0;
  int st = isoquant_step_workspace_size(ctx, batch, nq, num_q_heads, &need);
  if (st != ISOQUANT_OK) return st;
  int st_cache = check_cache(cache);
  if (st_cache != ISOQUANT_OK) return st_cache;
  if (batch == 0) {
    // nothing to attend; the new tokens are still appended
    return isoquant_compress_kv(ctx, cache, k, v, dtype, n_tok, slot_mapping, stream);
  }
  if (workspace == nullptr || out == nullptr || page_table == nullptr || seq_lens == nullptr || max_pages < 1)
    return ISOQUANT_ERR_INVALID_ARG;
  if (!aligned(workspace, 16) || !aligned(out, 16) || !aligned(page_table, 4) || !aligned(seq_lens, 4))
    return ISOQUANT_ERR_ALIGNMENT;
  if (ws_bytes < need) return ISOQUANT_ERR_WORKSPACE;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return ISOQUANT_ERR_INVALID_ARG;
  AttendShape s;
  st = make_shape(ctx, batch, nq, num_q_heads, cache->page_size, causal, &s);
  if (st != ISOQUANT_OK) return st;
  const size_t attend_bytes = round_up_256(attend_workspace_bytes(s));
  float *q_rot = reinterpret_cast<float *>(static_cast<char *>(workspace) + attend_bytes);
  st = isoquant_decode_prep(ctx, cache, k, v, n_tok, slot_mapping, q, dtype, batch * nq, num_q_heads, q_rot, stream);
  if (st != ISOQUANT_OK) return st;
  const int prep = ctx->last_launches;
  st = isoquant_attend_decode(ctx, cache, q_rot, batch, nq, num_q_heads, page_table, max_pages, seq_lens, causal,
                              scale, workspace, attend_bytes, out, stream);
  ctx->last_launches += prep;
  return st;
}

int isoquant_workspace_size(const isoquant_ctx *ctx, int batch, int nq, int num_q_heads, size_t *bytes) {
  return isoquant_workspace_size_paged(ctx, batch, nq, num_q_heads, 256, bytes);
}

int isoquant_workspace_size_paged(const isoquant_ctx *ctx, int batch, int nq, int num_q_heads, int page_size,
                                  size_t *bytes) {
  if (ctx == nullptr || bytes == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  if (!valid_page_size(page_size)) return ISOQUANT_ERR_UNSUPPORTED;
  AttendShape s;
  int st = make_shape(ctx, batch, nq, num_q_heads, page_size, 0, &s);
  if (st != ISOQUANT_OK) return st;
  *bytes = attend_workspace_bytes(s);
  return ISOQUANT_OK;
}

int isoquant_attend_partial(isoquant_ctx *ctx, const isoquant_cache *cache, const float *q_rot, int batch, int nq,
                            int num_q_heads, const int32_t *page_table, int max_pages, const int32_t *seq_lens,
                            int causal, float scale, void *workspace, size_t ws_bytes, void *stream) {
  ISOQUANT_TRACE("isoquant_attend_partial");
  if (ctx == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  int st = check_cache(cache);
  if (st != ISOQUANT_OK) return st;
  AttendShape s;
  st = make_shape(ctx, batch, nq, num_q_heads, cache->page_size, causal, &s);
  if (st != ISOQUANT_OK) return st;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return ISOQUANT_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = 1.0f / std::sqrt(static_cast<float>(kD));
  if (batch == 0) return ISOQUANT_OK;
  if (q_rot == nullptr || page_table == nullptr || seq_lens == nullptr || workspace == nullptr || max_pages < 1)
    return ISOQUANT_ERR_INVALID_ARG;
  if (!aligned(workspace, 16) || !aligned(q_rot, 4) || !aligned(page_table, 4) || !aligned(seq_lens, 4))
    return ISOQUANT_ERR_ALIGNMENT;
  if (ws_bytes < attend_workspace_min_bytes(s)) return ISOQUANT_ERR_WORKSPACE;
  // a sequence's pages of all KV heads (plus the tcgen05 kernels' work-free
  // pages, at most 16 per head) are counted in 32 bits
  if ((static_cast<int64_t>(max_pages) + 16) * ctx->num_kv_heads >= INT32_MAX) return ISOQUANT_ERR_INVALID_ARG;
  st = check_device(ctx);
  if (st != ISOQUANT_OK) return st;
  cudaError_t e = launch_attend_partial(ctx, cache, s, q_rot, page_table, max_pages, seq_lens, scale, workspace,
                                        ws_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return ISOQUANT_ERR_CUDA;
  ctx->last_launches = 1;
  return ISOQUANT_OK;
}

int isoquant_attend_combine(isoquant_ctx *ctx, int batch, int nq, int num_q_heads, const int32_t *seq_lens,
                            int page_size, const void *workspace, size_t ws_bytes, float *out, void *stream) {
  ISOQUANT_TRACE("isoquant_attend_combine");
  if (ctx == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  if (!valid_page_size(page_size)) return ISOQUANT_ERR_UNSUPPORTED;
  AttendShape s;
  int st = make_shape(ctx, batch, nq, num_q_heads, page_size, 0, &s);
  if (st != ISOQUANT_OK) return st;
  if (batch == 0) return ISOQUANT_OK;
  if (seq_lens == nullptr || workspace == nullptr || out == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  if (!aligned(workspace, 16) || !aligned(out, 16) || !aligned(seq_lens, 4)) return ISOQUANT_ERR_ALIGNMENT;
  if (ws_bytes < attend_workspace_min_bytes(s)) return ISOQUANT_ERR_WORKSPACE;
  st = check_device(ctx);
  if (st != ISOQUANT_OK) return st;
  cudaError_t e = launch_attend_combine(ctx, s, seq_lens, workspace, ws_bytes, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return ISOQUANT_ERR_CUDA;
  ctx->last_launches = 1;
  return ISOQUANT_OK;
}

int isoquant_attend_decode(isoquant_ctx *ctx, const isoquant_cache *cache, const float *q_rot, int batch, int nq,
                           int num_q_heads, const int32_t *page_table, int max_pages, const int32_t *seq_lens,
                           int causal, float scale, void *workspace, size_t ws_bytes, float *out, void *stream) {
  ISOQUANT_TRACE("isoquant_attend_decode");
  if (ctx == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  if (out == nullptr && batch > 0) return ISOQUANT_ERR_INVALID_ARG;
  if (out != nullptr && !aligned(out, 16)) return ISOQUANT_ERR_ALIGNMENT;
  int st = isoquant_attend_partial(ctx, cache, q_rot, batch, nq, num_q_heads, page_table, max_pages, seq_lens,
                                   causal, scale, workspace, ws_bytes, stream);
  if (st != ISOQUANT_OK) return st;
  const int first = ctx->last_launches;
  st = isoquant_attend_combine(ctx, batch, nq, num_q_heads, seq_lens, cache->page_size, workspace, ws_bytes, out,
                               stream);
  ctx->last_launches += first;
  return st;
}

int isoquant_get_status(isoquant_ctx *ctx, uint32_t *status, void *stream) {
  ISOQUANT_TRACE("isoquant_get_status");
  if (ctx == nullptr || status == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, ctx->status, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess || cudaMemsetAsync(ctx->status, 0, 16, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return ISOQUANT_ERR_CUDA;
  *status = host;
  return ISOQUANT_OK;
}

int isoquant_last_launch_count(const isoquant_ctx *ctx) { return ctx ? ctx->last_launches : 0; }

int isoquant_selftest_wait(isoquant_ctx *ctx, uint64_t limit_ns, uint64_t *elapsed_ns, void *stream) {
  ISOQUANT_TRACE("isoquant_selftest_wait");
  if (ctx == nullptr || limit_ns == 0 || limit_ns > kSelftestMaxNs) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 1;
  return launch_wait_selftest(ctx, limit_ns, elapsed_ns, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? ISOQUANT_OK
             : ISOQUANT_ERR_CUDA;
}

}  // extern "C"

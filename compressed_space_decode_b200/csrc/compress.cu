// compress.cu -- isoquant_compress_kv and isoquant_rotate_q kernels.
//
// RotaryQuant, Abstract: a Walsh-Hadamard transform followed by
// block-diagonal SO(4) rotations isotropizes each head vector before 3-bit
// scalar quantization.  One warp handles one d = 128 vector, lane l holding
// coordinates 4l..4l+3: the two smallest WHT strides stay inside the lane,
// the other five are warp shuffles, and SO(4) block l is lane l's own 4x4
// product, so the whole rotation stays in registers.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "isoquant_internal.cuh"

namespace isoquant {
namespace {

// Coordinates whose fp32 z lies closer than this to a threshold are
// re-derived in fp64.  The fp32 rotation error in z is below 1e-6 (7
// butterfly stages plus a 4-term product, each rounding at 2^-24 of
// quantities bounded by sqrt(128) |x| / n), so every code decided on the
// fast path is the code of the exact z.
constexpr float kRecheckBand = 1e-5f;

__device__ __forceinline__ void load4(const float *p, float (&x)[4]) {
  float4 v = *reinterpret_cast<const float4 *>(p);
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&x)[4]) {
  uint2 u = *reinterpret_cast<const uint2 *>(p);
  x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const __half *p, float (&x)[4]) {
  uint2 u = *reinterpret_cast<const uint2 *>(p);
  float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
  float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}

__device__ __forceinline__ uint32_t lane_sign_nibble(const HeadParams &hp, int lane) {
  return (hp.sign_bits[lane >> 3] >> (4 * (lane & 7))) & 0xFu;
}

// y = B * H * D * x (unnormalised H), 4 coordinates per lane, fp32.
__device__ __forceinline__ void rotate_f32(const HeadParams &hp, int lane, const float (&x)[4],
                                           float (&out)[4]) {
  const uint32_t sn = lane_sign_nibble(hp, lane);
  float y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = __uint_as_float(__float_as_uint(x[i]) ^ (((sn >> i) & 1u) << 31));
  wht128<float>(y, lane);
  const float4 *m = reinterpret_cast<const float4 *>(hp.m32[lane]);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float4 row = m[r];
    out[r] = fmaf(row.w, y[3], fmaf(row.z, y[2], fmaf(row.y, y[1], row.x * y[0])));
  }
}

__device__ __forceinline__ void rotate_f64(const HeadParams &hp, int lane, const float (&x)[4],
                                           double (&out)[4]) {
  const uint32_t sn = lane_sign_nibble(hp, lane);
  double y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = ((sn >> i) & 1u) ? -(double)x[i] : (double)x[i];
  wht128<double>(y, lane);
  const double *m = hp.m64[lane];
#pragma unroll
  for (int r = 0; r < 4; ++r)
    out[r] = fma(m[4 * r + 3], y[3], fma(m[4 * r + 2], y[2], fma(m[4 * r + 1], y[1], m[4 * r] * y[0])));
}

template <typename T>
__global__ void __launch_bounds__(256) k_compress(const HeadParams *__restrict__ params, Codebook cb,
                                                  const T *__restrict__ kin, const T *__restrict__ vin,
                                                  int n_tok, int H, const int64_t *__restrict__ slots,
                                                  uint32_t *__restrict__ codes,
                                                  uint16_t *__restrict__ norms, int num_pages,
                                                  int page_size, uint32_t *status) {
  const int lane = threadIdx.x & 31;
  const int64_t vec = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t per_kv = static_cast<int64_t>(n_tok) * H;
  if (vec >= 2 * per_kv) return;
  const int kv = static_cast<int>(vec / per_kv);
  const int64_t rem = vec - kv * per_kv;
  const int64_t t = rem / H;
  const int h = static_cast<int>(rem - t * H);
  const int64_t slot = slots[t];
  if (slot < 0) return;
  const int64_t page = slot / page_size;
  const int off = static_cast<int>(slot - page * page_size);
  if (page >= num_pages) {
    if (lane == 0) set_status(status, ISOQUANT_DEVERR_SLOT_RANGE);
    return;
  }
  const HeadParams &hp = params[h];

  float x[4];
  load4((kv ? vin : kin) + (t * H + h) * kD + 4 * lane, x);

  // ||x||_2 in fp64: squares of fp32 values are exact in fp64
  double ss = static_cast<double>(x[0]) * x[0] + static_cast<double>(x[1]) * x[1] +
              static_cast<double>(x[2]) * x[2] + static_cast<double>(x[3]) * x[3];
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  const double n = sqrt(ss);

  // z = (B H D x) / n; sqrt(128) of the normalised Hn cancels against the
  // sqrt(128) of z = sqrt(128) * y / n.
  float yr[4];
  rotate_f32(hp, lane, x, yr);
  const float inv = n > 0.0 ? static_cast<float>(1.0 / n) : 0.0f;
  uint32_t c[4];
  bool near = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float z = yr[i] * inv;
    uint32_t code = 0;
#pragma unroll
    for (int k = 0; k < kLevels - 1; ++k) {
      code += (z > cb.threshold[k]) ? 1u : 0u;
      near |= fabsf(z - cb.threshold[k]) < kRecheckBand;
    }
    c[i] = code;
  }
  if (__any_sync(0xffffffffu, near && n > 0.0)) {
    double y64[4];
    rotate_f64(hp, lane, x, y64);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double z = n > 0.0 ? y64[i] / n : 0.0;
      uint32_t code = 0;
#pragma unroll
      for (int k = 0; k < kLevels - 1; ++k) code += (z > cb.threshold64[k]) ? 1u : 0u;
      c[i] = code;
    }
  }

  // pack: word w holds codes 10w..10w+9, i.e. coordinates of lanes
  // floor(10w/4) .. +2; an odd word starts two codes into its first lane.
  const uint32_t c4 = c[0] | (c[1] << 3) | (c[2] << 6) | (c[3] << 9);
  const int w = lane;
  const int a = (5 * w) >> 1;
  const uint32_t s0 = __shfl_sync(0xffffffffu, c4, a & 31);
  const uint32_t s1 = __shfl_sync(0xffffffffu, c4, min(a + 1, 31));
  const uint32_t s2 = __shfl_sync(0xffffffffu, c4, min(a + 2, 31));
  const uint64_t comb = static_cast<uint64_t>(s0) | (static_cast<uint64_t>(s1) << 12) |
                        (static_cast<uint64_t>(s2) << 24);
  const uint32_t word =
      static_cast<uint32_t>(comb >> ((w & 1) ? 6 : 0)) & (w == 12 ? 0x00FFFFFFu : 0x3FFFFFFFu);

  const int64_t block = (page * 2 + kv) * H + h;
  if (lane < kWords) codes[block * kWords * page_size + static_cast<int64_t>(w) * page_size + off] = word;
  if (lane == 0) norms[block * page_size + off] = __half_as_ushort(__double2half(fmin(n, 65504.0)));
}

template <typename T>
__global__ void __launch_bounds__(256) k_rotate_q(const HeadParams *__restrict__ params,
                                                  const T *__restrict__ q, int n_rows, int Hq, int G,
                                                  float *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t vec = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (vec >= static_cast<int64_t>(n_rows) * Hq) return;
  const int hq = static_cast<int>(vec % Hq);
  float x[4], y[4];
  load4(q + vec * kD + 4 * lane, x);
  rotate_f32(params[hq / G], lane, x, y);
  const float s = 0.08838834764831845f;  // 1/sqrt(128): the normalisation of Hn
  *reinterpret_cast<float4 *>(out + vec * kD + 4 * lane) = make_float4(y[0] * s, y[1] * s, y[2] * s, y[3] * s);
}

}  // namespace

cudaError_t launch_compress(const isoquant_ctx *ctx, const isoquant_cache *cache, const void *k,
                            const void *v, int dtype, int n_tok, const int64_t *slot_mapping,
                            cudaStream_t stream) {
  const int H = ctx->num_kv_heads;
  const int64_t warps = 2LL * n_tok * H;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(blocks)), block(256);
  switch (dtype) {
    case ISOQUANT_F32:
      k_compress<float><<<grid, block, 0, stream>>>(ctx->params, ctx->codebook, static_cast<const float *>(k),
                                                    static_cast<const float *>(v), n_tok, H, slot_mapping,
                                                    cache->codes, cache->norms, cache->num_pages,
                                                    cache->page_size, ctx->status);
      break;
    case ISOQUANT_BF16:
      k_compress<__nv_bfloat16><<<grid, block, 0, stream>>>(
          ctx->params, ctx->codebook, static_cast<const __nv_bfloat16 *>(k),
          static_cast<const __nv_bfloat16 *>(v), n_tok, H, slot_mapping, cache->codes, cache->norms,
          cache->num_pages, cache->page_size, ctx->status);
      break;
    default:
      k_compress<__half><<<grid, block, 0, stream>>>(ctx->params, ctx->codebook, static_cast<const __half *>(k),
                                                     static_cast<const __half *>(v), n_tok, H, slot_mapping,
                                                     cache->codes, cache->norms, cache->num_pages,
                                                     cache->page_size, ctx->status);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_rotate_q(const isoquant_ctx *ctx, const void *q, int dtype, int n_rows,
                            int num_q_heads, float *q_rot, cudaStream_t stream) {
  const int G = num_q_heads / ctx->num_kv_heads;
  const int64_t warps = static_cast<int64_t>(n_rows) * num_q_heads;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(blocks)), block(256);
  switch (dtype) {
    case ISOQUANT_F32:
      k_rotate_q<float><<<grid, block, 0, stream>>>(ctx->params, static_cast<const float *>(q), n_rows,
                                                    num_q_heads, G, q_rot);
      break;
    case ISOQUANT_BF16:
      k_rotate_q<__nv_bfloat16><<<grid, block, 0, stream>>>(
          ctx->params, static_cast<const __nv_bfloat16 *>(q), n_rows, num_q_heads, G, q_rot);
      break;
    default:
      k_rotate_q<__half><<<grid, block, 0, stream>>>(ctx->params, static_cast<const __half *>(q), n_rows,
                                                     num_q_heads, G, q_rot);
      break;
  }
  return cudaGetLastError();
}

}  // namespace isoquant

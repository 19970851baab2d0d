// compress.cu -- isoquant_compress_kv and isoquant_rotate_q kernels.
//
// RotaryQuant, Abstract: a Walsh-Hadamard transform followed by
// block-diagonal SO(4) rotations isotropizes each head vector before 3-bit
// scalar quantization.  The compress kernels give each vector 8 lanes in two
// layouts (below); the query rotation and the fp64 path give it a warp, lane
// l holding coordinates 4l..4l+3 (two WHT strides inside the lane, five warp
// shuffles, SO(4) block l as the lane's own 4x4 product).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "isoquant_internal.cuh"

namespace isoquant {
namespace {

// Coordinates whose fp32 z lies closer than this to a threshold are
// re-derived in fp64.  The fp32 rotation error in z (7 butterfly stages, a
// 4-term product and 1/n, each rounding at 2^-24 of quantities bounded by
// sqrt(128) |x| / n) measures about 1e-6 at most (isoquant_debug_export_z
// against the exact z: 1.04e-6 for fp32 inputs, 7e-7 for bf16/fp16 ones),
// a tenth of this band, so every code decided on the fast path is the code
// of the exact z.
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

struct CompressArgs {
  const HeadParams *params;
  Codebook cb;
  const void *kin, *vin;
  int n_tok, H;
  const int64_t *slots;
  uint32_t *codes;
  uint16_t *norms;
  int num_pages, ps_shift;
  int strip;  // tokens per warp strip (a multiple of 4)
  uint32_t *status;
};

// ------------------------------------------------------------ two layouts
// A warp compresses four vectors of one head at a time: lane group
// g = lane / 8 holds one vector and its lane q = lane % 8 a sixteenth of it,
// in one of two layouts:
//   layout A (loads, signs, norm, WHT strides 16, 32 and 64): coordinates
//     16m + 2q and 16m + 2q + 1 for m = 0..7, as a[m] = (the two);
//   layout B (WHT strides 1, 2, 4 and 8, the SO(4) blocks, the codes):
//     coordinates 16q .. 16q + 15, as b[k] = (16q + 2k, 16q + 2k + 1).
// Each layout keeps its WHT strides inside the lane, so the transform needs
// no shuffles: the change of layout goes through a shared-memory tile per
// warp, and the lane's four SO(4) blocks 4q .. 4q + 3 stay in registers for
// the warp's whole strip of tokens.  Pairs of coordinates go through the
// packed fp32 instructions (two independent IEEE operations each).

// Shared tile of one warp: per vector 8 rows (m) of 16 floats, rows 20
// floats apart and vectors 176 apart, so that neither the 8-byte stores of
// layout A nor the 16-byte loads of layout B meet a bank conflict.
constexpr int kTileRow = 20;
constexpr int kTileVec = 8 * kTileRow + 16;
constexpr int kTileFloats = 4 * kTileVec;

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }

// One layout-A lane's 16 inputs as loaded: a 32-bit word per pair of 16-bit
// values, or the fp32 pair.
template <typename T>
struct RawA {
  uint32_t w[8];
};
template <>
struct RawA<float> {
  float2 w[8];
};
template <typename T>
__device__ __forceinline__ void load_a(const T *vec, int q, RawA<T> &r) {
#pragma unroll
  for (int m = 0; m < 8; ++m) r.w[m] = *reinterpret_cast<const uint32_t *>(vec + 16 * m + 2 * q);
}
__device__ __forceinline__ void load_a(const float *vec, int q, RawA<float> &r) {
#pragma unroll
  for (int m = 0; m < 8; ++m) r.w[m] = *reinterpret_cast<const float2 *>(vec + 16 * m + 2 * q);
}
// Unpack to fp32 with the signs D applied (sgn[m]: bit 15 and bit 31 flip
// coordinate 16m + 2q and 16m + 2q + 1).
__device__ __forceinline__ void unpack_a(const RawA<__nv_bfloat16> &r, const uint32_t (&sgn)[8], float2 (&a)[8]) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint32_t w = r.w[m] ^ sgn[m];
    a[m] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
}
__device__ __forceinline__ void unpack_a(const RawA<__half> &r, const uint32_t (&sgn)[8], float2 (&a)[8]) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint32_t w = r.w[m] ^ sgn[m];
    a[m] = __half22float2(*reinterpret_cast<const __half2 *>(&w));
  }
}
__device__ __forceinline__ void unpack_a(const RawA<float> &r, const uint32_t (&sgn)[8], float2 (&a)[8]) {
#pragma unroll
  for (int m = 0; m < 8; ++m)
    a[m] = make_float2(__uint_as_float(__float_as_uint(r.w[m].x) ^ (sgn[m] << 16)),
                       __uint_as_float(__float_as_uint(r.w[m].y) ^ (sgn[m] & 0x80000000u)));
}
// sum of the lane's 16 squares (signs do not matter): pairs, then a tree
__device__ __forceinline__ float lane_squares(const float2 (&a)[8]) {
  float2 s[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) s[i] = __ffma2_rn(a[2 * i + 1], a[2 * i + 1], __fmul2_rn(a[2 * i], a[2 * i]));
  const float2 t = add2(add2(s[0], s[1]), add2(s[2], s[3]));
  return t.x + t.y;
}
// The lane's strip constants: the sign masks of its layout-A coordinates and
// its SO(4) blocks 4q + k as column pairs, mc[k][r][j] = (M[r][2j], M[r][2j + 1]).
struct LaneConsts {
  uint32_t sgn[8];
  float2 mc[4][4][2];
};
__device__ __forceinline__ void lane_consts(const HeadParams &hp, int q, LaneConsts &c) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int j = 16 * m + 2 * q;  // even: both coordinates in one sign word
    const uint32_t bits = (hp.sign_bits[j >> 5] >> (j & 31)) & 3u;
    c.sgn[m] = ((bits & 1u) << 15) | ((bits >> 1) << 31);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 row = reinterpret_cast<const float4 *>(hp.m32[4 * q + k])[r];
      c.mc[k][r][0] = make_float2(row.x, row.y);
      c.mc[k][r][1] = make_float2(row.z, row.w);
    }
  }
}

__device__ __forceinline__ float group_sum(float s) {
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 4);
  return s;
}
// min of three (one instruction on sm_100)
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// The rotation of one lane group's vector, a in layout A with the signs D
// applied: the unnormalised Sylvester WHT (its sqrt(128) cancels against the
// one of z = sqrt(128) y / n) and the SO(4) blocks, leaving y[i] =
// coordinate 16q + i of B H D x.  The lower index of each butterfly keeps
// a + b, the upper one a - b.  `tile` is the warp's shared tile; every lane
// of the warp calls this together.
__device__ __forceinline__ void rotate_two_layouts(float2 (&a)[8], const LaneConsts &c, float *tile, int grp, int q,
                                                   float (&y)[16]) {
  // strides 16, 32, 64: bits 0, 1, 2 of m
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      if (m & s) continue;
      const float2 u = a[m], v = a[m + s];
      a[m] = add2(u, v);
      a[m + s] = sub2(u, v);
    }
  }
  // layout A -> layout B: row m of the vector's tile holds 16m .. 16m + 15
  float *tv = tile + grp * kTileVec;
  __syncwarp();
#pragma unroll
  for (int m = 0; m < 8; ++m) *reinterpret_cast<float2 *>(tv + m * kTileRow + 2 * q) = a[m];
  __syncwarp();
  float2 b[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 v = *reinterpret_cast<const float4 *>(tv + q * kTileRow + 4 * j);
    b[2 * j] = make_float2(v.x, v.y);
    b[2 * j + 1] = make_float2(v.z, v.w);
  }
  // stride 1 inside each pair; strides 2, 4, 8 between pairs
#pragma unroll
  for (int k = 0; k < 8; ++k) b[k] = make_float2(b[k].x + b[k].y, b[k].x - b[k].y);
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k & s) continue;
      const float2 u = b[k], v = b[k + s];
      b[k] = add2(u, v);
      b[k + s] = sub2(u, v);
    }
  }
  // SO(4) block 4q + k on coordinates 16q + 4k .. 16q + 4k + 3 = b[2k], b[2k + 1]
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float2 t = __ffma2_rn(c.mc[k][r][1], b[2 * k + 1], __fmul2_rn(c.mc[k][r][0], b[2 * k]));
      y[4 * k + r] = t.x + t.y;
    }
  }
}

// Pack the 128 codes of a lane group (lane q holding codes 16q..16q+15 at
// bits 3e of cbits) into the 13 canonical words (word w: codes 10w..10w+9 at
// bits 3(j - 10w)) and, if `store`, write the words that start in this lane
// to codes[(row0 + w) << ps_shift].  A word that straddles two lanes gets
// the second lane's part by one shuffle, which every lane executes.
__device__ __forceinline__ void pack_store_wide(uint64_t cbits, int q, bool store, uint32_t *codes, int64_t row0,
                                                int ps_shift) {
  const int d0 = 16 * q;
  const int wlo = d0 / 10, whi = (d0 + 15) / 10;
  uint32_t part[3];
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int w = wlo + r;
    const int j0 = max(10 * w, d0), j1 = min(10 * w + 10, d0 + 16);
    part[r] = 0u;
    if (w <= whi && j1 > j0) {
      const uint64_t bits = (cbits >> (3 * (j0 - d0))) & ((1ull << (3 * (j1 - j0))) - 1ull);
      part[r] = static_cast<uint32_t>(bits) << (3 * (j0 - 10 * w));
    }
  }
  // the next lane's share of its first word (when that word began here)
  const uint32_t nxt = __shfl_down_sync(0xffffffffu, part[0], 1);
  const bool spans = q < 7 && (d0 + 16) % 10 != 0;  // word whi continues in lane q + 1
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int w = wlo + r;
    if (w > whi) continue;
    uint32_t word = part[r];
    if (spans && w == whi) word |= nxt;
    if (store && 10 * w >= d0) codes[(row0 + w) << ps_shift] = word;
  }
}


// The fp64 path for one vector, by the whole warp (lane l: coordinates
// 4l..4l+3): norm, rotation and codes all in fp64.  Used for the few vectors
// whose fp16 norm rounding or codes the fp32 fast path cannot decide.
template <typename T, int BITS>
__device__ void compress_one_fp64(const HeadParams &hp, const Codebook &cb, const T *src, uint32_t *codes,
                                  uint16_t *norms, int64_t block, int off, int ps_shift, int lane) {
  float xv[4];
  load4(src + 4 * lane, xv);
  double ss = static_cast<double>(xv[0]) * xv[0] + static_cast<double>(xv[1]) * xv[1] +
              static_cast<double>(xv[2]) * xv[2] + static_cast<double>(xv[3]) * xv[3];
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  const double n = sqrt(ss);
  const uint16_t n16 = __half_as_ushort(__double2half(fmin(n, 65504.0)));
  double y64[4];
  rotate_f64(hp, lane, xv, y64);
  uint32_t c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const double z = n > 0.0 ? y64[k] / n : 0.0;
    uint32_t code = 0;
#pragma unroll
    for (int t = 0; t < (1 << BITS) - 1; ++t) code += (z > cb.threshold64[t]) ? 1u : 0u;
    c[k] = code;
  }
  if constexpr (BITS != 3) {
    // 2 bits: word w = codes 16w..16w+15 = lanes 4w..4w+3 (8 bits each);
    // 4 bits: word w = codes 8w..8w+7 = lanes 2w, 2w+1 (16 bits each)
    constexpr int kLanesPerWord = 32 / (4 * BITS);
    constexpr int kW = words_for(BITS);
    const uint32_t cl = c[0] | (c[1] << BITS) | (c[2] << (2 * BITS)) | (c[3] << (3 * BITS));
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < kLanesPerWord; ++i)
      word |= __shfl_sync(0xffffffffu, cl, (kLanesPerWord * lane + i) & 31) << (4 * BITS * i);
    if (lane < kW) codes[((block * kW + lane) << ps_shift) + off] = word;
    if (lane == 0) norms[(block << ps_shift) + off] = n16;
    return;
  }
  // word w holds codes 10w..10w+9, i.e. coordinates of lanes
  // floor(10w/4) .. +2; an odd word starts two codes into its first lane.
  const uint32_t c4 = c[0] | (c[1] << 3) | (c[2] << 6) | (c[3] << 9);
  const int wd = lane;
  const int a = (5 * wd) >> 1;
  const uint32_t s0 = __shfl_sync(0xffffffffu, c4, a & 31);
  const uint32_t s1 = __shfl_sync(0xffffffffu, c4, min(a + 1, 31));
  const uint32_t s2 = __shfl_sync(0xffffffffu, c4, min(a + 2, 31));
  const uint64_t comb = static_cast<uint64_t>(s0) | (static_cast<uint64_t>(s1) << 12) |
                        (static_cast<uint64_t>(s2) << 24);
  const uint32_t word =
      static_cast<uint32_t>(comb >> ((wd & 1) ? 6 : 0)) & (wd == 12 ? 0x00FFFFFFu : 0x3FFFFFFFu);
  if (lane < kWords) codes[((block * kWords + wd) << ps_shift) + off] = word;
  if (lane == 0) norms[(block << ps_shift) + off] = n16;
}


// Warp w of the K (kv = 0) or V (kv = 1) half: rotate, quantize and pack
// tokens strip * (w / H) .. + strip - 1 of head w % H, four at a time.
// `tile` is the warp's shared tile (kTileFloats floats).
template <typename T, int BITS>
__device__ __forceinline__ void compress_warp(const CompressArgs &g, int kv, uint32_t w, int lane, float *tile) {
  constexpr int kHalf = 1 << (BITS - 1);  // codes below kHalf are the negative levels
  constexpr int kPos = kHalf - 1;         // positive thresholds (the middle one is 0)
  constexpr uint32_t kAll = (1u << BITS) - 1u;
  constexpr int kW = words_for(BITS);
  const int H = g.H, n_tok = g.n_tok, ps_shift = g.ps_shift;
  const uint32_t strips = (static_cast<uint32_t>(n_tok) + g.strip - 1) / g.strip;
  const uint32_t sidx = w / static_cast<uint32_t>(H);
  if (sidx >= strips) return;
  const int h = static_cast<int>(w - sidx * static_cast<uint32_t>(H));
  const HeadParams &hp = g.params[h];
  const Codebook &cb = g.cb;
  const T *__restrict__ src = static_cast<const T *>(kv ? g.vin : g.kin);
  const int grp = lane >> 3, q = lane & 7;

  // this lane's sign masks and SO(4) blocks 4q..4q+3, for the whole strip
  LaneConsts lc;
  lane_consts(hp, q, lc);
  // the positive thresholds (the codebook is symmetric)
  float tp[kPos];
#pragma unroll
  for (int i = 0; i < kPos; ++i) tp[i] = cb.threshold[kHalf + i];

  const int t_begin = static_cast<int>(sidx) * g.strip;
  const int t_end = min(t_begin + g.strip, n_tok);
  // the inputs and slot of the group's next vector are loaded one iteration
  // ahead, so that their latency overlaps the current vector's rotation
  RawA<T> nraw{};
  int64_t nslot = -1;
  if (t_begin + grp < t_end) {
    nslot = g.slots[t_begin + grp];
    load_a(src + (static_cast<int64_t>(t_begin + grp) * H + h) * kD, q, nraw);
  }
  for (int tb = t_begin; tb < t_end; tb += 4) {
    const int t = tb + grp;
    const bool live = t < t_end;
    float2 a[8];
    int64_t slot = -1;
    if (live) {
      slot = nslot;
      unpack_a(nraw, lc.sgn, a);
    } else {
#pragma unroll
      for (int m = 0; m < 8; ++m) a[m] = make_float2(0.f, 0.f);
    }
    if (t + 4 < t_end) {
      nslot = g.slots[t + 4];
      load_a(src + (static_cast<int64_t>(t + 4) * H + h) * kD, q, nraw);
    }
    const int64_t page = slot >> ps_shift;
    const bool valid = live && slot >= 0 && page < g.num_pages;
    if (live && slot >= 0 && page >= g.num_pages && q == 0) set_status(g.status, ISOQUANT_DEVERR_SLOT_RANGE);

    // ||x||^2 in fp32: squares of bf16/fp16 inputs are exact and the tree
    // (4 levels in the lane, 3 across the group) is within 7 * 2^-24
    // relative; n32 = sqrt of it by sqrt.approx (within 2^-22), so n32 is
    // within ~5e-7 of the exact norm.  Its fp16 rounding is decided from
    // n32's bits: fp16 keeps the top 10 of fp32's 23 mantissa bits, so the
    // 13 below them place n32 inside an fp16 step, whose rounding midpoint
    // is 0x1000.  A pattern 16 or more fp32 units from it lies at least
    // 2^-20 (9.5e-7) relative from the midpoint, so the exact norm rounds
    // the same way; closer, or outside the fp16 normal range below 65000
    // (or not finite), the fp64 path decides.
    const float ssf = group_sum(lane_squares(a));
    float n32;
    asm("sqrt.approx.f32 %0, %1;" : "=f"(n32) : "f"(ssf));
    const uint16_t hb = __half_as_ushort(__float2half_rn(fminf(n32, 65504.f)));
    const int mid_off = static_cast<int>(__float_as_uint(n32) & 0x1FFFu) - 0x1000;
    bool slow = !(n32 >= 6.103515625e-05f && n32 < 65000.f && (mid_off >= 16 || mid_off <= -16));

    float y[16];
    rotate_two_layouts(a, lc, tile, grp, q, y);
    // codes: z = y / n against the thresholds t, decided as |y| against
    // t * n; neg = #{t : |y| < t * n} (the sign bits of the differences),
    // so the code is neg for y < 0 and 2^BITS - 1 - neg for y > 0.  A
    // coordinate within kRecheckBand of a threshold (0 included) in z units
    // sends the vector to the fp64 path, so the fast path's comparisons
    // (and its ties) only decide codes that the exact z decides the same way.
    float thr[kPos];
#pragma unroll
    for (int i = 0; i < kPos; ++i) thr[i] = tp[i] * n32;
    const float band = kRecheckBand * n32;
    uint64_t cbits = 0;
    float dmin = band;  // distance of the nearest coordinate to a threshold, capped
    if constexpr (BITS == 3) {
      // The code's three bits straight from sign bits: with s_k the sign bit
      // of |y| - t_k n (t ascending, so s_1 <= s_2 <= s_3) and p = (y > 0),
      // neg = s_1 + s_2 + s_3 has bit 0 = s_1 ^ s_2 ^ s_3 and bit 1 = s_2, so
      // the code neg ^ (p ? 7 : 0) has bits (s_1^s_2^s_3^p, s_2^p, p).  Bit
      // 31 of y is ~p, so the words below carry each bit inverted; funnel
      // shifts collect bit 31 of each, coordinates 0..9 into one word and
      // 10..15 into another (highest coordinate first, its bit 2 first), and
      // one XOR per word undoes the inversion.
      uint32_t wa = 0, wb = 0;
#pragma unroll
      for (int i = 15; i >= 0; --i) {
        const float av = fabsf(y[i]);
        const float r0 = av - thr[0], r1 = av - thr[1], r2 = av - thr[2];
        const uint32_t yb = __float_as_uint(y[i]);
        const uint32_t i0 = __float_as_uint(r0) ^ __float_as_uint(r1) ^ __float_as_uint(r2) ^ yb;
        const uint32_t i1 = __float_as_uint(r1) ^ yb;
        uint32_t &acc = i >= 10 ? wb : wa;
        acc = __funnelshift_l(yb, acc, 1);
        acc = __funnelshift_l(i1, acc, 1);
        acc = __funnelshift_l(i0, acc, 1);
        dmin = fmin3(dmin, fabsf(r0), fabsf(r1));
        dmin = fmin3(dmin, fabsf(r2), av);
      }
      cbits = static_cast<uint64_t>(wa ^ 0x3FFFFFFFu) | (static_cast<uint64_t>(wb ^ 0x3FFFFu) << 30);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float av = fabsf(y[i]);
        uint32_t neg = 0;
        float r[kPos];
#pragma unroll
        for (int j = 0; j < kPos; ++j) {
          r[j] = av - thr[j];
          neg += __float_as_uint(r[j]) >> 31;
        }
        const uint32_t c = neg ^ (kAll & ~static_cast<uint32_t>(__float_as_int(y[i]) >> 31));
        cbits |= static_cast<uint64_t>(c) << (BITS * i);
        if constexpr (kPos == 1) {
          dmin = fmin3(dmin, fabsf(r[0]), av);
        } else {
#pragma unroll
          for (int j = 0; j + 1 < kPos; j += 2) dmin = fmin3(dmin, fabsf(r[j]), fabsf(r[j + 1]));
          dmin = fmin3(dmin, fabsf(r[kPos - 1]), av);
        }
      }
    }
    const bool near = dmin < band;
    // the group's decision: any lane near a threshold sends the vector to
    // the fp64 path
    const uint32_t gmask = 0xFFu << (8 * grp);
    slow = (__ballot_sync(0xffffffffu, (near || slow) && valid) & gmask) != 0;
    const int off = static_cast<int>(slot & ((1 << ps_shift) - 1));
    const int64_t block = (page * 2 + kv) * H + h;
    const bool fast = valid && !slow;
    if constexpr (BITS == 3) {
      pack_store_wide(cbits, q, fast, g.codes + off, block * kWords, ps_shift);
    } else {
      // the lane's 16 codes are whole words: word q (2 bits) or words 2q,
      // 2q + 1 (4 bits)
      uint32_t *cw = g.codes + off;
      if (fast) {
        if constexpr (BITS == 2) {
          cw[(block * kW + q) << ps_shift] = static_cast<uint32_t>(cbits);
        } else {
          cw[(block * kW + 2 * q) << ps_shift] = static_cast<uint32_t>(cbits);
          cw[(block * kW + 2 * q + 1) << ps_shift] = static_cast<uint32_t>(cbits >> 32);
        }
      }
    }
    if (fast && q == 0) g.norms[(block << ps_shift) + off] = hb;
    // vectors for the fp64 path, one at a time by the whole warp
    uint32_t todo = __ballot_sync(0xffffffffu, valid && slow && q == 0);
    while (todo) {
      const int src_lane = __ffs(todo) - 1;
      todo &= todo - 1;
      const int gv = src_lane >> 3;
      const int tv = tb + gv;
      const int64_t sl = __shfl_sync(0xffffffffu, slot, src_lane);
      const int64_t pg = sl >> ps_shift;
      compress_one_fp64<T, BITS>(hp, cb, src + (static_cast<int64_t>(tv) * H + h) * kD, g.codes, g.norms,
                                 (pg * 2 + kv) * H + h, static_cast<int>(sl & ((1 << ps_shift) - 1)), ps_shift,
                                 lane);
    }
  }
}

// warps per compress block; blockIdx.y selects K or V.
#ifndef ISOQUANT_COMPRESS_WARPS
#define ISOQUANT_COMPRESS_WARPS 4
#endif
constexpr int kCompressWarps = ISOQUANT_COMPRESS_WARPS;  // warps per k_compress block
#ifndef ISOQUANT_COMPRESS_BLOCKS
#define ISOQUANT_COMPRESS_BLOCKS (kCompressWarps == 8 ? 2 : 3)
#endif
constexpr int kCompressBlocksPerSm = ISOQUANT_COMPRESS_BLOCKS;
template <typename T, int BITS>
__global__ void __launch_bounds__(kCompressWarps * 32, kCompressBlocksPerSm) k_compress(const CompressArgs g) {
  __shared__ __align__(16) float tile[kCompressWarps][kTileFloats];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5;
  compress_warp<T, BITS>(g, blockIdx.y, blockIdx.x * (blockDim.x >> 5) + warp, threadIdx.x & 31, tile[warp]);
}

// Debug export of the fast path's fp32 z: the same lane-group layouts and
// the same helpers as compress_warp, one vector per lane group, every
// coordinate's z = y / n (fp32, before any fp64 re-check; the compress
// kernel compares |y| with t * n instead) written to
// z[(t * H + h) * 128 + j].
template <typename T>
__global__ void __launch_bounds__(256) k_export_z(const HeadParams *params, const T *x, int n_tok, int H,
                                                  float *z) {
  __shared__ __align__(16) float tile[8][kTileFloats];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, grp = lane >> 3, q = lane & 7, warp = threadIdx.x >> 5;
  const int64_t vec = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp) * 4 + grp;
  // whole warps exit together (the helpers shuffle within the group)
  if ((vec & ~int64_t(3)) >= static_cast<int64_t>(n_tok) * H) return;
  const bool live = vec < static_cast<int64_t>(n_tok) * H;
  const int h = live ? static_cast<int>(vec % H) : 0;
  LaneConsts lc;
  lane_consts(params[h], q, lc);
  float2 a[8];
  if (live) {
    RawA<T> raw;
    load_a(x + vec * kD, q, raw);
    unpack_a(raw, lc.sgn, a);
  } else {
#pragma unroll
    for (int m = 0; m < 8; ++m) a[m] = make_float2(0.f, 0.f);
  }
  const float ssf = group_sum(lane_squares(a));
  // 1/n from the hardware reciprocal square root plus one Newton step
  const float rs = rsqrtf(ssf);
  const float inv = rs * (1.5f - 0.5f * ssf * rs * rs);
  float y[16];
  rotate_two_layouts(a, lc, tile[warp], grp, q, y);
  if (live) {
    float4 *dst = reinterpret_cast<float4 *>(z + vec * kD + 16 * q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = ssf > 0.f ? y[4 * i + e] * inv : 0.f;
      dst[i] = make_float4(o[0], o[1], o[2], o[3]);
    }
  }
}

struct RotateArgs {
  const HeadParams *params;
  const void *q;
  int n_rows, Hq, G;
  float *out;
};

// q_rot = R q for query vector `vec` (row vec / Hq, head vec % Hq).
template <typename T>
__device__ __forceinline__ void rotate_warp(const RotateArgs &g, uint32_t vec, int lane) {
  const HeadParams *__restrict__ params = g.params;
  const T *__restrict__ q = static_cast<const T *>(g.q);
  const int n_rows = g.n_rows, Hq = g.Hq, G = g.G;
  float *__restrict__ out = g.out;
  if (vec >= static_cast<uint32_t>(n_rows) * static_cast<uint32_t>(Hq)) return;
  const int hq = static_cast<int>(vec % static_cast<uint32_t>(Hq));
  float x[4], y[4];
  load4(q + static_cast<int64_t>(vec) * kD + 4 * lane, x);
  rotate_f32(params[hq / G], lane, x, y);
  const float s = 0.08838834764831845f;  // 1/sqrt(128): the normalisation of Hn
  *reinterpret_cast<float4 *>(out + static_cast<int64_t>(vec) * kD + 4 * lane) = make_float4(y[0] * s, y[1] * s, y[2] * s, y[3] * s);
}

template <typename T>
__global__ void __launch_bounds__(256) k_rotate_q(const RotateArgs g) {
  pdl_trigger();
  pdl_wait();
  rotate_warp<T>(g, (blockIdx.x * blockDim.x + threadIdx.x) >> 5, threadIdx.x & 31);
}

// One launch for the two independent halves of a decode step's preparation:
// blocks [0, 2 nbc) compress the new K (first nbc) and V tokens, the rest
// rotate the queries.  Their latency chains overlap instead of adding up.
template <typename T, int BITS>
__global__ void __launch_bounds__(256) k_decode_prep(const CompressArgs c, const RotateArgs r, int nbc) {
  __shared__ __align__(16) float tile[8][kTileFloats];
  pdl_trigger();
  pdl_wait();
  const uint32_t warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bx = static_cast<int>(blockIdx.x);
  if (bx < 2 * nbc) {
    const int kv = bx >= nbc ? 1 : 0;
    compress_warp<T, BITS>(c, kv, static_cast<uint32_t>(bx - kv * nbc) * (blockDim.x >> 5) + warp, lane, tile[warp]);
  } else {
    rotate_warp<T>(r, static_cast<uint32_t>(bx - 2 * nbc) * (blockDim.x >> 5) + warp, lane);
  }
}

}  // namespace

namespace {

// Tokens per warp strip.  A strip loads its head's signs and SO(4) blocks
// once, so long strips amortise that (bulk compression of 32768 x 8 vectors
// per half: 0.187 ms per layer at 16 tokens, 0.162 at 32, 0.154 at 64); a
// short batch (a decode step's few tokens) is spread over many warps
// instead.  The strip is the longest multiple of 4, up to kMaxStrip, that
// still gives each K/V half about as many warps as the SMs hold.
#ifndef ISOQUANT_COMPRESS_STRIP
#define ISOQUANT_COMPRESS_STRIP 64
#endif
constexpr int kMaxStrip = ISOQUANT_COMPRESS_STRIP;
int strip_tokens(const isoquant_ctx *ctx, int n_tok) {
  const int64_t vectors = static_cast<int64_t>(n_tok) * ctx->num_kv_heads;  // per K/V half
  const int64_t resident = static_cast<int64_t>(ctx->num_sms) * kCompressWarps * kCompressBlocksPerSm;  // warps the SMs hold
  const int64_t s = (vectors / resident) & ~int64_t(3);
  return static_cast<int>(s < 4 ? 4 : (s > kMaxStrip ? kMaxStrip : s));
}

CompressArgs compress_args(const isoquant_ctx *ctx, const isoquant_cache *cache, const void *k, const void *v,
                           int n_tok, const int64_t *slot_mapping) {
  CompressArgs g{};
  g.params = ctx->params;
  g.cb = ctx->codebook;
  g.kin = k;
  g.vin = v;
  g.n_tok = n_tok;
  g.H = ctx->num_kv_heads;
  g.slots = slot_mapping;
  g.codes = cache->codes;
  g.norms = cache->norms;
  g.num_pages = cache->num_pages;
  int ps_shift = 0;
  while ((1 << ps_shift) < cache->page_size) ++ps_shift;
  g.ps_shift = ps_shift;
  g.strip = strip_tokens(ctx, n_tok);
  g.status = ctx->status;
  return g;
}

// compress blocks per K/V half (warps_per_block warps each, one strip per warp)
int64_t compress_blocks(const isoquant_ctx *ctx, int n_tok, int warps_per_block) {
  const int strip = strip_tokens(ctx, n_tok);
  const int64_t warps = static_cast<int64_t>((n_tok + strip - 1) / strip) * ctx->num_kv_heads;
  return (warps + warps_per_block - 1) / warps_per_block;
}

RotateArgs rotate_args(const isoquant_ctx *ctx, const void *q, int n_rows, int num_q_heads, float *q_rot) {
  RotateArgs g{};
  g.params = ctx->params;
  g.q = q;
  g.n_rows = n_rows;
  g.Hq = num_q_heads;
  g.G = num_q_heads / ctx->num_kv_heads;
  g.out = q_rot;
  return g;
}

int64_t rotate_blocks(int n_rows, int num_q_heads) {
  return (static_cast<int64_t>(n_rows) * num_q_heads * 32 + 255) / 256;
}

}  // namespace

namespace {
template <int BITS>
cudaError_t launch_compress_t(int dtype, dim3 grid, dim3 block, cudaStream_t stream, const CompressArgs &g) {
  switch (dtype) {
    case ISOQUANT_F32: return launch_pdl(k_compress<float, BITS>, grid, block, 0, stream, g);
    case ISOQUANT_BF16: return launch_pdl(k_compress<__nv_bfloat16, BITS>, grid, block, 0, stream, g);
    default: return launch_pdl(k_compress<__half, BITS>, grid, block, 0, stream, g);
  }
}
template <int BITS>
cudaError_t launch_prep_t(int dtype, dim3 grid, dim3 block, cudaStream_t stream, const CompressArgs &c,
                          const RotateArgs &r, int nb) {
  switch (dtype) {
    case ISOQUANT_F32: return launch_pdl(k_decode_prep<float, BITS>, grid, block, 0, stream, c, r, nb);
    case ISOQUANT_BF16: return launch_pdl(k_decode_prep<__nv_bfloat16, BITS>, grid, block, 0, stream, c, r, nb);
    default: return launch_pdl(k_decode_prep<__half, BITS>, grid, block, 0, stream, c, r, nb);
  }
}
}  // namespace

cudaError_t launch_compress(const isoquant_ctx *ctx, const isoquant_cache *cache, const void *k,
                            const void *v, int dtype, int n_tok, const int64_t *slot_mapping,
                            cudaStream_t stream) {
  const int64_t blocks = compress_blocks(ctx, n_tok, kCompressWarps);
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const CompressArgs g = compress_args(ctx, cache, k, v, n_tok, slot_mapping);
  const dim3 grid(static_cast<unsigned>(blocks), 2), block(kCompressWarps * 32);
  switch (ctx->codebook.bits) {
    case 2: return launch_compress_t<2>(dtype, grid, block, stream, g);
    case 4: return launch_compress_t<4>(dtype, grid, block, stream, g);
    default: return launch_compress_t<3>(dtype, grid, block, stream, g);
  }
}

cudaError_t launch_rotate_q(const isoquant_ctx *ctx, const void *q, int dtype, int n_rows,
                            int num_q_heads, float *q_rot, cudaStream_t stream) {
  const int64_t blocks = rotate_blocks(n_rows, num_q_heads);
  if (blocks == 0) return cudaSuccess;
  const RotateArgs g = rotate_args(ctx, q, n_rows, num_q_heads, q_rot);
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
  switch (dtype) {
    case ISOQUANT_F32: return launch_pdl(k_rotate_q<float>, grid, block, 0, stream, g);
    case ISOQUANT_BF16: return launch_pdl(k_rotate_q<__nv_bfloat16>, grid, block, 0, stream, g);
    default: return launch_pdl(k_rotate_q<__half>, grid, block, 0, stream, g);
  }
}

cudaError_t launch_export_z(const isoquant_ctx *ctx, const void *x, int dtype, int n_tok, float *z,
                            cudaStream_t stream) {
  const int64_t warps = (static_cast<int64_t>(n_tok) * ctx->num_kv_heads + 3) / 4;
  const int64_t blocks = (warps + 7) / 8;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
  const int H = ctx->num_kv_heads;
  switch (dtype) {
    case ISOQUANT_F32:
      return launch_pdl(k_export_z<float>, grid, block, 0, stream, ctx->params, static_cast<const float *>(x), n_tok,
                        H, z);
    case ISOQUANT_BF16:
      return launch_pdl(k_export_z<__nv_bfloat16>, grid, block, 0, stream, ctx->params,
                        static_cast<const __nv_bfloat16 *>(x), n_tok, H, z);
    default:
      return launch_pdl(k_export_z<__half>, grid, block, 0, stream, ctx->params, static_cast<const __half *>(x),
                        n_tok, H, z);
  }
}

cudaError_t launch_decode_prep(const isoquant_ctx *ctx, const isoquant_cache *cache, const void *k, const void *v,
                               int n_tok, const int64_t *slot_mapping, const void *q, int dtype, int n_rows,
                               int num_q_heads, float *q_rot, cudaStream_t stream) {
  const int64_t nbc = compress_blocks(ctx, n_tok, 8);
  const int64_t nbr = rotate_blocks(n_rows, num_q_heads);
  const int64_t blocks = 2 * nbc + nbr;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const CompressArgs c = compress_args(ctx, cache, k, v, n_tok, slot_mapping);
  const RotateArgs r = rotate_args(ctx, q, n_rows, num_q_heads, q_rot);
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
  const int nb = static_cast<int>(nbc);
  switch (ctx->codebook.bits) {
    case 2: return launch_prep_t<2>(dtype, grid, block, stream, c, r, nb);
    case 4: return launch_prep_t<4>(dtype, grid, block, stream, c, r, nb);
    default: return launch_prep_t<3>(dtype, grid, block, stream, c, r, nb);
  }
}

}  // namespace isoquant

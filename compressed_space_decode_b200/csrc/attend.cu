// attend.cu -- isoquant_attend_partial / isoquant_attend_combine.
//
// RotaryQuant, Abstract: attention runs directly on the packed 3-bit
// tensors, without materialising full-precision KV.  Scores and the
// softmax-weighted V sum are formed in the rotated space from the codes; the
// output is rotated back once, in the combine step.
//
// Partial kernel (two CTAs per SM, persistent, split-K over pages):
//   * work = pages of (row group, batch, KV head) pairs, laid end to end;
//     CTA c takes pages [c*P/N, (c+1)*P/N) so that every SM streams the same
//     number of pages whatever the length mix, and writes one partial
//     (m, l, o) per pair it touches.
//   * warp 4 is a producer: per page it issues 28 bulk copies (13 K code
//     rows, 13 V code rows, 2 norm rows) into a 3-stage shared-memory ring
//     with an mbarrier per stage.
//   * warps 0..3 each take a 64-token unit of the page.  A GQA group of up to
//     8 query rows shares every KV tile: Q.K^T is an m16n8k16 tensor-core
//     product with the query split into fp16 high and low parts in the 16
//     rows (so the score keeps ~22 bits), K codes become fp16 centroids
//     through a 64-entry pair table held once per lane in shared memory, and
//     P.V is a second m16n8k16 product with V^T as the A operand.  The eight
//     4-token tiles of a unit run their mma chains interleaved.
//   * at the end of each pair, the warps merge their (m, l, o) in shared
//     memory and one record is written to the workspace.
// Combine kernel: one warp per output row merges the records of its pair,
// divides by l and applies R^-1 = D Hn B^T.
#include <cuda_fp16.h>

#include <cmath>
#include <mutex>

#include "isoquant_internal.cuh"

namespace isoquant {
namespace {

constexpr int kConsumerWarps = 4;
#ifndef ISOQUANT_ATTEND_CTAS_PER_SM
#define ISOQUANT_ATTEND_CTAS_PER_SM 2
#endif
constexpr int kCtasPerSm = ISOQUANT_ATTEND_CTAS_PER_SM;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
#ifndef ISOQUANT_ATTEND_STAGES
#define ISOQUANT_ATTEND_STAGES 3
#endif
constexpr int kStages = ISOQUANT_ATTEND_STAGES;
constexpr int kMaxPage = 256;
// Merge scratch (o[warps][8 rows][128], m[warps][8], l[warps][8], e[8]) is
// placed in the stage buffer being retired when a pair ends, after every
// consumer warp has finished reading it and before the stage is released.
constexpr int kScratchO = 0;
constexpr int kScratchM = kScratchO + kConsumerWarps * 8 * kD * 4;
constexpr int kScratchL = kScratchM + kConsumerWarps * 8 * 4;
constexpr int kScratchE = kScratchL + kConsumerWarps * 8 * 4;

// Shared memory of the mma.sync kernel for BITS-bit codes.  A stage holds one
// page of one (sequence, KV head): W code-word rows of K and of V (row w =
// word w of every token of the page) and the K and V norms.  Row strides (in
// 32-bit words): a quad's four threads read K rows {3t, 3t+1, 3t+2} (3 bits)
// or {t, t+4, ...} (2 and 4 bits) as 16-byte vectors, which a stride = 24 or
// 8 (mod 32) puts in distinct bank groups; V rows {g, g+1} are interleaved by
// a stride = 4 (mod 32).
template <int BITS>
struct DecLayout {
  static constexpr int W = words_for(BITS);
  static constexpr int kCpw = codes_per_word(BITS);                     // codes per word
  static constexpr int kPpw = kCpw / 2;                                 // code pairs per word
  static constexpr int kKWords = 4;                                     // K words a thread reads per token
  static constexpr int kVWords = BITS == 4 ? 2 : 1;                     // V words per token (2, 4 bits)
  static constexpr int kStages = BITS == 4 ? 2 : ::isoquant::kStages;  // 4 bits: 2 stages fit 2 CTAs/SM
  static constexpr int kStrideK = BITS == 3 ? kMaxPage + 24 : kMaxPage + 8;
  static constexpr int kStrideV = kMaxPage + 4;
  static constexpr int kStageKC = 0;
  static constexpr int kStageVC = kStageKC + W * kStrideK * 4;
  static constexpr int kStageKN = kStageVC + W * kStrideV * 4;
  static constexpr int kStageVN = kStageKN + kMaxPage * 2;
  static constexpr int kStageBytes = kStageVN + kMaxPage * 2;
  // query A fragments of the current pair (hi/lo fp16, 8 k-chunks x 32
  // lanes x 16 B) and the per-row power-of-two scale, shared by the warps
  static constexpr int kQFrag = kStages * kStageBytes;
  static constexpr int kQScale = kQFrag + 8 * 32 * 16;
  static constexpr int kBarriers = kQScale + 8 * 4;
  // abort flag (+0), CTA range and walk start (+8..+47)
  static constexpr int kLocate = kBarriers + 2 * kStages * 8;
  // Pair table, entry i = half2(C[i mod 2^BITS], C[i >> BITS]), one copy
  // per lane (entry i of lane l at byte 128 i + 4 l: 32 lanes with 32
  // different entries hit 32 different banks).  At 2 and 3 bits it sits in
  // this dynamic area at an address aligned to its span (2 KB, 8 KB), so an
  // entry's shared address is one AND-OR of the code bits with
  // (table base | 4 lane): no add per lookup.  The 4-bit table (32 KB) stays
  // a static array addressed from its base.
  static constexpr bool kAbsLut = BITS != 4;
  static constexpr int kLutSpan = (1 << (2 * BITS)) * 128;
  static constexpr int kLutArea = kLocate + 64;
  static constexpr int kSmemBytes = kAbsLut ? kLutArea + 2 * kLutSpan : kLocate + 64;
  // bytes a page's copies bring per token: K and V words, K and V norms
  static constexpr int kTxPerToken = 8 * W + 4;
  static constexpr int kLutWords = kAbsLut ? 4 : (1 << (2 * BITS)) * 32;
  static_assert(kScratchE + 8 * 4 <= kStageBytes, "merge scratch must fit in one stage");
  static_assert(kStageBytes % 16 == 0, "stage alignment");
};

struct PartialParams {
  const uint32_t *codes;
  const uint16_t *norms;
  int num_pages, page_size;
  const float *q_rot;
  const int32_t *page_table;
  int max_pages;
  const int32_t *seq_lens;
  int B, nq, Hq, H, G, R, RG, causal;
  float qfold;  // scale * log2(e) / sqrt(128)
  float level[kMaxLevels];
  int bits;  // code width of the cache (2, 3 or 4)
  float *records;
  uint32_t *status;
  int n_cta;
  int64_t *prefix;  // tcgen05 kernels: pages before each (stream, sequence) unit
  int vpages;       // tcgen05 kernels: work-free pages that follow each (unit, head) block
  uint32_t *plan;   // first word of the workspace header: receives plan_tag
  uint32_t plan_tag;
};

struct CombineParams {
  const float *records;
  const HeadParams *params;
  const int32_t *seq_lens;
  float *out;
  int B, nq, Hq, H, G, RG, page_size, n_cta;
  int rps;  // query rows per stream: 8 (mma.sync kernel), 64 or 128 (tcgen05 kernels)
  const int64_t *prefix;  // null for the mma.sync kernel
  int vpages;             // as in PartialParams
  uint32_t *status;
  const uint32_t *plan;   // the tag the partial kernel wrote
  uint32_t plan_tag;      // the tag of the plan this combine expects
};

// ------------------------------------------------------------------ PTX
// (mbarrier waits and bulk copies: isoquant_internal.cuh)
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// 2^x by the SFU (ex2.approx, relative error below 2^-22; 2^-inf = +0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// High part of w >= 0 for an fp16 high/low split: w with its 13 low
// mantissa bits cleared (exact in fp16 for 2^-14 <= w < 65520), or 0 below
// 2^-14, where all of w goes to the low part; w - high is exact in fp32 and
// below 2^-10 w, so the two fp16 parts keep ~21 bits.  Bit operations
// instead of a round trip through fp16 conversions.
__device__ __forceinline__ float hi_part(float w) {
  const float h = __uint_as_float(__float_as_uint(w) & 0xFFFFE000u);
  return w >= 6.103515625e-05f ? h : 0.f;
}
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// ------------------------------------------------------------ work walk
__device__ __forceinline__ int pages_of(int L, int ps) { return L > 0 ? (L + ps - 1) / ps : 0; }

__device__ __forceinline__ int64_t warp_sum64(int64_t v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// sum over b < b_end of pages_of(seq_lens[b]) (whole warp participates)
__device__ int64_t pages_before(const int32_t *seq_lens, int b_end, int ps, int lane) {
  int64_t s = 0;
  for (int b0 = 0; b0 < b_end; b0 += 32) {
    const int b = b0 + lane;
    s += (b < b_end) ? pages_of(seq_lens[b], ps) : 0;
  }
  return warp_sum64(s);
}

// Find the batch b whose pages (H per page index) contain offset `rem` of a
// row-group slab; returns b and H * (pages before b).
__device__ void locate_batch(const int32_t *seq_lens, int B, int H, int ps, int64_t rem, int lane, int &b_out,
                             int64_t &before_out) {
  int64_t base = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const int64_t np = (b < B) ? static_cast<int64_t>(H) * pages_of(seq_lens[b], ps) : 0;
    int64_t incl = np;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const int64_t excl = incl - np;
    const unsigned hit = __ballot_sync(0xffffffffu, base + excl <= rem && rem < base + incl);
    if (hit) {
      const int src = __ffs(hit) - 1;
      b_out = b0 + src;
      before_out = __shfl_sync(0xffffffffu, base + excl, src);
      return;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  b_out = B;
  before_out = base;
}

struct Walk {
  int rg, b, h, j, np, L;
  __device__ void advance(const int32_t *seq_lens, int B, int H, int ps) {
    if (++j < np) return;
    j = 0;
    if (++h < H) return;
    h = 0;
    do {
      if (++b == B) { b = 0; ++rg; }
      L = seq_lens[b];
      np = pages_of(L, ps);
    } while (np == 0);
  }
};

// ------------------------------------------------------------ unit walk
// The tcgen05 kernels split pages of (stream, sequence, KV head), a stream
// being `rps` consecutive query rows of a KV head.  Under causal masking
// stream rg of sequence b sees only the first L - nq + q_last + 1 tokens
// (q_last = its last query position), so it walks only the pages holding
// them: unit u = rg * B + b carries H * pages_of(horizon) pages.  Causal
// prefill thus costs the triangle, not the square.
__device__ __forceinline__ int unit_horizon(const PartialParams &p, int rps, int rg, int b) {
  const int L = p.seq_lens[b];
  if (!p.causal) return max(L, 0);
  const int q_last = min(p.nq - 1, (rg * rps + rps - 1) / p.G);
  return max(0, min(L, L - p.nq + q_last + 1));
}
// The CTAs split pages evenly; where a stream's switch in a CTA costs as
// much as a few pages of work (k_attend_wide: its queries are loaded, its
// record written, the pipeline drains), each (unit, head) block of np real
// pages is followed by vpages work-free ones, so that the split balances
// work rather than pages (a causal prefill's early streams are one or two
// tiles long).  (Units and the pages of one unit are counted in 32 bits:
// make_shape and isoquant_attend_partial refuse shapes where row groups x
// sequences x KV heads or (max_pages + 16) x KV heads reach 2^31 - 1.)
__device__ __forceinline__ int64_t unit_pages(const PartialParams &p, int rps, int u) {
  const int rg = u / p.B, b = u - rg * p.B;
  const int np = pages_of(unit_horizon(p, rps, rg, b), p.page_size);
  return np > 0 ? static_cast<int64_t>(p.H) * (np + p.vpages) : 0;
}

struct UWalk {
  int u, rg, b, h, j, np, nb, hz;  // j < nb = np + vpages; pages j >= np carry no work
  __device__ void set(const PartialParams &p, int rps, int u_) {
    u = u_;
    rg = u / p.B;
    b = u - rg * p.B;
    hz = unit_horizon(p, rps, rg, b);
    np = pages_of(hz, p.page_size);
    nb = np + p.vpages;
  }
  __device__ void start(const PartialParams &p, int rps, int u_, int off) {
    set(p, rps, u_);
    h = off / nb;
    j = off - h * nb;
  }
  __device__ void advance(const PartialParams &p, int rps) {
    if (++j < nb) return;
    j = 0;
    if (++h < p.H) return;
    h = 0;
    do set(p, rps, u + 1); while (np == 0);
  }
  // to page 0 of the next (unit, head) block that has pages
  __device__ void next_block(const PartialParams &p, int rps) {
    j = nb - 1;
    advance(p, rps);
  }
  __device__ bool real() const { return j < np; }
  // tokens of the current page this stream sees, and its 64-token tiles
  __device__ int page_tokens(int ps) const { return min(ps, hz - j * ps); }
};

// Every thread of the CTA: sum the pages of all units (each thread a slice
// of units, then a scan over the slices), take this CTA's range [gs, ge) of
// the total and find the unit and page offset where it starts:
// loc = {gs, ge, unit, offset}.  CTA 0 also writes prefix[u] (pages before
// unit u) and prefix[U] = total for the combine kernel.  Ends with
// __syncthreads.
template <int NT>
__device__ void tile_locate(const PartialParams &p, int rps, int64_t *scratch, int64_t *loc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int U = p.RG * p.B;
  const int u0 = static_cast<int>(static_cast<int64_t>(U) * tid / NT),
            u1 = static_cast<int>(static_cast<int64_t>(U) * (tid + 1) / NT);
  int64_t mine = 0;
  for (int u = u0; u < u1; ++u) mine += unit_pages(p, rps, u);
  int64_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int64_t before = 0, total = 0;
  for (int w = 0; w < NT / 32; ++w) {
    if (w < warp) before += scratch[w];
    total += scratch[w];
  }
  const int64_t excl = before + incl - mine;
  const int64_t gs = total * blockIdx.x / p.n_cta, ge = total * (blockIdx.x + 1) / p.n_cta;
  if (blockIdx.x == 0 && p.prefix != nullptr) {
    int64_t run = excl;
    for (int u = u0; u < u1; ++u) {
      p.prefix[u] = run;
      run += unit_pages(p, rps, u);
    }
    if (tid == NT - 1) p.prefix[U] = total;
  }
  if (gs < ge && excl <= gs && gs < excl + mine) {
    int64_t run = excl;
    for (int u = u0; u < u1; ++u) {
      const int64_t n = unit_pages(p, rps, u);
      if (gs < run + n) {
        loc[0] = gs;
        loc[1] = ge;
        loc[2] = u;
        loc[3] = gs - run;
        break;
      }
      run += n;
    }
  }
  if (tid == 0 && !(gs < ge)) {
    loc[0] = gs;
    loc[1] = ge;
  }
  __syncthreads();
}

// ------------------------------------------------------------ pair table
// s_lut[idx * 32 + lane] = half2(C[idx & 7], C[idx >> 3]): one copy per lane
// so that 32 lanes with 32 different indices hit 32 different banks.
__shared__ __align__(16) uint32_t s_lut[64 * 32];

// x >> SH for SH >= 0, x << -SH otherwise (SH a compile-time constant).
// (Shifting by multiplication on the FMA pipe instead, to unload the
// half-rate ALU pipe, was measured slower: the high-word multiplies stalled
// instruction dispatch.)
template <int SH>
__device__ __forceinline__ uint32_t shifted(uint32_t x) {
  static_assert(SH > -32 && SH < 32, "shift range");
  if constexpr (SH < 0) return x << (-SH);
  else return x >> SH;
}
// Byte offset of entry ((x >> (SH + 7)) & 63) for this lane: the entry index
// lands in bits 7..12 and the lane's bank in bits 2..6, so one AND-OR forms it.
template <int SH>
__device__ __forceinline__ uint32_t lut_off(uint32_t x, uint32_t lane4) {
  return (shifted<SH>(x) & 0x1F80u) | lane4;
}
__device__ __forceinline__ uint32_t lut_at(uint32_t off) {
  return *reinterpret_cast<const uint32_t *>(reinterpret_cast<const char *>(s_lut) + off);
}
// A table entry at a shared-window address (the decode kernel's aligned table).
__device__ __forceinline__ uint32_t plut(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// five adjacent-code pairs (2k, 2k+1), k = 0..4, of a packed word
// (lane4: the aligned table's base | 4 lane)
__device__ __forceinline__ void word_pairs(uint32_t w, uint32_t lane4, uint32_t *out) {
  out[0] = plut(lut_off<-7>(w, lane4));
  out[1] = plut(lut_off<-1>(w, lane4));
  out[2] = plut(lut_off<5>(w, lane4));
  out[3] = plut(lut_off<11>(w, lane4));
  out[4] = plut(lut_off<17>(w, lane4));
}

// The tcgen05 kernels' decode tables, one copy per lane: BITS = 3: entry i =
// half2(C[i & 7], C[i >> 3]) for the 64 code pairs; BITS = 2: the 16 pairs,
// half2(C[i & 3], C[i >> 2]); BITS = 4: the 16 single codes, C[i] in the
// low half (a pair is assembled from two entries).
template <int BITS>
__device__ __forceinline__ void fill_lut(const float *level, int tid, int nthreads) {
  constexpr int kEntries = BITS == 3 ? 64 : 16;
  for (int e = tid; e < kEntries * 32; e += nthreads) {
    const int idx = e >> 5;
    if constexpr (BITS == 3) s_lut[e] = pack_half2(level[idx & 7], level[idx >> 3]);
    else if constexpr (BITS == 2) s_lut[e] = pack_half2(level[idx & 3], level[idx >> 2]);
    else s_lut[e] = pack_half2(level[idx], 0.f);
  }
}
// One token's code words (word w at cw[w * ps + t]) ...
template <int BITS>
__device__ __forceinline__ void load_token_words(const uint32_t *cw, int ps, int t, uint32_t (&x)[words_for(BITS)]) {
#pragma unroll
  for (int w = 0; w < words_for(BITS); ++w) x[w] = __ldg(cw + w * ps + t);
}
// ... pair p of its codes (dims 2p, 2p + 1) as half2 ...
template <int BITS>
__device__ __forceinline__ uint32_t decode_pair(const uint32_t (&x)[words_for(BITS)], uint32_t lane4, int p) {
  if constexpr (BITS == 3) {
    return lut_at((((x[p / 5] >> (6 * (p % 5))) & 63u) << 7) | lane4);
  } else if constexpr (BITS == 2) {
    return lut_at((((x[p / 8] >> (4 * (p % 8))) & 15u) << 7) | lane4);
  } else {
    const uint32_t lo = lut_at((((x[p / 4] >> (8 * (p % 4))) & 15u) << 7) | lane4);
    const uint32_t hi = lut_at((((x[p / 4] >> (8 * (p % 4) + 4)) & 15u) << 7) | lane4);
    return __byte_perm(lo, hi, 0x5410);
  }
}
// ... or all 128 fp16 centroids as 64 half2 (dims 2i, 2i + 1 in out[i])
template <int BITS>
__device__ __forceinline__ void decode_token_words(const uint32_t (&x)[words_for(BITS)], uint32_t lane4,
                                                   uint32_t (&out)[64]) {
#pragma unroll
  for (int i = 0; i < 64; ++i) out[i] = decode_pair<BITS>(x, lane4, i);
}

__device__ __forceinline__ uint32_t u4_at(const uint4 &v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Q.K^T B-fragment register for pair k (0..15) of token j of a 4-token group:
// pairs 0..14 are adjacent codes (2(k%5), 2(k%5)+1) of words 3tq + k/5;
// pair 15 is codes (2tq, 2tq+1) of word 12 (shift sh12 = 6tq).
template <int K>
__device__ __forceinline__ uint32_t k_pair_c(const uint4 (&kw)[4], int j, uint32_t sh12, uint32_t lane4) {
  if constexpr (K < 15) {
    return plut(lut_off<6 * (K % 5) - 7>(u4_at(kw[K / 5], j), lane4));
  } else {
    return plut((((u4_at(kw[3], j) << 7) >> sh12) & 0x1F80u) | lane4);
  }
}
// 2 and 4 bits: pair k (0..15) is pair k mod P (P = pairs per word) of word
// k / P of the thread's words tq, tq + 4, ...: its 2 * BITS bits start at
// bit 2 * BITS * (k mod P); the table has 2^(2 BITS) entries.
template <int SH, uint32_t MASK>
__device__ __forceinline__ uint32_t lut_off_m(uint32_t x, uint32_t lane4) {
  return (shifted<SH>(x) & MASK) | lane4;
}
// 2 bits: off is a shared-window address (aligned table | 4 lane); 4 bits: a
// byte offset into the static table `lut`
template <int BITS>
__device__ __forceinline__ uint32_t lut_at2(const char *lut, uint32_t off) {
  if constexpr (BITS == 4) return *reinterpret_cast<const uint32_t *>(lut + off);
  else return plut(off);
}
template <int BITS, int K>
__device__ __forceinline__ uint32_t k_pair_w(const uint4 (&kw)[4], int j, uint32_t lane4, const char *lut) {
  constexpr int kPpw = 16 / BITS;
  constexpr uint32_t kMask = ((1u << (2 * BITS)) - 1u) << 7;
  return lut_at2<BITS>(lut, lut_off_m<2 * BITS * (K % kPpw) - 7, kMask>(u4_at(kw[K / kPpw], j), lane4));
}
// Slot K of a merged word, looked up
template <int BITS, uint32_t MASK, int K>
__device__ __forceinline__ uint32_t merged_pair(uint32_t e, uint32_t lane4, const char *lut) {
  return lut_at2<BITS>(lut, lut_off_m<2 * BITS * K - 7, MASK>(e, lane4));
}
// The kPpw 2*BITS-bit slots of a merged word, looked up in order
template <int BITS>
__device__ __forceinline__ void merged_pairs(uint32_t e, uint32_t lane4, const char *lut, uint32_t *out) {
  constexpr int kPpw = 16 / BITS;
  constexpr uint32_t kMask = ((1u << (2 * BITS)) - 1u) << 7;
  out[0] = merged_pair<BITS, kMask, 0>(e, lane4, lut);
  out[1] = merged_pair<BITS, kMask, 1>(e, lane4, lut);
  out[2] = merged_pair<BITS, kMask, 2>(e, lane4, lut);
  out[3] = merged_pair<BITS, kMask, 3>(e, lane4, lut);
  if constexpr (kPpw > 4) {
    out[4] = merged_pair<BITS, kMask, 4>(e, lane4, lut);
    out[5] = merged_pair<BITS, kMask, 5>(e, lane4, lut);
    out[6] = merged_pair<BITS, kMask, 6>(e, lane4, lut);
    out[7] = merged_pair<BITS, kMask, 7>(e, lane4, lut);
  }
}
template <int BITS>
__device__ __forceinline__ uint32_t k_pair(const uint4 (&kw)[4], int j, int k, uint32_t sh12, uint32_t lane4,
                                           const char *lut) {
  if constexpr (BITS == 3) {
    switch (k) {
      case 0: return k_pair_c<0>(kw, j, sh12, lane4);
      case 1: return k_pair_c<1>(kw, j, sh12, lane4);
      case 2: return k_pair_c<2>(kw, j, sh12, lane4);
      case 3: return k_pair_c<3>(kw, j, sh12, lane4);
      case 4: return k_pair_c<4>(kw, j, sh12, lane4);
      case 5: return k_pair_c<5>(kw, j, sh12, lane4);
      case 6: return k_pair_c<6>(kw, j, sh12, lane4);
      case 7: return k_pair_c<7>(kw, j, sh12, lane4);
      case 8: return k_pair_c<8>(kw, j, sh12, lane4);
      case 9: return k_pair_c<9>(kw, j, sh12, lane4);
      case 10: return k_pair_c<10>(kw, j, sh12, lane4);
      case 11: return k_pair_c<11>(kw, j, sh12, lane4);
      case 12: return k_pair_c<12>(kw, j, sh12, lane4);
      case 13: return k_pair_c<13>(kw, j, sh12, lane4);
      case 14: return k_pair_c<14>(kw, j, sh12, lane4);
      default: return k_pair_c<15>(kw, j, sh12, lane4);
    }
  } else {
    switch (k) {
      case 0: return k_pair_w<BITS, 0>(kw, j, lane4, lut);
      case 1: return k_pair_w<BITS, 1>(kw, j, lane4, lut);
      case 2: return k_pair_w<BITS, 2>(kw, j, lane4, lut);
      case 3: return k_pair_w<BITS, 3>(kw, j, lane4, lut);
      case 4: return k_pair_w<BITS, 4>(kw, j, lane4, lut);
      case 5: return k_pair_w<BITS, 5>(kw, j, lane4, lut);
      case 6: return k_pair_w<BITS, 6>(kw, j, lane4, lut);
      case 7: return k_pair_w<BITS, 7>(kw, j, lane4, lut);
      case 8: return k_pair_w<BITS, 8>(kw, j, lane4, lut);
      case 9: return k_pair_w<BITS, 9>(kw, j, lane4, lut);
      case 10: return k_pair_w<BITS, 10>(kw, j, lane4, lut);
      case 11: return k_pair_w<BITS, 11>(kw, j, lane4, lut);
      case 12: return k_pair_w<BITS, 12>(kw, j, lane4, lut);
      case 13: return k_pair_w<BITS, 13>(kw, j, lane4, lut);
      case 14: return k_pair_w<BITS, 14>(kw, j, lane4, lut);
      default: return k_pair_w<BITS, 15>(kw, j, lane4, lut);
    }
  }
}

// ------------------------------------------------------------ merging
// CTA that owns global page g when P pages are split as [c P / N, (c+1) P / N)
__device__ __forceinline__ int64_t cta_of_page(int64_t g, int64_t N, int64_t P) {
  return ((g + 1) * N + P - 1) / P - 1;
}
// The CTAs that hold a pair's pages [g0, g0 + np) of the P pages split over
// N CTAs: with P >= N every CTA of the range c_lo..c_hi holds at least one
// page; with fewer pages than CTAs each CTA holds at most one, so the owners
// are the np pages' CTAs, and the many CTAs in between (empty ranges, no
// record) are never visited.
struct Owners {
  int64_t c_lo, g0, N, P, count;
  bool dense;
  __device__ Owners(int64_t g0_, int np, int64_t N_, int64_t P_) : g0(g0_), N(N_), P(P_) {
    c_lo = cta_of_page(g0, N, P);
    dense = P >= N;
    count = dense ? cta_of_page(g0 + np - 1, N, P) - c_lo + 1 : np;
  }
  __device__ int64_t at(int64_t j) const { return dense ? c_lo + j : cta_of_page(g0 + j, N, P); }
};

// Merge the records that the owners of `pair`'s pages wrote for rows
// rr[0..NR), divide by l and apply R^-1 = D Hn B^T of head parameters hp;
// the warp stores row k's 128 outputs at dst[k] (lane holds dims 4 lane ..
// 4 lane + 3), or skips row k when dst[k] is null.  Latency, not bandwidth,
// bounds this: lane i fetches the (m, l) of owner i's record, and the o
// vectors are fetched 8 (record, row) pairs at a time before any is used.  Records are read through L2
// (ld.global.cg): in the fused path other CTAs of the running grid wrote
// them.
// Record of CTA c for the stream: slot (c + stream) * per + sub.
template <int NR>
__device__ __forceinline__ void merge_rows(const float *records, int64_t pair, int per, int sub, const Owners &own,
                                           const int (&rr)[NR], float *const (&dst)[NR], const HeadParams &hp,
                                           int lane) {
  // this lane's rows of B^T, fetched first so that their latency overlaps
  const float4 *mb4 = reinterpret_cast<const float4 *>(hp.m32[lane]);
  const float4 mb[4] = {mb4[0], mb4[1], mb4[2], mb4[3]};
  const uint32_t sn = (hp.sign_bits[lane >> 3] >> (4 * (lane & 7))) & 0xFu;

  // pass 1: running (max, sum) per lane over its records, then across lanes
  float mr[NR], lr[NR], m0[NR];
#pragma unroll
  for (int k = 0; k < NR; ++k) { mr[k] = -INFINITY; lr[k] = 0.f; m0[k] = -INFINITY; }
  const int64_t count = own.count;
  for (int64_t j0 = 0; j0 < count; j0 += 32) {
    const int64_t j = j0 + lane;
    if (j < count) {
      const float *rec = records + ((own.at(j) + pair) * per + sub) * kRecordFloats;
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(rec + 2 * rr[k]));
        if (j0 == 0) m0[k] = ml.x;
        if (ml.x > mr[k]) {
          lr[k] = lr[k] * ex2(mr[k] - ml.x) + ml.y;
          mr[k] = ml.x;
        } else if (ml.x != -INFINITY) {
          lr[k] += ml.y * ex2(ml.x - mr[k]);
        }
      }
    }
  }
  float M[NR], l[NR], o[NR][4];
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    M[k] = mr[k];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M[k] = fmaxf(M[k], __shfl_xor_sync(0xffffffffu, M[k], off));
    l[k] = (mr[k] == -INFINITY) ? 0.f : lr[k] * ex2(mr[k] - M[k]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) l[k] += __shfl_xor_sync(0xffffffffu, l[k], off);
    o[k][0] = o[k][1] = o[k][2] = o[k][3] = 0.f;
  }
  // pass 2: o = sum over records of 2^(m - M) o_c
  for (int64_t j0 = 0; j0 < count; j0 += 32) {
    const int64_t j = j0 + lane;
    const bool mine = j < count;
    // this lane's owner (record slot), handed to the other lanes below
    const int64_t slot = ((mine ? own.at(j) : own.c_lo) + pair) * per + sub;
    float sm[NR];
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      float mc = m0[k];
      if (j0 != 0) mc = mine ? __ldcg(records + slot * kRecordFloats + 2 * rr[k]) : -INFINITY;
      sm[k] = (!mine || M[k] == -INFINITY) ? 0.f : ex2(mc - M[k]);
    }
    const int n = static_cast<int>(count - j0 < 32 ? count - j0 : 32);
    constexpr int kBatch = 8 / NR;
    for (int i0 = 0; i0 < n; i0 += kBatch) {
      float sv[kBatch][NR];
      float4 v[kBatch][NR];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t sl = __shfl_sync(0xffffffffu, slot, (i0 + u) & 31);
        const float *rec = records + sl * kRecordFloats + 16 + 4 * lane;
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          sv[u][k] = __shfl_sync(0xffffffffu, sm[k], (i0 + u) & 31);
          v[u][k] = (i0 + u < n && sv[u][k] != 0.f) ? __ldcg(reinterpret_cast<const float4 *>(rec + rr[k] * kD))
                                                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          o[k][0] += sv[u][k] * v[u][k].x; o[k][1] += sv[u][k] * v[u][k].y;
          o[k][2] += sv[u][k] * v[u][k].z; o[k][3] += sv[u][k] * v[u][k].w;
        }
    }
  }
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    if (dst[k] == nullptr) continue;
    if (M[k] == -INFINITY || !(l[k] > 0.f)) {
      *reinterpret_cast<float4 *>(dst[k]) = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    // o~ = sum p n C / (l sqrt(128)); then R^-1 = D Hn B^T, Hn = H / sqrt(128)
    const float inv = 1.f / (l[k] * 128.f);
    float y[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float *b0 = reinterpret_cast<const float *>(&mb[0]), *b1 = reinterpret_cast<const float *>(&mb[1]);
      const float *b2 = reinterpret_cast<const float *>(&mb[2]), *b3 = reinterpret_cast<const float *>(&mb[3]);
      y[c] = fmaf(b3[c], o[k][3], fmaf(b2[c], o[k][2], fmaf(b1[c], o[k][1], b0[c] * o[k][0])));
    }
    wht128<float>(y, lane);
    float res[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) res[c] = __uint_as_float(__float_as_uint(y[c] * inv) ^ (((sn >> c) & 1u) << 31));
    *reinterpret_cast<float4 *>(dst[k]) = make_float4(res[0], res[1], res[2], res[3]);
  }
}

// The partial kernel of a call records which plan (kernel, rows per stream,
// streams, CTAs) laid out the records, so that a combine launched with
// another plan (a different workspace size passed to the two halves) sees
// the mismatch instead of merging the wrong records.
__device__ __forceinline__ void write_plan_tag(const PartialParams &p) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.plan = p.plan_tag;
}

// ------------------------------------------------------------ partial kernel
template <int BITS>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) k_attend_partial(const PartialParams p) {
  using L = DecLayout<BITS>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(16) uint32_t lutw[L::kLutWords];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tq = lane & 3;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarriers);
  uint64_t *empty = full + L::kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kLocate);
  int64_t *loc = reinterpret_cast<int64_t *>(smem + L::kLocate + 8);
  const int ps = p.page_size;

  uint32_t lut_lane = static_cast<uint32_t>(lane) * 4u;  // table base | 4 lane (4 bits: 4 lane)
  if constexpr (L::kAbsLut) {
    const uint32_t base = (smem_addr(smem + L::kLutArea) + L::kLutSpan - 1) & ~static_cast<uint32_t>(L::kLutSpan - 1);
    for (int e = tid; e < L::kLutSpan / 4; e += kThreads) {
      const int idx = e >> 5;
      const uint32_t v = pack_half2(p.level[idx & ((1 << BITS) - 1)], p.level[idx >> BITS]);
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(base + 4u * e), "r"(v) : "memory");
    }
    lut_lane |= base;
  } else {
    for (int e = tid; e < L::kLutWords; e += kThreads) {
      const int idx = e >> 5;
      lutw[e] = pack_half2(p.level[idx & ((1 << BITS) - 1)], p.level[idx >> BITS]);
    }
  }
  const char *lutb = reinterpret_cast<const char *>(lutw);
  if (tid == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the set-up above touches only shared memory; global memory from here on
  pdl_trigger();
  pdl_wait();
  write_plan_tag(p);
  // CTA's page range [gs, ge) and where it starts
  if (warp == 0) {
    const int64_t pb = pages_before(p.seq_lens, p.B, ps, lane);
    const int64_t p_rg = static_cast<int64_t>(p.H) * pb;
    const int64_t total = p_rg * p.RG;
    const int64_t gs = total * blockIdx.x / p.n_cta;
    const int64_t ge = total * (blockIdx.x + 1) / p.n_cta;
    int b = 0;
    int64_t before = 0;
    int64_t rem = 0, rg = 0;
    if (gs < ge) {
      rg = gs / p_rg;
      rem = gs - rg * p_rg;
      locate_batch(p.seq_lens, p.B, p.H, ps, rem, lane, b, before);
    }
    if (lane == 0) {
      loc[0] = gs;
      loc[1] = ge;
      loc[2] = rg;
      loc[3] = b;
      loc[4] = rem - before;  // offset inside batch b's H * np pages
    }
  }
  __syncthreads();
  const int64_t gs = loc[0], ge = loc[1];
  if (gs >= ge) return;
  Walk wk;
  wk.rg = static_cast<int>(loc[2]);
  wk.b = static_cast<int>(loc[3]);
  wk.L = p.seq_lens[wk.b];
  wk.np = pages_of(wk.L, ps);
  wk.h = static_cast<int>(loc[4] / wk.np);
  wk.j = static_cast<int>(loc[4] - static_cast<int64_t>(wk.h) * wk.np);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    int64_t it = 0;
    for (int64_t g = gs; g < ge; ++g, ++it) {
      const int stage = static_cast<int>(it % L::kStages);
      const uint32_t round = static_cast<uint32_t>(it / L::kStages);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[stage], (round & 1u) ^ 1u, p.status, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      int phys = -1;
      if (wk.j < p.max_pages) phys = p.page_table[static_cast<int64_t>(wk.b) * p.max_pages + wk.j];
      if (phys < 0 || phys >= p.num_pages) {
        if (lane == 0) set_status(p.status, ISOQUANT_DEVERR_PAGE_RANGE);
        phys = 0;
      }
      uint8_t *st = smem + static_cast<size_t>(stage) * L::kStageBytes;
      if (lane == 0) mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(L::kTxPerToken * ps));
      __syncwarp();
      const int64_t kblk = (static_cast<int64_t>(phys) * 2 + 0) * p.H + wk.h;
      const int64_t vblk = (static_cast<int64_t>(phys) * 2 + 1) * p.H + wk.h;
      // one bulk copy per code-word row of K and V, and the two norm rows
      for (int c = lane; c < 2 * L::W + 2; c += 32) {
        if (c < L::W) {
          bulk_g2s(st + L::kStageKC + c * L::kStrideK * 4, p.codes + (kblk * L::W + c) * ps,
                   static_cast<uint32_t>(ps * 4), &full[stage]);
        } else if (c < 2 * L::W) {
          const int w = c - L::W;
          bulk_g2s(st + L::kStageVC + w * L::kStrideV * 4, p.codes + (vblk * L::W + w) * ps,
                   static_cast<uint32_t>(ps * 4), &full[stage]);
        } else if (c == 2 * L::W) {
          bulk_g2s(st + L::kStageKN, p.norms + kblk * ps, static_cast<uint32_t>(ps * 2), &full[stage]);
        } else {
          bulk_g2s(st + L::kStageVN, p.norms + vblk * ps, static_cast<uint32_t>(ps * 2), &full[stage]);
        }
      }
      if (g + 1 < ge) wk.advance(p.seq_lens, p.B, p.H, ps);
    }
    // wait (bounded) for every copy still in flight before the CTA exits
    if (lane == 0) {
      const int64_t issued = it;
      for (int64_t k = (issued > L::kStages ? issued - L::kStages : 0); k < issued; ++k)
        mbar_wait(&full[k % L::kStages], static_cast<uint32_t>((k / L::kStages) & 1), p.status, nullptr);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const uint32_t lane4 = lut_lane;

  // dims this thread feeds to Q.K^T: pair k (k = 0..15) = coordinates
  // (kdim(k), kdim(k) + 1); pairs 0..14 come from words 3tq..3tq+2, pair 15
  // from word 12.
  // (2 and 4 bits: pairs of words tq, tq + 4, ..., kPpw pairs per word)
  auto kdim = [&](int k) -> int {
    if constexpr (BITS == 3) return k < 15 ? 10 * (3 * tq + k / 5) + 2 * (k % 5) : 120 + 2 * tq;
    else return (tq + 4 * (k / L::kPpw)) * L::kCpw + 2 * (k % L::kPpw);
  };
  // dims this thread feeds to P.V (rows gid / gid+8 of each 16-dim tile):
  // word gid fully, half of word 8 + gid/2, code gid of word 12.
  const int par = gid & 1;
  // 2 bits: word gid (even dims, then odd ones); 4 bits: words gid and
  // 8 + gid (each: even dims, then odd ones)
  auto vdim = [&](int k) -> int {
    if constexpr (BITS == 3) {
      if (k < 5) return 10 * gid + 2 * k;
      if (k < 10) return 10 * gid + 2 * (k - 5) + 1;
      if (k < 15) return 10 * (8 + (gid >> 1)) + par + 2 * (k - 10);
      return 120 + gid;
    } else if constexpr (BITS == 2) {
      return 16 * gid + (k < 8 ? 2 * k : 2 * (k - 8) + 1);
    } else {
      const int w = k < 8 ? gid : 8 + gid, kk = k & 7;
      return 8 * w + (kk < 4 ? 2 * kk : 2 * (kk - 4) + 1);
    }
  };

  uint4 *sq = reinterpret_cast<uint4 *>(smem + L::kQFrag);
  float *sq_scale = reinterpret_cast<float *>(smem + L::kQScale);
  float acc[8][4];
  float m_run = -INFINITY, l_run = 0.f, inv2e = 1.f;
  int lim = 0, lim_min = 0, lim_max = 0;

  int stage = 0;
  uint32_t phase = 0;
  for (int64_t g = gs; g < ge; ++g) {
    const bool seg_start = (g == gs) || (wk.j == 0);
    const bool seg_end = (g + 1 == ge) || (wk.j + 1 == wk.np);
    if (seg_start) {
      // every warp is done with the previous pair's query fragments
      named_bar_sync(1, kConsumerWarps * 32);
      const int r = wk.rg * 8 + gid;
      const bool valid = r < p.R;
      const int qi = valid ? r / p.G : 0;
      if (warp == 0) {
        // this pair's query rows as hi/lo fp16 A fragments, into shared memory
        const int hq = wk.h * p.G + (valid ? r % p.G : 0);
        const float *qp = p.q_rot + ((static_cast<int64_t>(wk.b) * p.nq + qi) * p.Hq + hq) * kD;
        float qv[32];
        float mx = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int d0 = kdim(k);
          qv[2 * k] = valid ? qp[d0] * p.qfold : 0.f;
          qv[2 * k + 1] = valid ? qp[d0 + 1] * p.qfold : 0.f;
          mx = fmaxf(mx, fmaxf(fabsf(qv[2 * k]), fabsf(qv[2 * k + 1])));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // power-of-two prescale: the largest |q| lands in [2^14, 2^15)
        int ex = 0;
        if (mx > 0.f) frexpf(mx, &ex);
        ex = max(ex, -100);
        const float up = ldexpf(1.f, 15 - ex);
        if (tq == 0) sq_scale[gid] = ldexpf(1.f, ex - 15);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t hl[4];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int k = 2 * c + e;
            const float a = qv[2 * k] * up, b = qv[2 * k + 1] * up;
            const __half ah = __float2half_rn(a), bh = __float2half_rn(b);
            hl[2 * e] = pack_half2(__half2float(ah), __half2float(bh));
            hl[2 * e + 1] = pack_half2(a - __half2float(ah), b - __half2float(bh));
          }
          sq[c * 32 + lane] = make_uint4(hl[0], hl[1], hl[2], hl[3]);
        }
      }
      named_bar_sync(1, kConsumerWarps * 32);
      inv2e = sq_scale[gid];
      const int L = wk.L;
      lim = valid ? (p.causal ? L - p.nq + qi + 1 : L) : L;
      lim = max(lim, 0);
      lim_min = p.causal ? max(L - p.nq + 1, 0) : L;
      lim_max = L;
#pragma unroll
      for (int m = 0; m < 8; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
      m_run = -INFINITY;
      l_run = 0.f;
    }

    bool ok = true;
    if (lane == 0) ok = mbar_wait(&full[stage], phase, p.status, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    const uint8_t *st = smem + static_cast<size_t>(stage) * L::kStageBytes;
    const uint32_t *kc = reinterpret_cast<const uint32_t *>(st + L::kStageKC);
    const uint32_t *vc = reinterpret_cast<const uint32_t *>(st + L::kStageVC);
    const __half *kn = reinterpret_cast<const __half *>(st + L::kStageKN);
    const __half *vn = reinterpret_cast<const __half *>(st + L::kStageVN);

    // each warp takes 64-token units: two 32-token halves whose independent
    // work interleaves, sharing one softmax reduction
    for (int sc = warp; ok && sc * 64 < ps; sc += kConsumerWarps) {
      const int t0 = sc * 64;                       // first token of the unit in the page
      const int tok0 = wk.j * ps + t0;              // absolute position
      if (tok0 >= lim_max) break;
      // tokens past a row's limit (or past the end of a 32-token page) exist
      // only in the last unit of a pair
      const bool tail = (tok0 + 64 > lim_min) || (t0 + 64 > ps);

      // ---- scores: tile t = 4h + j, column n = token t0 + 32h + 4n + j.  The
      // k-chunk loop is outermost so that the 8 tiles' mma chains interleave.
      constexpr int rsK = L::kStrideK, rsV = L::kStrideV;
      uint4 kw[2][4];  // words 3tq, 3tq+1, 3tq+2 and 12 (or tq + 4i) of tokens t0 + 32h + 4gid + {0..3}
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t *kb = kc + t0 + 32 * h + 4 * gid;
        if constexpr (BITS == 3) {
          kw[h][0] = *reinterpret_cast<const uint4 *>(kb + (3 * tq + 0) * rsK);
          kw[h][1] = *reinterpret_cast<const uint4 *>(kb + (3 * tq + 1) * rsK);
          kw[h][2] = *reinterpret_cast<const uint4 *>(kb + (3 * tq + 2) * rsK);
          kw[h][3] = *reinterpret_cast<const uint4 *>(kb + 12 * rsK);
        } else {
#pragma unroll
          for (int i = 0; i < L::kKWords; ++i) kw[h][i] = *reinterpret_cast<const uint4 *>(kb + (tq + 4 * i) * rsK);
        }
      }
      const uint32_t sh12 = 6 * tq;
      float d[8][4];
#pragma unroll
      for (int t = 0; t < 8; ++t) d[t][0] = d[t][1] = d[t][2] = d[t][3] = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 qa = sq[c * 32 + lane];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint32_t b0 = k_pair<BITS>(kw[t >> 2], t & 3, 2 * c, sh12, lane4, lutb);
          const uint32_t b1 = k_pair<BITS>(kw[t >> 2], t & 3, 2 * c + 1, sh12, lane4, lutb);
          mma16816(d[t], qa.x, qa.y, qa.z, qa.w, b0, b1);
        }
      }
      float x[16];  // x[8h + i] = token t0 + 32h + 8tq + i
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        x[8 * (t >> 2) + (t & 3)] = d[t][0] + d[t][2];      // hi + lo rows
        x[8 * (t >> 2) + 4 + (t & 3)] = d[t][1] + d[t][3];
      }
      // ---- norms, masking, online softmax (row gid)
      float nv[16];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 knv = *reinterpret_cast<const uint4 *>(kn + t0 + 32 * h + 8 * tq);
        const uint4 vnv = *reinterpret_cast<const uint4 *>(vn + t0 + 32 * h + 8 * tq);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&reinterpret_cast<const uint32_t *>(&knv)[i]));
          const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&reinterpret_cast<const uint32_t *>(&vnv)[i]));
          x[8 * h + 2 * i] *= a.x;
          x[8 * h + 2 * i + 1] *= a.y;
          nv[8 * h + 2 * i] = b.x;
          nv[8 * h + 2 * i + 1] = b.y;
        }
      }
      if (tail) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int tin = t0 + 32 * (i >> 3) + 8 * tq + (i & 7);
          if (wk.j * ps + tin >= lim || tin >= ps) x[i] = -INFINITY;
        }
      }
      // row maximum as a tree (depth 4, not a 15-long chain)
      float mt[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mt[i] = fmaxf(x[i], x[i + 8]);
#pragma unroll
      for (int i = 0; i < 4; ++i) mt[i] = fmaxf(mt[i], mt[i + 4]);
      float mx = fmaxf(fmaxf(mt[0], mt[2]), fmaxf(mt[1], mt[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      if (__any_sync(0xffffffffu, m_new > m_run)) {
        const float corr = (m_run == -INFINITY) ? 0.f : ex2((m_run - m_new) * inv2e);
        l_run *= corr;
        const float c0 = __shfl_sync(0xffffffffu, corr, (2 * tq) * 4);
        const float c1 = __shfl_sync(0xffffffffu, corr, (2 * tq + 1) * 4);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          acc[m][0] *= c0; acc[m][1] *= c1; acc[m][2] *= c0; acc[m][3] *= c1;
        }
        m_run = m_new;
      }
      const float mm = (m_run == -INFINITY) ? 0.f : m_run * inv2e;
      float pv[16], psum[4] = {0.f, 0.f, 0.f, 0.f};  // four short chains
      if (!tail) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float pr = ex2(fmaf(x[i], inv2e, -mm));
          psum[i & 3] += pr;
          pv[i] = pr * nv[i];
        }
      } else {
        // masked slots may hold stale norms: select, do not multiply
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float pr = ex2(fmaf(x[i], inv2e, -mm));
          psum[i & 3] += pr;
          pv[i] = pr > 0.f ? pr * nv[i] : 0.f;
        }
      }
      l_run += (psum[0] + psum[1]) + (psum[2] + psum[3]);

      // ---- P.V: O^T[16 dims x 8 rows] += V^T[16 dims x 16 tok] P^T
      if constexpr (BITS == 3) {
        constexpr uint32_t M = 0x071C71C7u;  // even-indexed 3-bit fields
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t *vb = vc + t0 + 32 * h + 8 * tq;
          const uint4 va0 = *reinterpret_cast<const uint4 *>(vb + gid * rsV);
          const uint4 va1 = *reinterpret_cast<const uint4 *>(vb + gid * rsV + 4);
          const uint4 vb0 = *reinterpret_cast<const uint4 *>(vb + (8 + (gid >> 1)) * rsV);
          const uint4 vb1 = *reinterpret_cast<const uint4 *>(vb + (8 + (gid >> 1)) * rsV + 4);
          const uint4 vz0 = *reinterpret_cast<const uint4 *>(vb + 12 * rsV);
          const uint4 vz1 = *reinterpret_cast<const uint4 *>(vb + 12 * rsV + 4);
#pragma unroll
          for (int kap = 0; kap < 2; ++kap) {
            uint32_t va[2][16];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const int tp = 2 * kap + half;  // token pair (2tp, 2tp+1) of this thread's 8
              const uint4 &A = tp < 2 ? va0 : va1;
              const uint4 &Bv = tp < 2 ? vb0 : vb1;
              const uint4 &Z = tp < 2 ? vz0 : vz1;
              const int e0 = (tp & 1) * 2;
              const uint32_t wa = u4_at(A, e0), wa1 = u4_at(A, e0 + 1);
              const uint32_t wb = u4_at(Bv, e0), wb1 = u4_at(Bv, e0 + 1);
              const uint32_t wz = u4_at(Z, e0), wz1 = u4_at(Z, e0 + 1);
              // merge two tokens' words: 6-bit slot k = (code of tok a, code of tok b)
              const uint32_t e_even = (wa & M) | (shifted<-3>(wa1) & ~M);
              const uint32_t e_odd = (shifted<3>(wa) & M) | (wa1 & ~M);
              const uint32_t e_half = ((wb >> (3 * par)) & M) | ((wb1 << (3 - 3 * par)) & ~M);
              word_pairs(e_even, lane4, va[half] + 0);
              word_pairs(e_odd, lane4, va[half] + 5);
              word_pairs(e_half, lane4, va[half] + 10);
              const uint32_t z12 = (((wz >> (3 * gid)) & 7u) << 7) | (((wz1 >> (3 * gid)) & 7u) << 10);
              va[half][15] = plut(z12 | lane4);
            }
            const uint32_t b0 = pack_half2(pv[8 * h + 4 * kap + 0], pv[8 * h + 4 * kap + 1]);
            const uint32_t b1 = pack_half2(pv[8 * h + 4 * kap + 2], pv[8 * h + 4 * kap + 3]);
#pragma unroll
            for (int m = 0; m < 8; ++m)
              mma16816(acc[m], va[0][2 * m], va[0][2 * m + 1], va[1][2 * m], va[1][2 * m + 1], b0, b1);
          }
        }
      } else {
        // 2 and 4 bits: the words of two tokens merge field by field, so
        // that slot k of the even (odd) merge is the pair (code of token a,
        // code of token b) of the word's field 2k (2k + 1)
        constexpr uint32_t M = BITS == 2 ? 0x33333333u : 0x0F0F0F0Fu;  // even-indexed fields
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t *vb = vc + t0 + 32 * h + 8 * tq;
          uint4 vw[L::kVWords][2];  // words gid (and 8 + gid) of the thread's 8 tokens
#pragma unroll
          for (int i = 0; i < L::kVWords; ++i) {
            vw[i][0] = *reinterpret_cast<const uint4 *>(vb + (gid + 8 * i) * rsV);
            vw[i][1] = *reinterpret_cast<const uint4 *>(vb + (gid + 8 * i) * rsV + 4);
          }
#pragma unroll
          for (int kap = 0; kap < 2; ++kap) {
            uint32_t va[2][16];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const int tp = 2 * kap + half;  // token pair (2tp, 2tp+1) of this thread's 8
              const int e0 = (tp & 1) * 2;
#pragma unroll
              for (int i = 0; i < L::kVWords; ++i) {
                const uint4 &A = tp < 2 ? vw[i][0] : vw[i][1];
                const uint32_t wa = u4_at(A, e0), wb = u4_at(A, e0 + 1);
                const uint32_t e_even = (wa & M) | (shifted<-BITS>(wb) & ~M);
                const uint32_t e_odd = (shifted<BITS>(wa) & M) | (wb & ~M);
                merged_pairs<BITS>(e_even, lane4, lutb, va[half] + 8 * i);
                merged_pairs<BITS>(e_odd, lane4, lutb, va[half] + 8 * i + L::kPpw);
              }
            }
            const uint32_t b0 = pack_half2(pv[8 * h + 4 * kap + 0], pv[8 * h + 4 * kap + 1]);
            const uint32_t b1 = pack_half2(pv[8 * h + 4 * kap + 2], pv[8 * h + 4 * kap + 3]);
#pragma unroll
            for (int m = 0; m < 8; ++m)
              mma16816(acc[m], va[0][2 * m], va[0][2 * m + 1], va[1][2 * m], va[1][2 * m + 1], b0, b1);
          }
        }
      }
    }
    if (seg_end) {
      // ---- merge the consumer warps' states and write one record
      const int64_t pair = (static_cast<int64_t>(wk.rg) * p.B + wk.b) * p.H + wk.h;
      // every warp is done reading this stage: reuse it as merge scratch
      named_bar_sync(1, kConsumerWarps * 32);
      uint8_t *scr = smem + static_cast<size_t>(stage) * L::kStageBytes;
      float *sm_o = reinterpret_cast<float *>(scr + kScratchO);
      float *sm_m = reinterpret_cast<float *>(scr + kScratchM);
      float *sm_l = reinterpret_cast<float *>(scr + kScratchL);
      float *sm_e = reinterpret_cast<float *>(scr + kScratchE);
      float l_tot = l_run;
      l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 1);
      l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 2);
      float *o_w = sm_o + warp * 8 * kD;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        o_w[(2 * tq) * kD + vdim(2 * m)] = acc[m][0];
        o_w[(2 * tq + 1) * kD + vdim(2 * m)] = acc[m][1];
        o_w[(2 * tq) * kD + vdim(2 * m + 1)] = acc[m][2];
        o_w[(2 * tq + 1) * kD + vdim(2 * m + 1)] = acc[m][3];
      }
      if (tq == 0) {
        sm_m[warp * 8 + gid] = m_run;
        sm_l[warp * 8 + gid] = l_tot;
        if (warp == 0) sm_e[gid] = inv2e;
      }
      named_bar_sync(1, kConsumerWarps * 32);
      float *rec = p.records + (blockIdx.x + pair) * static_cast<int64_t>(kRecordFloats);
      for (int e = tid; e < 8 * 32; e += kConsumerWarps * 32) {
        const int row = e >> 5, d0 = (e & 31) * 4;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * 8 + row]);
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float l = 0.f;
        if (M != -INFINITY) {
          const float e2 = sm_e[row];
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float s = ex2((sm_m[w * 8 + row] - M) * e2);
            l += s * sm_l[w * 8 + row];
            const float4 ow = *reinterpret_cast<const float4 *>(sm_o + (w * 8 + row) * kD + d0);
            o.x += s * ow.x; o.y += s * ow.y; o.z += s * ow.z; o.w += s * ow.w;
          }
          M *= e2;  // to log2 units
        }
        if ((e & 31) == 0) {
          rec[2 * row] = M;
          rec[2 * row + 1] = l;
        }
        *reinterpret_cast<float4 *>(rec + 16 + row * kD + d0) = o;
      }
      // the bulk copies that refill this stage must not overtake the
      // scratch accesses above
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      named_bar_sync(1, kConsumerWarps * 32);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == L::kStages) {
      stage = 0;
      phase ^= 1u;
    }

    if (g + 1 < ge) wk.advance(p.seq_lens, p.B, p.H, ps);
  }
}

// ------------------------------------------------------------ tcgen05 kernel
// Many query rows per KV head (speculative verification: nq positions x G
// heads, 64 rows and more).  The mma.sync kernel above decodes every KV
// tile once per group of 8 rows; this one decodes it once for 64 rows and
// runs both products on the fifth-generation tensor cores with the
// accumulators in tensor memory.
//
// Work = pages of (stream, sequence, KV head), a stream being 64 query rows;
// CTA c (two per SM) takes pages [c P / N, (c + 1) P / N) as above.  Per
// 64-token tile of a page, the CTA's 4 warps (128 threads):
//   1. decode the tile's K codes (threads 0..63, one token each, read from
//      global memory word by word: 32 tokens' word w are 128 contiguous
//      bytes) and V codes (threads 64..127) into fp16 centroid tiles in
//      shared memory, both in
//      the no-swizzle canonical layout: core matrix = 8 tokens x 8 dims
//      (16 B per token row), dim chunks 128 B apart, token groups 2 KB
//      apart.  K is read as a K-major B operand (N = tokens), V as an
//      MN-major B operand (N = dims, K = tokens);
//   2. S[128 x 64] = Q~ K^T with one tcgen05.mma per 16 dims: A = Q~, the
//      64 rows' fp16 high parts in rows 0..63 and low parts in rows 64..127,
//      so S's lanes 64..127 hold the low-part scores;
//   3. thread r < 64 (row r) adds its two score halves (the low half through
//      shared memory), applies the K norms, the row's prescale and the
//      limits and runs the online softmax; p * n_v goes to the A operand of
//      the next product as fp16 high part (row r) and low part (row r + 64),
//      so the weights keep ~22 bits at no extra tensor work; when the running
//      maximum moved, rows r and r + 64 of O in tensor memory are rescaled;
//   4. O[128 x 128] += P' V with one tcgen05.mma per 16 tokens.
// At the end of a stream's pages in this CTA, row r of the result is O's
// rows r + (r + 64), written with (m, l) as 8-row records for the combine.
constexpr int kTRows = 64;    // query rows per stream
constexpr int kTTok = 64;     // tokens per tile
constexpr int kTThreads = 4 * 32;
constexpr int kTCtasPerSm = 2;
constexpr int kTCols = 256;   // tensor memory per CTA: S at column 0, O at column 128
constexpr int kTQ = 0;                               // Q~ tile: 128 rows x 128 dims fp16
constexpr int kTK = kTQ + 128 * kD * 2;              // K tile: 64 tokens x 128 dims
constexpr int kTV = kTK + kTTok * kD * 2;            // V tile (right after K: the two hold O's low rows at the end)
constexpr int kTP = kTV + kTTok * kD * 2;            // P' tile: 128 rows x 64 tokens
constexpr int kTX = kTP + 128 * kTTok * 2;           // low-part scores: 64 rows x 64 tokens fp32
constexpr int kTKN = kTX + kTRows * kTTok * 4;       // K norms of the tile (fp32)
constexpr int kTVN = kTKN + kTTok * 4;               // V norms
constexpr int kTScale = kTVN + kTTok * 4;            // per-row prescale
constexpr int kTRed = kTScale + kTRows * 4;          // row maxima and sums of the two token halves
constexpr int kTBar = kTRed + 4 * kTRows * 4;        // s_done, pv_done
constexpr int kTMisc = kTBar + 2 * 8;                // tensor-memory base, abort flag
constexpr int kTSmemBytes = kTMisc + 16;
static_assert(kTK % 128 == 0 && kTV % 128 == 0 && kTP % 128 == 0, "UMMA tile alignment");

// shared-memory matrix descriptor, no swizzle (16-byte units)
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo16, uint32_t sbo16) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(lbo16 & 0x3FFFu) << 16) |
         (static_cast<uint64_t>(sbo16 & 0x3FFFu) << 32) | (1ull << 46);
}
// instruction descriptor: f16 A/B, f32 accumulator, M x N, B K- or MN-major
__host__ __device__ constexpr uint32_t umma_idesc(int m, int n, int b_mn_major) {
  return (1u << 4) | (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}
// One tensor-core product D (+)= A B (kind::f16, fp32 accumulator in tensor
// memory, A and B in shared memory), issued by the calling thread
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// Products with A in tensor memory (row m = lane m, column c = the packed
// fp16 pair k = 2c, 2c + 1 of a 16-wide K slice), issued by the calling
// thread as one asm block.
// The 16 score products of a tile (Q~ high parts, then low parts, against
// the K tile at descriptor bK: 8 K-slices of 16 dims each) in one asm block,
// issued by the calling thread: per product one address add, one descriptor
// add and the MMA.
__device__ __forceinline__ void umma_scores16(uint32_t d, uint32_t qh, uint32_t ql, uint64_t bK, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred pz, pa;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
      "setp.ne.b32 pz, %5, 0;\n\tsetp.eq.b32 pa, %5, 0;\n\t"
      "add.u32 a, %1, 0;\n\tadd.s64 b, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pz;\n\t"
      "add.u32 a, %1, 8;\n\tadd.s64 b, %3, 16;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 16;\n\tadd.s64 b, %3, 32;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 24;\n\tadd.s64 b, %3, 48;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 32;\n\tadd.s64 b, %3, 64;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 40;\n\tadd.s64 b, %3, 80;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 48;\n\tadd.s64 b, %3, 96;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 56;\n\tadd.s64 b, %3, 112;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 0;\n\tadd.s64 b, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 8;\n\tadd.s64 b, %3, 16;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 16;\n\tadd.s64 b, %3, 32;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 24;\n\tadd.s64 b, %3, 48;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 32;\n\tadd.s64 b, %3, 64;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 40;\n\tadd.s64 b, %3, 80;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 48;\n\tadd.s64 b, %3, 96;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %2, 56;\n\tadd.s64 b, %3, 112;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, {%5, %5, %5, %5}, pa;\n\t"
      "}\n"
      ::"r"(d), "r"(qh), "r"(ql), "l"(bK), "r"(idesc), "r"(0u)
      : "memory");
}
// The 8 products O (+)= P'V of a tile (P' high parts, then low parts, 4
// token slices of 16 each, against the V tile at descriptor bV); acc0 = 0
// starts O with the first one.
__device__ __forceinline__ void umma_pv8(uint32_t d, uint32_t pa, uint64_t bV, uint32_t idesc, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, pa;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\tsetp.eq.b32 pa, %5, 0;\n\t"
      "add.u32 a, %1, 0;\n\tadd.s64 b, %2, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, p0;\n\t"
      "add.u32 a, %1, 8;\n\tadd.s64 b, %2, 256;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 16;\n\tadd.s64 b, %2, 512;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 24;\n\tadd.s64 b, %2, 768;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 32;\n\tadd.s64 b, %2, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 40;\n\tadd.s64 b, %2, 256;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 48;\n\tadd.s64 b, %2, 512;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, pa;\n\t"
      "add.u32 a, %1, 56;\n\tadd.s64 b, %2, 768;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, {%5, %5, %5, %5}, pa;\n\t"
      "}\n"
      ::"r"(d), "r"(pa), "l"(bV), "r"(idesc), "r"(acc0), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void umma_commit_by(bool issue, uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\t"
      "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(smem_addr(bar)),
      "r"(static_cast<uint32_t>(issue))
      : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// byte offset of element (row, col) in a no-swizzle canonical tile whose
// 8-row groups are `group_bytes` apart and whose 8-column chunks are 128 B
// apart (row = M/N index, col = K index for K-major tiles)
__device__ __forceinline__ uint32_t canon_off(int row, int col, int group_bytes) {
  return static_cast<uint32_t>((row >> 3) * group_bytes + (col >> 3) * 128 + (row & 7) * 16 + (col & 7) * 2);
}

template <int BITS>
__global__ void __launch_bounds__(kTThreads, kTCtasPerSm) k_attend_tiles(const PartialParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t *bar_s = reinterpret_cast<uint64_t *>(smem + kTBar);
  uint64_t *bar_pv = bar_s + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kTMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kTMisc + 4);
  const int ps = p.page_size;

  fill_lut<BITS>(p.level, tid, kTThreads);
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_pv, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  pdl_trigger();
  pdl_wait();
  write_plan_tag(p);
  __shared__ int64_t tloc[4 + kTThreads / 32];
  tile_locate<kTThreads>(p, kTRows, tloc + 4, tloc);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t gs = tloc[0], ge = tloc[1];
  UWalk wk;
  if (gs < ge) wk.start(p, kTRows, static_cast<int>(tloc[2]), static_cast<int>(tloc[3]));

  const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
  const int r = tid & 63;        // row (softmax) or token (decode) of this thread
  const bool lo_half = tid >= 64;
  float *xchg = reinterpret_cast<float *>(smem + kTX);
  float *row_scale = reinterpret_cast<float *>(smem + kTScale);
  float *red_max = reinterpret_cast<float *>(smem + kTRed);  // [2][64]
  float *red_sum = red_max + 2 * kTRows;                      // [2][64]
  // descriptors built once (per product only constant start offsets are added)
  const uint64_t dQ = umma_desc(smem_addr(smem + kTQ), 8, 128), dK = umma_desc(smem_addr(smem + kTK), 8, 128),
                 dV = umma_desc(smem_addr(smem + kTV), 128, 8), dP = umma_desc(smem_addr(smem + kTP), 8, 64);
  constexpr uint32_t kIdescS = umma_idesc(128, kTTok, 0);
  constexpr uint32_t kIdescPV = umma_idesc(128, kD, 1);
  float m_run = -INFINITY, l_run = 0.f;
  int lim = 0;
  bool row_valid = false, first_pv = true, any_pv = false;
  uint32_t ph_s = 0, ph_pv = 0;
  bool ok = true;
  // Control flow depends on the page walk only, so the four warps meet at
  // every named barrier even after a bounded wait has given up (`ok` false:
  // the work is skipped, the barriers are not).
  for (int64_t g = gs; g < ge; ++g) {
    const bool seg_start = (g == gs) || (wk.j == 0);
    const bool seg_end = (g + 1 == ge) || (wk.j + 1 == wk.np);
    const int L = p.seq_lens[wk.b];
    if (seg_start) {
      // this stream's 64 rows as Q~: high parts in rows 0..63, low parts in
      // rows 64..127, each row prescaled by a power of two so that its
      // largest |q| lands in [2^14, 2^15).  The previous stream's products
      // have completed (its record was written).
      const int row = wk.rg * kTRows + r;
      row_valid = row < p.R;
      const int qi = row_valid ? row / p.G : 0;
      const int hq = wk.h * p.G + (row_valid ? row % p.G : 0);
      const float *qp = p.q_rot + ((static_cast<int64_t>(wk.b) * p.nq + qi) * p.Hq + hq) * kD;
      float mx = 0.f;
      for (int d = 0; d < kD; d += 4) {
        const float4 v = row_valid ? *reinterpret_cast<const float4 *>(qp + d) : make_float4(0.f, 0.f, 0.f, 0.f);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
      mx *= p.qfold;
      int ex = 0;
      if (mx > 0.f) frexpf(mx, &ex);
      ex = max(ex, -100);
      const float up = ldexpf(1.f, 15 - ex) * p.qfold;
      if (!lo_half) row_scale[r] = ldexpf(1.f, ex - 15);
      for (int c = 0; c < kD / 8; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = row_valid ? qp[8 * c + 2 * e] * up : 0.f;
          const float bb = row_valid ? qp[8 * c + 2 * e + 1] * up : 0.f;
          const __half ah = __float2half_rn(a), bh = __float2half_rn(bb);
          w4[e] = lo_half ? pack_half2(a - __half2float(ah), bb - __half2float(bh))
                          : pack_half2(__half2float(ah), __half2float(bh));
        }
        *reinterpret_cast<uint4 *>(smem + kTQ + canon_off(r + (lo_half ? 64 : 0), 8 * c, 2048)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      lim = row_valid ? (p.causal ? L - p.nq + qi + 1 : L) : 0;
      m_run = -INFINITY;
      l_run = 0.f;
      first_pv = true;
    }
    // this page's K (threads 0..63) or V (64..127) codes and norms in global
    // memory: word w of token t at cw[w * ps + t]
    int phys = -1;
    if (wk.j < p.max_pages) phys = p.page_table[static_cast<int64_t>(wk.b) * p.max_pages + wk.j];
    if (phys < 0 || phys >= p.num_pages) {
      if (tid == 0) set_status(p.status, ISOQUANT_DEVERR_PAGE_RANGE);
      phys = 0;
    }
    const int64_t blk = (static_cast<int64_t>(phys) * 2 + (lo_half ? 1 : 0)) * p.H + wk.h;
    const uint32_t *cw = p.codes + blk * words_for(BITS) * ps;
    const __half *nw = reinterpret_cast<const __half *>(p.norms) + blk * ps;

    const int ntile = (wk.page_tokens(ps) + kTTok - 1) / kTTok;  // tiles within the stream's horizon
    for (int ti = 0; ti < ntile; ++ti) {
      const int t0 = ti * kTTok;
      // the previous tile's P.V reads the V and P' tiles and O: the V warps
      // wait for it here, the K warps before they write P'
      bool pv_pending = any_pv;
      if (lo_half && pv_pending) {
        ok = mbar_wait(bar_pv, ph_pv, p.status, abort_flag) && ok;
        ok = __all_sync(0xffffffffu, ok);
        pv_pending = false;
        tc_fence_after();
      }
      if (any_pv) ph_pv ^= 1u;
      any_pv = false;
      // ---- 1. decode token t0 + r of K (threads 0..63) or V (64..127)
      {
        const int t = t0 + r;
        uint32_t x[words_for(BITS)];
        load_token_words<BITS>(cw, ps, t, x);
        const float nrm = __half2float(nw[t]);
        uint32_t out[64];
        decode_token_words<BITS>(x, lane4, out);
        uint8_t *tile = smem + (lo_half ? kTV : kTK);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          *reinterpret_cast<uint4 *>(tile + canon_off(r, 8 * c, 2048)) =
              make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
        reinterpret_cast<float *>(smem + (lo_half ? kTVN : kTKN))[r] = nrm;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      named_bar_sync(1, kTThreads);
      // ---- 2. S = Q~ K^T
      if (tid == 0 && ok) {
        tc_fence_after();
#pragma unroll
        for (int kc2 = 0; kc2 < kD / 16; ++kc2) umma_f16(tmem, dQ + kc2 * 16, dK + kc2 * 16, kIdescS, kc2 > 0 ? 1u : 0u);
        umma_commit(bar_s);
      }
      ok = mbar_wait(bar_s, ph_s, p.status, abort_flag) && ok;
      ok = __all_sync(0xffffffffu, ok);
      ph_s ^= 1u;
      tc_fence_after();
      // ---- 3. softmax: row r's tokens 0..31 by thread r (which holds the
      // high-part scores, lanes 0..63), tokens 32..63 by thread r + 64 (low
      // parts, lanes 64..127); each half sends the other the half it needs
      float sv[64];
      {
        const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        float tmp[32];
        tmem_ld32(ta, tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[i] = tmp[i];
        tmem_ld32(ta + 32, tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[32 + i] = tmp[i];
      }
      // xchg: [half][4-column group][row][4]; half 0 = high parts of tokens
      // 32..63 (for the low warps), half 1 = low parts of tokens 0..31
      const int own = lo_half ? 32 : 0;    // tokens this thread finishes
      {
        float *dst = xchg + (lo_half ? 1 : 0) * (32 * kTRows);
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(dst + (i * kTRows + 4 * r)) =
              lo_half ? make_float4(sv[i], sv[i + 1], sv[i + 2], sv[i + 3])
                      : make_float4(sv[32 + i], sv[33 + i], sv[34 + i], sv[35 + i]);
      }
      tc_fence_before();
      named_bar_sync(1, kTThreads);
      float mx = -INFINITY;
      {
        const float *kn_t = reinterpret_cast<const float *>(smem + kTKN) + own;
        const float *src = xchg + (lo_half ? 0 : 1) * (32 * kTRows);
        const float rs = row_scale[r];
        const int pos0 = wk.j * ps + t0 + own;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 o4 = *reinterpret_cast<const float4 *>(src + (i * kTRows + 4 * r));
          const float4 kn4 = *reinterpret_cast<const float4 *>(kn_t + i);
          const float x4[4] = {o4.x, o4.y, o4.z, o4.w}, k4[4] = {kn4.x, kn4.y, kn4.z, kn4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float sc = ((lo_half ? sv[32 + i + e] : sv[i + e]) + x4[e]) * rs * k4[e];
            if (!row_valid || pos0 + i + e >= lim) sc = -INFINITY;
            sv[i + e] = sc;  // compacted into sv[0..31]
            mx = fmaxf(mx, sc);
          }
        }
      }
      red_max[(lo_half ? kTRows : 0) + r] = mx;
      named_bar_sync(1, kTThreads);
      // P' and O may still be read by the previous tile's P.V
      if (!lo_half && pv_pending) {
        ok = mbar_wait(bar_pv, ph_pv ^ 1u, p.status, abort_flag) && ok;
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
      }
      const float m_new = fmaxf(m_run, fmaxf(red_max[r], red_max[kTRows + r]));
      const float corr = (m_run == -INFINITY || m_new == m_run) ? 1.f : ex2(m_run - m_new);
      {
        const float *vn_t = reinterpret_cast<const float *>(smem + kTVN) + own;
        const float mm = m_new == -INFINITY ? 0.f : m_new;
        float psum = 0.f;
        uint32_t pk[16], pl[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2(sv[i] - mm), p1 = ex2(sv[i + 1] - mm);
          psum += p0 + p1;
          // masked slots may hold stale norms: select, do not multiply
          const float w0 = p0 > 0.f ? p0 * vn_t[i] : 0.f, w1 = p1 > 0.f ? p1 * vn_t[i + 1] : 0.f;
          const __half h0 = __float2half_rn(w0), h1 = __float2half_rn(w1);
          pk[i >> 1] = pack_half2(__half2float(h0), __half2float(h1));
          pl[i >> 1] = pack_half2(w0 - __half2float(h0), w1 - __half2float(h1));
        }
        // p n_v: high part in row r, low part in row r + 64 of the A tile
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          *reinterpret_cast<uint4 *>(smem + kTP + canon_off(r, own + 8 * c, 1024)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          *reinterpret_cast<uint4 *>(smem + kTP + canon_off(r + 64, own + 8 * c, 1024)) =
              make_uint4(pl[4 * c], pl[4 * c + 1], pl[4 * c + 2], pl[4 * c + 3]);
        }
        red_sum[(lo_half ? kTRows : 0) + r] = psum;
      }
      named_bar_sync(1, kTThreads);
      // both threads of a row keep the same (m, l)
      l_run = l_run * corr + red_sum[r] + red_sum[kTRows + r];
      m_run = m_new;
      // rescale rows r (warps 0-1) and r + 64 (warps 2-3) of O when the row's
      // maximum moved (each warp loads and stores together)
      if (!first_pv && __any_sync(0xffffffffu, corr != 1.f)) {
        const uint32_t to = tmem + 128 + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float ov[32];
          tmem_ld32(to + 32 * c, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= corr;
          tmem_st32(to + 32 * c, ov);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      named_bar_sync(1, kTThreads);
      // ---- 4. O += P' V
      if (tid == 0 && ok) {
        tc_fence_after();
#pragma unroll
        for (int kc2 = 0; kc2 < kTTok / 16; ++kc2)
          umma_f16(tmem + 128, dP + kc2 * 16, dV + kc2 * 256, kIdescPV, (first_pv && kc2 == 0) ? 0u : 1u);
        umma_commit(bar_pv);
      }
      first_pv = false;
      any_pv = true;
    }
    if (seg_end) {
      // ---- the stream's record: wait for the last P.V, then row r of the
      // result is O's rows r + (r + 64); the low rows go through the K and V
      // tiles (every product has completed)
      if (any_pv) {
        ok = mbar_wait(bar_pv, ph_pv, p.status, abort_flag) && ok;
        ok = __all_sync(0xffffffffu, ok);
        ph_pv ^= 1u;
        any_pv = false;
      }
      tc_fence_after();
      float *olo = reinterpret_cast<float *>(smem + kTK);
      const uint32_t to = tmem + 128 + (static_cast<uint32_t>(32 * warp) << 16);
      if (lo_half) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float ov[32];
          tmem_ld32(to + 32 * c, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) olo[(32 * c + i) * kTRows + r] = ov[i];
        }
      }
      named_bar_sync(1, kTThreads);
      if (!lo_half) {
        const int row = wk.rg * kTRows + r;
        const int64_t stream = (static_cast<int64_t>(wk.rg) * p.B + wk.b) * p.H + wk.h;
        float *rec =
            p.records + ((blockIdx.x + stream) * (kTRows / 8) + (r >> 3)) * static_cast<int64_t>(kRecordFloats);
        const int rr = r & 7;
        const bool have = !first_pv;
        if (row < p.R) {
          rec[2 * rr] = have ? m_run : -INFINITY;
          rec[2 * rr + 1] = have ? l_run : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float ov[32];
          tmem_ld32(to + 32 * c, ov);
          if (row < p.R && have) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4 *>(rec + 16 + rr * kD + 32 * c + i) =
                  make_float4(ov[i] + olo[(32 * c + i) * kTRows + r], ov[i + 1] + olo[(32 * c + i + 1) * kTRows + r],
                              ov[i + 2] + olo[(32 * c + i + 2) * kTRows + r], ov[i + 3] + olo[(32 * c + i + 3) * kTRows + r]);
          }
        }
      }
      tc_fence_before();
      named_bar_sync(1, kTThreads);
    }
    if (g + 1 < ge) wk.advance(p, kTRows);
  }
  // the last P.V must finish before tensor memory is released
  if (any_pv) mbar_wait(bar_pv, ph_pv, p.status, nullptr);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTCols));
  }
}

// ------------------------------------------------------------ tcgen05 kernel, 128-row streams
// k_attend_wide: 128 or more query rows per KV head (causal prefill, long
// verification chunks).  One CTA per SM, warp-specialised, streams of 128
// query rows, 64-token tiles, the same unit walk as above:
//   * the decoder warps (after the softmax warps) unpack every tile into
//     stage T % kWStages of a shared-memory ring, a thread one token of K
//     and of V (2 warps) or of K or V (4 warps), as in k_attend_tiles; they
//     load a tile's code words before waiting for its stage;
//   * the last warp, one thread, issues the tensor-core products: S_T = Q~ K_T^T
//     into one of two score buffers in tensor memory (16 MMAs: the queries'
//     fp16 high parts, then their low parts, accumulated), and, once the
//     softmax of tile T - 1 is in shared memory, O += P'_{T-1} V_{T-1}
//     (8 MMAs: the weights' high parts, then their low parts).  S_{T+1} is
//     issued before P.V_T, so the tensor pipe computes the next scores while
//     the softmax warps work;
//   * warps 0 .. 4 kWParts - 1 run the online softmax: kWParts threads per
//     row r (tensor-memory lane r of S and O, reached by warps r / 32 + 4 k),
//     each with a slice of the tile's tokens and of the row's Q~ dims and O
//     columns, exchanging their maxima through shared memory (one warp per
//     row would leave each SM sub-partition a single latency-bound softmax
//     warp):
//     scores times the K norms and the row's prescale, causal and length
//     limits, running max and per-half sums, p * n_v split into fp16
//     high and low parts (the A operands of P.V, double-buffered so that
//     they are written while the previous P.V runs), and the rescale of its
//     O row when the row's maximum moved (after the previous P.V completed).
//     At a stream's last tile in this CTA it writes the row's (m, l, o)
//     record for the combine.
// Hand-offs are mbarriers: kv_full[s] (decoders -> MMA), kv_free[s] (P.V of
// the tile that used stage s completed -> decoders), s_full[b] (S in
// buffer b -> softmax), s_free[b] (softmax has read it -> MMA), p_full
// (P' written -> MMA), pv_done (P.V completed -> softmax) and q_full (the
// stream's Q~ written -> MMA).  Every wait is bounded; after one expires all
// roles skip their work and fall through to the end.
constexpr int kWRows = 128;
constexpr int kWTok = 64;
// softmax threads per row (one warpgroup each): a tile's tokens and a row's
// Q~ dims and O columns are split among them
#ifndef ISOQUANT_WIDE_PARTS
#define ISOQUANT_WIDE_PARTS 4
#endif
constexpr int kWParts = ISOQUANT_WIDE_PARTS;
static_assert(kWParts == 2 || kWParts == 4, "two or four softmax warpgroups");
constexpr int kWSoftWarps = 4 * kWParts;
constexpr int kWTpt = kWTok / kWParts;  // tokens of a tile per softmax thread
constexpr int kWDpt = kD / kWParts;     // Q~ dims / O columns per softmax thread
// decoder warps: 4 (a thread decodes one token of K or V per tile) or 2 (a
// thread decodes one token of K and of V).  At 4 bits a pair takes two
// table lookups, and two decoder warps become the bound (a 8192-token
// prefill: 3.2 ms with two, 2.1 with four); at 2 and 3 bits two keep the
// registers in budget at no cost
#ifndef ISOQUANT_WIDE_DEC
#define ISOQUANT_WIDE_DEC 0
#endif
template <int BITS>
constexpr int wide_dec_warps() {
  return ISOQUANT_WIDE_DEC ? ISOQUANT_WIDE_DEC : ((kWParts == 2 || BITS == 4) ? 4 : 2);
}
template <int BITS>
constexpr int wide_threads() {
  return (kWSoftWarps + wide_dec_warps<BITS>() + 1) * 32;  // softmax, decoder and MMA warps
}
// Tensor memory (512 columns, one CTA per SM): S buffers 0 and 1, O, then
// the A operands of both products, fp16 pairs packed per 32-bit column
// (row = lane): Q~ high and low parts (64 columns each) and two buffers of
// P' high and low parts (32 columns each).  With the A operands there, the
// products read only K and V from shared memory: fed from shared memory,
// an M = 128 product with N <= 128 is bound by shared-memory bandwidth.
constexpr int kWCols = 512;
constexpr uint32_t kWColS = 0, kWColO = 128, kWColQh = 256, kWColQl = 320, kWColP = 384;  // P buffer b: +64 b, low +32
#ifndef ISOQUANT_WIDE_STAGES
#define ISOQUANT_WIDE_STAGES 4
#endif
constexpr int kWStages = ISOQUANT_WIDE_STAGES;        // K/V tile ring
static_assert((kWStages & (kWStages - 1)) == 0 && kWStages >= 2, "power-of-two ring");
constexpr int kWStageBytes = kWTok * kD * 2;          // one 64-token tile of K or V, fp16
constexpr int kWK = 0;                                // kWStages K tiles
constexpr int kWV = kWK + kWStages * kWStageBytes;    // kWStages V tiles
constexpr int kWKN = kWV + kWStages * kWStageBytes;   // K norms, kWStages x 64 fp32
constexpr int kWVN = kWKN + kWStages * kWTok * 4;     // V norms
constexpr int kWRed = kWVN + kWStages * kWTok * 4;    // per part: row maxima [2 tiles], sums, |q| maxima
constexpr int kWBar = kWRed + 4 * kWParts * kWRows * 4;  // 2 kWStages + 8 mbarriers
constexpr int kWMisc = kWBar + (2 * kWStages + 8) * 8;  // tensor-memory base, abort flag, MMA-issued flag
constexpr int kWLoc = kWMisc + 16;                    // walk start + scan scratch
template <int BITS>
constexpr int wide_smem_bytes() {
  return kWLoc + (4 + wide_threads<BITS>() / 32) * 8;
}
static_assert(kWK % 128 == 0 && kWV % 128 == 0, "UMMA tile alignment");
static_assert(kWBar % 8 == 0 && kWLoc % 8 == 0, "barrier alignment");

// tensor-memory loads / stores by the width of the register array
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 16 || N == 32, "x16 or x32");
  if constexpr (N == 32) tmem_ld32(taddr, v);
  else tmem_ld16(taddr, v);
}
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t (&v)[N]) {
  static_assert(N == 8 || N == 16, "x8 or x16");
  if constexpr (N == 16) tmem_st16u(taddr, v);
  else tmem_st8u(taddr, v);
}

// the walk's tiles: for each page of [gs, ge), its 64-token tiles within the
// stream's horizon; f(wk, t0, first, last, more) with first / last = the
// stream's first / last tile in this CTA and more = another tile follows.
// Every role runs the same sequence.
template <typename F>
__device__ __forceinline__ void for_each_tile(const PartialParams &p, int64_t gs, int64_t ge, int u0, int off0,
                                              F &&f) {
  if (!(gs < ge)) return;
  const int ps = p.page_size;
  UWalk wk;
  wk.start(p, kWRows, u0, off0);
  for (int64_t g = gs; g < ge; ++g) {
    if (wk.real()) {
      const bool seg_start = (g == gs) || (wk.j == 0);
      const bool seg_end = (g + 1 == ge) || (wk.j + 1 == wk.np);
      // the next real page: the next one of this block, or the first of the
      // next block after the work-free pages
      const bool more_pages = g + 1 + (wk.j + 1 < wk.np ? 0 : p.vpages) < ge;
      const int nt = (wk.page_tokens(ps) + kWTok - 1) / kWTok;
      for (int ti = 0; ti < nt; ++ti)
        f(wk, ti * kWTok, seg_start && ti == 0, seg_end && ti == nt - 1, more_pages || ti + 1 < nt);
    }
    if (g + 1 < ge) wk.advance(p, kWRows);
  }
}

template <int BITS>
__global__ void __launch_bounds__(wide_threads<BITS>(), 1) k_attend_wide(const PartialParams p) {
  constexpr int kWDecWarps = wide_dec_warps<BITS>();
  static_assert(kWDecWarps == 2 || kWDecWarps == 4, "two or four decoder warps");
  constexpr int kWMmaWarp = kWSoftWarps + kWDecWarps;
  constexpr int kWThreads = wide_threads<BITS>();
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kWBar);
  uint64_t *kv_full = bars, *kv_free = bars + kWStages, *s_full = bars + 2 * kWStages, *s_free = s_full + 2;
  uint64_t *p_full = s_full + 4, *pv_done = s_full + 5, *q_full = s_full + 6, *mma_done = s_full + 7;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kWMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kWMisc + 4);
  volatile int *mma_issued = reinterpret_cast<volatile int *>(smem + kWMisc + 8);
  int64_t *loc = reinterpret_cast<int64_t *>(smem + kWLoc);
  const int ps = p.page_size;

  fill_lut<BITS>(p.level, tid, kWThreads);
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kWCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    tc_fence_before();
  }
  if (tid == 0) {
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(&kv_full[s], kWDecWarps);
      mbar_init(&kv_free[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], kWSoftWarps);
    }
    mbar_init(p_full, kWSoftWarps);
    mbar_init(pv_done, 1);
    mbar_init(q_full, kWSoftWarps);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *mma_issued = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  pdl_trigger();
  pdl_wait();
  write_plan_tag(p);
  tile_locate<kWThreads>(p, kWRows, loc + 4, loc);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t gs = loc[0], ge = loc[1];
  const int u0 = static_cast<int>(loc[2]), off0 = static_cast<int>(loc[3]);

  if (warp == kWMmaWarp) {
    // ---------------------------------------------------------------- MMA
    // the whole warp runs this role in step (waits included); lane 0 issues
    const bool leader = lane == 0;
    if (gs < ge) {
      // B descriptors built once; per product only the start address moves,
      // by whole 16-byte units that never carry out of its 14-bit field
      const uint64_t dK = umma_desc(smem_addr(smem + kWK), 8, 128), dV = umma_desc(smem_addr(smem + kWV), 128, 8);
      constexpr uint32_t kIdescS = umma_idesc(128, kWTok, 0);
      constexpr uint32_t kIdescPV = umma_idesc(128, kD, 1);
      bool ok = true;
      uint32_t T = 0, seg = 0, prev_T = 0;
      bool have_prev = false, prev_first = false;
      auto issue_pv = [&](uint32_t t, bool first) {
        ok = mbar_wait(p_full, t & 1u, p.status, abort_flag) && ok;
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (!ok) return;
        const uint64_t so = (t % kWStages) * static_cast<uint32_t>(kWStageBytes >> 4);
        const uint32_t pa = tmem + kWColP + (t & 1u) * 64;
        if (leader) {
          umma_pv8(tmem + kWColO, pa, dV + so, kIdescPV, first ? 0u : 1u);
          umma_commit(pv_done);
          umma_commit(&kv_free[t % kWStages]);
        }
        __syncwarp();
      };
      for_each_tile(p, gs, ge, u0, off0, [&](const UWalk &, int, bool first, bool last, bool) {
        const uint32_t st = T % kWStages, sb = T & 1u;
        if (first) ok = mbar_wait(q_full, seg & 1u, p.status, abort_flag) && ok;
        ok = mbar_wait(&kv_full[st], (T / kWStages) & 1u, p.status, abort_flag) && ok;
        if (T >= 2) ok = mbar_wait(&s_free[sb], ((T >> 1) + 1u) & 1u, p.status, abort_flag) && ok;
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (ok) {
          const uint64_t so = st * static_cast<uint32_t>(kWStageBytes >> 4);
          const uint32_t d = tmem + kWColS + 64 * sb;
          if (leader) {
            umma_scores16(d, tmem + kWColQh, tmem + kWColQl, dK + so, kIdescS);
            umma_commit(&s_full[sb]);
          }
          __syncwarp();
          *mma_issued = 1;
        }
        // the previous tile's P.V (same stream) after this tile's scores
        if (have_prev) issue_pv(prev_T, prev_first);
        have_prev = false;
        if (last) {
          issue_pv(T, first);
          ++seg;
        } else {
          have_prev = true;
          prev_T = T;
          prev_first = first;
        }
        ++T;
      });
      __syncwarp();
      if (*mma_issued) umma_commit_by(leader, mma_done);
    }
  } else if (warp >= kWSoftWarps) {
    // ------------------------------------------------------------ decoders
    // thread i: token r = i % 64 of the tile; with 4 warps K (i < 64) or V,
    // with 2 warps K then V
    constexpr int kJobs = kWDecWarps == 4 ? 1 : 2;
    const int i = tid - kWSoftWarps * 32;
    const int r = i & 63;
    const int kv0 = kWDecWarps == 4 ? (i >> 6) : 0;
    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    bool ok = true;
    uint32_t T = 0;
    int cur_page = -1, cur_h = -1, cur_u = -1;
    const uint32_t *cw[kJobs];
    const __half *nw[kJobs];
    for_each_tile(p, gs, ge, u0, off0, [&](const UWalk &wk, int t0, bool, bool, bool) {
      const uint32_t st = T % kWStages;
      if (wk.j != cur_page || wk.h != cur_h || wk.u != cur_u) {
        cur_page = wk.j;
        cur_h = wk.h;
        cur_u = wk.u;
        int phys = -1;
        if (wk.j < p.max_pages) phys = p.page_table[static_cast<int64_t>(wk.b) * p.max_pages + wk.j];
        if (phys < 0 || phys >= p.num_pages) {
          if (i == 0) set_status(p.status, ISOQUANT_DEVERR_PAGE_RANGE);
          phys = 0;
        }
#pragma unroll
        for (int jb = 0; jb < kJobs; ++jb) {
          const int64_t blk = (static_cast<int64_t>(phys) * 2 + kv0 + jb) * p.H + wk.h;
          cw[jb] = p.codes + blk * words_for(BITS) * ps;
          nw[jb] = reinterpret_cast<const __half *>(p.norms) + blk * ps;
        }
      }
      // the code words are loaded first: their latency overlaps the wait
      // for stage st, free once the P.V of tile T - kWStages has completed
      const int t = t0 + r;
      uint32_t x[kJobs][words_for(BITS)];
      __half nh[kJobs];
#pragma unroll
      for (int jb = 0; jb < kJobs; ++jb) {
        load_token_words<BITS>(cw[jb], ps, t, x[jb]);
        nh[jb] = nw[jb][t];
      }
      if (T >= kWStages)
        ok = mbar_wait(&kv_free[st], ((T / kWStages) + 1u) & 1u, p.status, abort_flag) && ok;
      if (ok) {
#pragma unroll
        for (int jb = 0; jb < kJobs; ++jb) {
          const bool is_v = kv0 + jb == 1;
          uint8_t *tile = smem + (is_v ? kWV : kWK) + st * kWStageBytes;
          // two halves of 64 dims, so that only 32 decoded words are live
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t out[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) out[q] = decode_pair<BITS>(x[jb], lane4, 32 * hh + q);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4 *>(tile + canon_off(r, 64 * hh + 8 * c, 2048)) =
                  make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
          }
          reinterpret_cast<float *>(smem + (is_v ? kWVN : kWKN))[st * kWTok + r] = __half2float(nh[jb]);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&kv_full[st]);
      ++T;
    });
  } else {
    // ------------------------------------------------------------- softmax
    // thread (r, part): row r of the stream (tensor-memory lane r), tokens
    // kWTpt * part .. + kWTpt - 1 of each tile, Q~ dims and O columns
    // kWDpt * part .. + kWDpt - 1
    const int r = tid & (kWRows - 1), part = tid >> 7;
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);  // this warp's lanes
    float *red = reinterpret_cast<float *>(smem + kWRed);
    float *rl = red + 2 * kWParts * kWRows;  // [part][row]: sums
    float *rq = red + 3 * kWParts * kWRows;  // [part][row]: |q| maxima
    // the parts of row r are warps r / 32 + 4 k, all on one SM sub-partition:
    // their exchanges (row maxima, |q| maxima, sums) use one named barrier per
    // lane quarter, so the four quarters do not wait on one another
    const int xbar = 1 + (warp & 3);
    constexpr int kXThreads = kWParts * 32;
    bool ok = true;
    uint32_t T = 0;
    float m_run = -INFINITY, l_part = 0.f, rs = 1.f;
    int lim = 0;
    bool row_valid = false;
    // this thread's dims of row r of stream (wk.rg, wk.b, wk.h)
    auto q_row = [&](const UWalk &wk) {
      const int row = wk.rg * kWRows + r;
      const bool valid = row < p.R;
      const int qi = valid ? row / p.G : 0;
      const int hq = wk.h * p.G + (valid ? row % p.G : 0);
      return p.q_rot + ((static_cast<int64_t>(wk.b) * p.nq + qi) * p.Hq + hq) * kD + kWDpt * part;
    };
    // Q~ of a stream into tensor memory (high parts, low parts), each row
    // prescaled by a power of two so that its largest |q| lands in
    // [2^14, 2^15); sets rs and releases the MMA warp.  The thread reads its
    // dims (independent 16-byte loads), takes the row's maximum with its
    // partners and reads them again from L1 to convert them.  Called when no
    // S of the previous stream is pending.
    auto build_q = [&](const UWalk &wk) {
      const bool valid = wk.rg * kWRows + r < p.R;
      const float4 *qp = reinterpret_cast<const float4 *>(q_row(wk));
      float mx = 0.f;
#pragma unroll
      for (int c = 0; c < kWDpt / 4; ++c) {
        const float4 v = valid ? __ldg(qp + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
      rq[part * kWRows + r] = mx;
      named_bar_sync(xbar, kXThreads);
      mx = 0.f;
#pragma unroll
      for (int q = 0; q < kWParts; ++q) mx = fmaxf(mx, rq[q * kWRows + r]);
      mx *= p.qfold;
      int ex = 0;
      if (mx > 0.f) frexpf(mx, &ex);
      ex = max(ex, -100);
      const float up = ldexpf(1.f, 15 - ex) * p.qfold;
      rs = ldexpf(1.f, ex - 15);
#pragma unroll
      for (int c16 = 0; c16 < kWDpt / 32; ++c16) {
        // dims kWDpt part + 32 c16 .. + 31: 16 packed columns of each part
        uint32_t wh[16], wl[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          // read again: the first pass left the line in L1
          const float4 v = valid ? __ldg(qp + 8 * c16 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
          const float a0 = v.x * up, a1 = v.y * up, a2 = v.z * up, a3 = v.w * up;
          const __half2 h0 = __floats2half2_rn(a0, a1), h1 = __floats2half2_rn(a2, a3);
          const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
          wh[2 * e] = *reinterpret_cast<const uint32_t *>(&h0);
          wh[2 * e + 1] = *reinterpret_cast<const uint32_t *>(&h1);
          wl[2 * e] = pack_half2(a0 - f0.x, a1 - f0.y);
          wl[2 * e + 1] = pack_half2(a2 - f1.x, a3 - f1.y);
        }
        tmem_st16u(tl + kWColQh + (kWDpt / 2) * part + 16 * c16, wh);
        tmem_st16u(tl + kWColQl + (kWDpt / 2) * part + 16 * c16, wl);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    };
    for_each_tile(p, gs, ge, u0, off0, [&](const UWalk &wk, int t0, bool first, bool last, bool more) {
      const uint32_t st = T % kWStages, sb = T & 1u;
      if (first) {
        // the CTA's first stream builds its Q~ here; every later one was
        // built at the end of the stream before it
        if (T == 0) build_q(wk);
        const int row = wk.rg * kWRows + r;
        row_valid = row < p.R;
        const int L = p.seq_lens[wk.b];
        lim = row_valid ? (p.causal ? L - p.nq + row / p.G + 1 : L) : 0;
        m_run = -INFINITY;
        l_part = 0.f;
      }
      if (last && more) {
        // the next stream: its queries are fetched into L2 now, so that
        // building its Q~ after this tile waits on L2, not on HBM
        UWalk nx = wk;
        nx.next_block(p, kWRows);
        const char *qn = reinterpret_cast<const char *>(q_row(nx));
        if (nx.rg * kWRows + r < p.R) {
#pragma unroll
          for (int ln = 0; ln < kWDpt * 4; ln += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(qn + ln));
        }
      }
      // ---- scores of tile T, this thread's tokens
      ok = mbar_wait(&s_full[sb], (T >> 1) & 1u, p.status, abort_flag) && ok;
      tc_fence_after();
      float sv[kWTpt];
      tmem_ld_n(tl + kWColS + 64 * sb + kWTpt * part, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      const float *kn = reinterpret_cast<const float *>(smem + kWKN) + st * kWTok + kWTpt * part;
      const float *vn = reinterpret_cast<const float *>(smem + kWVN) + st * kWTok + kWTpt * part;
      const int pos0 = wk.j * ps + t0 + kWTpt * part;
      const bool masked = __any_sync(0xffffffffu, pos0 + kWTpt > lim);
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four chains, not one
#pragma unroll
      for (int t = 0; t < kWTpt; t += 4) {
        const float4 k4 = *reinterpret_cast<const float4 *>(kn + t);
        const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x = sv[t + e] * kk[e];
          if (masked && pos0 + t + e >= lim) x = -INFINITY;
          sv[t + e] = x;
          mx4[e] = fmaxf(mx4[e], x);
        }
      }
      // the row's maximum over the parts (exchange buffer alternates by tile)
      float *rt = red + sb * (kWParts * kWRows);
      rt[part * kWRows + r] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      named_bar_sync(xbar, kXThreads);
      float mt = rt[r];
#pragma unroll
      for (int q = 1; q < kWParts; ++q) mt = fmaxf(mt, rt[q * kWRows + r]);
      const float m_new = fmaxf(m_run, mt * rs);
      const float corr = (m_run == -INFINITY || m_new == m_run) ? 1.f : ex2(m_run - m_new);
      const float mm = m_new == -INFINITY ? 0.f : m_new;
      float ps4[4] = {0.f, 0.f, 0.f, 0.f};
      // P' into tensor-memory buffer sb (its last reader, the P.V of tile
      // T - 2, has completed: this thread waited for it at tile T - 1 or at
      // the end of the previous stream)
      uint32_t ph[kWTpt / 2], pl[kWTpt / 2];
#pragma unroll
      for (int t = 0; t < kWTpt; t += 8) {
        const float4 va = *reinterpret_cast<const float4 *>(vn + t);
        const float4 vb = *reinterpret_cast<const float4 *>(vn + t + 4);
        const float vv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float pe = ex2(fmaf(sv[t + e], rs, -mm));
          ps4[e & 3] += pe;
          // masked slots may hold stale norms: select, do not multiply
          w[e] = masked ? (pe > 0.f ? pe * vv[e] : 0.f) : pe * vv[e];
        }
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float h0 = hi_part(w[e]), h1 = hi_part(w[e + 1]);
          ph[(t + e) >> 1] = pack_half2(h0, h1);
          pl[(t + e) >> 1] = pack_half2(w[e] - h0, w[e + 1] - h1);
        }
      }
      tmem_st_n(tl + kWColP + 64 * sb + (kWTpt / 2) * part, ph);
      tmem_st_n(tl + kWColP + 64 * sb + 32 + (kWTpt / 2) * part, pl);
      // O is still accumulated by the previous tile's P.V; this thread
      // rescales its O columns of its row
      if (!first) {
        ok = mbar_wait(pv_done, (T - 1u) & 1u, p.status, abort_flag) && ok;
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
          const uint32_t to = tl + kWColO + kWDpt * part;
#pragma unroll
          for (int c = 0; c < kWDpt / 32; ++c) {
            float ov[32];
            tmem_ld32(to + 32 * c, ov);
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] *= corr;
            tmem_st32(to + 32 * c, ov);
          }
        }
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      l_part = l_part * corr + ((ps4[0] + ps4[1]) + (ps4[2] + ps4[3]));
      m_run = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      if (last) {
        // ---- end of the stream in this CTA: once its last P.V completed,
        // the next stream's Q~ goes in (so that the MMA warp starts on it
        // while the record is written), then the record: (m, l) and O
        ok = mbar_wait(pv_done, T & 1u, p.status, abort_flag) && ok;
        tc_fence_after();
        if (more) {
          UWalk nx = wk;
          nx.next_block(p, kWRows);
          build_q(nx);
        }
        rl[part * kWRows + r] = l_part;
        named_bar_sync(xbar, kXThreads);
        const int64_t stream = static_cast<int64_t>(wk.u) * p.H + wk.h;
        float *rec = p.records + ((blockIdx.x + stream) * (kWRows / 8) + (r >> 3)) * static_cast<int64_t>(kRecordFloats);
        const int rr = r & 7;
        if (row_valid && part == 0) {
          float l = 0.f;
#pragma unroll
          for (int q = 0; q < kWParts; ++q) l += rl[q * kWRows + r];
          rec[2 * rr] = m_run;
          rec[2 * rr + 1] = l;
        }
        const uint32_t to = tl + kWColO + kWDpt * part;
#pragma unroll
        for (int c = 0; c < kWDpt / 32; ++c) {
          float ov[32];
          tmem_ld32(to + 32 * c, ov);
          if (row_valid) {
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<float4 *>(rec + 16 + rr * kD + kWDpt * part + 32 * c + k) =
                  make_float4(ov[k], ov[k + 1], ov[k + 2], ov[k + 3]);
          }
        }
        tc_fence_before();
      }
      ++T;
    });
  }
  // the products must complete before tensor memory is released
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (*mma_issued) mbar_wait(mma_done, 0, p.status, nullptr);
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kWCols));
  }
}

// ------------------------------------------------------------ combine kernel

// Small blocks, so that they fit beside partial-kernel CTAs as soon as any
// SM has room, and wait there for the partial kernel to complete.
constexpr int kCombineThreads = 128;

// One warp per NR consecutive query heads of a (sequence, position): NR
// divides the GQA group (up to 8), so the rows share a KV head, a stream and
// a record, and their loads overlap in one merge.
template <int NR>
__global__ void __launch_bounds__(kCombineThreads) k_attend_combine(const CombineParams p) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const uint32_t grp_id = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const bool plan_ok = __ldcg(p.plan) == p.plan_tag;
  const uint32_t per_bi = static_cast<uint32_t>(p.Hq / NR);
  const uint32_t n_groups = static_cast<uint32_t>(p.B) * p.nq * per_bi;
  if (grp_id >= n_groups) return;
  const int hq0 = static_cast<int>(grp_id % per_bi) * NR;
  const uint32_t bi = grp_id / per_bi;
  const int i = static_cast<int>(bi % static_cast<uint32_t>(p.nq));
  const int b = static_cast<int>(bi / static_cast<uint32_t>(p.nq));
  const int h = hq0 / p.G, gq = hq0 % p.G;
  // stream rg holds rows rg * rps .. ; record `sub` of a CTA holds 8 of them
  const int r0 = i * p.G + gq, rg = r0 / p.rps, sub = (r0 % p.rps) >> 3;
  const int ps = p.page_size;
  int rows[NR];
  float *dsts[NR];
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    rows[k] = (r0 + k) & 7;
    dsts[k] = p.out + (static_cast<int64_t>(bi) * p.Hq + hq0 + k) * kD + 4 * lane;
  }

  if (!plan_ok) {
    // the records were laid out by another plan (the two halves were given
    // different workspace sizes): flag it and output zeros, merge nothing
    if (lane == 0) set_status(p.status, ISOQUANT_DEVERR_PLAN_MISMATCH);
#pragma unroll
    for (int k = 0; k < NR; ++k) *reinterpret_cast<float4 *>(dsts[k]) = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  int np;
  int64_t g0, total;
  if (p.prefix != nullptr) {
    // tcgen05 kernels: the partial kernel wrote the pages before each unit
    const int64_t u = static_cast<int64_t>(rg) * p.B + b;
    const int64_t a0 = __ldcg(p.prefix + u), a1 = __ldcg(p.prefix + u + 1);
    const int nb = static_cast<int>(a1 - a0) / p.H;  // real pages + work-free ones, or 0
    np = nb > 0 ? nb - p.vpages : 0;
    g0 = a0 + static_cast<int64_t>(h) * nb;
    total = __ldcg(p.prefix + static_cast<int64_t>(p.RG) * p.B);
  } else {
    np = pages_of(p.seq_lens[b], ps);
    const int64_t p_rg = static_cast<int64_t>(p.H) * pages_before(p.seq_lens, p.B, ps, lane);
    total = p_rg * p.RG;
    g0 = rg * p_rg + static_cast<int64_t>(p.H) * pages_before(p.seq_lens, b, ps, lane) + static_cast<int64_t>(h) * np;
  }
  if (np == 0) {
#pragma unroll
    for (int k = 0; k < NR; ++k) *reinterpret_cast<float4 *>(dsts[k]) = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const Owners own(g0, np, p.n_cta, total);
  const int64_t pair = (static_cast<int64_t>(rg) * p.B + b) * p.H + h;
  merge_rows<NR>(p.records, pair, p.rps >> 3, sub, own, rows, dsts, p.params[h], lane);
}

}  // namespace

int attend_ctas_per_sm() { return kCtasPerSm; }

namespace {
// The tcgen05 kernels serve 64 or more query rows per KV head (pages of at
// least 64 tokens): k_attend_tiles (streams of 64 rows, two CTAs per SM)
// below kWideMinRows rows, k_attend_wide (streams of 128 rows, one CTA per
// SM) from there.  Their workspace: rps / 8 records per (CTA, stream) slot,
// then the unit prefix (streams * batch + 1 int64).
#ifndef ISOQUANT_WIDE_MIN_ROWS
#define ISOQUANT_WIDE_MIN_ROWS 128
#endif
constexpr int kWideMinRows = ISOQUANT_WIDE_MIN_ROWS;
static_assert(kWideMinRows >= kTRows, "the 128-row kernel serves shapes of 64+ rows");
struct TilePlan {
  int kind;  // 0: mma.sync kernel, 1: k_attend_tiles, 2: k_attend_wide
  int rps, streams, n_cta, vpages;
  size_t prefix_off, bytes;
};
TilePlan tile_plan(const AttendShape &s, int num_sms) {
  TilePlan t{};
  // the tcgen05 kernels from 64 rows per KV head (and 64-token pages); the
  // mma.sync kernel below that, at every code width
  if (s.rows < kTRows || s.page_size < kTTok) return t;
  t.kind = s.rows >= kWideMinRows ? 2 : 1;
  t.rps = t.kind == 2 ? kWRows : kTRows;
  t.n_cta = t.kind == 2 ? num_sms : num_sms * kTCtasPerSm;
  t.streams = (s.rows + t.rps - 1) / t.rps;
  // a stream switch in k_attend_wide costs about 6 tiles of work: 512 tokens
  // of work-free pages per (unit, head) block
  t.vpages = t.kind == 2 ? 512 / s.page_size : 0;
  const size_t slots = (static_cast<size_t>(t.n_cta) +
                        static_cast<size_t>(t.streams) * static_cast<size_t>(s.batch) * s.kv_heads) *
                       static_cast<size_t>(t.rps / 8);
  t.prefix_off = kWsHeader + slots * kRecordFloats * sizeof(float);
  t.bytes = t.prefix_off + (static_cast<size_t>(t.streams) * s.batch + 1) * sizeof(int64_t);
  return t;
}
// the mma.sync kernel's records (every shape can run on it)
size_t mma_bytes(const AttendShape &s) { return kWsHeader + s.slots * kRecordFloats * sizeof(float); }
// The plan a call runs: the tcgen05 kernel its shape selects when that
// kernel's records fit the workspace, else the mma.sync kernel.
TilePlan use_tiles(const isoquant_ctx *ctx, const AttendShape &s, size_t ws_bytes) {
  TilePlan t = tile_plan(s, ctx->num_sms);
  if (t.kind != 0 && t.bytes > ws_bytes) t.kind = 0;
  return t;
}
// Tag of a plan, written to the workspace header by the partial kernel and
// checked by the combine kernel.
uint32_t plan_tag(const AttendShape &s, const TilePlan &t, int n_cta, int rg) {
  uint64_t h = 0x9E3779B97F4A7C15ull;
  const int64_t f[] = {t.kind, t.kind ? t.rps : 8, rg, n_cta, t.vpages, s.batch, s.nq, s.q_heads, s.kv_heads,
                       s.page_size};
  for (int64_t v : f) {
    h ^= static_cast<uint64_t>(v) + 0x632BE59BD9B4E019ull + (h << 6) + (h >> 2);
  }
  return static_cast<uint32_t>(h ^ (h >> 32)) | 1u;
}
}  // namespace

size_t attend_workspace_min_bytes(const AttendShape &s) {
  // the smaller of the two plans: any workspace of at least this size runs
  // one of them
  const size_t mma = mma_bytes(s);
  const TilePlan t = tile_plan(s, s.n_cta / kCtasPerSm);
  return t.kind != 0 && t.bytes < mma ? t.bytes : mma;
}

size_t attend_workspace_bytes(const AttendShape &s) {
  // the records of the kernel the shape runs on: the tcgen05 plan from 64
  // query rows per KV head (pages of 64 tokens or more), else the mma.sync
  // kernel's
  const TilePlan t = tile_plan(s, s.n_cta / kCtasPerSm);
  return t.kind != 0 ? t.bytes : mma_bytes(s);
}

namespace {
// kernel attributes of one code width (the mma.sync and both tcgen05 kernels)
template <int BITS>
cudaError_t configure_width() {
  cudaError_t e = cudaFuncSetAttribute(k_attend_partial<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DecLayout<BITS>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attend_partial<BITS>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attend_tiles<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attend_tiles<BITS>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attend_wide<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, wide_smem_bytes<BITS>());
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_attend_wide<BITS>, cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared);
}
template <int BITS>
cudaError_t launch_tcgen05(int kind, const PartialParams &p, cudaStream_t stream) {
  if (kind == 2)
    return launch_pdl(k_attend_wide<BITS>, dim3(p.n_cta), dim3(wide_threads<BITS>()), wide_smem_bytes<BITS>(), stream, p);
  return launch_pdl(k_attend_tiles<BITS>, dim3(p.n_cta), dim3(kTThreads), kTSmemBytes, stream, p);
}

// Kernel attributes are per device: set them once on each device (the one
// current at the call, which the entry points check is the context's).
constexpr int kMaxConfigDevices = 64;
std::mutex g_config_mutex;
bool g_configured[kMaxConfigDevices] = {};
cudaError_t configure_device(int device) {
  if (device < 0 || device >= kMaxConfigDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_config_mutex);
  if (g_configured[device]) return cudaSuccess;
  cudaError_t e = configure_width<3>();
  if (e == cudaSuccess) e = configure_width<2>();
  if (e == cudaSuccess) e = configure_width<4>();
  if (e == cudaSuccess) g_configured[device] = true;
  return e;
}
}  // namespace

cudaError_t launch_attend_partial(const isoquant_ctx *ctx, const isoquant_cache *cache, const AttendShape &s,
                                  const float *q_rot, const int32_t *page_table, int max_pages,
                                  const int32_t *seq_lens, float scale, void *ws, size_t ws_bytes,
                                  cudaStream_t stream) {
  cudaError_t ce = configure_device(ctx->device);
  if (ce != cudaSuccess) return ce;
  PartialParams p{};
  p.codes = cache->codes;
  p.norms = cache->norms;
  p.num_pages = cache->num_pages;
  p.page_size = cache->page_size;
  p.q_rot = q_rot;
  p.page_table = page_table;
  p.max_pages = max_pages;
  p.seq_lens = seq_lens;
  p.B = s.batch;
  p.nq = s.nq;
  p.Hq = s.q_heads;
  p.H = s.kv_heads;
  p.G = s.group;
  p.R = s.rows;
  p.RG = s.row_groups;
  p.causal = s.causal;
  p.qfold = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634 / std::sqrt(128.0));
  for (int i = 0; i < kMaxLevels; ++i) p.level[i] = ctx->codebook.level[i];
  p.bits = ctx->codebook.bits;
  p.records = reinterpret_cast<float *>(static_cast<char *>(ws) + kWsHeader);
  p.status = ctx->status;
  p.n_cta = s.n_cta;
  p.prefix = nullptr;
  p.plan = static_cast<uint32_t *>(ws);
  const TilePlan t = use_tiles(ctx, s, ws_bytes);
  if (t.kind != 0) {
    p.RG = t.streams;
    p.n_cta = t.n_cta;
    p.vpages = t.vpages;
    p.prefix = reinterpret_cast<int64_t *>(static_cast<char *>(ws) + t.prefix_off);
  }
  p.plan_tag = plan_tag(s, t, p.n_cta, p.RG);
  if (t.kind != 0) {
    switch (p.bits) {
      case 2: return launch_tcgen05<2>(t.kind, p, stream);
      case 4: return launch_tcgen05<4>(t.kind, p, stream);
      default: return launch_tcgen05<3>(t.kind, p, stream);
    }
  }
  switch (p.bits) {
    case 2: return launch_pdl(k_attend_partial<2>, dim3(s.n_cta), dim3(kThreads), DecLayout<2>::kSmemBytes, stream, p);
    case 4: return launch_pdl(k_attend_partial<4>, dim3(s.n_cta), dim3(kThreads), DecLayout<4>::kSmemBytes, stream, p);
    default: return launch_pdl(k_attend_partial<3>, dim3(s.n_cta), dim3(kThreads), DecLayout<3>::kSmemBytes, stream, p);
  }
}

cudaError_t launch_attend_combine(const isoquant_ctx *ctx, const AttendShape &s, const int32_t *seq_lens,
                                  const void *ws, size_t ws_bytes, float *out, cudaStream_t stream) {
  CombineParams p{};
  p.records = reinterpret_cast<const float *>(static_cast<const char *>(ws) + kWsHeader);
  p.params = ctx->params;
  p.seq_lens = seq_lens;
  p.out = out;
  p.B = s.batch;
  p.nq = s.nq;
  p.Hq = s.q_heads;
  p.H = s.kv_heads;
  p.G = s.group;
  p.RG = s.row_groups;
  p.page_size = s.page_size;
  p.n_cta = s.n_cta;
  p.rps = 8;
  p.prefix = nullptr;
  p.status = ctx->status;
  p.plan = static_cast<const uint32_t *>(ws);
  const TilePlan t = use_tiles(ctx, s, ws_bytes);
  if (t.kind != 0) {
    p.RG = t.streams;
    p.n_cta = t.n_cta;
    p.rps = t.rps;
    p.vpages = t.vpages;
    p.prefix = reinterpret_cast<const int64_t *>(static_cast<const char *>(ws) + t.prefix_off);
  }
  p.plan_tag = plan_tag(s, t, p.n_cta, p.RG);
  // rows per warp: one while there are few rows (decode: a row's merge has
  // many split records, and more warps overlap more of them); with many
  // rows (prefill: one or two records each), the largest of 8, 4, 2 that
  // divides the GQA group, so a warp's rows overlap their loads
  const int64_t n_rows = static_cast<int64_t>(s.batch) * s.nq * s.q_heads;
  const bool many = n_rows >= static_cast<int64_t>(64) * ctx->num_sms;
  const int nr = !many ? 1 : s.group % 8 == 0 ? 8 : s.group % 4 == 0 ? 4 : s.group % 2 == 0 ? 2 : 1;
  const int64_t warps = static_cast<int64_t>(s.batch) * s.nq * (s.q_heads / nr);
  const int64_t blocks = (warps * 32 + kCombineThreads - 1) / kCombineThreads;
  if (blocks == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(blocks)), block(kCombineThreads);
  switch (nr) {
    case 8: return launch_pdl(k_attend_combine<8>, grid, block, 0, stream, p);
    case 4: return launch_pdl(k_attend_combine<4>, grid, block, 0, stream, p);
    case 2: return launch_pdl(k_attend_combine<2>, grid, block, 0, stream, p);
    default: return launch_pdl(k_attend_combine<1>, grid, block, 0, stream, p);
  }
}

namespace {
// Failure-path self-test: one thread waits on a barrier that nothing
// arrives on, so the bounded wait runs out after limit_ns, raises the
// timeout bit and returns; the elapsed time goes to *elapsed_ns.
__global__ void k_wait_selftest(uint32_t *status, uint64_t limit_ns, uint64_t *elapsed_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const uint64_t t0 = global_ns();
  const bool done = mbar_wait(&bar, 0, status, nullptr, limit_ns);
  if (elapsed_ns != nullptr) *elapsed_ns = done ? 0 : global_ns() - t0;
}
}  // namespace

cudaError_t launch_wait_selftest(const isoquant_ctx *ctx, uint64_t limit_ns, uint64_t *elapsed_ns,
                                 cudaStream_t stream) {
  k_wait_selftest<<<1, 32, 0, stream>>>(ctx->status, limit_ns, elapsed_ns);
  return cudaGetLastError();
}

}  // namespace isoquant

// isoquant_internal.cuh -- shared definitions of the CUDA library (sm_100a).
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via
// Fused Compressed-Space Attention", Abstract (WHT + block-diagonal SO(4)
// isotropization, 3-bit scalar quantization, attention on packed codes).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/isoquant.h"

namespace isoquant {

constexpr int kD = 128;
constexpr int kBlocks = 32;
constexpr int kWords = 13;  // 3-bit codes (the method's): words per vector
constexpr int kLevels = 8;
constexpr int kMaxLevels = 16;

// Code formats: `bits` in {2, 3, 4}, floor(32 / bits) codes per 32-bit word
// (16, 10, 8; code j at bits bits * (j % per_word) of word j / per_word),
// ceil(128 / per_word) words per vector (8, 13, 16).
__host__ __device__ constexpr int codes_per_word(int bits) { return 32 / bits; }
__host__ __device__ constexpr int words_for(int bits) {
  return (kD + codes_per_word(bits) - 1) / codes_per_word(bits);
}

// Per-head parameter block in device memory.
struct HeadParams {
  float m32[kBlocks][16];    // SO(4) block matrices, row-major, y' = M y
  double m64[kBlocks][16];   // same in fp64 (exact re-check near thresholds)
  uint32_t sign_bits[4];     // bit j set <=> sign_j = -1
  uint32_t pad[4];
};

// Codebook handed to the kernels by value (2^bits levels used).
struct Codebook {
  float level[kMaxLevels];       // fp16-rounded Lloyd-Max levels, ascending
  float threshold[kMaxLevels - 1];
  double threshold64[kMaxLevels - 1];
  uint16_t level16[kMaxLevels];  // fp16 bits of the levels
  int bits;
};

}  // namespace isoquant

struct isoquant_ctx {
  int device;
  int num_kv_heads;
  int num_sms;
  isoquant::HeadParams *params;  // device [num_kv_heads]
  uint32_t *status;              // device, 16 bytes
  isoquant::Codebook codebook;
  int last_launches;
};

namespace isoquant {

// ------------------------------------------------------------ host helpers
int build_codebook(Codebook *cb, int bits);

// launchers (defined in compress.cu / attend.cu)
cudaError_t launch_compress(const isoquant_ctx *ctx, const isoquant_cache *cache, const void *k,
                            const void *v, int dtype, int n_tok, const int64_t *slot_mapping,
                            cudaStream_t stream);
cudaError_t launch_rotate_q(const isoquant_ctx *ctx, const void *q, int dtype, int n_rows,
                            int num_q_heads, float *q_rot, cudaStream_t stream);
cudaError_t launch_export_z(const isoquant_ctx *ctx, const void *x, int dtype, int n_tok, float *z,
                            cudaStream_t stream);
cudaError_t launch_decode_prep(const isoquant_ctx *ctx, const isoquant_cache *cache, const void *k,
                               const void *v, int n_tok, const int64_t *slot_mapping, const void *q,
                               int dtype, int n_rows, int num_q_heads, float *q_rot, cudaStream_t stream);

struct AttendShape {
  int batch, nq, q_heads, kv_heads, group, rows, row_groups, page_size, causal;
  int bits;  // code width of the context
  int n_cta;
  size_t slots;       // partial records
};
constexpr size_t kWsHeader = 256;
constexpr size_t kRecordFloats = 8 * 2 + 8 * kD;  // (m,l) x 8 rows, o[8][128]

// Workspace sizes: the records of the kernel the shape runs on with an
// ample workspace, and the minimum any call accepts (the smaller of the
// tcgen05 plan and the mma.sync records).
size_t attend_workspace_bytes(const AttendShape &s);
size_t attend_workspace_min_bytes(const AttendShape &s);
int attend_workspace_min(const isoquant_ctx *ctx, int batch, int nq, int num_q_heads, size_t *bytes);
int attend_ctas_per_sm();
cudaError_t launch_attend_partial(const isoquant_ctx *ctx, const isoquant_cache *cache,
                                  const AttendShape &s, const float *q_rot, const int32_t *page_table,
                                  int max_pages, const int32_t *seq_lens, float scale, void *ws,
                                  size_t ws_bytes, cudaStream_t stream);
cudaError_t launch_attend_combine(const isoquant_ctx *ctx, const AttendShape &s,
                                  const int32_t *seq_lens, const void *ws, size_t ws_bytes, float *out,
                                  cudaStream_t stream);
cudaError_t launch_wait_selftest(const isoquant_ctx *ctx, uint64_t limit_ns, uint64_t *elapsed_ns,
                                 cudaStream_t stream);

// ------------------------------------------------------------ launch chain
// Every kernel of the library is a programmatic dependent launch: it may be
// scheduled while the kernel before it in the stream is still running, and
// it calls pdl_wait() before it touches global memory, which returns once
// that kernel has completed and its writes are visible.  pdl_trigger() at
// the top of each CTA lets the next kernel's CTAs be scheduled as early as
// resources allow, so a step's launch latencies overlap the running kernels.
// After a kernel that never triggers (any other library's), the launch is
// an ordinary stream-ordered one.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, A... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<P>(args)...);
}

// ------------------------------------------------------------ device helpers
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t bits) {
  atomicOr(status, bits);
}


// ------------------------------------------------------------ mbarriers, bulk copies
constexpr uint32_t kSpinLimit = 1u << 25;  // polls (a backstop: the time limit ends a wait first)
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// try_wait with a suspend-time hint: a thread whose phase is not complete is
// suspended until the phase completes or `ns` nanoseconds pass, so a waiting
// warp neither takes issue slots from the working ones nor wakes late.
__device__ __forceinline__ bool mbar_try_wait_for(uint64_t *bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait: polls with a 1 us suspend hint (the hardware resumes the
// thread as soon as the phase completes) and gives up after limit_ns,
// raising the timeout bit, or as soon as another thread of the CTA has
// raised the abort flag.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *status,
                                          volatile int *abort_flag, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait_for(bar, parity, 1000u)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (global_ns() - t0 > limit_ns) break;
  }
  set_status(status, ISOQUANT_DEVERR_WAIT_TIMEOUT);
  if (abort_flag != nullptr) *abort_flag = 1;
  return false;
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Sylvester WHT (unnormalised) of 128 values held 4 per lane, lane l holding
// elements 4l..4l+3.  Strides 1 and 2 are inside a lane; strides 4..64 pair
// lanes l and l^(stride/4).  The lower index of each butterfly keeps a+b,
// the upper one a-b.
template <typename T>
__device__ __forceinline__ void wht128(T (&v)[4], int lane) {
  T a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2; v[1] = a1 + a3; v[2] = a0 - a2; v[3] = a1 - a3;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    // lower lane: v + p; upper lane: p - v; one fused op either way
    const T sgn = (lane & m) ? T(-1) : T(1);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const T p = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = fma(sgn, v[i], p);
    }
  }
}

}  // namespace isoquant

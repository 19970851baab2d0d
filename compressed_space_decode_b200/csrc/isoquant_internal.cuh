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

// trace.cuh -- optional NVTX ranges around the C-ABI calls.
//
// Built with -DISOQUANT_NVTX (python compressed_space_decode_b200/build.py
// --nvtx), every call that launches work opens an NVTX range named after
// the call for its host-side duration, so that a timeline (Nsight Systems,
// or any NVTX consumer) shows which call issued which kernels.  NVTX v3 is
// header-only; without a tool attached a range costs a few nanoseconds.
// Without the flag the macro expands to nothing.
#pragma once

#ifdef ISOQUANT_NVTX
#include <nvtx3/nvToolsExt.h>
namespace isoquant {
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace isoquant
#define ISOQUANT_TRACE(name) ::isoquant::NvtxRange isoquant_nvtx_range_(name)
#else
#define ISOQUANT_TRACE(name) static_cast<void>(0)
#endif

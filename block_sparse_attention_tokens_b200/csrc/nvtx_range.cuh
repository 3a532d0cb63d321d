// NVTX range around a library entry point, so a timeline or profiler (Nsight
// Systems, ncu --nvtx range filters) shows which call enqueued which kernels.
// NVTX v3 is header-only: with no tool attached the push and pop return at once.
// Build with -DBSA_NO_NVTX to leave the ranges out.
#pragma once

#ifndef BSA_NO_NVTX
#include <nvtx3/nvToolsExt.h>

namespace bsa {
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace bsa

#define BSA_NVTX_RANGE(name) ::bsa::NvtxRange bsa_nvtx_range_(name)
#else
#define BSA_NVTX_RANGE(name) ((void)0)
#endif

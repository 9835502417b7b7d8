// nvtx_range.h -- one NVTX range per C-ABI call, named after the call.  A profiler then
// shows which call launched which kernels, and can capture by call: for example
// `ncu --nvtx --nvtx-include "duo_decode_attention/" ...` profiles only the kernels
// that duo_decode_attention launched.
// NVTX v3 is header-only.  With no tool attached, a range costs one call through a
// function pointer that does nothing.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace duo {

struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

}  // namespace duo

// the range covers the rest of the enclosing scope (every return path included)
#define DUO_NVTX_RANGE(name) const ::duo::NvtxRange duo_nvtx_range_(name)

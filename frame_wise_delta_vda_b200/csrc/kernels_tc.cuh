// kernels_tc.cuh - tcgen05 / TMA tensor-core kernels of the VDA path (d = 128,
// bf16 I/O).  Not yet enabled: every size runs on the SIMT kernels.
#pragma once

#include "common.cuh"
#include "vda.h"

namespace vda {

inline bool tc_path_supported(int d, int dtype) { (void)d; (void)dtype; return false; }
inline size_t tc_extra_workspace_bytes(bool tc, size_t FH, int d) { (void)tc; (void)FH; (void)d; return 0; }
inline int tc_launches_per_forward() { return 4; }

template <typename MarkFn>
int launch_tc(size_t, int, int, int, int, int, const vda_args&, char*, char*, char*, char*,
              cudaStream_t, float*, MarkFn) {
  return VDA_ERR_UNSUPPORTED;
}

}  // namespace vda

// Tensor-core vocabulary-attention path (placeholder until the tcgen05 kernels land).
#include "dg_tc.h"

namespace dg {

bool tc_supported(int, int, int) { return false; }
int tc_stat_tiles(int, int V, int) { return V / 256; }
size_t tc_workspace_bytes(int, int, int) { return 0; }
int tc_plan_init(TcPlan*, int, int, int, const void*, void*, float*, TileStat*, void*, char* err,
                 size_t errn) {
  if (err && errn) err[0] = 0;
  return -5;
}
void tc_plan_free(TcPlan*) {}
int tc_launches(const TcPlan&) { return 1; }
cudaError_t launch_tc_attention(cudaStream_t, const TcPlan&, DevState*, const void*, const void*,
                                const float*, const float*, TileStat*, float*, void*) {
  return cudaErrorNotSupported;
}
cudaError_t launch_tc_redo(cudaStream_t, const TcPlan&, DevState*, const void*, const void*,
                           const float*, const RowStat*, const int32_t*, float*) {
  return cudaErrorNotSupported;
}

}  // namespace dg

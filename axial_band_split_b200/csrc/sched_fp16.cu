// fp16 tensor-core schedule (placeholder until the tcgen05 kernels land).
#include "mrf_handle.h"

namespace mrf {

std::string fp16_supported(const mrf_config &, const BandTables &) {
  return "the fp16 tensor-core schedule is not built yet";
}
mrf_status pack_fp16(mrf_handle *, WeightMap &) { return MRF_EUNSUPPORTED; }
void schedule_fp16(mrf_handle *, const float *, float *, int, int) {}
void destroy_fp16(mrf_handle *) {}

}  // namespace mrf

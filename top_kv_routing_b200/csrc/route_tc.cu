// Tensor-core (tcgen05) routing score path.
#include "route_tc.cuh"

namespace route_tc {

bool supported(int n_kv_heads) { (void)n_kv_heads; return false; }

int launch(const LaunchArgs& a, cudaStream_t s, int* launches, const char** why) {
  (void)a; (void)s;
  *launches = 0;
  *why = "tensor-core routing path not available in this build";
  return 1;
}

}  // namespace route_tc

// Instances of the quad-per-row route kernel with float-image selection words.
#include "route_quad.cuh"

namespace moe {
void *route_quad_fn_float(int P, int nch) { return quad_fn<false>(P, nch); }
}  // namespace moe

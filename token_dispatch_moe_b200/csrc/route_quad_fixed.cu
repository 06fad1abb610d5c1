// Instances of the quad-per-row route kernel with fixed-point selection words (sigmoid and softmax keys).
#include "route_quad.cuh"

namespace moe {
void *route_quad_fn_fixed(int P, int nch) { return quad_fn<true>(P, nch); }
}  // namespace moe

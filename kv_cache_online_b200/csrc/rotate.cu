// Coordinate rotation dispatch (iS-KV reading notes, Algorithm 2 step 7; Section 4.4 for the
// re-orthogonalisation): U[0:n] <- U[0:n] G[0:k] in place over every history row.
#include "kernels.h"

namespace iskv {

cudaError_t launch_rotate_coords(const char *jobs, const RotParams &p, int64_t n_cap_max,
                                 cudaStream_t s) {
  return launch_rotate_coords_ffma(jobs, p, n_cap_max, s);
}

}  // namespace iskv

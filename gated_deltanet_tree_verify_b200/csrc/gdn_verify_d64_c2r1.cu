// gdn_verify_d64_c2r1.cu -- the verify kernels instantiated for d_k = 64
// and lane shape C = 2 chunks, RL = 1 rows per lane.

#include "gdn_verify.cuh"

namespace gdn {
namespace verify {
template cudaError_t launch_dk<64, 2, 1>(const KParams&, const VerifyArgs&, const VerifyGeom&,
                                           cudaStream_t);
}  // namespace verify
}  // namespace gdn

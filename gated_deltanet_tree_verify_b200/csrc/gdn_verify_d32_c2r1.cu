// gdn_verify_d32_c2r1.cu -- the verify kernels instantiated for d_k = 32
// and lane shape C = 2 chunks, RL = 1 rows per lane.

#include "gdn_verify.cuh"

namespace gdn {
namespace verify {
template cudaError_t launch_dk<32, 2, 1>(const KParams&, const VerifyArgs&, const VerifyGeom&,
                                           cudaStream_t);
}  // namespace verify
}  // namespace gdn

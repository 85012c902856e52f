// gdn_verify_d64.cu -- the verify kernels instantiated for d_k = 64.

#include "gdn_verify.cuh"

namespace gdn {
namespace verify {
template cudaError_t launch_dk<64>(const KParams&, const VerifyArgs&, const VerifyGeom&, cudaStream_t);
}  // namespace verify
}  // namespace gdn

// gdn_verify_d32.cu -- the verify kernels instantiated for d_k = 32.

#include "gdn_verify.cuh"

namespace gdn {
namespace verify {
template cudaError_t launch_dk<32>(const KParams&, const VerifyArgs&, const VerifyGeom&, cudaStream_t);
}  // namespace verify
}  // namespace gdn

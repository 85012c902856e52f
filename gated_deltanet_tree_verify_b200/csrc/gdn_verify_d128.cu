// gdn_verify_d128.cu -- the verify kernels instantiated for d_k = 128.

#include "gdn_verify.cuh"

namespace gdn {
namespace verify {
template cudaError_t launch_dk<128>(const KParams&, const VerifyArgs&, const VerifyGeom&, cudaStream_t);
}  // namespace verify
}  // namespace gdn

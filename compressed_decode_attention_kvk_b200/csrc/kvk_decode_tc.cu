// kvk_decode_tc.cu -- tensor-core (tcgen05) split decode; see the kernel's header comment.
#include "kvk_decode_common.cuh"

namespace kvk {

bool tc_supported(const kvk_layout*, const AnchorDesc&, int, int) { return false; }

cudaError_t launch_decode_tc(const DecodeArgs&, const AnchorDesc&, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kvk

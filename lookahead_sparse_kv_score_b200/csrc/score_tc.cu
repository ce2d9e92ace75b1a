// Tensor-core scoring path (tcgen05 + TMA); placeholder until the kernel lands.
#include "lsa_common.cuh"

namespace lsa {
size_t tc_image_bytes(int, int, int) { return 0; }
bool tc_supported(int, int, int, int) { return false; }
int launch_score_tc(const TcArgs&, cudaStream_t) {
  return fail(LSA_ERR_UNSUPPORTED, "tensor-core scoring not built");
}
}  // namespace lsa

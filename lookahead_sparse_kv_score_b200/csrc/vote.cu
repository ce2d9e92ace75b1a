// Cross-layer majority-vote labels; placeholder until the kernel lands.
#include "lsa_common.cuh"

namespace lsa {
int launch_vote(const VoteArgs&, cudaStream_t) {
  return fail(LSA_ERR_UNSUPPORTED, "vote labels not built");
}
}  // namespace lsa

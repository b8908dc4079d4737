// score_tc.cu -- tensor-core scoring path (tcgen05 + TMA); not yet enabled.
#include "kvc_internal.cuh"

namespace kvc {

bool tc_score_supported(const ScoreJob&) { return false; }
size_t tc_score_workspace(int, int, int) { return 0; }
cudaError_t tc_score(const ScoreJob&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kvc

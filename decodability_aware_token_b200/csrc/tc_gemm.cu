#include "tc_gemm.h"

namespace focus {
struct TcPlan {};
int tc_plan_create(TcPlan** out, const Dims&, const TcWeights&, void*, void*, void*, int, int, int) {
    *out = nullptr;
    return FOCUS_OK;
}
void tc_plan_destroy(TcPlan*) {}
int tc_splits(const TcPlan*, int, int) { return 1; }
int tc_lm_tiles(const TcPlan*) { return 0; }
int tc_gemm(TcPlan*, Epi, int, const GemmArgs&, cudaStream_t) { return 0; }
}  // namespace focus

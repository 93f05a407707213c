// tcgen05 / TMEM / TMA GEMM for the bf16 step: weights' tensor maps are built once at init.
#pragma once
#include "launch.h"

namespace focus {

struct TcWeights {
    int L;
    const void* const* wqkv;
    const void* const* wo;
    const void* const* wgate;
    const void* const* wup;
    const void* const* wdown;
    const void* lm_head;
};

struct TcPlan;

// Build the plan (tensor maps of every weight and activation operand).  *out may be left null,
// in which case bf16 GEMMs run on the CUDA-core kernel.
int tc_plan_create(TcPlan** out, const Dims& dm, const TcWeights& w, void* h, void* o, void* act, int rows_full,
                   int rows_c, int lm_tiles_cap, int* err);
void tc_plan_destroy(TcPlan* p);
int tc_lm_tiles(const TcPlan* p);
int tc_gemm(TcPlan* p, Epi epi, const GemmArgs& g, cudaStream_t s);
// GEMMs of at most this many rows run on the swapped few-row kernel
constexpr int kTcFewRows = 256;

}  // namespace focus

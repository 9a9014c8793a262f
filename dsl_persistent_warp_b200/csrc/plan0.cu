// plan0.cu -- kernels of tile plan 0 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(0)

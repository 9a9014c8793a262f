// plan8.cu -- kernels of tile plan 8 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(8)

// plan1.cu -- kernels of tile plan 1 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(1)

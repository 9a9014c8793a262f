// plan2.cu -- kernels of tile plan 2 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(2)

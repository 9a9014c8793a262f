// plan3.cu -- kernels of tile plan 3 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(3)

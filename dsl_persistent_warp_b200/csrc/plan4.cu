// plan4.cu -- kernels of tile plan 4 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(4)

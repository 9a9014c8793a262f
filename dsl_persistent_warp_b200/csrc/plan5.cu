// plan5.cu -- kernels of tile plan 5 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(5)

// plan7.cu -- kernels of tile plan 7 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(7)

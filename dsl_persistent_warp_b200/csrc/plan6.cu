// plan6.cu -- kernels of tile plan 6 (see plans.h).
#include "launch.cuh"

PW_DEFINE_PLAN(6)

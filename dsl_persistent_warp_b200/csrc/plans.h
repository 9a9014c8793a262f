// plans.h -- the tile plans of the persistent GEMM, one line each, shared by the host planner
// (api.cu) and the translation units that instantiate each plan's kernels (plan*.cu).
//
// Fields, in the order of gemm_persistent's template parameters:
//   CG      CTAs per cluster tile (2: tcgen05.mma.cta_group::2, 256-row tiles)
//   BN      N of one MMA = columns of one TMEM accumulator slot
//   NSUB    MMA sub-tiles along N sharing the A stage (tile N = BN * NSUB)
//   STAGES  shared-memory ring stages
//   BK      K per stage (64 = 128-byte swizzled rows)
//   ARES    1: the A panel stays resident in shared memory (M <= 128*CG, K <= 512)
#pragma once

#define PW_PLAN0_ARGS 1, 128, 1, 6, 64, 0  // 128x128, one CTA
#define PW_PLAN1_ARGS 1, 256, 1, 4, 64, 0  // 128x256, one CTA
#define PW_PLAN2_ARGS 2, 256, 1, 6, 64, 0  // 256x256, 2-CTA cluster
#define PW_PLAN3_ARGS 2, 128, 1, 8, 64, 0  // 256x128, 2-CTA cluster
#define PW_PLAN4_ARGS 2, 256, 2, 4, 64, 0  // 256x512, 2-CTA cluster, two 256-column sub-tiles
#define PW_PLAN5_ARGS 2, 128, 1, 8, 64, 1  // 256x128, 2-CTA cluster, A resident
#define PW_PLAN6_ARGS 1, 128, 1, 4, 64, 1  // 128x128, one CTA, A resident
#define PW_PLAN7_ARGS 2, 256, 1, 4, 64, 1  // 256x256, 2-CTA cluster, A resident
#define PW_PLAN8_ARGS 1, 64, 1, 8, 64, 0   // 128x64, one CTA (thin problems)
#define PW_NUM_PLANS 9

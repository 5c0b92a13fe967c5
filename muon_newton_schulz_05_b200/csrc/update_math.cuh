// Element arithmetic of the parameter update (the update pass and the
// standalone EMA).
//   decoupled : theta <- theta (1 - lr wd) - lr s O         ("Muonとは")
//   cautious  : theta <- theta - lr wd mask theta - lr s O,
//               mask = [O M_slow > 0]                        ("ANVIL II와 가중치 평균")
//   EMA       : ema <- beta ema + (1 - beta) theta           (same section)
#pragma once

#include <cuda_bf16.h>

#include "muon_b200.h"

namespace muon {

enum UpdMode : int { kUpdDecoupled = 0, kUpdCautious = 1, kUpdWriteO = 2 };

// value as stored (bf16 values are rounded to nearest even)
__device__ __forceinline__ float stored(int dtype, float x) {
  return dtype == MUON_BF16 ? __bfloat162float(__float2bfloat16_rn(x)) : x;
}

// theta after the step (before rounding to the parameter's dtype);
// step_scale = lr * max(1, R/C)^(1/2), lr_wd = lr * weight_decay.
__device__ __forceinline__ float param_update(int mode, float th, float o, float ms,
                                              float step_scale, float lr_wd) {
  if (mode == kUpdCautious) {
    const float mask = (o * ms > 0.0f) ? 1.0f : 0.0f;
    return fmaf(-step_scale, o, fmaf(-lr_wd * mask, th, th));
  }
  return fmaf(-step_scale, o, th * (1.0f - lr_wd));
}

__device__ __forceinline__ float ema_elem(float beta, float ema, float th) {
  return fmaf(beta, ema, (1.0f - beta) * th);
}

}  // namespace muon

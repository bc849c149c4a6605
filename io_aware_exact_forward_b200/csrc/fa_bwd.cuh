// fa_bwd.cuh -- backward kernels (placeholder until the tcgen05 kernels land).
#pragma once
#include "fa_ptx.cuh"
namespace fa {
static int bwd_setup() { return FA_OK; }
}  // namespace fa

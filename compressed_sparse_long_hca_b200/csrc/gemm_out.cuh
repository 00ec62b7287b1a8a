// Output description of the projection GEMM, shared by its kernels and the
// C ABI: Y is written as up to kGemmMaxSeg row segments, rows
// [seg_end[s-1], seg_end[s]) to y[s] as a contiguous [n_tok][rows] matrix,
// BF16 when bit s of bf16_mask is set, else fp32.
#pragma once
#include <stdint.h>

namespace csa {

constexpr int kGemmMaxSeg = 8;

struct GemmOut {
  int n_seg;
  int seg_end[kGemmMaxSeg];
  void* y[kGemmMaxSeg];
  uint32_t bf16_mask;
};

}  // namespace csa

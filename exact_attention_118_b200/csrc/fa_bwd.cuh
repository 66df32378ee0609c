// fa_bwd.cuh - attention backward for sm_100a (placeholder until the kernels land).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include "fa.h"
#include "fa_ptx.cuh"

namespace fa {

inline size_t bwd_workspace_bytes(int BH, int N, int d) {
  const size_t rows = static_cast<size_t>(BH) * N;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return up(rows * d * sizeof(float)) + up(rows * sizeof(float));
}

template <typename MakeTile, typename MakeMap>
fa_status bwd_launch(const void*, const void*, const void*, const void*, const float*, const void*, void*, void*,
                     void*, void*, int, int, int, float, int, cudaStream_t, MakeTile, MakeMap) {
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa

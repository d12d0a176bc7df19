// Where the append kernels store a token's packed codes.
#pragma once
#include <cstdint>

namespace fsq {

// Token t's R code bytes go to codes + t * ldc, or, with per_row > 0, to
// codes + (t / per_row) * row_stride + (t % per_row) * ldc: the tokens form
// groups of per_row consecutive tokens (the new tokens of one row of a
// [B, T_max, R] cache), each group at its own row of the cache.
struct CodeRows {
  uint8_t *codes;
  int64_t ldc;
  int64_t per_row;
  int64_t row_stride;
  __device__ __forceinline__ uint8_t *row(int64_t t) const {
    if (per_row <= 0) return codes + t * ldc;
    return codes + (t / per_row) * row_stride + (t % per_row) * ldc;
  }
};

}  // namespace fsq

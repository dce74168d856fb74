// row_max.cuh - the maximum of one thread's BN scores (its query row's share of
// a KV block), the first step of each online-softmax block.  A NaN score makes
// the maximum NaN, so that the whole row's results are NaN (a NaN input is never
// dropped).  The maximum is exact whatever the tree's shape, so the shape is a
// pure speed choice:
//   FP8ATTN_MAX_TREE 2: 8 independent chains of two-input max, then a tree;
//   FP8ATTN_MAX_TREE 3: 16 chains of the three-input max, then a tree.
#pragma once
#include <cuda_runtime.h>

#include "sm100.cuh"

#ifndef FP8ATTN_MAX_TREE
#define FP8ATTN_MAX_TREE 2
#endif

namespace fp8attn {

template <int BN>
__device__ __forceinline__ float row_max(const float* s) {
  if constexpr (FP8ATTN_MAX_TREE == 2) {
    float m8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m8[i] = fmax_nan(s[i], s[8 + i]);
#pragma unroll
    for (int j = 16; j < BN; j += 8)
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = fmax_nan(m8[i], s[j + i]);
    return fmax_nan(fmax_nan(fmax_nan(m8[0], m8[1]), fmax_nan(m8[2], m8[3])),
                    fmax_nan(fmax_nan(m8[4], m8[5]), fmax_nan(m8[6], m8[7])));
  } else {
    float mx16[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) mx16[i] = s[i];
#pragma unroll
    for (int j = 16; j + 16 < BN; j += 32)
#pragma unroll
      for (int i = 0; i < 16; ++i) mx16[i] = fmax3(mx16[i], s[j + i], s[j + 16 + i]);
    if constexpr ((BN - 16) % 32 != 0) {
#pragma unroll
      for (int i = 0; i < 16; ++i) mx16[i] = fmax_nan(mx16[i], s[BN - 16 + i]);
    }
    float mx = fmax3(fmax3(mx16[0], mx16[1], mx16[2]), fmax3(mx16[3], mx16[4], mx16[5]),
                     fmax3(mx16[6], mx16[7], mx16[8]));
    mx = fmax3(mx, fmax3(mx16[9], mx16[10], mx16[11]), fmax3(mx16[12], mx16[13], mx16[14]));
    return fmax_nan(mx, mx16[15]);
  }
}

}  // namespace fp8attn

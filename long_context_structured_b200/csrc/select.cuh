// select.cuh -- small top-k selection helpers shared by the selector's exact
// rescan and the decoding step's top-k: a per-thread descending list and k
// rounds of a block-wide argmax over the threads' lists, both ordering by
// (logit desc, position asc).
#pragma once

#include <math_constants.h>

namespace sattn {

// insert (v, j) into the descending list (vals, idxs); strict > keeps the
// earlier (smaller j) entry first among equal scores
template <int KC>
__device__ __forceinline__ void list_insert(float v, int j, float (&vals)[KC], int (&idxs)[KC]) {
#pragma unroll
  for (int x = 0; x < KC; ++x) {
    if (v > vals[x]) {
      const float tv = vals[x];
      const int tj = idxs[x];
      vals[x] = v;
      idxs[x] = j;
      v = tv;
      j = tj;
    }
  }
}

// (oz, oj) precedes (bz, bj): larger logit, or equal with the smaller
// position; an empty slot (j < 0) precedes nothing
__device__ __forceinline__ bool sel_before(float oz, int oj, float bz, int bj) {
  return oj >= 0 && (bj < 0 || oz > bz || (oz == bz && oj < bj));
}

// k rounds of a block-wide argmax over every thread's sorted list (vals,
// idxs); round r hands (logit, position) of the r-th pick to out(r, z, j)
// on thread 0 (j = -1 once the lists are exhausted).  red_z / red_j: one
// slot per warp of the block.  Every thread of the block must call it.
template <int KC, class Out>
__device__ __forceinline__ void block_topk_rounds(int k, const float (&vals)[KC], const int (&idxs)[KC],
                                                  float* red_z, int* red_j, Out out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  int head = 0;  // next unused entry of this thread's list
  for (int r = 0; r < k; ++r) {
    float bz = -CUDART_INF_F;
    int bj = -1;
#pragma unroll
    for (int y = 0; y < KC; ++y)
      if (y == head) {
        bz = vals[y];
        bj = idxs[y];
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (sel_before(oz, oj, bz, bj)) {
        bz = oz;
        bj = oj;
      }
    }
    if (lane == 0) {
      red_z[warp] = bz;
      red_j[warp] = bj;
    }
    __syncthreads();
    float wz = red_z[0];
    int wj = red_j[0];
    for (int w = 1; w < nw; ++w) {
      const float oz = red_z[w];
      const int oj = red_j[w];
      if (sel_before(oz, oj, wz, wj)) {
        wz = oz;
        wj = oj;
      }
    }
    __syncthreads();
    if (wj >= 0 && head < KC) {
      int hj = -2;
#pragma unroll
      for (int y = 0; y < KC; ++y)
        if (y == head) hj = idxs[y];
      if (hj == wj) ++head;
    }
    if (threadIdx.x == 0) out(r, wz, wj);
  }
}

}  // namespace sattn

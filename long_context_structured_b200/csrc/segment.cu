// segment.cu -- K7: retrieval for segmented execution.
//
// "Training-Inference Consistent Segmented Execution for Long-Context LLMs"
// (sections 整体框架 and 关键设计): before segment s, each long head takes
// the top-k from a detached, read-only pool of earlier keys using the
// segment-end query, and prepends the retrieved R keys as a prefix at
// positions 0..P-1 while the segment moves to P + t.
//
// Reading used here (the pages leave the score open): the pool is every key
// j < sS of the head's kv head, unrotated; it is cut into blocks of
// `blk` keys; a block scores max_{j in block} <q_{sS-1}, k_j> with the
// unrotated query of the previous segment's last token; the best R/blk
// blocks are taken (ties to the lower block) and laid out in ascending
// block order.
//
// Rotary re-basing: only distances enter a rotary logit, so the segment's
// queries and keys keep their global positions and each prefix key p is
// rotated to the virtual position sS - P + p, which puts it at distance
// P + t - p from the query at sS + t, exactly as positions p and P + t do.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 256;

// grid (N - 1, n_long, B): segment s = blockIdx.x + 1
__global__ void __launch_bounds__(kThreads) block_select_kernel(SegRetrArgs a) {
  extern __shared__ float sm[];
  const int s = blockIdx.x + 1;
  const int slot = blockIdx.y;
  const int b = blockIdx.z;
  const int h = a.long_heads[slot];
  const int g = h / (a.Hq / a.Hkv);
  const int nb = a.R / a.blk;
  const int nblocks = s * a.S / a.blk;
  float* q = sm;                         // [d]
  float* score = sm + a.d;               // [nblocks]
  __shared__ float red_z[kThreads / 32];
  __shared__ int red_u[kThreads / 32];
  __shared__ int chosen[1024];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* qp = a.Q + b * a.q_sb + h * a.q_sh + (int64_t)(s * a.S - 1) * a.q_st;
  for (int c = threadIdx.x; c < a.d; c += blockDim.x) q[c] = __bfloat162float(qp[c]);
  __syncthreads();
  const __nv_bfloat16* kb = a.K + b * a.k_sb + g * a.k_sh;
  for (int u = warp; u < nblocks; u += kThreads / 32) {
    float best = -CUDART_INF_F;
    for (int x = lane; x < a.blk; x += 32) {
      const __nv_bfloat16* kp = kb + (int64_t)(u * a.blk + x) * a.k_st;
      float acc = 0.f;
      for (int c = 0; c < a.d; c += 2) {
        const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kp + c));
        acc = fmaf(q[c], kv.x, fmaf(q[c + 1], kv.y, acc));
      }
      best = fmaxf(best, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0) score[u] = best;
  }
  __syncthreads();
  const int nsel = min(nb, nblocks);
  for (int r = 0; r < nsel; ++r) {
    float bz = -CUDART_INF_F;
    int bu = -1;
    for (int u = threadIdx.x; u < nblocks; u += blockDim.x) {
      const float z = score[u];
      if (z == -CUDART_INF_F) continue;  // taken (scores of real blocks are finite)
      if (bu < 0 || z > bz) {
        bz = z;
        bu = u;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
      const int ou = __shfl_xor_sync(0xffffffffu, bu, o);
      if (ou >= 0 && (bu < 0 || oz > bz || (oz == bz && ou < bu))) {
        bz = oz;
        bu = ou;
      }
    }
    if (lane == 0) {
      red_z[warp] = bz;
      red_u[warp] = bu;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float wz = red_z[0];
      int wu = red_u[0];
      for (int w = 1; w < kThreads / 32; ++w) {
        const float oz = red_z[w];
        const int ou = red_u[w];
        if (ou >= 0 && (wu < 0 || oz > wz || (oz == wz && ou < wu))) {
          wz = oz;
          wu = ou;
        }
      }
      chosen[r] = wu;
      score[wu] = -CUDART_INF_F;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    // ascending block order
    for (int x = 1; x < nsel; ++x) {
      const int v = chosen[x];
      int y = x - 1;
      while (y >= 0 && chosen[y] > v) {
        chosen[y + 1] = chosen[y];
        --y;
      }
      chosen[y + 1] = v;
    }
    a.prefix_cnt[((size_t)b * a.n_long + slot) * a.N + s] = nsel * a.blk;
  }
  __syncthreads();
  int32_t* out = a.prefix_blocks + (((size_t)b * a.Hq + h) * a.N + s) * nb;
  for (int x = threadIdx.x; x < nb; x += blockDim.x) out[x] = x < nsel ? chosen[x] : -1;
}

// grid (Rpad / 8, (N - 1) * n_long, B); one warp per prefix row
__global__ void prefix_assemble_kernel(SegRetrArgs a, int Rpad) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + warp;
  const int s = blockIdx.y % (a.N - 1) + 1;
  const int slot = blockIdx.y / (a.N - 1);
  const int b = blockIdx.z;
  if (p >= Rpad) return;
  const int h = a.long_heads[slot];
  const int g = h / (a.Hq / a.Hkv);
  const int cnt = a.prefix_cnt[((size_t)b * a.n_long + slot) * a.N + s];
  const size_t orow = ((((size_t)b * a.n_long + slot) * a.N + s) * Rpad + p) * a.d;
  const int half = a.d / 2;
  const int nb = a.R / a.blk;
  if (p >= cnt) {
    for (int c = lane; c < a.d; c += 32) {
      a.Kpre[orow + c] = __float2bfloat16_rn(0.f);
      a.Vpre[orow + c] = __float2bfloat16_rn(0.f);
    }
    return;
  }
  const int blk_id = a.prefix_blocks[(((size_t)b * a.Hq + h) * a.N + s) * nb + p / a.blk];
  const int j = blk_id * a.blk + p % a.blk;
  const int vpos = s * a.S - cnt + p;
  const __nv_bfloat16* kp = a.K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
  const __nv_bfloat16* vp = a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st;
  for (int c = lane; c < half; c += 32) {
    const float k0 = __bfloat162float(kp[c]), k1 = __bfloat162float(kp[c + half]);
    const float2 cs = a.tab ? a.tab[(int64_t)vpos * half + c] : make_float2(1.f, 0.f);
    a.Kpre[orow + c] = __float2bfloat16_rn(k0 * cs.x - k1 * cs.y);
    a.Kpre[orow + c + half] = __float2bfloat16_rn(k1 * cs.x + k0 * cs.y);
  }
  for (int c = lane; c < a.d; c += 32) a.Vpre[orow + c] = vp[c];
}

}  // namespace

cudaError_t launch_segment_retrieval(const SegRetrArgs& a, cudaStream_t st) {
  if (a.N <= 1 || a.n_long == 0 || a.R == 0 || a.B == 0) return cudaSuccess;
  const int nblocks_max = (a.N - 1) * a.S / a.blk;
  const size_t smem = (size_t)(a.d + nblocks_max) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 g1(a.N - 1, a.n_long, a.B);
  block_select_kernel<<<g1, kThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int Rpad = (a.R + kTile - 1) / kTile * kTile;
  dim3 g2(Rpad / 8, (a.N - 1) * a.n_long, a.B);
  prefix_assemble_kernel<<<g2, 256, 0, st>>>(a, Rpad);
  return cudaGetLastError();
}

}  // namespace sattn

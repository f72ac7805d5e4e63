// tree.cu -- SharedLLM's tree cross-attention ("SharedLLM", sections 关键设计
// 2 and 4): the compressed context and the rotated queries.
//
// Each context chunk of length l is a binary tree.  With the
// language-modelling policy the right child is always the one expanded, so
// levels w = 1..D keep their left child and level D also its right child
// (D = 0 keeps the root).  A node is split at b = floor(m/2) (the split
// noise is 0 at test time) and a kept node of length m at level w keeps
// m' = max(1, floor(m / alpha_w)) rows at equally spaced (fractional-stride)
// offsets floor(k m / m'), with alpha_w = alpha_D 2^(D - w): coarse high
// levels, fine low ones.  The kept rows of chunk c, in text order, take the
// chunk-level rotary position c; every query takes position n = the number
// of chunks.  The attention itself then runs in the prefill kernel as
// dense cross-attention over the gathered rows.
//
//   tree_prep_kernel   one thread per 4 rotary pairs of a row: queries
//                      rotated to position n; kept K rows rotated to their
//                      chunk's position and V rows copied into dense
//                      [B, Hkv, Spad, d] arrays (rows >= n * n_kept zeroed).
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

// Offset within its chunk of the k-th kept row (text order); -1 if k is out
// of range.  rate = alpha_leaf << (depth - w) at level w.
__host__ __device__ inline int kept_offset(int l, int depth, int alpha_leaf, int k) {
  if (depth == 0) {
    const int kept = l / alpha_leaf > 1 ? l / alpha_leaf : 1;
    return k < kept ? (int)((long long)k * l / kept) : -1;
  }
  int start = 0, len = l;
  for (int w = 1; w <= depth; ++w) {
    const int b = len >> 1;
    const int rate = alpha_leaf << (depth - w);
    if (b > 0) {
      const int kept = b / rate > 1 ? b / rate : 1;
      if (k < kept) return start + (int)((long long)k * b / kept);
      k -= kept;
    }
    if (w == depth) {
      const int m = len - b;
      if (m > 0) {
        const int kept = m / rate > 1 ? m / rate : 1;
        if (k < kept) return start + b + (int)((long long)k * m / kept);
      }
      return -1;
    }
    start += b;
    len -= b;
  }
  return -1;
}

constexpr int kPairsPerThread = 4;

__device__ __forceinline__ void rotate_store(const __nv_bfloat16* src, __nv_bfloat16* dst, const float2* tab,
                                             int64_t pos, int half, int c0) {
  float x0[kPairsPerThread], x1[kPairsPerThread];
#pragma unroll
  for (int e = 0; e < kPairsPerThread; ++e) {
    x0[e] = __bfloat162float(src[c0 + e]);
    x1[e] = __bfloat162float(src[c0 + e + half]);
  }
#pragma unroll
  for (int e = 0; e < kPairsPerThread; ++e) {
    const float2 cs = tab ? tab[pos * half + c0 + e] : make_float2(1.f, 0.f);
    dst[c0 + e] = __float2bfloat16_rn(x0[e] * cs.x - x1[e] * cs.y);
    dst[c0 + e + half] = __float2bfloat16_rn(x1[e] * cs.x + x0[e] * cs.y);
  }
}

// Threads [0, q_threads) rotate query rows, the rest build the kept K/V rows;
// threads per row = d / (2 kPairsPerThread).
__global__ void tree_prep_kernel(TreeArgs a) {
  const int half = a.d / 2;
  const int tpr = half / kPairsPerThread;
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t q_threads = (int64_t)a.B * a.Hq * a.Tq * tpr;
  const int64_t kv_threads = (int64_t)a.B * a.Hkv * a.Spad * tpr;
  if (tid < q_threads) {
    const int c0 = (int)(tid % tpr) * kPairsPerThread;
    const int64_t row = tid / tpr;
    const int i = (int)(row % a.Tq);
    const int64_t bh = row / a.Tq;
    const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
    rotate_store(a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st, a.Qr + row * a.d, a.tab, a.n_chunks, half, c0);
    return;
  }
  const int64_t t2 = tid - q_threads;
  if (t2 >= kv_threads) {
    const int64_t t3 = t2 - kv_threads;
    if (a.kept_index && t3 < a.n_kept) a.kept_index[t3] = kept_offset(a.chunk_len, a.depth, a.alpha_leaf, (int)t3);
    return;
  }
  const int c0 = (int)(t2 % tpr) * kPairsPerThread;
  const int64_t row = t2 / tpr;
  const int s = (int)(row % a.Spad);
  const int64_t bg = row / a.Spad;
  const int g = (int)(bg % a.Hkv), b = (int)(bg / a.Hkv);
  __nv_bfloat16* kd = a.Kt + row * a.d;
  __nv_bfloat16* vd = a.Vt + row * a.d;
  if (s >= a.n_chunks * a.n_kept) {  // padding rows: zero keeps masked products finite
#pragma unroll
    for (int e = 0; e < kPairsPerThread; ++e) {
      kd[c0 + e] = kd[c0 + e + half] = __float2bfloat16_rn(0.f);
      vd[c0 + e] = vd[c0 + e + half] = __float2bfloat16_rn(0.f);
    }
    return;
  }
  const int c = s / a.n_kept;
  const int j = c * a.chunk_len + kept_offset(a.chunk_len, a.depth, a.alpha_leaf, s % a.n_kept);
  rotate_store(a.K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st, kd, a.tab, c, half, c0);
  const __nv_bfloat16* vs = a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st;
#pragma unroll
  for (int e = 0; e < kPairsPerThread; ++e) {
    vd[c0 + e] = vs[c0 + e];
    vd[c0 + e + half] = vs[c0 + e + half];
  }
}

}  // namespace

int tree_kept_count(int chunk_len, int depth, int alpha_leaf) {
  if (chunk_len < 1 || depth < 0 || depth > 20 || alpha_leaf < 1 || alpha_leaf > 1024) return -1;
  int n = 0;
  while (kept_offset(chunk_len, depth, alpha_leaf, n) >= 0) ++n;
  return n;
}

cudaError_t launch_tree_prep(const TreeArgs& a, cudaStream_t st) {
  const int tpr = a.d / 2 / kPairsPerThread;
  const int64_t total = ((int64_t)a.B * a.Hq * a.Tq + (int64_t)a.B * a.Hkv * a.Spad) * tpr + a.n_kept;
  if (total == 0) return cudaSuccess;
  tree_prep_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sattn

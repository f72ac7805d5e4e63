// attn_f32.cu -- K6: the same structured attention in fp32 on CUDA cores.
//
// One warp per query row.  The row's key set is walked part by part: sink
// span j < n_start, window [max(n_start, i - w), i], separators j < i - w
// from the compacted list, then the top-k keys (with their given logits).
// The parts are disjoint by construction.  Logits follow the capped rule:
// <R(L) q_i, k_j> when L > 0 and i - j > L, else <R(i) q_i, R(j) k_j>
// ("LM-Infinite", section 方法).  Online softmax in fp32.
#include <math_constants.h>

#include "kernels.cuh"

namespace sattn {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// PP pairs per lane (d = 64 * PP).  Lane owns elements c and c + d/2 for
// c = lane * PP + e.
template <int PP>
__global__ void attn_f32_kernel(AttnF32Args a) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  if (wid >= nrows) return;
  const int half = a.d / 2;
  const int i = (int)(wid % a.T);
  const int64_t bh = wid / a.T;
  const int h = (int)(bh % a.Hq);
  const int b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const float scale = rsqrtf((float)a.d);

  const float* qp = a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st;
  float qi0[PP], qi1[PP], qc0[PP], qc1[PP];
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    const float x0 = qp[c], x1 = qp[c + half];
    const float2 cs = a.tab ? a.tab[(int64_t)i * half + c] : make_float2(1.f, 0.f);
    qi0[e] = x0 * cs.x - x1 * cs.y;
    qi1[e] = x1 * cs.x + x0 * cs.y;
    const float2 cl = (a.tab && a.L > 0) ? a.tab[(int64_t)a.L * half + c] : make_float2(1.f, 0.f);
    qc0[e] = x0 * cl.x - x1 * cl.y;
    qc1[e] = x1 * cl.x + x0 * cl.y;
  }
  const float* kb = a.K + b * a.k_sb + g * a.k_sh;
  const float* vb = a.V + b * a.v_sb + g * a.v_sh;

  float m = -CUDART_INF_F, l = 0.f, o0[PP], o1[PP];
#pragma unroll
  for (int e = 0; e < PP; ++e) o0[e] = o1[e] = 0.f;

  auto logit = [&](int j) -> float {
    const float* kp = kb + (int64_t)j * a.k_st;
    const bool capped = a.L > 0 && (i - j) > a.L;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      const float k0 = kp[c], k1 = kp[c + half];
      if (capped) {
        acc = fmaf(qc0[e], k0, fmaf(qc1[e], k1, acc));
      } else {
        const float2 cs = a.tab ? a.tab[(int64_t)j * half + c] : make_float2(1.f, 0.f);
        acc = fmaf(qi0[e], k0 * cs.x - k1 * cs.y, fmaf(qi1[e], k1 * cs.x + k0 * cs.y, acc));
      }
    }
    return warp_sum(acc);
  };
  // ALiBi: -m_h * min(i - j, L) (no clip when L = 0), m_h = 2^(-8 (h+1) / Hq)
  const float slope = a.alibi ? exp2f(-8.f * (float)(h + 1) / (float)a.Hq) : 0.f;
  auto add = [&](int j, float z) {
    const int dist = (a.L > 0) ? min(i - j, a.L) : (i - j);
    const float s = z * scale - slope * (float)dist;
    const float mn = fmaxf(m, s);
    const float al = expf(m - mn);  // m = -inf -> 0
    const float p = expf(s - mn);
    l = l * al + p;
    const float* vp = vb + (int64_t)j * a.v_st;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      o0[e] = fmaf(p, vp[c], o0[e] * al);
      o1[e] = fmaf(p, vp[c + half], o1[e] * al);
    }
    m = mn;
  };

  const int n_sink = min(a.n_start, i + 1);
  for (int j = 0; j < n_sink; ++j) add(j, logit(j));
  const int w_lo = max(a.n_start, i - a.window);
  for (int j = max(0, w_lo); j <= i; ++j) add(j, logit(j));
  if (a.sep_pos) {
    const int cnt = a.sep_count[b];
    const int32_t* sp = a.sep_pos + (size_t)b * a.T;
    for (int r = 0; r < cnt; ++r) {
      const int j = sp[r];
      if (j >= i - a.window) break;  // ascending; the rest lie in the window or later
      add(j, logit(j));
    }
  }
  if (a.tk_idx) {
    const int64_t row = wid * a.topk;
    for (int x = 0; x < a.topk; ++x) {
      const int j = a.tk_idx[row + x];
      if (j >= 0 && j < a.T) add(j, a.tk_z[row + x]);
    }
  }
  float* op = a.O + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    op[c] = o0[e] * inv;
    op[c + half] = o1[e] * inv;
  }
  if (lane == 0) a.lse[wid] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
}

}  // namespace

cudaError_t launch_attn_f32(const AttnF32Args& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  if (rows == 0) return cudaSuccess;
  const int threads = 128;
  const int64_t blocks = (rows * 32 + threads - 1) / threads;
  if (a.d == 128)
    attn_f32_kernel<2><<<(unsigned)blocks, threads, 0, st>>>(a);
  else if (a.d == 64)
    attn_f32_kernel<1><<<(unsigned)blocks, threads, 0, st>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace sattn

// bwd_f32.cu -- backward pass of the structured attention in fp32 on CUDA
// cores: the gradients of sum(dO . O) with respect to Q, K and V ("SepLLM",
// section 6.2: training runs the forward and the backward pass through the
// masked product).
//
// Per row i and kept key j (the same key set and logits as the forward):
//   P_ij = exp(s_ij - LSE_i),  dP_ij = dO_i . v_j,  D_i = dO_i . O_i,
//   dz_ij = P_ij (dP_ij - D_i) / sqrt(d),
//   dV_j += P_ij dO_i;
//   uncapped pair (z = <R(i)q_i, R(j)k_j>): dq_i += R(i)^T dz R(j)k_j,
//                                          dk_j += R(j)^T dz R(i)q_i;
//   capped pair (L > 0, i - j > L; z = <R(L)q_i, k_j>): dq_i += R(L)^T dz k_j,
//                                          dk_j += dz R(L)q_i
// ("LM-Infinite", section 方法: the distance cap and its RoPE realisation).
// The top-k sets are the forward's (a constant of the backward pass).
//
// Two kernels, no atomics (deterministic):
//   bwd_f32_dq_kernel   one warp per query row: walks the row's key set
//                       (sinks, window, separators, top-k) and writes dq_i
//                       and D_i;
//   bwd_f32_dkv_kernel  one warp per key: walks the rows that keep the key
//                       (every row of the group's query heads at or after j
//                       for a sink or separator; the window rows
//                       [j, j + w]; rows whose top-k list names j) and
//                       writes dk_j and dv_j.
#include <math_constants.h>

#include "kernels.cuh"

namespace sattn {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float2 tab_at(const float2* tab, int64_t pos, int half, int c) {
  return tab ? tab[pos * half + c] : make_float2(1.f, 0.f);
}

// x -> R x on the pair (x0, x1) = (x_c, x_{c+d/2})
__device__ __forceinline__ void rot(float x0, float x1, float2 cs, float& y0, float& y1) {
  y0 = x0 * cs.x - x1 * cs.y;
  y1 = x1 * cs.x + x0 * cs.y;
}
// y -> R^T y
__device__ __forceinline__ void rot_t(float y0, float y1, float2 cs, float& x0, float& x1) {
  x0 = y0 * cs.x + y1 * cs.y;
  x1 = y1 * cs.x - y0 * cs.y;
}

// PP pairs per lane (d = 64 * PP); lane owns elements c and c + d/2 for c = lane * PP + e
template <int PP>
__global__ void bwd_f32_dq_kernel(BwdF32Args a) {
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
  const float* op = a.O + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
  const float* gp = a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
  float qi0[PP], qi1[PP], qc0[PP], qc1[PP], g0[PP], g1[PP];
  float dd = 0.f;
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    const float x0 = qp[c], x1 = qp[c + half];
    rot(x0, x1, tab_at(a.tab, i, half, c), qi0[e], qi1[e]);
    rot(x0, x1, a.L > 0 ? tab_at(a.tab, a.L, half, c) : make_float2(1.f, 0.f), qc0[e], qc1[e]);
    g0[e] = gp[c];
    g1[e] = gp[c + half];
    dd = fmaf(g0[e], op[c], fmaf(g1[e], op[c + half], dd));
  }
  const float D = warp_sum(dd);
  const float lse = a.lse[wid];
  const float* kb = a.K + b * a.k_sb + g * a.k_sh;
  const float* vb = a.V + b * a.v_sb + g * a.v_sh;
  // ALiBi: -m_h * min(i - j, L) (no clip when L = 0), m_h = 2^(-8 (h+1) / Hq)
  const float slope = a.alibi ? exp2f(-8.f * (float)(h + 1) / (float)a.Hq) : 0.f;

  float ar0[PP], ar1[PP], ac0[PP], ac1[PP];  // sums of dz * R(j)k_j and dz * k_j
#pragma unroll
  for (int e = 0; e < PP; ++e) ar0[e] = ar1[e] = ac0[e] = ac1[e] = 0.f;

  auto key = [&](int j) {
    const float* kp = kb + (int64_t)j * a.k_st;
    const float* vp = vb + (int64_t)j * a.v_st;
    const bool capped = a.L > 0 && (i - j) > a.L;
    float k0[PP], k1[PP], z = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      const float x0 = kp[c], x1 = kp[c + half];
      if (capped) {
        k0[e] = x0;
        k1[e] = x1;
        z = fmaf(qc0[e], x0, fmaf(qc1[e], x1, z));
      } else {
        rot(x0, x1, tab_at(a.tab, j, half, c), k0[e], k1[e]);
        z = fmaf(qi0[e], k0[e], fmaf(qi1[e], k1[e], z));
      }
      dp = fmaf(g0[e], vp[c], fmaf(g1[e], vp[c + half], dp));
    }
    z = warp_sum(z);
    dp = warp_sum(dp);
    const int dist = (a.L > 0) ? min(i - j, a.L) : (i - j);
    const float p = expf(z * scale - slope * (float)dist - lse);
    const float dz = p * (dp - D) * scale;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      if (capped) {
        ac0[e] = fmaf(dz, k0[e], ac0[e]);
        ac1[e] = fmaf(dz, k1[e], ac1[e]);
      } else {
        ar0[e] = fmaf(dz, k0[e], ar0[e]);
        ar1[e] = fmaf(dz, k1[e], ar1[e]);
      }
    }
  };

  const int n_sink = min(a.n_start, i + 1);
  for (int j = 0; j < n_sink; ++j) key(j);
  const int w_lo = max(a.n_start, i - a.window);
  for (int j = max(0, w_lo); j <= i; ++j) key(j);
  if (a.sep_pos) {
    const int cnt = a.sep_count[b];
    const int32_t* sp = a.sep_pos + (size_t)b * a.T;
    for (int r = 0; r < cnt; ++r) {
      const int j = sp[r];
      if (j >= i - a.window) break;  // ascending; the rest lie in the window or later
      key(j);
    }
  }
  if (a.tk_idx) {
    const int64_t row = wid * a.topk;
    for (int x = 0; x < a.topk; ++x) {
      const int j = a.tk_idx[row + x];
      if (j >= 0 && j < a.T) key(j);
    }
  }
  float* dq = a.dQ + b * a.dq_sb + h * a.dq_sh + (int64_t)i * a.dq_st;
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    float x0, x1, y0, y1;
    rot_t(ar0[e], ar1[e], tab_at(a.tab, i, half, c), x0, x1);
    rot_t(ac0[e], ac1[e], a.L > 0 ? tab_at(a.tab, a.L, half, c) : make_float2(1.f, 0.f), y0, y1);
    dq[c] = x0 + y0;
    dq[c + half] = x1 + y1;
  }
  if (lane == 0) a.Dsum[wid] = D;
}

template <int PP>
__global__ void bwd_f32_dkv_kernel(BwdF32Args a) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nkeys = (int64_t)a.B * a.Hkv * a.T;
  if (wid >= nkeys) return;
  const int half = a.d / 2;
  const int j = (int)(wid % a.T);
  const int64_t bg = wid / a.T;
  const int g = (int)(bg % a.Hkv);
  const int b = (int)(bg / a.Hkv);
  const int rep = a.Hq / a.Hkv;
  const float scale = rsqrtf((float)a.d);

  const float* kp = a.K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
  const float* vp = a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st;
  float kr0[PP], kr1[PP], kw0[PP], kw1[PP], v0[PP], v1[PP];
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    kw0[e] = kp[c];
    kw1[e] = kp[c + half];
    rot(kw0[e], kw1[e], tab_at(a.tab, j, half, c), kr0[e], kr1[e]);
    v0[e] = vp[c];
    v1[e] = vp[c + half];
  }
  const bool all_later = j < a.n_start || (a.is_sep && a.is_sep[(size_t)b * a.T + j]);
  float gr0[PP], gr1[PP], gw0[PP], gw1[PP], gv0[PP], gv1[PP];
#pragma unroll
  for (int e = 0; e < PP; ++e) gr0[e] = gr1[e] = gw0[e] = gw1[e] = gv0[e] = gv1[e] = 0.f;

  for (int h = g * rep; h < (g + 1) * rep; ++h) {
    const float slope = a.alibi ? exp2f(-8.f * (float)(h + 1) / (float)a.Hq) : 0.f;
    const int64_t rowbase = ((int64_t)b * a.Hq + h) * a.T;
    const int i_end = (all_later || a.topk > 0) ? a.T : min(a.T, j + a.window + 1);
    for (int i = j; i < i_end; ++i) {
      bool keep = all_later || (i - j <= a.window);
      if (!keep && a.tk_idx) {
        const int32_t* tl = a.tk_idx + (rowbase + i) * a.topk;
        for (int x = 0; x < a.topk; ++x) keep = keep || (tl[x] == j);
      }
      if (!keep) continue;
      const bool capped = a.L > 0 && (i - j) > a.L;
      const float* qp = a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st;
      const float* gp = a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
      float q0[PP], q1[PP], g0[PP], g1[PP], z = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < PP; ++e) {
        const int c = lane * PP + e;
        const float2 cs = capped ? tab_at(a.tab, a.L, half, c) : tab_at(a.tab, i, half, c);
        rot(qp[c], qp[c + half], cs, q0[e], q1[e]);
        z = capped ? fmaf(q0[e], kw0[e], fmaf(q1[e], kw1[e], z)) : fmaf(q0[e], kr0[e], fmaf(q1[e], kr1[e], z));
        g0[e] = gp[c];
        g1[e] = gp[c + half];
        dp = fmaf(g0[e], v0[e], fmaf(g1[e], v1[e], dp));
      }
      z = warp_sum(z);
      dp = warp_sum(dp);
      const int dist = (a.L > 0) ? min(i - j, a.L) : (i - j);
      const float p = expf(z * scale - slope * (float)dist - a.lse[rowbase + i]);
      const float dz = p * (dp - a.Dsum[rowbase + i]) * scale;
#pragma unroll
      for (int e = 0; e < PP; ++e) {
        gv0[e] = fmaf(p, g0[e], gv0[e]);
        gv1[e] = fmaf(p, g1[e], gv1[e]);
        if (capped) {
          gw0[e] = fmaf(dz, q0[e], gw0[e]);
          gw1[e] = fmaf(dz, q1[e], gw1[e]);
        } else {
          gr0[e] = fmaf(dz, q0[e], gr0[e]);
          gr1[e] = fmaf(dz, q1[e], gr1[e]);
        }
      }
    }
  }
  float* dk = a.dK + b * a.dk_sb + g * a.dk_sh + (int64_t)j * a.dk_st;
  float* dv = a.dV + b * a.dv_sb + g * a.dv_sh + (int64_t)j * a.dv_st;
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    float x0, x1;
    rot_t(gr0[e], gr1[e], tab_at(a.tab, j, half, c), x0, x1);
    dk[c] = x0 + gw0[e];
    dk[c + half] = x1 + gw1[e];
    dv[c] = gv0[e];
    dv[c + half] = gv1[e];
  }
}

template <int PP>
cudaError_t launch_pp(const BwdF32Args& a, cudaStream_t st) {
  const int threads = 128;
  const int64_t rows = (int64_t)a.B * a.Hq * a.T, keys = (int64_t)a.B * a.Hkv * a.T;
  bwd_f32_dq_kernel<PP><<<(unsigned)((rows * 32 + threads - 1) / threads), threads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_f32_dkv_kernel<PP><<<(unsigned)((keys * 32 + threads - 1) / threads), threads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_f32(const BwdF32Args& a, cudaStream_t st) {
  if ((int64_t)a.B * a.Hq * a.T == 0) return cudaSuccess;
  if (a.d == 128) return launch_pp<2>(a, st);
  if (a.d == 64) return launch_pp<1>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn

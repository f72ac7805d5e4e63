// bwd_simt.cu -- the CUDA-core parts of the bf16 backward pass ("SepLLM",
// section 6.2: training runs the forward and the backward pass through the
// masked product).
//
//   bwd_rowstats_kernel    D_i = dO_i . O_i and -LSE_i log2(e) per row,
//                          padded to whole 128-row tiles;
//   bwd_sink_rows_kernel   the starting-span keys j < n_start ("LM-Infinite",
//                          section 方法) are fp32 side keys in the forward, and
//                          here too: per row, P and dS of its sink pairs and
//                          their dq (capped pairs through R(L)^T, others
//                          through R(i)^T of R(j) k_j);
//   bwd_sink_keys_kernel   dk and dv of the sink keys: fixed-order sums over
//                          row blocks (no atomics);
//   bwd_combine_kernel     dk_j, dv_j = band-tile part + separator part (its
//                          compacted slot) + sink part, rounded to bf16.
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSinkRowBlock = 256;  // rows per partial sum of the sink-key reduction

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float2 tab_at(const float2* tab, int64_t pos, int half, int c) {
  return tab ? tab[pos * half + c] : make_float2(1.f, 0.f);
}
__device__ __forceinline__ void rot(float x0, float x1, float2 cs, float& y0, float& y1) {
  y0 = x0 * cs.x - x1 * cs.y;
  y1 = x1 * cs.x + x0 * cs.y;
}
__device__ __forceinline__ void rot_t(float y0, float y1, float2 cs, float& x0, float& x1) {
  x0 = y0 * cs.x + y1 * cs.y;
  x1 = y1 * cs.x - y0 * cs.y;
}
__device__ __forceinline__ float bf(const __nv_bfloat16* p, int64_t idx) { return __bfloat162float(p[idx]); }

// one warp per padded row
__global__ void bwd_rowstats_kernel(BwdArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.Tpad;
  if (wid >= nrows) return;
  const int i = (int)(wid % a.Tpad);
  const int64_t bh = wid / a.Tpad;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  float dd = 0.f, nl = -CUDART_INF_F;
  if (i < a.T) {
    const __nv_bfloat16* o = a.O + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
    const __nv_bfloat16* g = a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
    for (int c = lane; c < a.d; c += 32) dd = fmaf(bf(o, c), bf(g, c), dd);
    dd = warp_sum(dd);
    nl = -a.lse[bh * a.T + i] * kLog2e;
  }
  if (lane == 0) {
    a.Dsum[wid] = dd;
    a.nlse2[wid] = nl;
  }
}

// one warp per row; PP rotary pairs per lane (d = 64 PP)
template <int PP>
__global__ void bwd_sink_rows_kernel(BwdArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  if (wid >= nrows) return;
  const int half = a.d / 2;
  const int i = (int)(wid % a.T);
  const int64_t bh = wid / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const int64_t prow = bh * a.Tpad + i;
  const float D = a.Dsum[prow], nl2 = a.nlse2[prow];
  const __nv_bfloat16* gp = a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
  float g0[PP], g1[PP], ar0[PP], ar1[PP], ac0[PP], ac1[PP];
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    g0[e] = bf(gp, c);
    g1[e] = bf(gp, c + half);
    ar0[e] = ar1[e] = ac0[e] = ac1[e] = 0.f;
  }
  const int ns = min(a.n_sink, i + 1);
  for (int j = 0; j < ns; ++j) {
    const __nv_bfloat16* vp = a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st;
    const __nv_bfloat16* kp = a.K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
    float dp = 0.f;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      dp = fmaf(g0[e], bf(vp, c), fmaf(g1[e], bf(vp, c + half), dp));
    }
    dp = warp_sum(dp);
    const float p = exp2f(fmaf(a.sink_z[wid * a.n_sink + j], a.scale_log2, nl2));
    const float ds = p * (dp - D);
    if (lane == 0) {
      a.sink_ds[wid * a.n_sink + j] = ds;
      a.sink_p[wid * a.n_sink + j] = p;
    }
    const bool capped = a.L > 0 && (i - j) > a.L;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      const float x0 = bf(kp, c), x1 = bf(kp, c + half);
      if (capped) {
        ac0[e] = fmaf(ds, x0, ac0[e]);
        ac1[e] = fmaf(ds, x1, ac1[e]);
      } else {
        float y0, y1;
        rot(x0, x1, tab_at(a.tab, j, half, c), y0, y1);
        ar0[e] = fmaf(ds, y0, ar0[e]);
        ar1[e] = fmaf(ds, y1, ar1[e]);
      }
    }
  }
  const float scale = rsqrtf((float)a.d);
  float* out = a.dq_side + wid * a.d;
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const int c = lane * PP + e;
    float x0, x1, y0, y1;
    rot_t(ar0[e], ar1[e], tab_at(a.tab, i, half, c), x0, x1);
    rot_t(ac0[e], ac1[e], a.L > 0 ? tab_at(a.tab, a.L, half, c) : make_float2(1.f, 0.f), y0, y1);
    out[c] = (x0 + y0) * scale;
    out[c + half] = (x1 + y1) * scale;
  }
}

// One CTA per (b, g, sink j, row block), d/2 threads, thread p owning pair
// (p, p + d/2): sums over the block's rows i >= j of every query head of
// the group of dS_ij R(i) q_i (uncapped pairs) and dS_ij R(L) q_i (capped),
// and of P_ij dO_i.  Writes the raw-frame dk part (R(j)^T applied to the
// uncapped sum; unscaled) and the dv part.
__global__ void bwd_sink_keys_kernel(BwdArgs a) {
  const int p = threadIdx.x;
  const int half = a.d / 2;
  int64_t x = blockIdx.x;
  const int rb = (int)(x % a.nRB);
  x /= a.nRB;
  const int j = (int)(x % a.n_sink);
  x /= a.n_sink;
  const int g = (int)(x % a.Hkv), b = (int)(x / a.Hkv);
  const int rep = a.Hq / a.Hkv;
  float ur0 = 0.f, ur1 = 0.f, uc0 = 0.f, uc1 = 0.f, v0 = 0.f, v1 = 0.f;
  const int i_lo = max(j, rb * kSinkRowBlock), i_hi = min(a.T, (rb + 1) * kSinkRowBlock);
  const float2 cl = a.L > 0 ? tab_at(a.tab, a.L, half, p) : make_float2(1.f, 0.f);
  for (int h = g * rep; h < (g + 1) * rep; ++h) {
    const int64_t bh = (int64_t)b * a.Hq + h;
    for (int i = i_lo; i < i_hi; ++i) {
      const int64_t wid = bh * a.T + i;
      const float ds = a.sink_ds[wid * a.n_sink + j];
      const float pj = a.sink_p[wid * a.n_sink + j];
      const __nv_bfloat16* qp = a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st;
      const __nv_bfloat16* gp = a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
      const float q0 = bf(qp, p), q1 = bf(qp, p + half);
      const bool capped = a.L > 0 && (i - j) > a.L;
      float y0, y1;
      rot(q0, q1, capped ? cl : tab_at(a.tab, i, half, p), y0, y1);
      if (capped) {
        uc0 = fmaf(ds, y0, uc0);
        uc1 = fmaf(ds, y1, uc1);
      } else {
        ur0 = fmaf(ds, y0, ur0);
        ur1 = fmaf(ds, y1, ur1);
      }
      v0 = fmaf(pj, bf(gp, p), v0);
      v1 = fmaf(pj, bf(gp, p + half), v1);
    }
  }
  float x0, x1;
  rot_t(ur0, ur1, tab_at(a.tab, j, half, p), x0, x1);
  float* part = a.sink_part + (size_t)blockIdx.x * 2 * a.d;
  part[p] = x0 + uc0;
  part[p + half] = x1 + uc1;
  part[a.d + p] = v0;
  part[a.d + p + half] = v1;
}

// one thread per 8 consecutive elements of one key row
__global__ void bwd_combine_kernel(BwdArgs a) {
  const int per_row = a.d / 8;
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)a.B * a.Hkv * a.T * per_row;
  if (tid >= total) return;
  const int c0 = (int)(tid % per_row) * 8;
  const int64_t key = tid / per_row;
  const int j = (int)(key % a.T);
  const int64_t bg = key / a.T;
  const int g = (int)(bg % a.Hkv), b = (int)(bg / a.Hkv);
  float k[8], v[8];
  const float* kb = a.dk_band + key * a.d + c0;
  const float* vb = a.dv_band + key * a.d + c0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    k[e] = kb[e];
    v[e] = vb[e];
  }
  if (a.gather && j >= a.n_start) {
    const int32_t* pre = a.sep_prefix + (size_t)b * (a.T + 1);
    const int r = pre[j];
    if (pre[j + 1] > r) {  // j is a separator: its compacted slot r
      const float* ks = a.dk_sep + (bg * a.Tpad + r) * a.d + c0;
      const float* vs = a.dv_sep + (bg * a.Tpad + r) * a.d + c0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        k[e] += ks[e];
        v[e] += vs[e];
      }
    }
  }
  if (j < a.n_sink) {
    const float scale = rsqrtf((float)a.d);
    const float* part = a.sink_part + (size_t)((bg * a.n_sink + j) * a.nRB) * 2 * a.d;
    for (int rb = 0; rb < a.nRB; ++rb) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        k[e] = fmaf(part[(size_t)rb * 2 * a.d + c0 + e], scale, k[e]);
        v[e] += part[(size_t)rb * 2 * a.d + a.d + c0 + e];
      }
    }
  }
  __nv_bfloat16* dk = a.dK + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st + c0;
  __nv_bfloat16* dv = a.dV + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st + c0;
  uint4 ko, vo;
  ko.x = pack_bf16x2(k[0], k[1]);
  ko.y = pack_bf16x2(k[2], k[3]);
  ko.z = pack_bf16x2(k[4], k[5]);
  ko.w = pack_bf16x2(k[6], k[7]);
  vo.x = pack_bf16x2(v[0], v[1]);
  vo.y = pack_bf16x2(v[2], v[3]);
  vo.z = pack_bf16x2(v[4], v[5]);
  vo.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dk) = ko;
  *reinterpret_cast<uint4*>(dv) = vo;
}

}  // namespace

int bwd_sink_row_block() { return kSinkRowBlock; }

cudaError_t launch_bwd_rowstats(const BwdArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Hq * a.Tpad;
  if (rows == 0) return cudaSuccess;
  bwd_rowstats_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_sink_rows(const BwdArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  if (rows == 0 || a.n_sink == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows * 32 + 127) / 128);
  if (a.d == 128)
    bwd_sink_rows_kernel<2><<<blocks, 128, 0, st>>>(a);
  else if (a.d == 64)
    bwd_sink_rows_kernel<1><<<blocks, 128, 0, st>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_bwd_sink_keys(const BwdArgs& a, cudaStream_t st) {
  const int64_t blocks = (int64_t)a.B * a.Hkv * a.n_sink * a.nRB;
  if (blocks == 0) return cudaSuccess;
  bwd_sink_keys_kernel<<<(unsigned)blocks, a.d / 2, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_combine(const BwdArgs& a, cudaStream_t st) {
  const int64_t total = (int64_t)a.B * a.Hkv * a.T * (a.d / 8);
  if (total == 0) return cudaSuccess;
  bwd_combine_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sattn

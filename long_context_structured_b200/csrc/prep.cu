// prep.cu -- K1: rotary table and the elementwise prep pass.
//
// Rotary convention: rotate-half; pair (c, c + d/2) turns by the angle
// p * theta^(-2c/d).  The capped logit ("LM-Infinite", section 方法, RoPE
// realisation of d'_ij = min(d_ij, L)) needs, besides R(i) q_i and R(j) k_j,
// the query rotated to the cap, R(L) q_i, paired with the unrotated key.
//
// Outputs (all optional): Qr = R(i) q_i, Qc = R(L) q_i, Kr = R(j) k_j as bf16
// tensor-core operands; the fp32 logits of the starting-span ("sink") keys,
// computed from fp32 rotations of the exact inputs so that the large sink
// logits do not inherit bf16 operand rounding; and per (batch, kv head) the
// largest key norm, used by the top-k selector to bound bf16 scoring error.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"

namespace sattn {

namespace {

__global__ void rope_table_kernel(float2* tab, int npos, int half, int d, double theta) {
  const int64_t n = (int64_t)npos * half;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(x / half);
    const int c = (int)(x % half);
    const double inv_freq = pow(theta, -2.0 * (double)c / (double)d);
    double s, co;
    sincos((double)p * inv_freq, &s, &co);
    tab[x] = make_float2((float)co, (float)s);
  }
}

template <typename Tin>
__device__ __forceinline__ float ld_in(const Tin* p);
template <>
__device__ __forceinline__ float ld_in<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float ld_in<float>(const float* p) {
  return *p;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// PP = pairs per lane = d / 64.  Lane l owns pairs c = l*PP + e, e < PP,
// i.e. elements c and c + d/2.
template <typename Tin, int PP>
__global__ void prep_kernel(PrepArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int half = a.d / 2;
  const int64_t nq = (int64_t)a.B * a.Hq * a.T;
  const int64_t nk = (int64_t)a.B * a.Hkv * a.T;
  const Tin* Q = reinterpret_cast<const Tin*>(a.Q);
  const Tin* K = reinterpret_cast<const Tin*>(a.K);
  if (wid < nq) {
    const int i = (int)(wid % a.T);
    const int64_t bh = wid / a.T;
    const int h = (int)(bh % a.Hq);
    const int b = (int)(bh / a.Hq);
    const int g = h / (a.Hq / a.Hkv);
    const Tin* qp = Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st;
    float x0[PP], x1[PP], r0[PP], r1[PP], c0[PP], c1[PP];
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      x0[e] = ld_in(qp + c);
      x1[e] = ld_in(qp + c + half);
      float2 cs = a.tab ? a.tab[(int64_t)i * half + c] : make_float2(1.f, 0.f);
      r0[e] = x0[e] * cs.x - x1[e] * cs.y;
      r1[e] = x1[e] * cs.x + x0[e] * cs.y;
      float2 cl = (a.tab && a.L > 0) ? a.tab[(int64_t)a.L * half + c] : make_float2(1.f, 0.f);
      c0[e] = x0[e] * cl.x - x1[e] * cl.y;
      c1[e] = x1[e] * cl.x + x0[e] * cl.y;
    }
    const int64_t orow = wid * a.d;
    if (a.Qr) {
#pragma unroll
      for (int e = 0; e < PP; ++e) {
        const int c = lane * PP + e;
        a.Qr[orow + c] = __float2bfloat16_rn(r0[e]);
        a.Qr[orow + c + half] = __float2bfloat16_rn(r1[e]);
      }
    }
    if (a.Qc) {
#pragma unroll
      for (int e = 0; e < PP; ++e) {
        const int c = lane * PP + e;
        a.Qc[orow + c] = __float2bfloat16_rn(c0[e]);
        a.Qc[orow + c + half] = __float2bfloat16_rn(c1[e]);
      }
    }
    if (a.sink_z) {
      const Tin* kb = K + b * a.k_sb + g * a.k_sh;
      for (int j = 0; j < a.n_sink; ++j) {
        float z;
        if (j > i || j >= a.T) {
          z = -CUDART_INF_F;
        } else {
          const Tin* kp = kb + (int64_t)j * a.k_st;
          const bool capped = a.L > 0 && (i - j) > a.L;
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < PP; ++e) {
            const int c = lane * PP + e;
            const float k0 = ld_in(kp + c), k1 = ld_in(kp + c + half);
            if (capped) {
              acc = fmaf(c0[e], k0, acc);
              acc = fmaf(c1[e], k1, acc);
            } else {
              const float2 cs = a.tab ? a.tab[(int64_t)j * half + c] : make_float2(1.f, 0.f);
              const float kr0 = k0 * cs.x - k1 * cs.y;
              const float kr1 = k1 * cs.x + k0 * cs.y;
              acc = fmaf(r0[e], kr0, acc);
              acc = fmaf(r1[e], kr1, acc);
            }
          }
          z = warp_sum(acc);
        }
        if (lane == 0) a.sink_z[wid * a.n_sink + j] = z;
      }
    }
  } else if (wid < nq + nk) {
    const int64_t kw = wid - nq;
    const int j = (int)(kw % a.T);
    const int64_t bg = kw / a.T;
    const int g = (int)(bg % a.Hkv);
    const int b = (int)(bg / a.Hkv);
    const Tin* kp = K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      const float k0 = ld_in(kp + c), k1 = ld_in(kp + c + half);
      ss = fmaf(k0, k0, fmaf(k1, k1, ss));
      if (a.Kr) {
        const float2 cs = a.tab ? a.tab[(int64_t)j * half + c] : make_float2(1.f, 0.f);
        a.Kr[kw * a.d + c] = __float2bfloat16_rn(k0 * cs.x - k1 * cs.y);
        a.Kr[kw * a.d + c + half] = __float2bfloat16_rn(k1 * cs.x + k0 * cs.y);
      }
    }
    if (a.kmax) {
      ss = warp_sum(ss);
      if (lane == 0) atomicMax(a.kmax + bg, __float_as_uint(sqrtf(ss)));
    }
  }
}

template <typename Tin>
cudaError_t launch_prep_t(const PrepArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * (a.Hq + a.Hkv) * a.T;
  const int threads = 256;
  const int64_t blocks = (rows * 32 + threads - 1) / threads;
  if (blocks == 0) return cudaSuccess;
  if (a.d == 128)
    prep_kernel<Tin, 2><<<(unsigned)blocks, threads, 0, st>>>(a);
  else if (a.d == 64)
    prep_kernel<Tin, 1><<<(unsigned)blocks, threads, 0, st>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope_table(float2* tab, int npos, int d, double theta, cudaStream_t st) {
  const int half = d / 2;
  const int64_t n = (int64_t)npos * half;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 148 * 16);
  rope_table_kernel<<<(unsigned)blocks, threads, 0, st>>>(tab, npos, half, d, theta);
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st) {
  return a.f32 ? launch_prep_t<float>(a, st) : launch_prep_t<__nv_bfloat16>(a, st);
}

}  // namespace sattn
